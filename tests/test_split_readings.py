"""Pins of the arithmetic behind the e4m3 kernel's exactness readings (CPU).

These check the two splits the e4m3 kernel relies on, from their
definitions, with torch's float8_e4m3fn cast (round to nearest even) as the
e4m3 encoder; neither the CUDA path nor the oracle is involved.

* Q split: a head's bf16 query times 2^a, with the frame a chosen so that the
  largest |q 2^a| lies in [128, 256), equals hi + lo exactly (hi = e4m3(x),
  lo = e4m3(x - hi)) for every element of at least 2^-9 of the largest; at
  2^-10 that no longer holds for all elements.
* P split: an fp16 P is hi = its sign, exponent and three leading mantissa
  bits (exact in e4m3 from 2^-6 up) plus lo = the rest rounded to e4m3, and
  |P - (hi + lo)| <= max(2^-7 P, 2^-9) over every fp16 value in [0, 256):
  relative 2^-7 from 2^-3 up, absolute below, where lo and then hi fall into
  e4m3's subnormal range.
"""
import math

import torch


def _e4m3(x: torch.Tensor) -> torch.Tensor:
    return x.to(torch.float8_e4m3fn).float()


def _q_split(q: torch.Tensor):
    amax = q.abs().max().item()
    a = min(120, max(-120, 7 - math.floor(math.log2(amax))))
    x = q * 2.0 ** a                                   # exact: a power of two
    hi = _e4m3(x)
    lo = _e4m3(x - hi)
    return x, hi, lo


def _q_rows(seed: int, n: int = 300):
    g = torch.Generator().manual_seed(seed)
    for _ in range(n):
        spread = float(torch.rand(1, generator=g) * 4)
        q = torch.randn(512, generator=g) * torch.exp(torch.randn(512, generator=g) * spread)
        q = q * 2.0 ** int(torch.randint(-30, 30, (1,), generator=g))
        yield q.to(torch.bfloat16).float()


def test_q_frame_puts_the_largest_in_128_256():
    for q in _q_rows(1, 100):
        x, _, _ = _q_split(q)
        assert 128 <= x.abs().max().item() < 256


def test_q_split_exact_above_2_pow_minus_9_of_the_largest():
    for q in _q_rows(2):
        x, hi, lo = _q_split(q)
        big = x.abs() >= 2.0 ** -9 * x.abs().max()
        assert torch.equal((hi + lo)[big], x[big])
        # and never off by more than the e4m3 subnormal step below it
        assert (x - hi - lo).abs().max().item() <= 2.0 ** -10


def test_q_split_is_not_exact_at_2_pow_minus_10():
    # the bound above is the boundary: some element at 2^-10 of the largest
    # (a residual on a 2^-10 grid, below e4m3's smallest subnormal) is lost
    lost = False
    for q in _q_rows(3):
        x, hi, lo = _q_split(q)
        band = (x.abs() >= 2.0 ** -10 * x.abs().max()) & (x.abs() < 2.0 ** -9 * x.abs().max())
        lost |= bool(((hi + lo) != x)[band].any())
    assert lost


def _p_split(p16: torch.Tensor):
    bits = p16.view(torch.int16)
    hi16 = (bits & torch.tensor(0xFF80 - 0x10000, dtype=torch.int16)).view(torch.float16)
    rest = p16.float() - hi16.float()
    assert torch.equal(rest.to(torch.float16).float(), rest)     # exact in fp16
    return _e4m3(hi16.float()), _e4m3(rest), hi16.float()


def test_p_split_bound_over_every_fp16_below_256():
    p16 = torch.arange(0, 0x5C00, dtype=torch.int32).to(torch.int16).view(torch.float16)
    p = p16.float()
    hi, lo, hi16 = _p_split(p16)
    err = (p - hi - lo).abs()
    assert bool((err <= torch.maximum(2.0 ** -7 * p, torch.full_like(p, 2.0 ** -9))).all())
    upper = p >= 2.0 ** -3
    assert bool((err[upper] <= 2.0 ** -7 * p[upper]).all())
    # hi is exact in e4m3 wherever it is normal there
    normal = hi16 >= 2.0 ** -6
    assert torch.equal(hi[normal], hi16[normal])


def test_p_split_relative_bound_fails_below_2_pow_minus_3():
    # the relative 2^-7 does not extend below 2^-3 (lo becomes subnormal)
    p16 = torch.arange(0x2400, 0x3000, dtype=torch.int32).to(torch.int16).view(torch.float16)
    p = p16.float()                                             # [2^-6, 2^-3)
    hi, lo, _ = _p_split(p16)
    assert bool(((p - hi - lo).abs() > 2.0 ** -7 * p).any())
