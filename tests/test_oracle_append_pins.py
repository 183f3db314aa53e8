"""Pins of the cache-write oracle (``oracle/cache_write.py``) against facts that
do not come from the oracle itself: the E4M3 value table and an independent
library cast, exact midpoint ties and saturation, the defining properties of
the per-group quantiser, an independent torch packing of the same rule, and
the decode oracle's own row fetch for placement and ownership.  Planted
mistakes at the end check that these pins catch plausible errors."""
import numpy as np
import pytest
import torch

import oracle
from oracle import cache_write as ka
from long_context_decode_mla_b200 import workload as wl

ALL_FINITE = [c for c in range(256) if (c & 0x7F) != 0x7F]


def _bf16_bits(x: torch.Tensor) -> np.ndarray:
    return x.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


# ------------------------------------------------------------- E4M3 encoder --

def test_every_finite_code_round_trips():
    vals = np.array([oracle.e4m3_value(c) for c in ALL_FINITE], dtype=np.float32)
    codes = oracle.encode_e4m3(vals)
    for c, got in zip(ALL_FINITE, codes):
        assert int(got) == c, (hex(c), hex(int(got)))


def test_midpoints_tie_to_the_even_code():
    pos = [c for c in range(0x7F)]
    for a, b in zip(pos[:-1], pos[1:]):
        mid = (oracle.e4m3_value(a) + oracle.e4m3_value(b)) / 2
        even = a if a % 2 == 0 else b
        assert int(oracle.encode_e4m3(np.float32(mid))) == even
        assert int(oracle.encode_e4m3(np.float32(-mid))) == even | 0x80
        # just off the midpoint goes to the nearer value
        below = np.nextafter(np.float32(mid), np.float32(0))
        above = np.nextafter(np.float32(mid), np.float32(1e9))
        assert int(oracle.encode_e4m3(below)) == a
        assert int(oracle.encode_e4m3(above)) == b


def test_saturation_and_signed_zero():
    assert int(oracle.encode_e4m3(np.float32(448.0))) == 0x7E
    for v in (449.0, 464.0, 480.0, 1e6, np.float32(3.4e38)):
        assert int(oracle.encode_e4m3(np.float32(v))) == 0x7E
        assert int(oracle.encode_e4m3(np.float32(-v))) == 0xFE
    assert int(oracle.encode_e4m3(np.float32(0.0))) == 0x00
    assert int(oracle.encode_e4m3(np.float32(-0.0))) == 0x80
    # below half the smallest subnormal (2^-9 / 2) rounds to zero, at it ties to zero
    assert int(oracle.encode_e4m3(np.float32(2.0 ** -10))) == 0x00
    assert int(oracle.encode_e4m3(np.float32(2.0 ** -10 * 1.0001))) == 0x01


def test_matches_an_independent_library_cast():
    g = torch.Generator().manual_seed(7)
    x = torch.cat([torch.randn(20000, generator=g) * s for s in (0.01, 1.0, 30.0, 200.0)])
    x = x.clamp(-448, 448)
    ref = x.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = oracle.encode_e4m3(x.numpy())
    assert np.array_equal(got, ref)


# --------------------------------------------------------------- quantiser --

def test_quantised_row_layout_and_defining_properties():
    g = torch.Generator().manual_seed(11)
    group_scale = torch.tensor([0.001, 1.0, 50.0, 0.0]).repeat_interleave(128)
    lat = torch.randn(512, generator=g) * group_scale
    rope = torch.randn(64, generator=g)
    lb, rb = _bf16_bits(lat), _bf16_bits(rope)
    row = oracle.quantize_fp8_row(lb, rb)
    assert row.shape == (656,) and row.dtype == np.uint8
    scales = row[512:528].view("<f4")
    x = oracle.decode_bf16(lb).astype(np.float32)
    for grp in range(4):
        part = x[128 * grp:128 * grp + 128]
        amax = np.float32(np.abs(part).max())
        if amax == 0:
            assert scales[grp] == 1.0 and not (row[128 * grp:128 * grp + 128] & 0x7F).any()
            continue
        assert scales[grp] == np.float32(amax / np.float32(448))
        codes = row[128 * grp:128 * grp + 128]
        dec = oracle.decode_e4m3(codes) * np.float64(scales[grp])
        # the largest magnitude maps to +-448 (within one code of saturation)
        k = int(np.argmax(np.abs(part)))
        assert abs(oracle.e4m3_value(int(codes[k]) & 0x7F) - 448.0) <= 32.0
        # every value within half a step of E4M3 (relative 2^-4 for normals,
        # absolute 2^-10 * scale for subnormals)
        tol = np.maximum(np.abs(part) * 2.0 ** -4, 2.0 ** -10 * float(scales[grp])) * 1.0001
        assert np.all(np.abs(dec - part) <= tol)
    assert np.array_equal(row[528:].view("<u2"), rb)


def test_quantiser_matches_the_independent_torch_packing():
    """workload.pack_fp8_rows applies the same rule with torch ops (fp32
    division and the library cast); the bytes must agree exactly."""
    g = torch.Generator().manual_seed(12)
    x = torch.randn(200, 576, generator=g) * torch.rand(200, 1, generator=g) * 100
    x[3, :128] = 0.0                                    # a zero group
    xb = x.to(torch.bfloat16)
    ref = wl.pack_fp8_rows(xb[:, :512].float(), xb[:, 512:]).numpy()
    for i in range(200):
        got = oracle.quantize_fp8_row(_bf16_bits(xb[i, :512]), _bf16_bits(xb[i, 512:]))
        assert np.array_equal(got, ref[i]), i


# ---------------------------------------------------- ownership and placement --

def _tables(B, N, nblk, seed):
    rng = np.random.default_rng(seed)
    perm = rng.permutation(N * B * nblk).astype(np.int32)
    return perm.reshape(N, B, nblk)


@pytest.mark.parametrize("kv_dtype", ["bf16", "fp8"])
@pytest.mark.parametrize("N", [1, 2, 3, 4, 8])
def test_each_token_lands_once_on_its_owner_where_decode_reads_it(kv_dtype, N):
    B, nblk = 3, 4
    tables = _tables(B, N, nblk, seed=N)
    rb = oracle.FP8_ROW_BYTES if kv_dtype == "fp8" else oracle.BF16_ROW_BYTES
    pool = np.zeros((N * B * nblk, 64, rb), dtype=np.uint8)
    g = torch.Generator().manual_seed(100 + N)
    T = 40
    pos = torch.randint(0, 64 * nblk, (T,), generator=g).numpy().astype(np.int32)
    req = torch.randint(0, B, (T,), generator=g).numpy().astype(np.int32)
    # distinct (request, position) pairs so each row is written once
    _, keep = np.unique(req.astype(np.int64) * 100000 + pos, return_index=True)
    pos, req = pos[keep], req[keep]
    lat = _bf16_bits(torch.randn(len(pos), 512, generator=g))
    rope = _bf16_bits(torch.randn(len(pos), 64, generator=g))
    cache = pool
    for s in range(N):
        before = cache.copy()
        cache, flags = oracle.kv_append(cache, kv_dtype, lat, rope, pos, req, tables[s], s, N)
        assert flags == 0
        changed = np.argwhere((cache != before).any(axis=2))
        owned = [(i, int(pos[i]) // N) for i in range(len(pos)) if pos[i] % N == s]
        # rows that changed are exactly the owned tokens' rows
        expect = {(int(tables[s][req[i], j // 64]), j % 64) for i, j in owned}
        assert {(int(a), int(b)) for a, b in changed} <= expect
    for i in range(len(pos)):
        s, j = int(pos[i]) % N, int(pos[i]) // N
        got = oracle.fetch_rows(cache, kv_dtype, tables[s][req[i]], np.array([pos[i]]), N, 64)
        want_row = oracle.quantize_fp8_row(lat[i], rope[i]) if kv_dtype == "fp8" else \
            oracle.bf16_row(lat[i], rope[i])
        want = oracle.decode_rows(want_row[None, :], kv_dtype)
        assert np.array_equal(got, want)


def test_skips_and_flags():
    N, B, nblk = 2, 2, 2
    tables = _tables(B, N, nblk, seed=5)
    pool = np.zeros((N * B * nblk, 64, oracle.FP8_ROW_BYTES), dtype=np.uint8)
    lat = _bf16_bits(torch.ones(5, 512))
    rope = _bf16_bits(torch.ones(5, 64))
    bad = tables.copy()
    bad[0, 1, 0] = 10 ** 6
    # pad, ok, beyond the table, bad block row, non-owner
    pos = np.array([-1, 0, 2 * 64 * nblk, 4, 1], dtype=np.int32)
    req = np.array([0, 0, 0, 1, 0], dtype=np.int32)
    out, flags = oracle.kv_append(pool, "fp8", lat, rope, pos, req, bad[0], 0, N)
    assert flags == ka.FLAG_BAD_LENGTH | ka.FLAG_BAD_BLOCK
    assert (out != pool).any(axis=2).sum() == 1          # only position 0 was written
    out2, flags2 = oracle.kv_append(pool, "fp8", lat, rope, np.array([0], np.int32),
                                    np.array([7], np.int32), bad[0], 0, N)
    assert flags2 == ka.FLAG_BAD_LENGTH and np.array_equal(out2, pool)


# -------------------------------------------------------- planted mistakes --

def test_planted_truncating_encoder_is_caught(monkeypatch):
    def truncating(x):
        x = np.asarray(x, dtype=np.float32)
        a = np.minimum(np.abs(x.astype(np.float64)), 448.0)
        idx = np.searchsorted(ka._POS_VALUES, a, side="right") - 1
        return (np.clip(idx, 0, 0x7E).astype(np.uint8) | (np.signbit(x).astype(np.uint8) << 7))
    monkeypatch.setattr(ka, "encode_e4m3", truncating)
    monkeypatch.setattr(oracle, "encode_e4m3", truncating)
    with pytest.raises(AssertionError):
        test_midpoints_tie_to_the_even_code()


def test_planted_odd_tie_rule_is_caught(monkeypatch):
    real = ka.encode_e4m3

    def odd_ties(x):
        c = real(x)
        x = np.asarray(x, dtype=np.float32)
        a = np.abs(x.astype(np.float64))
        lo = np.clip(np.searchsorted(ka._POS_VALUES, a, side="left") - 1, 0, 0x7E)
        hi = np.clip(lo + 1, 0, 0x7E)
        tie = np.isclose(a, (ka._POS_VALUES[lo] + ka._POS_VALUES[hi]) / 2, rtol=0, atol=0)
        return np.where(tie & (lo % 2 == 1), lo, np.where(tie, hi, c & 0x7F)).astype(np.uint8) | \
            (c & 0x80)
    monkeypatch.setattr(oracle, "encode_e4m3", odd_ties)
    with pytest.raises(AssertionError):
        test_midpoints_tie_to_the_even_code()


def test_planted_write_on_every_shard_is_caught(monkeypatch):
    real = ka.kv_append

    def everywhere(kv_cache, kv_dtype, latent_bits, rope_bits, positions, req_idx, block_table,
                   shard_id, num_shards):
        # writes every token on every shard, at the owner's local row
        p = np.asarray(positions).copy()
        fake = p - (p % num_shards) + shard_id
        return real(kv_cache, kv_dtype, latent_bits, rope_bits, fake, req_idx, block_table,
                    shard_id, num_shards)
    monkeypatch.setattr(oracle, "kv_append", everywhere)
    with pytest.raises(AssertionError):
        test_each_token_lands_once_on_its_owner_where_decode_reads_it("fp8", 2)
