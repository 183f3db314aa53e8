"""Exact addressing over whole full-size batches, on the GPU, through the C ABI.

Id-coded caches (the row of global token t carries the bits of t, every
query is zero) at the agentic configuration's length mix (64 requests,
lognormal lengths up to 200,000, N = 1 and 8 shards) and at the million-token
configuration (one request of 2^20 tokens, N = 8, split over many CTAs per
shard).  Every query weighs every token of its shard equally, so for shard s
of request b with n tokens the LSE is ln n and n * O[d] is the number of the
shard's token ids with bit d set: both are known in closed form, so every
request, shard and head of the batch is checked, with no oracle run.  This
covers the CTA slices, segment batches and split-slot bookkeeping that
sampled parity checks leave out.
"""
import math

import numpy as np
import pytest
import torch

from long_context_decode_mla_b200 import dcpmla
from long_context_decode_mla_b200 import workload as wl

pytestmark = pytest.mark.gpu

BITS = wl.ID_BITS


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    dcpmla.lib()
    torch.cuda.set_device(0)


def _expected(L, s, N):
    """(n, per-bit counts) of the token ids t < L with t mod N == s."""
    ids = np.arange(s, L, N, dtype=np.int64)
    if ids.size == 0:
        return 0, np.zeros(BITS, dtype=np.int64)
    return ids.size, ((ids[:, None] >> np.arange(BITS)[None, :]) & 1).sum(axis=0)


def _check(lens, N, num_splits=0):
    prob = wl.id_coded_problem_device(lens, N, "fp8", heads=64, seed=7 + N)
    dec = dcpmla.DcpDecoder(prob.batch, prob.heads, N, num_splits=num_splits)
    dec.step(prob)
    torch.cuda.synchronize()
    assert dec.flags() == 0
    parts = dec.partials[:, :, :, :BITS].double().cpu().numpy()
    rest_zero = bool((dec.partials[:, :, :, BITS:] == 0).all())
    lses = dec.lses.double().cpu().numpy()
    assert rest_zero, "values beyond the id bits must be 0"
    for b, L in enumerate(lens):
        for s in range(N):
            n, cnt = _expected(int(L), s, N)
            if n == 0:
                assert np.all(np.isneginf(lses[s, b])) and not parts[s, b].any()
                continue
            assert np.abs(lses[s, b] - math.log(n)).max() < 1e-5, (b, s)
            scaled = parts[s, b] * n                      # [heads, bits]
            assert np.all(np.rint(scaled) == cnt[None, :]), (b, s)
            assert np.abs(scaled - cnt[None, :]).max() <= 1e-4 * n + 1e-3, (b, s)
    # the merge of N equal-weight shards: LSE ln L and L * O[d] = all ids' bits
    out = dec.out[:, :, :BITS].double().cpu().numpy()
    lse = dec.out_lse.double().cpu().numpy()
    for b, L in enumerate(lens):
        n, cnt = _expected(int(L), 0, 1)
        assert np.abs(lse[b] - math.log(n)).max() < 1e-5
        assert np.all(np.rint(out[b] * n) == cnt[None, :]), b


@pytest.mark.parametrize("N", [1, 8])
def test_agentic_length_mix_every_request(N):
    lens = wl.lognormal_lengths(64, wl.CONFIGS["agentic"]["seed"]).tolist()
    _check(lens, N)


def test_million_token_request_over_split_ctas():
    _check([1 << 20], 8, num_splits=max(1, dcpmla.device_sm_count() // 8))
