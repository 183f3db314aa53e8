"""PCP host logic (no GPU): the library's chunk plan against the oracle's, and
the PCP entry points failing closed before any launch."""
import ctypes

import numpy as np
import pytest

import oracle
from long_context_decode_mla_b200 import dcpmla

EINVAL, EUNSUP, EWS, EALIGN = -1, -2, -3, -4
FAKE = 0x10000          # aligned, never dereferenced


@pytest.mark.parametrize("P", [1, 2, 3, 8])
@pytest.mark.parametrize("T", [0, 1, 5, 15, 16, 17, 100, 1000, 65537])
def test_rank_tokens_match_the_oracle_plan(T, P):
    got = [dcpmla.pcp_rank_tokens(T, P, r) for r in range(P)]
    for r in range(P):
        assert got[r] == oracle.pcp_rank_tokens(T, P, r).tolist()
    # the ranks' tokens partition the prompt
    assert sorted(t for g in got for t in g) == list(range(T))


def test_rank_tokens_refuse_bad_arguments():
    L = dcpmla.lib()
    n = ctypes.c_int(0)
    assert L.pcp_rank_tokens(-1, 8, 0, None, 0, ctypes.byref(n)) == EINVAL
    assert L.pcp_rank_tokens(10, 0, 0, None, 0, ctypes.byref(n)) == EINVAL
    assert L.pcp_rank_tokens(10, 8, 8, None, 0, ctypes.byref(n)) == EINVAL
    assert L.pcp_rank_tokens(100, 8, 0, None, 0, ctypes.byref(n)) == 0 and n.value == 13
    buf = (ctypes.c_int32 * 4)()
    assert L.pcp_rank_tokens(100, 8, 0, buf, 4, ctypes.byref(n)) == EINVAL   # too small


def test_gathered_size_is_whole_blocks():
    assert dcpmla.pcp_gathered_bytes(1, "fp8") == 64 * 656
    assert dcpmla.pcp_gathered_bytes(64, "bf16") == 64 * 1152
    assert dcpmla.pcp_gathered_bytes(65, "fp8") == 128 * 656
    assert dcpmla.pcp_gathered_bytes(0, "fp8") == 0


def test_gather_fails_closed_before_any_launch():
    L = dcpmla.lib()

    def call(kvd=1, nb=16, bs=64, stride=4, N=8, T=100, out=FAKE, nbytes=1 << 20, kv=FAKE):
        return L.pcp_gather_rows(kv, kvd, nb, bs, FAKE, stride, N, T, out, nbytes, None, None)

    assert call(kvd=3) == EINVAL and call(nb=0) == EINVAL and call(stride=0) == EINVAL
    assert call(N=0) == EINVAL and call(T=-1) == EINVAL and call(bs=16) == EUNSUP
    assert call(nbytes=100) == EWS and call(out=FAKE + 4) == EALIGN
    assert call(T=0) == 0                                   # nothing to do


def test_prefill_attention_fails_closed_before_any_launch():
    L = dcpmla.lib()

    def call(n=10, H=16, nblk=4, ws_bytes=0, positions=FAKE, q=FAKE):
        return L.pcp_prefill_attention(q, positions, n, H, FAKE, 1, nblk, 0.07, FAKE, FAKE,
                                       FAKE, ws_bytes, 4, 0, None)

    assert call(n=-1) == EINVAL and call(nblk=0) == EINVAL and call(positions=None) == EINVAL
    assert call(H=65) == EUNSUP
    assert call() == EWS                                    # empty workspace
    assert call(q=FAKE + 2, ws_bytes=1 << 30) == EALIGN
    assert call(n=0) == 0
