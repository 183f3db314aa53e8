"""Pins of the multi-query oracle (``oracle/multi_query.py``).

Facts used, none of them the oracle restated: q_len = 1 is the single-query
oracle; query row i is single-query decode over the prefix of L - q_len + i + 1
tokens (a different call path: the cached length changes, not a mask);
merging the shard partials gives the unsharded result; a brute force over the
logical rows in token order, with plain Python sums, gives the same values.
A planted off-by-one in the causal limit must be caught.
"""
import math

import numpy as np
import pytest

import oracle
from oracle import multi_query as mq
from long_context_decode_mla_b200 import workload as wl

SCALE = 192 ** -0.5


def _problem(lens, N, kv_dtype, H, q_len, seed):
    prob, rows = wl.logical_problem(lens, N, kv_dtype, H * q_len, seed)
    ni = prob.numpy_inputs()
    q = ni["q"].reshape(len(lens), q_len, H, 576)
    return ni, q, rows


@pytest.mark.parametrize("kv_dtype", ["bf16", "fp8"])
def test_one_query_is_the_single_query_oracle(kv_dtype):
    ni, q, _ = _problem([300, 64, 1, 129], 3, kv_dtype, 8, 1, seed=1)
    for s in range(3):
        o1, l1 = mq.mla_decode_partial_multi(q, ni["kv_cache"], kv_dtype, ni["block_tables"][s],
                                             ni["seq_lens"], s, 3, SCALE)
        o0, l0 = oracle.mla_decode_partial(q[:, 0], ni["kv_cache"], kv_dtype,
                                           ni["block_tables"][s], ni["seq_lens"], s, 3, SCALE)
        assert np.array_equal(o1[:, 0], o0) and np.array_equal(l1[:, 0], l0)


@pytest.mark.parametrize("N", [1, 2, 3, 8])
@pytest.mark.parametrize("q_len", [2, 4])
def test_each_row_is_decode_over_its_prefix(N, q_len):
    lens = [500, q_len, 1, 64 * N + 1, 3]
    ni, q, _ = _problem(lens, N, "fp8", 4, q_len, seed=N + q_len)
    parts, ls, out, lse = mq.dcp_decode_multi(q, ni["kv_cache"], "fp8", ni["block_tables"],
                                              ni["seq_lens"], N, SCALE)
    for i in range(q_len):
        prefix = np.maximum(np.asarray(lens) - q_len + i + 1, 0)
        p1, l1, o1, e1 = oracle.dcp_decode(q[:, i], ni["kv_cache"], "fp8", ni["block_tables"],
                                           prefix, N, SCALE)
        assert np.allclose(parts[:, :, i], p1, rtol=0, atol=1e-12)
        assert np.array_equal(np.isneginf(ls[:, :, i]), np.isneginf(l1))
        fin = np.isfinite(l1)
        assert np.allclose(ls[:, :, i][fin], l1[fin], rtol=0, atol=1e-12)
        assert np.allclose(out[:, i], o1, rtol=0, atol=1e-12)


def test_queries_before_the_start_are_empty():
    ni, q, _ = _problem([1, 2], 2, "bf16", 2, 4, seed=3)
    _, _, out, lse = mq.dcp_decode_multi(q, ni["kv_cache"], "bf16", ni["block_tables"],
                                         ni["seq_lens"], 2, SCALE)
    # request 0 (L = 1): only query 3 (position 0) sees a token; request 1: queries 2 and 3
    assert np.all(np.isneginf(lse[0, :3])) and np.isfinite(lse[0, 3]).all()
    assert not out[0, :3].any()
    assert np.all(np.isneginf(lse[1, :2])) and np.isfinite(lse[1, 2:]).all()


@pytest.mark.parametrize("N", [2, 3, 8])
def test_merge_of_shards_equals_one_shard(N):
    lens = [700, 5, 130]
    prob, rows = wl.logical_problem(lens, N, "bf16", 8, seed=40)
    cache1, tables1, lens1 = wl.place_rows(rows, 1, "bf16", seed=41)
    q = prob.numpy_inputs()["q"].reshape(3, 2, 4, 576)
    _, _, outN, lseN = mq.dcp_decode_multi(q, prob.kv_cache.numpy(), "bf16",
                                           prob.block_tables.numpy(), prob.seq_lens.numpy(), N,
                                           SCALE)
    _, _, out1, lse1 = mq.dcp_decode_multi(q, cache1.numpy(), "bf16", tables1.numpy(),
                                           lens1.numpy(), 1, SCALE)
    assert np.allclose(outN, out1, rtol=0, atol=1e-12)
    assert np.allclose(lseN, lse1, rtol=0, atol=1e-12)


def test_brute_force_over_logical_rows():
    """Causal softmax over the rows in token order, plain Python arithmetic."""
    lens, q_len, H, N = [37, 3], 3, 2, 3
    prob, rows = wl.logical_problem(lens, N, "bf16", H * q_len, seed=9)
    ni = prob.numpy_inputs()
    q = oracle.decode_bf16(ni["q"]).reshape(2, q_len, H, 576)
    _, _, out, lse = mq.dcp_decode_multi(ni["q"].reshape(2, q_len, H, 576), ni["kv_cache"], "bf16",
                                         ni["block_tables"], ni["seq_lens"], N, SCALE)
    for b, L in enumerate(lens):
        keys = oracle.decode_rows(rows[b].numpy(), "bf16")
        for i in range(q_len):
            for h in range(H):
                n = L - q_len + i + 1
                if n <= 0:
                    assert math.isinf(lse[b, i, h]) and lse[b, i, h] < 0
                    continue
                s = [SCALE * math.fsum(float(a) * float(c) for a, c in zip(q[b, i, h], keys[t]))
                     for t in range(n)]
                m = max(s)
                z = math.fsum(math.exp(x - m) for x in s)
                want_lse = m + math.log(z)
                assert abs(lse[b, i, h] - want_lse) < 1e-10
                for d in (0, 7, 300, 511):
                    want = math.fsum(math.exp(s[t] - want_lse) * float(keys[t][d])
                                     for t in range(n))
                    assert abs(out[b, i, h, d] - want) < 1e-10


def test_planted_off_by_one_limit_is_caught(monkeypatch):
    real = mq.mla_decode_partial_multi

    def strict(q, kv_cache, kv_dtype, block_table, seq_lens, shard_id, num_shards, softmax_scale,
               block_size=64):
        # sees one token fewer: t < L - q_len + i instead of t <= ...
        return real(q, kv_cache, kv_dtype, block_table, np.asarray(seq_lens) - 1, shard_id,
                    num_shards, softmax_scale, block_size)
    monkeypatch.setattr(mq, "mla_decode_partial_multi", strict)
    with pytest.raises(AssertionError):
        test_each_row_is_decode_over_its_prefix(2, 2)
