"""Pins of the PCP prefill oracle (``oracle/pcp.py``), on the CPU.

Each pin checks the oracle against something other than itself:

* the chunk plan against the definition (2P contiguous chunks in prompt
  order, sizes within one) and the page's geometry (``tests/golden/
  pcp_geometry.json``: 8 ranks, 16 chunks, all 64 heads per rank);
* the front/back pairing against its closed form: with c tokens per chunk,
  every rank's causal work sum_{i in rank}(i + 1) is (2P - 1) c^2 + c (c + 1),
  and the ranks add up to T (T + 1) / 2;
* the gathered cache against the raw cache bytes read through each shard's
  block table by hand;
* every prefill row against DCP decode of that token over its prefix (the
  decode oracle's shard partials and LSE merge: an independent call path);
* token 0 against its own value row (a softmax over one key is exactly 1);
* tiny prompts against brute force with math.fsum;
* a planted off-by-one (a query that does not see itself) against the
  decode path, which it must fail.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import pcp
from long_context_decode_mla_b200 import workload as wl


@pytest.mark.parametrize("T", [0, 1, 5, 15, 16, 17, 100, 4096, 4099])
@pytest.mark.parametrize("P", [1, 2, 8])
def test_chunk_plan_partitions_the_prompt(T, P):
    chunks = pcp.pcp_chunks(T, P)
    assert len(chunks) == 2 * P
    assert chunks[0][0] == 0 and chunks[-1][1] == T
    for (a, b), (c, _) in zip(chunks, chunks[1:]):
        assert b == c and a <= b
    sizes = [b - a for a, b in chunks]
    assert max(sizes) - min(sizes) <= 1
    assert sizes == sorted(sizes, reverse=True)          # the larger chunks come first
    seen = np.concatenate([pcp.pcp_rank_tokens(T, P, r) for r in range(P)])
    assert sorted(seen.tolist()) == list(range(T))       # every token on exactly one rank


def test_page_geometry_and_pairing():
    with open(os.path.join(os.path.dirname(__file__), "golden", "pcp_geometry.json")) as f:
        g = json.load(f)
    P, n = g["ranks"], g["chunks"]
    T = 100 * n
    chunks = pcp.pcp_chunks(T, P)
    assert len(chunks) == n and all(b - a == 100 for a, b in chunks)
    # rank r holds chunk r (front) and chunk n - 1 - r (back)
    for r in range(P):
        tok = pcp.pcp_rank_tokens(T, P, r)
        assert tok.tolist() == list(range(100 * r, 100 * r + 100)) + \
            list(range(100 * (n - 1 - r), 100 * (n - 1 - r) + 100))
    with pytest.raises(ValueError):
        pcp.pcp_rank_tokens(T, P, P)
    # every rank computes all heads for its tokens: the oracle's rank step
    # returns every head of the query rows it is given
    rows = np.random.default_rng(0).standard_normal((3, 576))
    q = np.random.default_rng(1).standard_normal((3, g["heads_per_rank"], 576))
    o, lse = pcp.pcp_prefill_rank(q, rows, np.array([0, 2]), 0.05)
    assert o.shape == (2, g["heads_per_rank"], 512) and lse.shape == (2, g["heads_per_rank"])


@pytest.mark.parametrize("P,c", [(1, 7), (2, 5), (8, 64), (8, 4096)])
def test_paired_chunks_balance_causal_work_exactly(P, c):
    T = 2 * P * c
    work = [int((pcp.pcp_rank_tokens(T, P, r) + 1).sum()) for r in range(P)]
    assert work == [(2 * P - 1) * c * c + c * (c + 1)] * P
    assert sum(work) == T * (T + 1) // 2


def _prompt(T, H, N, kv_dtype, seed):
    name = "agentic" if kv_dtype == "fp8" else "dense"
    prob = wl.make_problem(name, num_shards=N, batch=1, heads=H, seq_len=[T], seed=seed)
    ni = prob.numpy_inputs()
    q = wl.random_q(T, H, seed + 50).view(torch.int16).numpy().view(np.uint16)
    return ni, q, ni["block_tables"][:, 0]


@pytest.mark.parametrize("kv_dtype", ["bf16", "fp8"])
def test_gathered_rows_follow_the_round_robin_layout(kv_dtype):
    T, N = 300, 4
    ni, _, bt = _prompt(T, 2, N, kv_dtype, 11)
    rows = pcp.gather_prompt_rows(ni["kv_cache"], kv_dtype, bt, T, N)
    for t in (0, 1, 3, 4, 63, 255, 256, 257, 299):
        s, j = t % N, t // N
        raw = ni["kv_cache"][bt[s][j // 64], j % 64]
        assert np.array_equal(rows[t], oracle.decode_rows(raw[None], kv_dtype)[0])


@pytest.mark.parametrize("kv_dtype,T,N,P", [("bf16", 300, 4, 4), ("fp8", 257, 8, 2),
                                            ("fp8", 40, 2, 8)])
def test_every_prefill_row_is_dcp_decode_of_its_token(kv_dtype, T, N, P):
    H = 8
    ni, q, bt = _prompt(T, H, N, kv_dtype, 20 + T)
    per_rank = pcp.pcp_prefill(q, ni["kv_cache"], kv_dtype, bt, T, P, N, ni["softmax_scale"])
    o = np.zeros((T, H, 512))
    lse = np.zeros((T, H))
    for tokens, o_r, l_r in per_rank:
        o[tokens], lse[tokens] = o_r, l_r
    # decode path: token i as its own request, length i + 1, same shard tables
    tables = np.repeat(ni["block_tables"][:, :1], T, axis=1)
    _, _, o_dec, l_dec = oracle.dcp_decode(q, ni["kv_cache"], kv_dtype, tables,
                                           np.arange(1, T + 1), N, ni["softmax_scale"])
    assert np.abs(o - o_dec).max() <= 1e-12 * np.abs(o_dec).max()
    assert np.abs(lse - l_dec).max() <= 1e-12 * np.abs(l_dec).max()


def test_first_token_sees_only_its_own_row():
    T, H, N = 70, 4, 2
    ni, q, bt = _prompt(T, H, N, "fp8", 5)
    rows = pcp.gather_prompt_rows(ni["kv_cache"], "fp8", bt, T, N)
    o, lse = pcp.pcp_prefill_rank(q, rows, np.array([0]), ni["softmax_scale"])
    qf = oracle.decode_bf16(q)
    for h in range(H):
        assert np.array_equal(o[0, h], rows[0, :512])
        assert lse[0, h] == pytest.approx(ni["softmax_scale"] * float(qf[0, h] @ rows[0]),
                                          rel=1e-14, abs=1e-14)


def test_tiny_prompt_brute_force():
    rng = np.random.default_rng(3)
    T, H = 5, 2
    q = rng.standard_normal((T, H, 576))
    rows = rng.standard_normal((T, 576))
    scale = 0.07
    o, lse = pcp.pcp_prefill_rank(q, rows, np.arange(T), scale)
    for i in range(T):
        for h in range(H):
            s = [scale * math.fsum(q[i, h, d] * rows[t, d] for d in range(576))
                 for t in range(i + 1)]
            m = max(s)
            want_lse = m + math.log(math.fsum(math.exp(x - m) for x in s))
            assert lse[i, h] == pytest.approx(want_lse, rel=1e-12, abs=1e-12)
            for d in (0, 1, 255, 511):
                want = math.fsum(math.exp(s[t] - want_lse) * rows[t, d] for t in range(i + 1))
                assert o[i, h, d] == pytest.approx(want, rel=1e-10, abs=1e-12)


def test_a_query_that_misses_itself_is_caught():
    """Plant an off-by-one causal limit (query i sees rows 0..i-1) in a copy of
    the rank step: the decode pin must reject it."""
    T, H, N = 50, 4, 2
    ni, q, bt = _prompt(T, H, N, "bf16", 9)
    rows = pcp.gather_prompt_rows(ni["kv_cache"], "bf16", bt, T, N)
    qf = oracle.decode_bf16(q)
    wrong = np.stack([oracle.attention_with_lse(qf[i], rows[:i], ni["softmax_scale"])[0]
                      for i in range(1, T)])
    tables = np.repeat(ni["block_tables"][:, :1], T, axis=1)
    _, _, o_dec, _ = oracle.dcp_decode(q, ni["kv_cache"], "bf16", tables, np.arange(1, T + 1), N,
                                       ni["softmax_scale"])
    assert np.abs(wrong - o_dec[1:]).max() > 1e-3
