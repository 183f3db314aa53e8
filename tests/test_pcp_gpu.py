"""PCP prefill on the GPU, through the C ABI, against ``oracle.pcp_prefill``.

A prompt of T tokens sits in a DCP-sharded cache (N = 8 round-robin shards,
each with its own permuted block table).  ``pcp_gather_rows`` must rebuild
the prompt's rows in token order bit for bit; ``pcp_prefill_attention`` then
runs every PCP rank's query tokens (8 ranks, 16 chunks: chunk r and chunk
15 - r) causally over the gathered rows, and each rank's O and LSE must match
the oracle within the decode tolerances (bf16 rows 2e-3 max|O| and 1e-4 LSE;
fp8 rows 2e-2 and 1e-3, the e4m3 kernel's exact scores).
"""
import numpy as np
import pytest
import torch

import oracle
from long_context_decode_mla_b200 import dcpmla
from long_context_decode_mla_b200 import workload as wl

pytestmark = pytest.mark.gpu

TOL = {"bf16": (2e-3, 1e-4), "fp8": (2e-2, 1e-3)}
P, N = 8, 8


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    dcpmla.lib()
    torch.cuda.set_device(0)


def _prompt(T, H, kv_dtype, seed):
    name = "agentic" if kv_dtype == "fp8" else "dense"
    prob = wl.make_problem(name, num_shards=N, batch=1, heads=H, seq_len=[T], seed=seed)
    q = wl.random_q(T, H, seed + 1)                        # every prompt token's query
    return prob, q


def _raw_rows(prob, T):
    """The prompt's row bytes in token order, read through the shard tables by hand."""
    kv = prob.kv_cache.numpy()
    tab = prob.block_tables.numpy()
    out = np.zeros((T, kv.shape[2]), dtype=np.uint8)
    for t in range(T):
        s, j = t % N, t // N
        out[t] = kv[tab[s, 0, j // 64], j % 64]
    return out


@pytest.mark.parametrize("kv_dtype,T,H", [("fp8", 2000, 16), ("bf16", 2000, 16),
                                          ("fp8", 700, 64), ("fp8", 13, 8), ("bf16", 13, 8)])
@pytest.mark.parametrize("splits", [0, 7])
def test_pcp_prefill_matches_the_oracle(kv_dtype, T, H, splits):
    prob, q = _prompt(T, H, kv_dtype, seed=500 + T + H)
    pre = dcpmla.PcpPrefill(T, H, P, kv_dtype, num_splits=splits)
    kv = prob.kv_cache.cuda()
    tables = prob.block_tables[:, 0].contiguous().cuda()   # [N, stride]: each shard's row
    pre.gather(kv, tables)
    pre.attend(q.cuda(), prob.softmax_scale)
    torch.cuda.synchronize()
    assert int(pre.flags.item()) == 0
    # the gathered copy is the prompt's rows, bit for bit
    rb = wl.ROW_BYTES[kv_dtype]
    got = pre.gathered[:T * rb].view(T, rb).cpu().numpy()
    assert np.array_equal(got, _raw_rows(prob, T))
    # every rank's attention
    ni = prob.numpy_inputs()
    qn = q.view(torch.int16).numpy().view("uint16")
    ref = oracle.pcp_prefill(qn, ni["kv_cache"], kv_dtype, ni["block_tables"][:, 0], T, P, N,
                             prob.softmax_scale)
    rel_o, abs_l = TOL[kv_dtype]
    for r, (tokens, o_ref, l_ref) in enumerate(ref):
        assert pre.tokens[r].cpu().numpy().tolist() == tokens.tolist()
        if tokens.size == 0:
            continue
        o = pre.out[r].double().cpu().numpy()
        l = pre.out_lse[r].double().cpu().numpy()
        assert np.abs(o - o_ref).max() <= rel_o * np.abs(o_ref).max(), r
        assert np.abs(l - l_ref).max() <= abs_l, r


def test_bad_table_entry_is_flagged_and_zeroed():
    T, H = 1200, 8                                          # 150 local rows per shard
    prob, q = _prompt(T, H, "fp8", seed=77)
    tables = prob.block_tables[:, 0].contiguous().clone()
    tables[3, 1] = 1 << 30                                  # shard 3, local rows 64..127
    pre = dcpmla.PcpPrefill(T, H, P, "fp8")
    pre.gather(prob.kv_cache.cuda(), tables.cuda())
    torch.cuda.synchronize()
    assert int(pre.flags.item()) & dcpmla.FLAG_BAD_BLOCK
    rb = wl.ROW_BYTES["fp8"]
    got = pre.gathered[:T * rb].view(T, rb).cpu().numpy()
    bad = [t for t in range(T) if t % N == 3 and (t // N) // 64 == 1]
    assert bad and not got[bad].any()
    good = [t for t in range(T) if t not in set(bad)]
    assert np.array_equal(got[good], _raw_rows(prob, T)[good])
