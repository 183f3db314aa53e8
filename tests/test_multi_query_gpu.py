"""GPU parity of multi-query decode (``mla_decode_partial_multi``) through the C ABI.

Each row (query i of q_len, head h) attends causally to the cached tokens up
to position L_b - q_len + i; partials per shard and the merged result must
match the oracle within the single-query tolerances (bf16 cache 2e-3 max|O|
and 1e-4 LSE, fp8 cache 2e-2 max|O| and 1e-3 LSE: fp8 rows run one query per
pass through the e4m3-direct kernel, whose scores are exact), with exact
(0, -inf) for rows that see no token of a shard.  Rows beyond one 64-row tile
(64 heads x q_len 2..4, the models' head count) run as several passes over
the cache.
"""
import numpy as np
import pytest
import torch

import oracle
from long_context_decode_mla_b200 import dcpmla
from long_context_decode_mla_b200 import workload as wl

pytestmark = pytest.mark.gpu

TOL = {"bf16": (2e-3, 1e-4), "fp8": (2e-2, 1e-3)}


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    dcpmla.lib()
    torch.cuda.set_device(0)


# fp8 on the explicitly chosen fp16-operand kernel: e4m3 * scale is rounded
# to fp16 before its MMAs (the parity tests derive the 5e-3 LSE bound)
TOL_FP8_FP16_OPERANDS = (2e-2, 5e-3)


def _compare(o, l, o_ref, l_ref, kv_dtype, what, tol=None):
    rel_o, abs_l = TOL[kv_dtype] if tol is None else tol
    fin = np.isfinite(l_ref)
    assert np.array_equal(fin, np.isfinite(l)), f"{what}: -inf pattern differs"
    assert not o[~fin].any(), f"{what}: empty rows must have O == 0"
    if fin.any():
        assert np.abs(o - o_ref).max() <= rel_o * np.abs(o_ref).max(), what
        assert np.abs(l[fin] - l_ref[fin]).max() <= abs_l, what


def _run_and_check(lens, N, kv_dtype, H, q_len, splits, seed, impl="auto"):
    name = "agentic" if kv_dtype == "fp8" else "dense"
    prob = wl.make_problem(name, num_shards=N, batch=len(lens), heads=H * q_len, seq_len=lens,
                           seed=seed)
    dec = dcpmla.DcpDecoder(prob.batch, H, N, num_splits=splits, q_len=q_len, impl=impl)
    dec.step(prob.to("cuda"))
    torch.cuda.synchronize()
    assert dec.flags() == 0
    ni = prob.numpy_inputs()
    q = ni["q"].reshape(prob.batch, q_len, H, 576)
    rp, rl, ro, rlse = oracle.dcp_decode_multi(q, ni["kv_cache"], kv_dtype, ni["block_tables"],
                                               ni["seq_lens"], N, ni["softmax_scale"])
    B = prob.batch
    parts = dec.partials.double().cpu().numpy().reshape(N, B, q_len, H, 512)
    lses = dec.lses.double().cpu().numpy().reshape(N, B, q_len, H)
    tol = TOL_FP8_FP16_OPERANDS if (impl == "tc16" and kv_dtype == "fp8") else None
    for s in range(N):
        _compare(parts[s], lses[s], rp[s], rl[s], kv_dtype, f"shard {s}", tol)
    out = dec.out.double().cpu().numpy().reshape(B, q_len, H, 512)
    lse = dec.out_lse.double().cpu().numpy().reshape(B, q_len, H)
    _compare(out, lse, ro, rlse, kv_dtype, "merged", tol)


@pytest.mark.parametrize("kv_dtype", ["fp8", "bf16"])
@pytest.mark.parametrize("H,q_len", [(16, 4), (32, 2), (8, 8), (64, 2), (64, 3), (64, 4)])
@pytest.mark.parametrize("N", [1, 2, 8])
def test_multi_query_matches_the_oracle(kv_dtype, H, q_len, N):
    lens = [1, q_len - 1 if q_len > 1 else 1, q_len, 64 * N, 64 * N + 1, 2000, 4099]
    _run_and_check(lens, N, kv_dtype, H, q_len, splits=0, seed=200 + N + q_len)


@pytest.mark.parametrize("splits", [1, 3, 148])
def test_multi_query_across_split_counts(splits):
    _run_and_check([5000, 70, 3, 64 * 4 + 2], 4, "fp8", 16, 4, splits=splits, seed=300 + splits)


def test_one_query_through_the_multi_entry_point_is_plain_decode():
    prob = wl.make_problem("agentic", num_shards=2, batch=3, heads=64, seq_len=[3000, 7, 129],
                           seed=310).to("cuda")
    a = dcpmla.DcpDecoder(3, 64, 2)
    a.step(prob)
    outs = []
    for s in range(2):
        o = torch.empty(3, 64, 512, device="cuda")
        l = torch.empty(3, 64, device="cuda")
        ws = torch.zeros(dcpmla.mla_decode_workspace_size(3, 64), dtype=torch.uint8, device="cuda")
        dcpmla.mla_decode_partial_multi(prob.q.view(3, 1, 64, 576), prob.kv_cache, "fp8",
                                        prob.block_tables[s], prob.seq_lens, s, 2,
                                        prob.softmax_scale, o, l, ws)
        outs.append((o, l))
    torch.cuda.synchronize()
    for s in range(2):
        assert torch.equal(outs[s][0], a.partials[s]) and torch.equal(outs[s][1], a.lses[s])


@pytest.mark.parametrize("impl,kv_dtype", [("simt", "fp8"), ("simt", "bf16"), ("tc16", "fp8")])
def test_multi_query_passes_on_every_kernel(impl, kv_dtype):
    # the CUDA-core kernel runs one query per pass; the fp16-operand kernel
    # packs whole queries into 64-row tiles (here 2 passes of 32 x 2 rows)
    _run_and_check([1, 3, 4, 130, 2000], 2, kv_dtype, 32 if impl == "tc16" else 64, 4,
                   splits=0, seed=330, impl=impl)


def test_unsupported_shapes_fail_closed():
    prob = wl.make_problem("agentic", num_shards=2, batch=1, heads=64, seq_len=[100], seed=5)
    p = prob.to("cuda")
    o = torch.empty(1, 2, 65, 512, device="cuda")
    l = torch.empty(1, 2, 65, device="cuda")
    ws = torch.zeros(dcpmla.mla_decode_workspace_size(1, 130), dtype=torch.uint8, device="cuda")
    q65 = torch.zeros(1, 2, 65, 576, dtype=torch.bfloat16, device="cuda")     # 65 heads
    with pytest.raises(dcpmla.DcpMlaError) as e:
        dcpmla.mla_decode_partial_multi(q65, p.kv_cache, "fp8", p.block_tables[0], p.seq_lens, 0,
                                        2, p.softmax_scale, o, l, ws)
    assert e.value.code == -2
    q0 = torch.zeros(1, 0, 64, 576, dtype=torch.bfloat16, device="cuda")      # no query
    with pytest.raises(dcpmla.DcpMlaError) as e:
        dcpmla.mla_decode_partial_multi(q0, p.kv_cache, "fp8", p.block_tables[0], p.seq_lens, 0,
                                        2, p.softmax_scale, o, l, ws)
    assert e.value.code == -1
