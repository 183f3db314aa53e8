"""dcpmla.HostPipeline: decode steps from pinned host buffers, copies overlapped.

Each step's host results must equal (bit for bit: same kernels, same inputs)
a direct DcpDecoder step on device copies of the same inputs.  The steps use
different queries (and for one case different lengths and sparse lists), so
that a slot that read or returned another step's buffers would show; five
steps reuse both slots at least twice.  One step is also checked against the
fp64 oracle.
"""
import numpy as np
import pytest
import torch

import oracle
from long_context_decode_mla_b200 import dcpmla
from long_context_decode_mla_b200 import workload as wl

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    dcpmla.lib()
    torch.cuda.set_device(0)


def _step_inputs(prob, k):
    """Host inputs of step k: the problem's tables with a fresh query (and,
    for odd k, shorter lengths and shuffled sparse lists)."""
    g = torch.Generator().manual_seed(1000 + k)
    q = torch.randn(prob.q.shape, generator=g).to(torch.bfloat16)
    lens = prob.seq_lens.cpu().clone()
    if k % 2 == 1:
        lens = torch.clamp(lens - 37 * (k + 1), min=0)
    idx = None
    if prob.sparse_idx is not None:
        idx = prob.sparse_idx.cpu().clone()
        idx = idx[:, torch.randperm(idx.shape[1], generator=g)].contiguous()
    return (q.pin_memory(), lens.pin_memory(), prob.block_tables.cpu().pin_memory(),
            None if idx is None else idx.pin_memory())


@pytest.mark.parametrize("case", ["dense-fp8", "dense-bf16", "sparse-fp8"])
def test_pipeline_matches_direct_steps(case):
    if case == "sparse-fp8":
        prob = wl.make_problem("sparse", num_shards=4, batch=6, seq_len=5000, topk=400, seed=7,
                               device="cuda", kv_device="cuda")
    else:
        kv = case.split("-")[1]
        prob = wl.make_problem("dense", num_shards=4, batch=5, heads=64,
                               seq_len=[3000, 64, 1, 9000, 700], kv_dtype=kv, seed=11,
                               device="cuda", kv_device="cuda")
    topk = 0 if prob.sparse_idx is None else prob.sparse_idx.shape[1]
    pipe = dcpmla.HostPipeline(prob, topk=topk, num_splits=3)
    steps = 5
    inputs = [_step_inputs(prob, k) for k in range(steps)]
    outs = [(torch.empty(prob.batch, prob.heads, dcpmla.V_DIM).pin_memory(),
             torch.empty(prob.batch, prob.heads).pin_memory()) for _ in range(steps)]
    for k in range(steps):
        pipe.submit(*inputs[k], *outs[k])
    pipe.join()
    torch.cuda.synchronize()
    assert pipe.flags() == 0

    direct = dcpmla.DcpDecoder(prob.batch, prob.heads, prob.num_shards, topk=topk, num_splits=3)
    for k in range(steps):
        q, lens, tables, idx = inputs[k]
        dp = wl.DecodeProblem(q.cuda(), prob.kv_cache, prob.kv_dtype, tables.cuda(), lens.cuda(),
                              prob.num_shards, prob.softmax_scale,
                              None if idx is None else idx.cuda(), prob.block_size)
        o, lse = direct.step(dp)
        torch.cuda.synchronize()
        assert torch.equal(outs[k][0], o.cpu()), f"step {k}: O differs from a direct step"
        assert torch.equal(outs[k][1], lse.cpu()), f"step {k}: LSE differs from a direct step"
        if k == steps - 1:
            ni = dp.numpy_inputs()
            _, _, ro, rlse = oracle.dcp_decode(ni["q"], ni["kv_cache"], ni["kv_dtype"],
                                               ni["block_tables"], ni["seq_lens"],
                                               ni["num_shards"], ni["softmax_scale"],
                                               ni["sparse_idx"], ni["block_size"])
            out = outs[k][0].double().numpy()
            lse_h = outs[k][1].double().numpy()
            fin = np.isfinite(rlse)
            assert np.array_equal(fin, np.isfinite(lse_h))
            tol_o, tol_l = (2e-3, 1e-4) if prob.kv_dtype == "bf16" else (2e-2, 1e-3)
            assert np.abs(out - ro).max() <= tol_o * max(np.abs(ro).max(), 1e-30)
            if fin.any():
                assert np.abs(lse_h[fin] - rlse[fin]).max() <= tol_l
