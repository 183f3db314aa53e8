"""The bounded-wait (timeout) path of the tensor-core kernel, on the GPU.

With DCPMLA_TEST_WITHHOLD_ARRIVAL the fp16-operand kernel's converter warps
withhold their first arrival (the e4m3 kernel's producer withholds its first
tile), so nothing ever completes the first stage: every waiting role of
every CTA gives up after its clock budget (about 2 s), the CTA drains, frees
its tensor memory and sets DCPMLA_FLAG_TIMEOUT.  No trap, fault or unbounded
wait is involved, and the context must stay usable: a normal call right after
must succeed and match the oracle.
"""
import numpy as np
import pytest
import torch

import oracle
from long_context_decode_mla_b200 import dcpmla
from long_context_decode_mla_b200 import workload as wl

pytestmark = pytest.mark.gpu

WITHHOLD = 0x100          # DCPMLA_TEST_WITHHOLD_ARRIVAL


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    dcpmla.lib()
    torch.cuda.set_device(0)


def test_withheld_arrival_times_out_and_the_context_survives():
    prob = wl.make_problem("tiny", num_shards=2).to("cuda")        # 8 tiles per shard
    B, H = prob.batch, prob.heads
    o = torch.empty(B, H, 512, device="cuda")
    l = torch.empty(B, H, device="cuda")
    ws = torch.zeros(dcpmla.mla_decode_workspace_size(B, H, 8), dtype=torch.uint8, device="cuda")
    # one tile per CTA: only the MMA and softmax waits run out, once each
    dcpmla.mla_decode_partial(prob.q, prob.kv_cache, "bf16", prob.block_tables[0], prob.seq_lens,
                              0, 2, None, prob.softmax_scale, o, l, ws, 8,
                              dcpmla.IMPLS["tc"] | WITHHOLD)
    torch.cuda.synchronize()
    flags = int(ws[:4].view(torch.int32).item())
    assert flags & dcpmla.FLAG_TIMEOUT

    # the context is intact: a normal step gives the oracle's result
    dec = dcpmla.DcpDecoder(B, H, 2, impl="tc")
    dec.step(prob)
    torch.cuda.synchronize()
    assert dec.flags() == 0
    ni = wl.make_problem("tiny", num_shards=2).numpy_inputs()
    _, _, ref, ref_lse = oracle.dcp_decode(ni["q"], ni["kv_cache"], "bf16", ni["block_tables"],
                                           ni["seq_lens"], 2, ni["softmax_scale"])
    out = dec.out.double().cpu().numpy()
    assert np.abs(out - ref).max() <= 2e-3 * np.abs(ref).max()


def test_withheld_tile_times_out_on_the_e4m3_kernel():
    # fp8 single-token decode runs on the e4m3-direct kernel: the producer
    # withholds every CTA's first tile, so staging, scores, softmax and PV
    # waits run out; the CTAs drain, free TMEM and flag the timeout
    prob = wl.make_problem("agentic", num_shards=2, batch=3, seq_len=[1500, 300, 64],
                           seed=41).to("cuda")
    B, H = prob.batch, prob.heads
    o = torch.empty(B, H, 512, device="cuda")
    l = torch.empty(B, H, device="cuda")
    ws = torch.zeros(dcpmla.mla_decode_workspace_size(B, H, 6), dtype=torch.uint8, device="cuda")
    dcpmla.mla_decode_partial(prob.q, prob.kv_cache, "fp8", prob.block_tables[0], prob.seq_lens,
                              0, 2, None, prob.softmax_scale, o, l, ws, 6,
                              dcpmla.IMPLS["tc"] | WITHHOLD)
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32).item()) & dcpmla.FLAG_TIMEOUT

    dec = dcpmla.DcpDecoder(B, H, 2, impl="tc")
    dec.step(prob)
    torch.cuda.synchronize()
    assert dec.flags() == 0
    ni = wl.make_problem("agentic", num_shards=2, batch=3, seq_len=[1500, 300, 64],
                         seed=41).numpy_inputs()
    _, _, ref, ref_lse = oracle.dcp_decode(ni["q"], ni["kv_cache"], "fp8", ni["block_tables"],
                                           ni["seq_lens"], 2, ni["softmax_scale"])
    assert np.abs(dec.out.double().cpu().numpy() - ref).max() <= 2e-2 * np.abs(ref).max()
    assert np.abs(dec.out_lse.double().cpu().numpy() - ref_lse).max() <= 1e-3


def test_withhold_needs_the_tensor_core_kernel():
    prob = wl.make_problem("tiny", num_shards=2).to("cuda")
    o = torch.empty(1, 8, 512, device="cuda")
    l = torch.empty(1, 8, device="cuda")
    ws = torch.zeros(dcpmla.mla_decode_workspace_size(1, 8, 8), dtype=torch.uint8, device="cuda")
    for impl in (dcpmla.IMPLS["simt"] | WITHHOLD, dcpmla.IMPLS["auto"] | WITHHOLD):
        with pytest.raises(dcpmla.DcpMlaError) as e:
            dcpmla.mla_decode_partial(prob.q, prob.kv_cache, "bf16", prob.block_tables[0],
                                      prob.seq_lens, 0, 2, None, prob.softmax_scale, o, l, ws, 8,
                                      impl)
        assert e.value.code == -1


def test_withheld_tile_times_out_on_the_listed_e4m3_kernel():
    # sparse fp8 decode runs on the listed instantiation of the e4m3 kernel
    # (row lists, TMA gathers and cp.async): its producer withholds every
    # CTA's first tile, the waits run out, the copies of the tiles it did
    # issue are drained, and the next call is correct
    prob = wl.make_problem("sparse", num_shards=2, batch=4, seq_len=3000, topk=300,
                           seed=43).to("cuda")
    B, H = prob.batch, prob.heads
    topk = prob.sparse_idx.shape[1]
    o = torch.empty(B, H, 512, device="cuda")
    l = torch.empty(B, H, device="cuda")
    ws = torch.zeros(dcpmla.mla_decode_workspace_size(B, H, 2, topk), dtype=torch.uint8,
                     device="cuda")
    dcpmla.mla_decode_partial(prob.q, prob.kv_cache, "fp8", prob.block_tables[0], prob.seq_lens,
                              0, 2, prob.sparse_idx, prob.softmax_scale, o, l, ws, 2,
                              dcpmla.IMPLS["tc"] | WITHHOLD)
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32).item()) & dcpmla.FLAG_TIMEOUT

    dec = dcpmla.DcpDecoder(B, H, 2, topk=topk, impl="tc")
    dec.step(prob)
    torch.cuda.synchronize()
    assert dec.flags() == 0
    ni = wl.make_problem("sparse", num_shards=2, batch=4, seq_len=3000, topk=300,
                         seed=43).numpy_inputs()
    _, _, ref, ref_lse = oracle.dcp_decode(ni["q"], ni["kv_cache"], "fp8", ni["block_tables"],
                                           ni["seq_lens"], 2, ni["softmax_scale"],
                                           ni["sparse_idx"], ni["block_size"])
    out = dec.out.double().cpu().numpy()
    lse = dec.out_lse.double().cpu().numpy()
    assert np.abs(out - ref).max() <= 2e-2 * np.abs(ref).max()
    fin = np.isfinite(ref_lse)
    assert np.array_equal(fin, np.isfinite(lse))
    assert np.abs(lse[fin] - ref_lse[fin]).max() <= 1e-3
