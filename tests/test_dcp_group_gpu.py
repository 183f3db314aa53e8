"""Real multi-GPU DCP decode, checked on one GPU.

1. ``dcp_merge_heads`` over per-rank exchange buffers.  Shard s's partial
   (``mla_decode_partial``) is written into its own buffer from
   ``dcp_exchange_alloc``, as rank s would write it; each rank's slice of
   heads is merged by ``dcp_merge_heads`` reading all N buffers through the
   pointer table.  The slices put together must be bit-identical to
   ``dcp_merge`` of the same partials stacked (same arithmetic, same order),
   -inf LSEs included, and match the oracle within the decode tolerances.
2. ``DcpRankDecoder`` in a one-rank NCCL group: the whole per-rank step
   (query all-gather, partial into the exchange slot, the stream-ordered
   all-reduce, the head-sliced merge) over two steps, so both slots are used,
   against the oracle.

Ranks on several GPUs are not run here (one GPU); the peer mapping is the
CUDA IPC path of ``dcp_exchange_open``.
"""
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import oracle
from long_context_decode_mla_b200 import dcp_group, dcpmla
from long_context_decode_mla_b200 import workload as wl

pytestmark = pytest.mark.gpu

# fp8 LSE: 1e-3 (exact scores: dense, and sparse over the gathered selections)
TOL = {"bf16": (2e-3, 1e-4), "fp8": (2e-2, 1e-3), "fp8-sparse": (2e-2, 1e-3)}


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    dcpmla.lib()
    torch.cuda.set_device(0)


def _compare(o, l, o_ref, l_ref, kv_dtype):
    rel_o, abs_l = TOL[kv_dtype]
    fin = np.isfinite(l_ref)
    assert np.array_equal(fin, np.isfinite(l))
    assert not o[~fin].any()
    if fin.any():
        assert np.abs(o - o_ref).max() <= rel_o * np.abs(o_ref).max()
        assert np.abs(l[fin] - l_ref[fin]).max() <= abs_l


@pytest.mark.parametrize("name,N,H,lens", [
    ("agentic", 8, 64, [5000, 3, 1, 64 * 8 + 5, 0]),
    ("dense", 2, 16, [700, 1, 64, 2]),
    ("agentic", 4, 8, [9000, 130]),
    ("sparse", 8, 64, [20000, 300]),
])
def test_merge_heads_over_exchange_buffers(name, N, H, lens):
    over = dict(batch=len(lens), heads=H, seq_len=lens, seed=700 + N)
    if name == "sparse":
        over["topk"] = 256
    prob = wl.make_problem(name, num_shards=N, **over)
    p = prob.to("cuda")
    B = prob.batch
    lse_off, slot = dcp_group.slot_layout(B, H)
    bufs = [dcpmla.dcp_exchange_alloc(slot)[0] for _ in range(N)]
    try:
        topk = 0 if p.sparse_idx is None else p.sparse_idx.shape[1]
        ws = torch.zeros(dcpmla.mla_decode_workspace_size(B, H, 0, topk), dtype=torch.uint8,
                         device="cuda")
        parts = [dcp_group.device_view(a, (B, H, 512)) for a in bufs]
        lses = [dcp_group.device_view(a + lse_off, (B, H)) for a in bufs]
        for s in range(N):
            dcpmla.mla_decode_partial(p.q, p.kv_cache, p.kv_dtype, p.block_tables[s], p.seq_lens,
                                      s, N, p.sparse_idx, p.softmax_scale, parts[s], lses[s], ws)
        ref = torch.empty(B, H, 512, device="cuda")
        ref_lse = torch.empty(B, H, device="cuda")
        dcpmla.dcp_merge(torch.stack(parts), torch.stack(lses), ref, ref_lse)
        out = torch.empty(B, H, 512, device="cuda")
        out_lse = torch.empty(B, H, device="cuda")
        for r in range(N):
            h0, hn = dcp_group.head_slice(r, N, H)
            o_r = torch.empty(B, hn, 512, device="cuda")
            l_r = torch.empty(B, hn, device="cuda")
            dcpmla.dcp_merge_heads(bufs, [a + lse_off for a in bufs], B, H, h0, hn, o_r, l_r)
            out[:, h0:h0 + hn] = o_r
            out_lse[:, h0:h0 + hn] = l_r
        torch.cuda.synchronize()
        assert int(ws[:4].view(torch.int32).item()) == 0
        assert torch.equal(out, ref) and torch.equal(out_lse, ref_lse)
        ni = prob.numpy_inputs()
        if prob.sparse_idx is None:
            _, _, o_ref, l_ref = oracle.dcp_decode(ni["q"], ni["kv_cache"], prob.kv_dtype,
                                                   ni["block_tables"], ni["seq_lens"], N,
                                                   ni["softmax_scale"])
        else:
            _, _, o_ref, l_ref = oracle.dcp_decode(ni["q"], ni["kv_cache"], prob.kv_dtype,
                                                   ni["block_tables"], ni["seq_lens"], N,
                                                   ni["softmax_scale"],
                                                   sparse_idx=ni["sparse_idx"])
        _compare(out.double().cpu().numpy(), out_lse.double().cpu().numpy(), o_ref, l_ref,
                 prob.kv_dtype + ("-sparse" if prob.kv_dtype == "fp8" and prob.sparse_idx is not None
                                  else ""))
    finally:
        torch.cuda.synchronize()
        for a in bufs:
            dcpmla.dcp_exchange_free(a)


def test_merge_heads_one_head_slices_and_a_single_shard():
    prob = wl.make_problem("dense", num_shards=1, batch=2, heads=8, seq_len=[300, 5], seed=77)
    p = prob.to("cuda")
    part = torch.empty(1, 2, 8, 512, device="cuda")
    lse = torch.empty(1, 2, 8, device="cuda")
    ws = torch.zeros(dcpmla.mla_decode_workspace_size(2, 8), dtype=torch.uint8, device="cuda")
    dcpmla.mla_decode_partial(p.q, p.kv_cache, "bf16", p.block_tables[0], p.seq_lens, 0, 1, None,
                              p.softmax_scale, part[0], lse[0], ws)
    for h in range(8):
        o = torch.empty(2, 1, 512, device="cuda")
        l = torch.empty(2, 1, device="cuda")
        dcpmla.dcp_merge_heads([part[0]], [lse[0]], 2, 8, h, 1, o, l)
        torch.cuda.synchronize()
        # one shard: the merge returns the shard's own result (w = 1, ln 1 = 0)
        assert torch.equal(o[:, 0], part[0, :, h]) and torch.equal(l[:, 0], lse[0, :, h])


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def test_rank_decoder_in_a_one_rank_nccl_group():
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0,
                            world_size=1, device_id=torch.device("cuda", 0))
    dec = None
    try:
        dec = dcp_group.DcpRankDecoder(3, 64, topk=0)
        for seed in (801, 802):
            prob = wl.make_problem("agentic", num_shards=1, batch=3, heads=64,
                                   seq_len=[6000, 70, 1], seed=seed)
            p = prob.to("cuda")
            out, lse = dec.step(p.q, p.kv_cache, "fp8", p.block_tables[0], p.seq_lens,
                                p.softmax_scale)
            torch.cuda.synchronize()
            assert dec.flags() == 0
            ni = prob.numpy_inputs()
            _, _, o_ref, l_ref = oracle.dcp_decode(ni["q"], ni["kv_cache"], "fp8",
                                                   ni["block_tables"], ni["seq_lens"], 1,
                                                   ni["softmax_scale"])
            _compare(out.double().cpu().numpy(), lse.double().cpu().numpy(), o_ref, l_ref, "fp8")
            o_s, l_s = dec.partial()
            assert torch.equal(o_s, out) and torch.equal(l_s, lse)
        assert dec.steps == 2
    finally:
        if dec is not None:
            dec.close()
        dist.destroy_process_group()
