"""mla_decode_partial_noalloc against mla_decode_partial, through the C ABI.

The no-alloc entry point runs the same kernels on a scratch array built into
the library (one per device) instead of a caller's workspace.  This file is
named to be collected last, so that it runs both alone and after every other
GPU test in the same process.  Both entry points run the same kernels, so
the parity tests' tolerances hold with room (bf16 cache: max|dO| <= 2e-3
max|O|, |dLSE| <= 1e-4; fp8 cache: 2e-2 and 1e-3).
"""
import numpy as np
import pytest
import torch

from long_context_decode_mla_b200 import dcpmla
from long_context_decode_mla_b200 import workload as wl

pytestmark = pytest.mark.gpu

TOL = {"bf16": (2e-3, 1e-4), "fp8": (2e-2, 1e-3)}


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    dcpmla.lib()
    torch.cuda.set_device(0)


def _outputs(prob):
    return (torch.full((prob.batch, prob.heads, dcpmla.V_DIM), float("nan"), device="cuda"),
            torch.full((prob.batch, prob.heads), float("nan"), device="cuda"))


def _with_workspace(prob, shard, num_splits, impl):
    o, l = _outputs(prob)
    topk = 0 if prob.sparse_idx is None else prob.sparse_idx.shape[1]
    ws = torch.zeros(dcpmla.mla_decode_workspace_size(prob.batch, prob.heads, num_splits, topk),
                     dtype=torch.uint8, device="cuda")
    dcpmla.mla_decode_partial(prob.q, prob.kv_cache, prob.kv_dtype, prob.block_tables[shard],
                              prob.seq_lens, shard, prob.num_shards, prob.sparse_idx,
                              prob.softmax_scale, o, l, ws, num_splits, impl)
    return o, l, ws[:4].view(torch.int32)


def _no_alloc(prob, shard, num_splits, impl):
    o, l = _outputs(prob)
    flags = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    dcpmla.mla_decode_partial_noalloc(prob.q, prob.kv_cache, prob.kv_dtype,
                                      prob.block_tables[shard], prob.seq_lens, shard,
                                      prob.num_shards, prob.sparse_idx, prob.softmax_scale, o, l,
                                      flags, num_splits, impl)
    return o, l, flags


def _close(a, b, kv_dtype):
    (o, l), (o_ref, l_ref) = [(x.double().cpu().numpy(), y.double().cpu().numpy())
                              for x, y in (a, b)]
    fin = np.isfinite(l_ref)
    assert np.array_equal(fin, np.isfinite(l))
    assert not o[~fin].any()
    if fin.any():
        rel_o, abs_l = TOL[kv_dtype]
        assert np.abs(o - o_ref).max() <= rel_o * max(np.abs(o_ref).max(), 1e-30)
        assert np.abs(l[fin] - l_ref[fin]).max() <= abs_l


PROBLEMS = {
    "bf16-dense": lambda: wl.make_problem("dense", num_shards=2, batch=3, heads=64,
                                          seq_len=[5000, 64, 3]),
    "fp8-agentic": lambda: wl.make_problem("agentic", num_shards=4, batch=5,
                                           seq_len=[9000, 4342, 130, 2, 20000]),
    "fp8-sparse": lambda: wl.make_problem("sparse", num_shards=2, batch=6, seq_len=3000,
                                          topk=300, seed=4),
}


@pytest.mark.parametrize("impl", ["auto", "simt"])
@pytest.mark.parametrize("name", sorted(PROBLEMS))
@pytest.mark.parametrize("num_splits", [0, 37])
def test_two_calls_in_a_row_match_the_workspace_entry_point(name, impl, num_splits):
    prob = PROBLEMS[name]().to("cuda")
    ref = [_with_workspace(prob, s, num_splits, impl) for s in (0, 1)]
    got = [_no_alloc(prob, s, num_splits, impl) for s in (0, 1)]    # back to back, one stream
    torch.cuda.synchronize()
    for (o, l, f), (o_ref, l_ref, f_ref) in zip(got, ref):
        assert int(f.item()) == 0 and int(f_ref.item()) == 0
        _close((o, l), (o_ref, l_ref), prob.kv_dtype)


def test_flags_belong_to_one_call():
    bad = wl.make_problem("tiny", num_shards=2).to("cuda")
    bad.seq_lens[0] = 10 ** 6                       # needs more blocks than the row has
    good = wl.make_problem("tiny", num_shards=2).to("cuda")
    _, _, f_bad = _no_alloc(bad, 0, 0, "simt")
    o, l, f_good = _no_alloc(good, 0, 0, "simt")
    o_ref, l_ref, _ = _with_workspace(good, 0, 0, "simt")
    torch.cuda.synchronize()
    assert int(f_bad.item()) & dcpmla.FLAG_BAD_LENGTH
    assert int(f_good.item()) == 0
    _close((o, l), (o_ref, l_ref), good.kv_dtype)


def test_request_beyond_the_scratch_is_refused():
    prob = wl.make_problem("tiny", num_shards=1).to("cuda")
    heads = 64
    batch = 600              # (600 + 148) slots x 64 heads x 2 KB > 32 MiB
    assert dcpmla.mla_decode_workspace_size(batch, heads, 148) > dcpmla.NOALLOC_SCRATCH_BYTES
    q = torch.zeros(batch, heads, dcpmla.HEAD_DIM, dtype=torch.bfloat16, device="cuda")
    o = torch.full((batch, heads, dcpmla.V_DIM), 7.0, device="cuda")
    l = torch.full((batch, heads), 7.0, device="cuda")
    bt = prob.block_tables[0].expand(batch, -1).contiguous()
    lens = prob.seq_lens.expand(batch).contiguous()
    with pytest.raises(dcpmla.DcpMlaError) as e:
        dcpmla.mla_decode_partial_noalloc(q, prob.kv_cache, prob.kv_dtype, bt, lens, 0, 1, None,
                                          prob.softmax_scale, o, l, None, 148, "auto")
    assert e.value.code == -3
    torch.cuda.synchronize()
    assert bool((o == 7.0).all()) and bool((l == 7.0).all())
