"""GPU-vs-oracle parity of the whole emulated DCP step, through the C ABI.

Tolerances, applied to every shard's partials and to the merged result: bf16
cache max|dO| <= 2e-3 * max|O| and |dLSE| <= 1e-4, fp8 cache max|dO| <=
2e-2 * max|O| (the required accuracy of the decode path) and |dLSE| <= 1e-3.
The fp8 path (dense, and sparse over the gathered selections) multiplies the
e4m3 codes exactly and applies each per-128 scale in fp32, so its scores
carry only fp32 accumulation error (the CUDA-core kernel likewise).  Only the
explicitly chosen fp16-operand kernel rounds e4m3 * scale once to fp16 before
the MMA (relative error <= 2^-11 per value, independent across values), so a
score moves by about 0.072 * 2^-11 * sqrt(sum_d q_d^2 k_d^2) ~ 0.9e-3 (rms,
N(0,1) data, 512 latent values); its LSE bound is 5e-3.
Empty shards must return exactly (0, -inf).  Addressing and sparse selection
are checked bit-exactly with id-coded rows.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from long_context_decode_mla_b200 import dcpmla
from long_context_decode_mla_b200 import workload as wl

pytestmark = pytest.mark.gpu

TOL = {"bf16": (2e-3, 1e-4), "fp8": (2e-2, 1e-3)}
TOL_FP8_FP16_OPERANDS = (2e-2, 5e-3)     # fp8 on the fp16-operand kernel (tc16)


def _tol(kv_dtype, impl, sparse):
    if kv_dtype == "fp8" and impl == "tc16":
        return TOL_FP8_FP16_OPERANDS
    return TOL[kv_dtype]
IMPLS = ["simt", "auto"]


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    dcpmla.lib()
    torch.cuda.set_device(0)


def _run(prob, impl="auto", num_splits=0, streams=None):
    dp = prob.to("cuda")
    topk = 0 if prob.sparse_idx is None else prob.sparse_idx.shape[1]
    dec = dcpmla.DcpDecoder(prob.batch, prob.heads, prob.num_shards, topk=topk,
                            num_splits=num_splits, impl=impl, streams=streams)
    dec.step(dp)
    torch.cuda.synchronize()
    assert dec.flags() == 0
    return (dec.partials.double().cpu().numpy(), dec.lses.double().cpu().numpy(),
            dec.out.double().cpu().numpy(), dec.out_lse.double().cpu().numpy())


def _oracle(prob, batch_ids=None):
    ni = prob.numpy_inputs()
    return oracle.dcp_decode(ni["q"], ni["kv_cache"], ni["kv_dtype"], ni["block_tables"],
                             ni["seq_lens"], ni["num_shards"], ni["softmax_scale"],
                             ni["sparse_idx"], ni["block_size"], batch_ids)


def _compare(o, l, o_ref, l_ref, kv_dtype, what, tol=None):
    rel_o, abs_l = TOL[kv_dtype] if tol is None else tol
    fin = np.isfinite(l_ref)
    assert np.array_equal(fin, np.isfinite(l)), f"{what}: -inf pattern differs"
    assert np.all(np.isneginf(l[~fin])), f"{what}: empty rows must have LSE -inf"
    empty_rows = ~fin
    assert not o[empty_rows].any(), f"{what}: empty rows must have O == 0"
    if not fin.any():
        return 0.0, 0.0
    scale = np.abs(o_ref).max()
    eo = np.abs(o - o_ref).max() / scale
    el = np.abs(l[fin] - l_ref[fin]).max()
    assert eo <= rel_o, f"{what}: max|dO|/max|O| = {eo:.3g} > {rel_o}"
    assert el <= abs_l, f"{what}: max|dLSE| = {el:.3g} > {abs_l}"
    return eo, el


def _check_problem(prob, impl="auto", batch_ids=None, num_splits=0, streams=None):
    parts, lses, out, lse = _run(prob, impl, num_splits, streams)
    rp, rl, ro, rlse = _oracle(prob, batch_ids)
    ids = list(range(prob.batch)) if batch_ids is None else list(batch_ids)
    tol = _tol(prob.kv_dtype, impl, prob.sparse_idx is not None)
    for s in range(prob.num_shards):
        _compare(parts[s, ids], lses[s, ids], rp[s], rl[s], prob.kv_dtype, f"shard {s}", tol)
    return _compare(out[ids], lse[ids], ro, rlse, prob.kv_dtype, "merged", tol)


# --------------------------------------------------------------- small ------

@pytest.mark.parametrize("impl", IMPLS)
@pytest.mark.parametrize("N", [1, 2, 4, 8])
def test_tiny_config(impl, N):
    _check_problem(wl.make_problem("tiny", num_shards=N), impl)


@pytest.mark.parametrize("impl", IMPLS)
@pytest.mark.parametrize("kv_dtype", ["bf16", "fp8"])
@pytest.mark.parametrize("N", [1, 3, 8])
def test_ragged_lengths_and_empty_shards(impl, kv_dtype, N):
    lens = [0, 1, N - 1, N, 63, 64, 65, 130, 1000, 4097]
    prob = wl.make_problem("dense", num_shards=N, batch=len(lens), heads=64, seq_len=lens,
                           kv_dtype=kv_dtype, seed=77)
    _check_problem(prob, impl)


@pytest.mark.parametrize("impl", IMPLS)
@pytest.mark.parametrize("heads", [1, 8, 17, 64])
def test_head_counts(impl, heads):
    prob = wl.make_problem("dense", num_shards=2, batch=3, heads=heads, seq_len=[700, 64, 3],
                           seed=5)
    _check_problem(prob, impl)


@pytest.mark.parametrize("impl", IMPLS)
@pytest.mark.parametrize("splits", [1, 3, 148, 400])
def test_split_counts_agree(impl, splits):
    prob = wl.make_problem("agentic", num_shards=4, batch=5,
                           seq_len=[9000, 200, 64, 20000, 5], seed=9)
    _check_problem(prob, impl, num_splits=splits)


# splits: 0 gives every request its own CTA; 2 puts three whole requests,
# empty ones among them, on each CTA of the request-aligned schedule
@pytest.mark.parametrize("impl", IMPLS)
@pytest.mark.parametrize("N", [1, 2, 8])
@pytest.mark.parametrize("splits", [0, 2])
def test_sparse_small(impl, N, splits):
    prob = wl.make_problem("sparse", num_shards=N, batch=6, seq_len=3000, topk=300, seed=4)
    idx = prob.sparse_idx
    idx[1] = -1                                   # empty list
    idx[2, :] = (torch.arange(300) * N) % 3000    # everything on shard 0
    idx[3, :150] = torch.arange(150) + 3000       # half out of range
    _check_problem(prob, impl, num_splits=splits)


# more requests than one CTA of the request-aligned schedule takes (32): a
# single requested CTA becomes ceil(70 / 32) = 3, each with empty lists
@pytest.mark.parametrize("impl", IMPLS)
def test_sparse_many_requests_per_cta(impl):
    prob = wl.make_problem("sparse", num_shards=2, batch=70, seq_len=1500, topk=100, seed=33)
    idx = prob.sparse_idx
    idx[5] = -1
    idx[40] = -1
    idx[69, 1:] = -1
    _check_problem(prob, impl, num_splits=1)


# bf16 rows: the auto path copies the selected rows into whole blocks for the
# fp16-operand kernel; the others select in-kernel
@pytest.mark.parametrize("impl", IMPLS + ["tc16"])
@pytest.mark.parametrize("N", [1, 4])
@pytest.mark.parametrize("splits", [0, 3])
def test_sparse_bf16_rows(impl, N, splits):
    prob = wl.make_problem("sparse", num_shards=N, batch=5, seq_len=2500, topk=260,
                           kv_dtype="bf16", seed=41)
    idx = prob.sparse_idx
    idx[0, 100:] = -1                             # a short list
    idx[2, :] = -1                                # empty list
    idx[4, :50] = torch.arange(50) + 2500         # some out of range
    _check_problem(prob, impl, num_splits=splits)


# --------------------------------------------------------------- addressing -

def _id_expect(ids):
    return [sum((t >> d) & 1 for t in ids) for d in range(21)]


@pytest.mark.parametrize("impl", IMPLS)
@pytest.mark.parametrize("kv_dtype", ["bf16", "fp8"])
@pytest.mark.parametrize("N", [1, 2, 3, 4, 8])
def test_block_table_addressing_is_exact(impl, kv_dtype, N):
    lens = [1, max(1, N - 1), N, 63, 64, 65, 1000, 5000]
    prob = wl.id_coded_problem(lens, N, kv_dtype, heads=8, seed=N)
    parts, lses, out, lse = _run(prob, impl)
    for b, L in enumerate(lens):
        for s in range(N):
            ids = [t for t in range(L) if t % N == s]
            if not ids:
                assert np.all(np.isneginf(lses[s, b])) and not parts[s, b].any()
                continue
            n = len(ids)
            assert np.abs(lses[s, b] - math.log(n)).max() < 1e-5
            counts = np.rint(parts[s, b, :, :21] * n)
            assert np.all(np.abs(parts[s, b, :, :21] * n - counts) < 1e-3)
            assert all(counts[h].tolist() == _id_expect(ids) for h in range(8))
            assert not parts[s, b, :, 21:].any()


@pytest.mark.parametrize("impl", IMPLS)
@pytest.mark.parametrize("N", [1, 2, 4, 8])
@pytest.mark.parametrize("splits", [0, 2])
def test_sparse_selection_is_exact(impl, N, splits):
    L = 6000
    rng = np.random.default_rng(N)
    idx = np.full((5, 512), -1, dtype=np.int32)
    idx[0] = rng.choice(L, 512, replace=False)
    idx[1, :64] = np.arange(64) * N + (N - 1)      # all on the last shard
    idx[2, :4] = [L, -5, 10 * L, -1]               # nothing valid
    idx[3, :300] = rng.choice(L, 300, replace=False)
    idx[4, :] = rng.choice(L, 512, replace=False)
    prob = wl.id_coded_problem([L] * 5, N, "fp8", heads=8, seed=N, sparse_idx=idx)
    parts, lses, out, lse = _run(prob, impl, num_splits=splits)
    for b in range(5):
        for s in range(N):
            ids = [int(t) for t in idx[b] if 0 <= t < L and t % N == s]
            if not ids:
                assert np.all(np.isneginf(lses[s, b])) and not parts[s, b].any()
                continue
            n = len(ids)
            assert np.abs(lses[s, b] - math.log(n)).max() < 1e-5
            counts = np.rint(parts[s, b, :, :21] * n)
            assert all(counts[h].tolist() == _id_expect(ids) for h in range(8))
    assert np.all(np.isneginf(lse[2])) and not out[2].any()


# --------------------------------------------------------------- merge ------

def test_dcp_merge_kernel_matches_oracle():
    rng = np.random.default_rng(7)
    N, B, H = 8, 5, 64
    parts = rng.standard_normal((N, B, H, 512)).astype(np.float32)
    lses = (rng.standard_normal((N, B, H)) * 4).astype(np.float32)
    lses[2, 1] = -np.inf
    lses[:, 3] = -np.inf                     # every shard empty
    parts[:, 3] = 0
    lses[1:, 4] = -np.inf                    # only shard 0 contributes
    o = torch.empty(B, H, 512, device="cuda")
    ol = torch.empty(B, H, device="cuda")
    dcpmla.dcp_merge(torch.from_numpy(parts).cuda(), torch.from_numpy(lses).cuda(), o, ol)
    torch.cuda.synchronize()
    ro, rl = oracle.dcp_merge(parts.astype(np.float64), lses.astype(np.float64))
    o, ol = o.double().cpu().numpy(), ol.double().cpu().numpy()
    assert np.array_equal(np.isneginf(ol), np.isneginf(rl))
    assert not o[3].any()
    fin = np.isfinite(rl)
    assert np.abs(o - ro).max() < 1e-5 * np.abs(ro).max()
    assert np.abs(ol[fin] - rl[fin]).max() < 1e-5


# --------------------------------------------------------------- faults -----

def test_bad_block_entry_is_flagged_not_read():
    prob = wl.make_problem("tiny", num_shards=2).to("cuda")
    prob.block_tables[1, 0, 2] = 10 ** 6           # outside the pool
    prob.block_tables[0, 0, 0] = -7
    dec = dcpmla.DcpDecoder(1, 8, 2, impl="simt")
    dec.step(prob)
    torch.cuda.synchronize()
    assert dec.flags() & dcpmla.FLAG_BAD_BLOCK


@pytest.mark.parametrize("impl", IMPLS)
@pytest.mark.parametrize("splits", [0, 2])
def test_sparse_bad_block_entry_is_flagged_and_skipped(impl, splits):
    # one table entry of shard 1 points outside the pool: the selections in
    # that block are flagged and left out, the rest decode as usual
    N, bad_b, bad_k = 2, 1, 2
    prob = wl.make_problem("sparse", num_shards=N, batch=4, seq_len=3000, topk=300, seed=21)
    expect = wl.DecodeProblem(prob.q, prob.kv_cache, prob.kv_dtype, prob.block_tables.clone(),
                              prob.seq_lens, N, prob.softmax_scale, prob.sparse_idx.clone(),
                              prob.block_size)
    idx = expect.sparse_idx[bad_b]
    hit = (idx >= 0) & (idx % N == 1) & ((idx // N) // prob.block_size == bad_k)
    assert hit.any()
    idx[hit] = -1
    prob.block_tables[1, bad_b, bad_k] = 10 ** 6
    dp = prob.to("cuda")
    dec = dcpmla.DcpDecoder(prob.batch, prob.heads, N, topk=prob.sparse_idx.shape[1],
                            num_splits=splits, impl=impl)
    dec.step(dp)
    torch.cuda.synchronize()
    assert dec.flags() & dcpmla.FLAG_BAD_BLOCK
    rp, rl, ro, rlse = _oracle(expect)
    parts, lses = dec.partials.double().cpu().numpy(), dec.lses.double().cpu().numpy()
    for s in range(N):
        _compare(parts[s], lses[s], rp[s], rl[s], prob.kv_dtype, f"shard {s}")
    _compare(dec.out.double().cpu().numpy(), dec.out_lse.double().cpu().numpy(), ro, rlse,
             prob.kv_dtype, "merged")


def test_length_beyond_table_is_flagged():
    prob = wl.make_problem("tiny", num_shards=2).to("cuda")
    prob.seq_lens[0] = 10 ** 6                       # needs more blocks than the row has
    dec = dcpmla.DcpDecoder(1, 8, 2, impl="simt")
    dec.step(prob)
    torch.cuda.synchronize()
    assert dec.flags() & dcpmla.FLAG_BAD_LENGTH


# --------------------------------------------------------------- full size --

def _sample(prob, k=3):
    lens = prob.seq_lens.tolist()
    order = sorted(range(len(lens)), key=lambda b: lens[b])
    return sorted(set([order[0], order[-1], order[len(order) // 2]][:k]))


@pytest.mark.parametrize("N", [1, 2, 4, 8])
def test_dense_config_full_size(N):
    prob = wl.make_problem("dense", num_shards=N, kv_device="cuda")
    _check_problem(prob, "auto", batch_ids=[0, 13, 31])


@pytest.mark.parametrize("N", [1, 2, 4, 8])
def test_agentic_config_full_size(N):
    prob = wl.make_problem("agentic", num_shards=N, kv_device="cuda")
    _check_problem(prob, "auto", batch_ids=_sample(prob))


@pytest.mark.parametrize("N", [1, 2, 4, 8])
def test_million_config_full_size(N):
    prob = wl.make_problem("million", num_shards=N, kv_device="cuda")
    streams = [torch.cuda.Stream() for _ in range(N)]
    _check_problem(prob, "auto", batch_ids=[0], num_splits=max(1, 148 // N), streams=streams)


@pytest.mark.parametrize("N", [1, 2, 4, 8])
def test_sparse_config_full_size(N):
    prob = wl.make_problem("sparse", num_shards=N, kv_device="cuda")
    _check_problem(prob, "auto", batch_ids=[0, 64, 127])


def test_sparse_config_full_size_sm_share():
    # the bench's launch: 8 shards, each given 148 / 8 CTAs (seven or eight
    # whole requests each)
    prob = wl.make_problem("sparse", num_shards=8, kv_device="cuda")
    _check_problem(prob, "auto", batch_ids=[0, 6, 7, 127], num_splits=18)


@pytest.mark.parametrize("impl", IMPLS)
@pytest.mark.parametrize("kv_dtype", ["bf16", "fp8"])
def test_growing_scores_force_mixed_rescales(impl, kv_dtype):
    """Rows grow along the sequence, so the running max jumps tile after tile
    for most heads, while heads with a zero query never move: the output
    rescaling is exercised with different decisions across heads."""
    g = torch.Generator().manual_seed(21)
    L = 3000
    rows = []
    for b in range(2):
        x = torch.randn(L, 576, generator=g) * (1.0 + torch.arange(L)[:, None] / 1500.0)
        if kv_dtype == "bf16":
            rows.append(x.to(torch.bfloat16).view(torch.uint8).view(L, 1152))
        else:
            rows.append(wl.pack_fp8_rows(x[:, :512], x[:, 512:]))
    cache, tables, lens = wl.place_rows(rows, 2, kv_dtype, seed=3)
    q = wl.random_q(2, 64, 21)
    q[:, ::3] = 0                                     # every third head never rescales
    prob = wl.DecodeProblem(q, cache, kv_dtype, tables, lens, 2)
    _check_problem(prob, impl, num_splits=1)


@pytest.mark.parametrize("impl", IMPLS)
def test_fp8_scales_outside_the_fp16_fast_path(impl):
    """Group scales above 65504 / 448 (codes capped at +-384 so every product
    stays finite) and below 2^-14 take the fp32 conversion path of the
    tensor-core kernel; they must match the oracle like any other scale.
    Request 0 has every scale at 160, request 1 every scale at 3e-5, request
    2 a random mix of 160, 3e-5 and ordinary scales.  The queries of requests
    0 and 2 are scaled down so that scores stay O(1)."""
    g = torch.Generator().manual_seed(31)
    L = 2500
    rows = []
    for b in range(3):
        x = torch.randn(L, 576, generator=g)
        r = wl.pack_fp8_rows(x[:, :512], x[:, 512:])
        codes = r[:, :512]
        big = codes & 0x7F > 0x7C                      # |value| > 384 -> 384, sign kept
        r[:, :512] = torch.where(big, (codes & 0x80) | 0x7C, codes)
        scales = r[:, 512:528].contiguous().view(torch.float32).view(L, 4)
        if b == 0:
            scales = torch.full_like(scales, 160.0)
        elif b == 1:
            scales = torch.full_like(scales, 3e-5)
        else:
            choice = torch.randint(0, 3, (L, 4), generator=g)
            scales = torch.where(choice == 0, torch.full_like(scales, 160.0),
                                 torch.where(choice == 1, torch.full_like(scales, 3e-5), scales))
        r[:, 512:528] = scales.contiguous().view(torch.uint8).view(L, 16)
        rows.append(r)
    cache, tables, lens = wl.place_rows(rows, 2, "fp8", seed=5)
    q = wl.random_q(3, 64, 31).float()
    q[0] *= 1e-4
    q[2] *= 1e-4
    prob = wl.DecodeProblem(q.to(torch.bfloat16), cache, "fp8", tables, lens, 2)
    _check_problem(prob, impl, num_splits=3)
