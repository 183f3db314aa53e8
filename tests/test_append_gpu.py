"""GPU parity of the DCP cache write (``mla_kv_append``) through the C ABI.

The written cache bytes must equal the oracle's bit for bit (the quantised
codes and scales are integer/byte results of a fixed fp32 rule), tokens a
shard does not own must leave its blocks untouched, and a decode over the
appended rows must match the oracle's decode over the oracle-written cache.
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


def _bits(x: torch.Tensor) -> np.ndarray:
    return x.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _tokens(T, seed):
    g = torch.Generator().manual_seed(seed)
    lat = torch.randn(T, 512, generator=g)
    lat = lat * torch.exp(torch.randn(T, 4, generator=g) * 2).repeat_interleave(128, 1)
    lat[0, :128] = 0.0                       # an all-zero group
    lat[1, 128:256] = -0.0                   # negative zeros
    lat[2, 256:384] *= 1e-30                 # tiny values (bf16 subnormal range)
    lat[3, 384:] *= 1e4                      # large values
    rope = torch.randn(T, 64, generator=g)
    return lat.to(torch.bfloat16), rope.to(torch.bfloat16)


def _pool_and_tables(N, B, nblk, kv_dtype, seed):
    rng = np.random.default_rng(seed)
    tables = rng.permutation(N * B * nblk).astype(np.int32).reshape(N, B, nblk)
    rb = oracle.FP8_ROW_BYTES if kv_dtype == "fp8" else oracle.BF16_ROW_BYTES
    pool = rng.integers(0, 256, size=(N * B * nblk, 64, rb), dtype=np.uint8)   # junk to overwrite
    return pool, tables


def _append_all_shards_gpu(pool, tables, lat, rope, pos, req, kv_dtype, N):
    d_pool = torch.from_numpy(pool.copy()).cuda()
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    d_lat, d_rope = lat.cuda(), rope.cuda()
    d_pos = torch.from_numpy(pos).cuda()
    d_req = torch.from_numpy(req).cuda()
    for s in range(N):
        dcpmla.mla_kv_append(d_lat, d_rope, d_pos, d_req, torch.from_numpy(tables[s]).cuda(), s, N,
                             d_pool, kv_dtype, flags)
    torch.cuda.synchronize()
    return d_pool.cpu().numpy(), int(flags.item())


def _append_all_shards_oracle(pool, tables, lat, rope, pos, req, kv_dtype, N):
    cache, flags = pool, 0
    for s in range(N):
        cache, f = oracle.kv_append(cache, kv_dtype, _bits(lat), _bits(rope), pos, req,
                                    tables[s], s, N)
        flags |= f
    return cache, flags


@pytest.mark.parametrize("kv_dtype", ["fp8", "bf16"])
@pytest.mark.parametrize("N", [1, 2, 4, 8])
def test_written_bytes_match_the_oracle(kv_dtype, N):
    B, nblk, T = 3, 3, 96
    pool, tables = _pool_and_tables(N, B, nblk, kv_dtype, seed=N)
    g = torch.Generator().manual_seed(50 + N)
    pos = torch.randint(0, 64 * nblk * N, (T,), generator=g).numpy().astype(np.int32)
    req = torch.randint(0, B, (T,), generator=g).numpy().astype(np.int32)
    _, keep = np.unique(req.astype(np.int64) * 10 ** 6 + pos, return_index=True)
    keep = np.sort(keep)
    pos, req = pos[keep], req[keep]
    pos[-1] = -1                                        # padding entry
    lat, rope = _tokens(len(pos), seed=60 + N)
    got, gflags = _append_all_shards_gpu(pool, tables, lat, rope, pos, req, kv_dtype, N)
    want, wflags = _append_all_shards_oracle(pool, tables, lat, rope, pos, req, kv_dtype, N)
    assert gflags == wflags == 0
    diff = np.argwhere(got != want)
    assert diff.size == 0, f"{len(diff)} bytes differ, first at {diff[:4].tolist()}"
    # rows no shard owns a token for are untouched
    assert (got != pool).any(axis=2).sum() == len(pos) - 1


def test_out_of_range_entries_are_flagged_and_skipped():
    N, B, nblk = 2, 2, 2
    pool, tables = _pool_and_tables(N, B, nblk, "fp8", seed=9)
    bad = tables.copy()
    bad[0, 1, 0] = 10 ** 6                              # block outside the pool
    lat, rope = _tokens(4, seed=1)
    # ok, beyond the table, bad block, ok
    pos = np.array([0, 2 * 64 * nblk, 2, 4], dtype=np.int32)
    req = np.array([0, 0, 1, 5], dtype=np.int32)                  # last: request outside [0, B)
    d_pool = torch.from_numpy(pool.copy()).cuda()
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    dcpmla.mla_kv_append(lat.cuda(), rope.cuda(), torch.from_numpy(pos).cuda(),
                         torch.from_numpy(req).cuda(), torch.from_numpy(bad[0]).cuda(), 0, N,
                         d_pool, "fp8", flags)
    torch.cuda.synchronize()
    got = d_pool.cpu().numpy()
    want, wflags = oracle.kv_append(pool, "fp8", _bits(lat), _bits(rope), pos, req, bad[0], 0, N)
    assert int(flags.item()) == wflags == dcpmla.FLAG_BAD_BLOCK | dcpmla.FLAG_BAD_LENGTH
    assert np.array_equal(got, want)


@pytest.mark.parametrize("kv_dtype", ["fp8", "bf16"])
@pytest.mark.parametrize("N", [2, 8])
def test_decode_after_append_matches_the_oracle(kv_dtype, N):
    """Each request's next token (position L_b) is written on its owner shard,
    then the N shard partials and the merge run over L_b + 1 tokens."""
    lens = [3000, 1, 64 * N, 64 * N - 1, 777]
    name = "agentic" if kv_dtype == "fp8" else "dense"
    prob = wl.make_problem(name, num_shards=N, batch=len(lens), seq_len=[L + 1 for L in lens],
                           seed=77)
    B = prob.batch
    pos = np.array(lens, dtype=np.int32)
    req = np.arange(B, dtype=np.int32)
    # N(0,1) tokens like the rest of the cache: the tolerances above are
    # derived for such data (the byte-exact test covers extreme values)
    g = torch.Generator().manual_seed(78)
    lat = torch.randn(B, 512, generator=g).to(torch.bfloat16)
    rope = torch.randn(B, 64, generator=g).to(torch.bfloat16)
    pool = prob.kv_cache.numpy()
    tables = prob.block_tables.numpy()
    want_pool, wflags = _append_all_shards_oracle(pool, tables, lat, rope, pos, req, kv_dtype, N)
    got_pool, gflags = _append_all_shards_gpu(pool, tables, lat, rope, pos, req, kv_dtype, N)
    assert gflags == wflags == 0
    assert np.array_equal(got_pool, want_pool)
    # decode over the appended cache (GPU reads its own write; the oracle reads its own)
    dp = prob.to("cuda")
    dp.kv_cache = torch.from_numpy(got_pool).cuda()
    dec = dcpmla.DcpDecoder(B, prob.heads, N)
    dec.step(dp)
    torch.cuda.synchronize()
    assert dec.flags() == 0
    ni = prob.numpy_inputs()
    _, _, ro, rl = oracle.dcp_decode(ni["q"], want_pool, kv_dtype, ni["block_tables"],
                                     ni["seq_lens"], N, ni["softmax_scale"], None, 64)
    o = dec.out.double().cpu().numpy()
    lse = dec.out_lse.double().cpu().numpy()
    rel_o, abs_l = (2e-2, 5e-3) if kv_dtype == "fp8" else (2e-3, 1e-4)
    assert np.abs(o - ro).max() <= rel_o * np.abs(ro).max()
    assert np.abs(lse - rl).max() <= abs_l
