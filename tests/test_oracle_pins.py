"""Pins for the fp64 CPU oracle, independent of the oracle's own code.

Every check here compares the oracle with something it does not contain:
high-precision decimal brute force, closed forms, merge identities, a library
decoder for the E4M3 code table, id-coded rows whose expected outputs follow
from the round-robin ownership rule, and figures printed on the pages.  The
``planted`` tests at the end swap a plausible mistake into a copy of the
oracle and check that at least one pin catches it.
"""
import importlib.util
import json
import math
import os
from decimal import Decimal, getcontext

import numpy as np
import pytest
import torch

import oracle
from long_context_decode_mla_b200 import workload as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
SCALE = 192 ** -0.5


# ------------------------------------------------------------ helpers ------

def _lib_rows(rows_u8: torch.Tensor, kv_dtype: str):
    """Decode rows with torch's own dtypes (independent of the oracle's decoder).

    Returns a list of rows, each a list of 576 exact Python floats.
    """
    n = rows_u8.shape[0]
    if kv_dtype == "bf16":
        vals = rows_u8.contiguous().view(torch.bfloat16).view(n, 576).double()
        return vals.tolist(), None
    codes = rows_u8[:, :512].contiguous().view(torch.float8_e4m3fn).double().view(n, 4, 128)
    scales = rows_u8[:, 512:528].contiguous().view(torch.float32).view(n, 4).double()
    rope = rows_u8[:, 528:].contiguous().view(torch.bfloat16).view(n, 64).double()
    return codes, scales, rope


def _decimal_rows(rows_u8, kv_dtype):
    """Exact decimal values of each row (fp8: code * scale computed in Decimal)."""
    if kv_dtype == "bf16":
        vals, _ = _lib_rows(rows_u8, kv_dtype)
        return [[Decimal(x) for x in r] for r in vals]
    codes, scales, rope = _lib_rows(rows_u8, kv_dtype)
    out = []
    for i in range(rows_u8.shape[0]):
        r = []
        for g in range(4):
            sc = Decimal(float(scales[i, g]))
            r.extend(Decimal(float(c)) * sc for c in codes[i, g].tolist())
        r.extend(Decimal(x) for x in rope[i].tolist())
        out.append(r)
    return out


def _decimal_attention(q_rows, k_rows, scale):
    """Direct softmax attention in 60-digit decimal: no max shift, no blocking."""
    getcontext().prec = 60
    sc = Decimal(scale)
    H = len(q_rows)
    if not k_rows:
        return np.zeros((H, 512)), np.full(H, -np.inf)
    O = np.zeros((H, 512))
    L = np.zeros(H)
    for h in range(H):
        s = [sc * sum(qa * kb for qa, kb in zip(q_rows[h], k)) for k in k_rows]
        e = [x.exp() for x in s]
        z = sum(e)
        L[h] = float(z.ln())
        for d in range(512):
            O[h, d] = float(sum(ei * k[d] for ei, k in zip(e, k_rows)) / z)
    return O, L


def _assert_close(o, lse, o_ref, lse_ref, rel=1e-12):
    scale_o = max(1e-300, float(np.abs(o_ref).max()))
    assert np.abs(o - o_ref).max() <= rel * scale_o
    fin = np.isfinite(lse_ref)
    assert np.array_equal(fin, np.isfinite(lse))
    assert np.all(np.isneginf(lse[~fin]))
    if fin.any():
        assert np.abs(lse[fin] - lse_ref[fin]).max() <= rel * max(1.0, np.abs(lse_ref[fin]).max())


def _run_oracle(prob, shard_id=None, batch_ids=None, mod=oracle):
    ni = prob.numpy_inputs()
    if shard_id is None:
        return mod.dcp_decode(ni["q"], ni["kv_cache"], ni["kv_dtype"], ni["block_tables"],
                              ni["seq_lens"], ni["num_shards"], ni["softmax_scale"],
                              ni["sparse_idx"], ni["block_size"], batch_ids)
    return mod.mla_decode_partial(ni["q"], ni["kv_cache"], ni["kv_dtype"],
                                  ni["block_tables"][shard_id], ni["seq_lens"], shard_id,
                                  ni["num_shards"], ni["softmax_scale"], ni["sparse_idx"],
                                  ni["block_size"], batch_ids)


# ------------------------------------------------------------ decoders -----

def test_e4m3_table_matches_library_decoder():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    lib = codes.view(torch.float8_e4m3fn).double().numpy()
    ours = oracle.decode_e4m3(np.arange(256, dtype=np.uint8))
    nan = np.isnan(lib)
    assert np.array_equal(nan, np.isnan(ours))
    assert nan.sum() == 2                          # 0x7F and 0xFF
    assert np.array_equal(lib[~nan], ours[~nan])
    assert ours[0x7E] == 448.0 and ours[0x01] == 2.0 ** -9 and ours[0x38] == 1.0


def test_bf16_decode_matches_library():
    g = torch.Generator().manual_seed(3)
    x = (torch.randn(4096, generator=g) * 1e3).to(torch.bfloat16)
    bits = x.view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(oracle.decode_bf16(bits), x.double().numpy())


# ------------------------------------------------------------ brute force --

@pytest.mark.parametrize("kv_dtype", ["bf16", "fp8"])
@pytest.mark.parametrize("N", [1, 3])
def test_brute_force_decimal(kv_dtype, N):
    """Each shard's partial and the merge equal direct decimal softmax attention."""
    lens = [37, 5]
    prob, rows = wl.logical_problem(lens, N, kv_dtype, heads=3, seed=11)
    q = prob.q.double().tolist()
    q_dec = [[[Decimal(x) for x in h] for h in b] for b in q]
    parts, lses, out, lse = _run_oracle(prob)
    for b, L in enumerate(lens):
        k_all = _decimal_rows(rows[b], kv_dtype)
        o_ref, l_ref = _decimal_attention(q_dec[b], k_all, SCALE)
        _assert_close(out[b], lse[b], o_ref, l_ref)
        for s in range(N):
            sub = [k_all[t] for t in range(L) if t % N == s]
            o_ref, l_ref = _decimal_attention(q_dec[b], sub, SCALE)
            _assert_close(parts[s, b], lses[s, b], o_ref, l_ref)


def test_lse_is_log_of_sum_of_exp_without_shift():
    """LSE = ln sum exp(score) computed directly in extended precision."""
    prob, rows = wl.logical_problem([50], 1, "bf16", heads=4, seed=12)
    ni = prob.numpy_inputs()
    o, lse = _run_oracle(prob, shard_id=0)
    k = oracle.decode_rows(rows[0].numpy(), "bf16").astype(np.longdouble)
    qv = prob.q[0].double().numpy().astype(np.longdouble)
    s = np.longdouble(SCALE) * (qv @ k.T)
    direct = np.log(np.exp(s).sum(axis=1))
    assert np.abs(lse[0] - direct.astype(np.float64)).max() < 1e-12


# ------------------------------------------------------------ closed forms -

def test_zero_query_gives_mean_and_log_count():
    prob, rows = wl.logical_problem([77], 1, "bf16", heads=2, seed=13)
    prob.q.zero_()
    o, lse = _run_oracle(prob, shard_id=0)
    v = rows[0].view(torch.bfloat16).view(77, 576)[:, :512].double().numpy()
    assert np.allclose(lse[0], math.log(77), rtol=0, atol=1e-13)
    assert np.abs(o[0] - v.mean(axis=0)[None]).max() < 1e-13


def test_single_and_pair_of_tokens():
    prob, rows = wl.logical_problem([1, 2], 1, "bf16", heads=3, seed=14)
    o, lse = _run_oracle(prob, shard_id=0)
    for b, L in [(0, 1), (1, 2)]:
        k = rows[b].view(torch.bfloat16).view(L, 576).double().numpy()
        q = prob.q[b].double().numpy()
        s = SCALE * q @ k.T
        if L == 1:
            assert np.array_equal(o[b], np.repeat(k[:1, :512], 3, axis=0))
            assert np.abs(lse[b] - s[:, 0]).max() < 1e-13
        else:
            sig = 1.0 / (1.0 + np.exp(s[:, 1] - s[:, 0]))     # weight of token 0
            ref = sig[:, None] * k[0, :512] + (1 - sig)[:, None] * k[1, :512]
            assert np.abs(o[b] - ref).max() < 1e-13
            assert np.abs(lse[b] - np.logaddexp(s[:, 0], s[:, 1])).max() < 1e-13


def test_identical_keys_give_uniform_weights():
    rows = [wl.random_logical_rows([1], "bf16", 15)[0].repeat(40, 1)]
    cache, tables, lens = wl.place_rows(rows, 4, "bf16", 15)
    q = wl.random_q(1, 2, 15)
    prob = wl.DecodeProblem(q, cache, "bf16", tables, lens, 4)
    parts, lses, out, lse = _run_oracle(prob)
    k = rows[0][:1].view(torch.bfloat16).double().numpy()
    s = SCALE * q[0].double().numpy() @ k.T
    assert np.abs(out[0] - k[0, :512][None]).max() < 1e-14
    assert np.abs(lse[0] - (s[:, 0] + math.log(40))).max() < 1e-12
    for sh in range(4):     # 10 tokens per shard
        assert np.abs(lses[sh, 0] - (s[:, 0] + math.log(10))).max() < 1e-12


# ------------------------------------------------------------ merge --------

def _random_partials(rng, N, shape=(3, 5)):
    parts = rng.standard_normal((N, *shape, 512))
    lses = rng.standard_normal((N, *shape)) * 5
    return parts, lses


@pytest.mark.parametrize("N", [1, 2, 3, 4, 8])
def test_merge_of_shards_equals_unsharded(N):
    prob, rows = wl.logical_problem([300, 41, 7], N, "bf16", heads=4, seed=20 + N)
    parts, lses, out, lse = _run_oracle(prob)
    cache1, tables1, lens1 = wl.place_rows(rows, 1, "bf16", 99)
    prob1 = wl.DecodeProblem(prob.q, cache1, "bf16", tables1, lens1, 1)
    o1, l1 = _run_oracle(prob1, shard_id=0)
    assert np.abs(out - o1).max() < 1e-12 * np.abs(o1).max()
    assert np.abs(lse - l1).max() < 1e-12 * max(1.0, np.abs(l1).max())


def test_merge_is_order_independent_and_associative():
    rng = np.random.default_rng(0)
    parts, lses = _random_partials(rng, 6)
    o, l = oracle.dcp_merge(parts, lses)
    perm = rng.permutation(6)
    o2, l2 = oracle.dcp_merge(parts[perm], lses[perm])
    assert np.abs(o - o2).max() < 1e-13 and np.abs(l - l2).max() < 1e-13
    oa, la = oracle.dcp_merge(parts[:2], lses[:2])
    ob, lb = oracle.dcp_merge(parts[2:], lses[2:])
    o3, l3 = oracle.dcp_merge(np.stack([oa, ob]), np.stack([la, lb]))
    assert np.abs(o - o3).max() < 1e-13 and np.abs(l - l3).max() < 1e-13


def test_merge_identity_and_all_empty():
    rng = np.random.default_rng(1)
    parts, lses = _random_partials(rng, 3)
    o, l = oracle.dcp_merge(parts, lses)
    z = np.zeros((1, *parts.shape[1:]))
    ninf = np.full((1, *lses.shape[1:]), -np.inf)
    o2, l2 = oracle.dcp_merge(np.concatenate([parts, z]), np.concatenate([lses, ninf]))
    assert np.array_equal(o, o2) and np.array_equal(l, l2)
    oe, le = oracle.dcp_merge(np.zeros((4, 2, 512)), np.full((4, 2), -np.inf))
    assert np.array_equal(oe, np.zeros((2, 512))) and np.all(np.isneginf(le))
    # a single finite shard among empty ones passes through unchanged
    o1, l1 = oracle.dcp_merge(np.stack([z[0], parts[0], z[0]]),
                              np.stack([ninf[0], lses[0], ninf[0]]))
    assert np.abs(o1 - parts[0]).max() < 1e-15 and np.array_equal(l1, lses[0])


# ------------------------------------------------------------ addressing ---

@pytest.mark.parametrize("kv_dtype", ["bf16", "fp8"])
@pytest.mark.parametrize("N", [1, 2, 3, 8])
def test_id_coded_dense_addressing(kv_dtype, N):
    """Shard s reads exactly the tokens t < L with t mod N = s."""
    lens = [1, N - 1 if N > 1 else 2, N, 63, 64, 65, 1000]
    prob = wl.id_coded_problem(lens, N, kv_dtype, heads=2, seed=N)
    parts, lses, out, lse = _run_oracle(prob)
    for b, L in enumerate(lens):
        for s in range(N):
            ids = [t for t in range(L) if t % N == s]
            if not ids:
                assert np.all(np.isneginf(lses[s, b])) and not parts[s, b].any()
                continue
            assert np.allclose(lses[s, b], math.log(len(ids)), rtol=0, atol=1e-13)
            counts = np.rint(parts[s, b, 0, :21] * len(ids))
            exp = [sum((t >> d) & 1 for t in ids) for d in range(21)]
            assert counts.tolist() == exp
            assert not parts[s, b, :, 21:].any()


@pytest.mark.parametrize("N", [1, 2, 4, 8])
def test_id_coded_sparse_selection(N):
    L = 500
    rng = np.random.default_rng(N)
    idx = np.full((4, 64), -1, dtype=np.int32)
    idx[0, :40] = rng.choice(L, 40, replace=False)             # spread over shards
    idx[1, :10] = np.arange(10) * N                            # all on shard 0
    idx[2, :5] = [L, L + 7, -3, 2 * L, -1]                     # all invalid
    idx[3, :] = rng.choice(L, 64, replace=False)               # full list
    prob = wl.id_coded_problem([L] * 4, N, "fp8", heads=2, seed=N, sparse_idx=idx)
    parts, lses, out, lse = _run_oracle(prob)
    for b in range(4):
        for s in range(N):
            ids = [int(t) for t in idx[b] if 0 <= t < L and t % N == s]
            if not ids:
                assert np.all(np.isneginf(lses[s, b])) and not parts[s, b].any()
                continue
            assert np.allclose(lses[s, b], math.log(len(ids)), rtol=0, atol=1e-13)
            counts = np.rint(parts[s, b, 0, :21] * len(ids))
            assert counts.tolist() == [sum((t >> d) & 1 for t in ids) for d in range(21)]
    assert np.all(np.isneginf(lse[2]))


# ------------------------------------------------------------ page figures -

def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def test_golden_row_bytes():
    g = _golden("mla_row_bytes.json")
    assert g["kv_lora_rank"] == oracle.LATENT_DIM and g["qk_rope_head_dim"] == oracle.ROPE_DIM
    assert oracle.BF16_ROW_BYTES == g["bytes_per_token_per_layer"]
    assert oracle.BF16_ROW_BYTES * g["layers"] // g["gpus"] == g["bytes_per_token_per_gpu"]
    rows = wl.random_logical_rows([3], "bf16", 1)[0]
    assert rows.shape[1] == g["bytes_per_token_per_layer"]
    assert oracle.decode_rows(rows.numpy(), "bf16").shape == (3, 576)


def test_golden_round_robin_share():
    g = _golden("round_robin_share.json")
    L, N = g["request_tokens"], g["num_shards"]
    sets = [oracle.local_positions(L, N, s) for s in range(N)]
    assert all(len(x) == L // N for x in sets)
    allpos = np.sort(np.concatenate(sets))
    assert np.array_equal(allpos, np.arange(L))
    assert round(g["total_gib"] * len(sets[0]) / L, 1) == g["per_gpu_gib_rounded"]


# ------------------------------------------------------------ planted ------

def _oracle_copy():
    spec = importlib.util.spec_from_file_location(
        "oracle_copy", os.path.join(os.path.dirname(oracle.__file__), "mla_decode.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _brute_force_error(mod, kv_dtype="fp8", N=2):
    lens = [23]
    prob, rows = wl.logical_problem(lens, N, kv_dtype, heads=2, seed=31)
    q_dec = [[[Decimal(x) for x in h] for h in b] for b in prob.q.double().tolist()]
    parts, lses, out, lse = _run_oracle(prob, mod=mod)
    k_all = _decimal_rows(rows[0], kv_dtype)
    o_ref, l_ref = _decimal_attention(q_dec[0], k_all, SCALE)
    err = np.abs(out[0] - o_ref).max() / np.abs(o_ref).max()
    for s in range(N):
        sub = [k_all[t] for t in range(lens[0]) if t % N == s]
        o_s, l_s = _decimal_attention(q_dec[0], sub, SCALE)
        err = max(err, np.abs(parts[s, 0] - o_s).max() / np.abs(o_s).max(),
                  np.abs(lses[s, 0] - l_s).max())
    return err


def test_planted_mistakes_are_caught():
    base = _brute_force_error(_oracle_copy())
    assert base < 1e-12

    m = _oracle_copy()                        # scores without the rope part
    orig = m.attention_with_lse

    def no_rope(q, keys, scale):
        k2 = keys.copy()
        k2[:, 512:] = 0
        o, l = orig(q, k2, scale)
        if keys.shape[0]:
            s = scale * (q @ keys.T)
            p = np.exp(scale * (q @ k2.T) - l[:, None])
            o = p @ keys[:, :512]
        return o, l
    m.attention_with_lse = no_rope
    assert _brute_force_error(m) > 1e-6

    m = _oracle_copy()                        # fp8 scale also applied to rope
    dec = m.decode_rows

    def scaled_rope(raw, kv_dtype):
        out = dec(raw, kv_dtype)
        sc = raw[:, 512:516].copy().view("<f4").astype(np.float64)
        out[:, 512:] *= sc
        return out
    m.decode_rows = scaled_rope
    assert _brute_force_error(m) > 1e-6

    m = _oracle_copy()                        # contiguous (not round-robin) ownership
    def blocked(seq_len, num_shards, shard_id, sparse_idx=None):
        per = -(-seq_len // num_shards)
        return np.arange(shard_id * per, min(seq_len, (shard_id + 1) * per))
    m.local_positions = blocked
    assert _brute_force_error(m) > 1e-6

    m = _oracle_copy()                        # base-2 log-sum-exp
    orig2 = m.attention_with_lse
    m.attention_with_lse = lambda q, k, s: (lambda o, l: (o, l / math.log(2)))(*orig2(q, k, s))
    assert _brute_force_error(m) > 1e-6

    m = _oracle_copy()                        # E4M3 with the wrong exponent bias
    m._E4M3_TABLE = m._E4M3_TABLE * 2.0
    ours = m.decode_e4m3(np.arange(256, dtype=np.uint8))
    lib = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).double()
    fin = ~np.isnan(ours)
    assert not np.array_equal(ours[fin], lib.numpy()[fin])

    m = _oracle_copy()                        # merge that ignores empty shards' -inf
    def naive_merge(parts, lses):
        w = np.exp(lses - lses.max(axis=0))
        return (w[..., None] * parts).sum(0) / w.sum(0)[..., None], np.log(np.exp(lses).sum(0))
    m.dcp_merge = naive_merge
    with np.errstate(all="ignore"):
        oe, le = m.dcp_merge(np.zeros((2, 1, 512)), np.full((2, 1), -np.inf))
    assert np.isnan(oe).any()
