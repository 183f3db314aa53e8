"""Plain fp64 CPU oracle for decode-context-parallel (DCP) absorbed-MLA decode.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import or call this
module: it exists so that the tests, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` can check the CUDA
kernels against an independent, obviously correct statement of what they
compute.  It shares no code, constants or helpers with the CUDA path.

Sources (web pages, cited by title and section):

* "GLM-5.2 vLLM Decode Context Parallelism", section "See why vLLM 0.26.0
  fails": each rank computes attention over its local part of the cache, and
  the partial results are combined with the softmax normalisation, which needs
  the log-sum-exp (LSE) of decode attention.
* same page, section "Separate the backend merge from stable": the LSE comes
  back in token/head form; global sparse top-K indices are localised to the
  rank that owns each position; a row with no selected local token yields the
  neutral pair (O = 0, LSE = -inf) so that it drops out of the merge.
* same page, "Frequently asked questions" ("Why does DCP need softmax LSE?"):
  the LSE is the stable statistic used for the cross-rank merge.
* "How vLLM Serves GLM-5.3 with Million-Token Contexts on 16 H200s", section
  "The core design": the decode cache is spread over the ranks round-robin, so
  each of N ranks holds 1/N of the tokens.
* "The 3.3x Belongs to the Model, Not the Flag", section "What is being
  sharded": each rank stores and reads only its part of the sequence.
* "The Final Verification: Confirming a 200k Context Deployment on GLM-5",
  section "The Decision-Making Process Visible in the Reasoning": one MLA row
  per token and layer is kv_lora_rank + qk_rope_head_dim = 512 + 64 values.

Readings where the pages are silent (each is also listed in the design notes):

* Absorbed MLA: the query is already multiplied into the latent space, so one
  576-wide latent row serves as the key (all 576 values) and its first 512
  values as the value.  Output is the 512-wide latent attention output.
* Token t of request b belongs to shard t mod N at local index j = t div N.
  Each shard has its own block table over local indices; row j sits in
  physical block ``block_table[b][j // block_size]``, row ``j % block_size``.
* The LSE is the natural logarithm of sum_t exp(score_t), scores including
  the softmax scale.
* fp8 row layout (656 bytes): 512 OCP E4M3 codes in dimension order, four
  little-endian fp32 scales (one per 128 latent dimensions), 64 bf16 rope
  values.  Value of latent dimension d = e4m3(code[d]) * scale[d // 128].
  bf16 row layout (1152 bytes): 576 bf16 values.
* Sparse index lists hold global token positions; entries outside [0, L_b)
  (e.g. -1 padding) are skipped; each listed entry counts once as listed.

Parity status: every function here is pinned by the CPU tests (brute force in
high-precision decimal arithmetic, closed forms, merge invariants, the full
E4M3 code table against an independent library decoder, and id-coded
addressing checks).
"""
from __future__ import annotations

import math

import numpy as np

LATENT_DIM = 512          # kv_lora_rank: also the value / output width
ROPE_DIM = 64             # qk_rope_head_dim
ROW_DIM = LATENT_DIM + ROPE_DIM   # 576 values per cached token row
BF16_ROW_BYTES = ROW_DIM * 2      # 1152
FP8_ROW_BYTES = LATENT_DIM + 4 * 4 + ROPE_DIM * 2   # 512 + 16 + 128 = 656
FP8_SCALE_GROUP = 128


# ---------------------------------------------------------------- decoding --

def e4m3_value(code: int) -> float:
    """Value of one OCP FP8 E4M3 ("fn" flavour) byte, from the format itself.

    Bit 7 is the sign, bits 6..3 the exponent (bias 7), bits 2..0 the
    mantissa.  Exponent 0 encodes subnormals m * 2^-9.  Exponent 15 with
    mantissa 7 is NaN; there are no infinities, so 0x7E encodes 448.
    """
    sign = -1.0 if (code >> 7) & 1 else 1.0
    exp = (code >> 3) & 0xF
    man = code & 0x7
    if exp == 0xF and man == 0x7:
        return math.nan
    if exp == 0:
        return sign * man * 2.0 ** -9
    return sign * (1.0 + man / 8.0) * 2.0 ** (exp - 7)


_E4M3_TABLE = np.array([e4m3_value(c) for c in range(256)], dtype=np.float64)


def decode_e4m3(codes: np.ndarray) -> np.ndarray:
    """Decode an array of uint8 E4M3 codes to float64 (elementwise e4m3_value)."""
    return _E4M3_TABLE[np.asarray(codes, dtype=np.uint8)]


def decode_bf16(bits: np.ndarray) -> np.ndarray:
    """Decode uint16 bf16 bit patterns: they are the top half of an fp32."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def decode_rows(raw_rows: np.ndarray, kv_dtype: str) -> np.ndarray:
    """Turn raw cache rows (uint8 [n, row_bytes]) into float64 [n, 576]."""
    raw_rows = np.ascontiguousarray(raw_rows, dtype=np.uint8)
    n = raw_rows.shape[0]
    if kv_dtype == "bf16":
        assert raw_rows.shape[1] == BF16_ROW_BYTES
        return decode_bf16(raw_rows.view(np.uint16).reshape(n, ROW_DIM))
    if kv_dtype == "fp8":
        assert raw_rows.shape[1] == FP8_ROW_BYTES
        codes = raw_rows[:, :LATENT_DIM]
        scales = raw_rows[:, LATENT_DIM:LATENT_DIM + 16].copy().view("<f4")
        scales = scales.reshape(n, 4).astype(np.float64)
        rope = raw_rows[:, LATENT_DIM + 16:].copy().view("<u2").reshape(n, ROPE_DIM)
        out = np.empty((n, ROW_DIM), dtype=np.float64)
        latent = decode_e4m3(codes).reshape(n, 4, FP8_SCALE_GROUP)
        out[:, :LATENT_DIM] = (latent * scales[:, :, None]).reshape(n, LATENT_DIM)
        out[:, LATENT_DIM:] = decode_bf16(rope)
        return out
    raise ValueError(f"unknown kv dtype {kv_dtype!r}")


# ---------------------------------------------------------------- sharding --

def local_positions(seq_len: int, num_shards: int, shard_id: int,
                    sparse_idx: np.ndarray | None = None) -> np.ndarray:
    """Global token positions that shard ``shard_id`` attends over.

    Dense: every t in [0, seq_len) with t mod N == shard_id (round-robin
    ownership).  Sparse: the listed positions that are inside [0, seq_len)
    and owned by this shard, in list order.
    """
    if sparse_idx is None:
        return np.arange(shard_id, seq_len, num_shards, dtype=np.int64)
    idx = np.asarray(sparse_idx, dtype=np.int64)
    keep = (idx >= 0) & (idx < seq_len) & (idx % num_shards == shard_id)
    return idx[keep]


def fetch_rows(kv_cache: np.ndarray, kv_dtype: str, block_table_row: np.ndarray,
               positions: np.ndarray, num_shards: int, block_size: int) -> np.ndarray:
    """Rows (float64 [n, 576]) of the given global positions from one shard.

    ``kv_cache`` is the raw byte pool uint8 [num_blocks, block_size, row_bytes];
    ``block_table_row`` is this shard's table for the request, indexed by the
    local position j = t div N.
    """
    j = np.asarray(positions, dtype=np.int64) // num_shards
    blocks = np.asarray(block_table_row, dtype=np.int64)[j // block_size]
    rows = kv_cache[blocks, j % block_size]
    return decode_rows(rows, kv_dtype)


# --------------------------------------------------------------- attention --

def attention_with_lse(q: np.ndarray, keys: np.ndarray, softmax_scale: float):
    """Softmax attention of all heads over one set of latent rows.

    q: float64 [H, 576]; keys: float64 [n, 576].  Scores
    s[h, t] = softmax_scale * sum_d q[h, d] * keys[t, d]; values are the first
    512 columns of the same rows.  Returns (O [H, 512], LSE [H]) with
    LSE = m + ln sum_t exp(s - m), m = max_t s, and
    O = sum_t exp(s - LSE) * v_t.  An empty set gives O = 0, LSE = -inf.
    """
    H = q.shape[0]
    if keys.shape[0] == 0:
        return np.zeros((H, LATENT_DIM)), np.full(H, -np.inf)
    s = softmax_scale * (q @ keys.T)                 # [H, n]
    m = s.max(axis=1, keepdims=True)
    lse = m[:, 0] + np.log(np.exp(s - m).sum(axis=1))
    p = np.exp(s - lse[:, None])
    return p @ keys[:, :LATENT_DIM], lse


def mla_decode_partial(q: np.ndarray, kv_cache: np.ndarray, kv_dtype: str,
                       block_table: np.ndarray, seq_lens: np.ndarray,
                       shard_id: int, num_shards: int, softmax_scale: float,
                       sparse_idx: np.ndarray | None = None, block_size: int = 64,
                       batch_ids=None):
    """Partial attention of one shard for every request (or ``batch_ids``).

    q: bf16 bits uint16 [B, H, 576] or float array [B, H, 576];
    kv_cache: uint8 [num_blocks, block_size, row_bytes]; block_table: int32
    [B, max_blocks] of this shard; seq_lens: global lengths [B];
    sparse_idx: int32 [B, topk] global positions or None.
    Returns (O float64 [len(batch_ids), H, 512], LSE float64 [len(batch_ids), H]).
    """
    qf = decode_bf16(q) if q.dtype == np.uint16 else np.asarray(q, dtype=np.float64)
    ids = range(qf.shape[0]) if batch_ids is None else batch_ids
    outs, lses = [], []
    for b in ids:
        pos = local_positions(int(seq_lens[b]), num_shards, shard_id,
                              None if sparse_idx is None else sparse_idx[b])
        keys = fetch_rows(kv_cache, kv_dtype, block_table[b], pos, num_shards, block_size)
        o, lse = attention_with_lse(qf[b], keys, softmax_scale)
        outs.append(o)
        lses.append(lse)
    return np.stack(outs), np.stack(lses)


def dcp_merge(partials: np.ndarray, lses: np.ndarray):
    """LSE-weighted merge of N partial results.

    partials: [N, ..., 512]; lses: [N, ...].  With M = max_i LSE_i and
    w_i = exp(LSE_i - M): O = sum_i w_i O_i / sum_i w_i and
    LSE = M + ln sum_i w_i.  Entries with LSE_i = -inf weigh exactly 0; if all
    are -inf the result is (0, -inf).
    """
    partials = np.asarray(partials, dtype=np.float64)
    lses = np.asarray(lses, dtype=np.float64)
    M = lses.max(axis=0)
    empty = np.isneginf(M)
    M_safe = np.where(empty, 0.0, M)
    w = np.where(np.isneginf(lses), 0.0, np.exp(lses - M_safe[None]))
    wsum = w.sum(axis=0)
    wsum_safe = np.where(empty, 1.0, wsum)
    out = (w[..., None] * partials).sum(axis=0) / wsum_safe[..., None]
    out = np.where(empty[..., None], 0.0, out)
    lse = np.where(empty, -np.inf, M_safe + np.log(wsum_safe))
    return out, lse


def dcp_decode(q, shard_caches, kv_dtype, block_tables, seq_lens, num_shards,
               softmax_scale, sparse_idx=None, block_size=64, batch_ids=None):
    """Whole DCP step: every shard's partial, then the merge.

    ``shard_caches`` is either one pool shared by all shards or a list of N
    pools; ``block_tables`` is [N, B, max_blocks].  Returns
    (partials [N, b, H, 512], lses [N, b, H], O [b, H, 512], LSE [b, H]).
    """
    parts, ls = [], []
    for s in range(num_shards):
        cache = shard_caches[s] if isinstance(shard_caches, (list, tuple)) else shard_caches
        o, lse = mla_decode_partial(q, cache, kv_dtype, block_tables[s], seq_lens, s,
                                    num_shards, softmax_scale, sparse_idx, block_size,
                                    batch_ids)
        parts.append(o)
        ls.append(lse)
    parts = np.stack(parts)
    ls = np.stack(ls)
    out, lse = dcp_merge(parts, ls)
    return parts, ls, out, lse
