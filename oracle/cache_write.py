"""CPU oracle for the DCP cache write of new decode tokens.

TEST INFRASTRUCTURE ONLY, like the rest of ``oracle/``: the tests,
``__graft_entry__.smoke()`` and ``bench.py``'s CPU legs may call it; the
product path never does.  It shares no code with the CUDA path.

Sources (web pages, cited by title and section):

* "GLM-5.2 vLLM Decode Context Parallelism", section "Keep the current-main
  correctness blocker visible" (sub-heading "Query work is skipped with an
  owner-remote KV slot"): under DCP a token whose cache slot is owned by
  another rank gets no cache write on this rank (the slot guard stays), while
  its query is still processed.  Ownership suppresses the write, not the query.
* same page, section "Stable H200 control: no DCP candidate": the fp8 cache
  dtype resolves to the DeepSeek sparse-MLA packed layout.
* "How vLLM Serves GLM-5.3 with Million-Token Contexts on 16 H200s", section
  "The core design": tokens are distributed to the ranks round-robin.

Readings where the pages are silent (also listed in the design notes):

* Token t of request b is owned by shard t mod N and lands at local row
  j = t div N: physical block ``block_table[b][j // 64]``, row ``j % 64``.
  A shard skips every token it does not own; a negative position means "no
  token" and is skipped as well.
* fp8 row (656 bytes) from a bf16 latent row x (512 values) and bf16 rope
  (64 values): for each group g of 128 latent values, amax_g = max |x| (exact
  in fp32), scale_g = fp32(amax_g / 448), or 1.0 when amax_g = 0; code =
  E4M3 of fp32(x / scale_g), rounded to nearest with ties to the even code and
  saturated at +-448.  Bytes: the 512 codes, the 4 scales as little-endian
  fp32, the 64 rope values as bf16.  bf16 row (1152 bytes): the 576 bf16
  values as given.
* A block-table entry outside [0, num_blocks) is not written and sets flag
  bit 1; a token whose local block index is beyond the table row, or whose
  request index is outside [0, batch), is not written and sets flag bit 2.

Parity status: pinned by the CPU tests (the encoder against the E4M3 value
table and an independent library cast, exact midpoint ties and saturation;
the quantiser's defining properties; ownership and placement against the
decode oracle's row fetch).
"""
from __future__ import annotations

import numpy as np

from .mla_decode import BF16_ROW_BYTES, FP8_ROW_BYTES, LATENT_DIM, decode_bf16, e4m3_value

BLOCK_ROWS = 64
FLAG_BAD_BLOCK = 1
FLAG_BAD_LENGTH = 2
E4M3_MAX = 448.0

# The 127 non-negative finite E4M3 values in code order (codes 0x00 .. 0x7E);
# they increase with the code, so nearest-value search is a sorted search.
_POS_VALUES = np.array([e4m3_value(c) for c in range(0x7F)], dtype=np.float64)


def encode_e4m3(x: np.ndarray) -> np.ndarray:
    """fp32 values -> OCP E4M3 ("fn") codes: nearest value, ties to the even
    code, magnitudes above 448 saturate to 448, the sign bit follows x."""
    x = np.asarray(x, dtype=np.float32)
    a = np.abs(x.astype(np.float64))
    a = np.minimum(a, E4M3_MAX)
    hi = np.searchsorted(_POS_VALUES, a, side="left")          # first value >= a
    hi = np.clip(hi, 0, 0x7E)
    lo = np.clip(hi - 1, 0, 0x7E)
    d_lo = a - _POS_VALUES[lo]
    d_hi = _POS_VALUES[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo).astype(np.uint8)
    code = np.where(a == _POS_VALUES[hi], hi, code).astype(np.uint8)   # exact hits
    sign = np.signbit(x).astype(np.uint8) << 7
    return (code | sign).astype(np.uint8)


def quantize_fp8_row(latent_bits: np.ndarray, rope_bits: np.ndarray) -> np.ndarray:
    """One 656-byte fp8 row from bf16 bit patterns (512 latent, 64 rope)."""
    x = decode_bf16(np.asarray(latent_bits, dtype=np.uint16)).astype(np.float32)
    codes = np.empty(LATENT_DIM, dtype=np.uint8)
    scales = np.empty(4, dtype=np.float32)
    for g in range(4):
        grp = x[128 * g:128 * g + 128]
        amax = np.float32(np.max(np.abs(grp)))
        scale = np.float32(1.0) if amax == 0 else np.float32(amax / np.float32(E4M3_MAX))
        scales[g] = scale
        codes[128 * g:128 * g + 128] = encode_e4m3((grp / scale).astype(np.float32))
    out = np.empty(FP8_ROW_BYTES, dtype=np.uint8)
    out[:512] = codes
    out[512:528] = scales.astype("<f4").view(np.uint8)
    out[528:] = np.asarray(rope_bits, dtype="<u2").view(np.uint8)
    return out


def bf16_row(latent_bits: np.ndarray, rope_bits: np.ndarray) -> np.ndarray:
    """One 1152-byte bf16 row: the 576 values as given."""
    bits = np.concatenate([np.asarray(latent_bits, dtype="<u2"),
                           np.asarray(rope_bits, dtype="<u2")])
    out = bits.view(np.uint8)
    assert out.size == BF16_ROW_BYTES
    return out


def kv_append(kv_cache: np.ndarray, kv_dtype: str, latent_bits: np.ndarray, rope_bits: np.ndarray,
              positions: np.ndarray, req_idx: np.ndarray, block_table: np.ndarray,
              shard_id: int, num_shards: int):
    """Shard ``shard_id``'s cache write of T new tokens.

    kv_cache [num_blocks][64][row bytes] uint8 (not modified; a copy is
    returned), latent_bits [T][512] and rope_bits [T][64] bf16 bit patterns,
    positions [T] global token positions, req_idx [T] request of each token,
    block_table [B][stride] this shard's table.  Returns (new cache, flags).
    """
    cache = np.array(kv_cache, copy=True)
    num_blocks = cache.shape[0]
    batch, stride = block_table.shape
    flags = 0
    for i in range(len(positions)):
        t, b = int(positions[i]), int(req_idx[i])
        if t < 0 or t % num_shards != shard_id:
            continue
        if not 0 <= b < batch:
            flags |= FLAG_BAD_LENGTH
            continue
        j = t // num_shards
        k = j // BLOCK_ROWS
        if k >= stride:
            flags |= FLAG_BAD_LENGTH
            continue
        blk = int(block_table[b, k])
        if not 0 <= blk < num_blocks:
            flags |= FLAG_BAD_BLOCK
            continue
        row = quantize_fp8_row(latent_bits[i], rope_bits[i]) if kv_dtype == "fp8" else \
            bf16_row(latent_bits[i], rope_bits[i])
        cache[blk, j % BLOCK_ROWS, :] = row
    return cache, flags
