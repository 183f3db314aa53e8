"""CPU oracle for multi-query (speculative / multi-token prediction) DCP decode.

TEST INFRASTRUCTURE ONLY, like the rest of ``oracle/``.

Sources (web pages, cited by title and section):

* "GLM-5.2 vLLM Decode Context Parallelism", section "Add MTP only after plain
  decode passes": multi-token prediction adds draft-token query shapes to the
  same decode attention, and is verified after plain decode.
* "vLLM 0.28.0 Decode Context Parallel: The End of the Context-Length Tax in
  2026", section "DFlash2 Speculative Decoding": speculative decoding verifies
  several draft tokens per step.
* The DCP sources of ``mla_decode.py`` for sharding, LSE and the merge.

Readings where the pages are silent (also listed in the design notes):

* A step carries q_len query tokens per request; their keys are already in
  the cache, which holds L_b tokens in total.  Query i (0 <= i < q_len) sits at
  position L_b - q_len + i and attends causally to every cached token t with
  t <= L_b - q_len + i.  Queries at negative positions attend to nothing and
  give the neutral pair (O = 0, LSE = -inf).
* Rows are laid out [q_len][H]: q is [B][q_len][H][576], partial outputs
  [B][q_len][H][512] and LSEs [B][q_len][H]; sharding, LSE and the merge are
  those of single-query decode, per row.

Parity status: pinned by the CPU tests (q_len = 1 is the single-query oracle;
every row equals single-query decode over the prefix it may see, which is an
independent call path; the merge over shards equals the unsharded result;
brute force on tiny inputs).
"""
from __future__ import annotations

import numpy as np

from .mla_decode import (attention_with_lse, dcp_merge, decode_bf16, fetch_rows,
                         local_positions)


def mla_decode_partial_multi(q: np.ndarray, kv_cache: np.ndarray, kv_dtype: str,
                             block_table: np.ndarray, seq_lens: np.ndarray, shard_id: int,
                             num_shards: int, softmax_scale: float, block_size: int = 64):
    """One shard's partials for q_len query tokens per request.

    q: bf16 bits uint16 or floats [B, q_len, H, 576].  Returns
    (O float64 [B, q_len, H, 512], LSE float64 [B, q_len, H]).
    """
    qf = decode_bf16(q) if q.dtype == np.uint16 else np.asarray(q, dtype=np.float64)
    B, q_len, H = qf.shape[:3]
    outs = np.zeros((B, q_len, H, 512))
    lses = np.full((B, q_len, H), -np.inf)
    for b in range(B):
        L = int(seq_lens[b])
        pos = local_positions(L, num_shards, shard_id)
        keys = fetch_rows(kv_cache, kv_dtype, block_table[b], pos, num_shards, block_size)
        for i in range(q_len):
            limit = L - q_len + i                      # last position query i may see
            keep = pos <= limit
            o, lse = attention_with_lse(qf[b, i], keys[keep], softmax_scale)
            outs[b, i], lses[b, i] = o, lse
    return outs, lses


def dcp_decode_multi(q, kv_cache, kv_dtype, block_tables, seq_lens, num_shards, softmax_scale,
                     block_size=64):
    """All N shard partials, then the merge, for multi-query decode.

    Returns (partials [N, B, q_len, H, 512], lses [N, B, q_len, H],
    O [B, q_len, H, 512], LSE [B, q_len, H]).
    """
    parts, ls = [], []
    for s in range(num_shards):
        o, lse = mla_decode_partial_multi(q, kv_cache, kv_dtype, block_tables[s], seq_lens, s,
                                          num_shards, softmax_scale, block_size)
        parts.append(o)
        ls.append(lse)
    parts, ls = np.stack(parts), np.stack(ls)
    out, lse = dcp_merge(parts, ls)
    return parts, ls, out, lse
