"""CPU oracle for prefill context parallelism (PCP) over a DCP-sharded cache.

TEST INFRASTRUCTURE ONLY, like the rest of ``oracle/``.

Sources (web pages, cited by title and section):

* "How vLLM Serves GLM-5.3 with Million-Token Contexts on 16 H200s", section
  "The core design": PCP splits a prompt's queries by token over the ranks;
  each rank computes all attention heads for its own tokens.  Causal
  attention makes later tokens dearer, so the prompt is cut into twice as
  many chunks as ranks and a front chunk is paired with a back chunk on each
  rank to even out the work (16 chunks for 8 ranks).  DCP keeps the cache
  distributed round-robin; since the query layout and the cache layout
  differ, prefill gathers the distributed cache for the layer, attends
  locally, and then drops the gathered copy.
* The DCP sources of ``mla_decode.py`` for the cache layout (token t on shard
  t mod N at local index t div N) and for attention with LSE.

Readings where the pages are silent (also listed in the design notes):

* Chunks are contiguous and in prompt order; with T tokens and 2P chunks (P
  ranks) the first T mod 2P chunks hold ceil(T / 2P) tokens and the rest
  floor(T / 2P) (so chunks may be empty when T < 2P).  Rank r owns chunks r
  and 2P - 1 - r; its queries are chunk r's tokens followed by chunk
  2P - 1 - r's.
* Attention is the absorbed-MLA form of the decode path (the only form the
  latent cache supports without model weights): query token i, head h,
  attends causally to every prompt token t <= i, scores softmax_scale *
  <q_i,h, k_t> over all 576 values, values the first 512; LSE in natural log.
* The prompt's rows are already in the distributed cache (the cache write of
  the prompt precedes its attention), one request at a time.

Parity status: pinned by the CPU tests (the chunk plan partitions the prompt
and balances causal work exactly, by its closed form; every prefill row
equals DCP decode of that token over its prefix, an independent call path
through the shard partials and the merge; token 0 reduces to its own value
row; brute force with math.fsum on tiny inputs).
"""
from __future__ import annotations

import numpy as np

from .mla_decode import attention_with_lse, decode_bf16, fetch_rows


def pcp_chunks(num_tokens: int, pcp_size: int) -> list[tuple[int, int]]:
    """The 2P contiguous chunks [start, stop) of a T-token prompt."""
    if pcp_size < 1 or num_tokens < 0:
        raise ValueError("pcp_size must be >= 1 and num_tokens >= 0")
    n = 2 * pcp_size
    base, extra = divmod(num_tokens, n)
    chunks, start = [], 0
    for k in range(n):
        size = base + (1 if k < extra else 0)
        chunks.append((start, start + size))
        start += size
    return chunks


def pcp_rank_tokens(num_tokens: int, pcp_size: int, rank: int) -> np.ndarray:
    """Query tokens of ``rank``: chunk ``rank`` then chunk 2P - 1 - rank."""
    if not 0 <= rank < pcp_size:
        raise ValueError(f"rank {rank} outside a PCP group of {pcp_size}")
    chunks = pcp_chunks(num_tokens, pcp_size)
    front = chunks[rank]
    back = chunks[2 * pcp_size - 1 - rank]
    return np.concatenate([np.arange(*front), np.arange(*back)]).astype(np.int64)


def gather_prompt_rows(kv_cache: np.ndarray, kv_dtype: str, block_tables: np.ndarray,
                       num_tokens: int, num_shards: int, block_size: int = 64) -> np.ndarray:
    """The gathered cache of one request: float64 [T, 576] in token order.

    ``block_tables`` [N, max_blocks]: each shard's table row for the request;
    token t is read from shard t mod N at local index t div N.
    """
    rows = np.zeros((num_tokens, 576))
    for s in range(num_shards):
        pos = np.arange(s, num_tokens, num_shards, dtype=np.int64)
        if pos.size:
            rows[pos] = fetch_rows(kv_cache, kv_dtype, block_tables[s], pos, num_shards,
                                   block_size)
    return rows


def pcp_prefill_rank(q: np.ndarray, rows: np.ndarray, tokens: np.ndarray,
                     softmax_scale: float):
    """Causal attention of the given query tokens over the gathered rows.

    q: [T, H, 576] (bf16 bits or floats) of the whole prompt; rows: float64
    [T, 576]; tokens: the rank's query positions.  Returns
    (O float64 [n, H, 512], LSE float64 [n, H]); query i sees rows 0..i.
    """
    qf = decode_bf16(q) if q.dtype == np.uint16 else np.asarray(q, dtype=np.float64)
    H = qf.shape[1]
    outs = np.zeros((len(tokens), H, 512))
    lses = np.zeros((len(tokens), H))
    for n, i in enumerate(tokens):
        outs[n], lses[n] = attention_with_lse(qf[i], rows[:i + 1], softmax_scale)
    return outs, lses


def pcp_prefill(q, kv_cache, kv_dtype, block_tables, num_tokens, pcp_size, num_shards,
                softmax_scale, block_size=64):
    """Every PCP rank's share of one request's prefill attention.

    Each rank gathers the distributed cache of the prompt, then attends with
    its own query tokens.  Returns a list over ranks of
    (tokens [n_r], O [n_r, H, 512], LSE [n_r, H]).
    """
    rows = gather_prompt_rows(kv_cache, kv_dtype, block_tables, num_tokens, num_shards,
                              block_size)
    out = []
    for r in range(pcp_size):
        tokens = pcp_rank_tokens(num_tokens, pcp_size, r)
        o, lse = pcp_prefill_rank(q, rows, tokens, softmax_scale)
        out.append((tokens, o, lse))
    return out
