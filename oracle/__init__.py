"""fp64 CPU oracle for DCP absorbed-MLA decode (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline legs of
``bench.py`` may import this package.  The CUDA path never does.
"""
from .mla_decode import (  # noqa: F401
    BF16_ROW_BYTES, FP8_ROW_BYTES, LATENT_DIM, ROPE_DIM, ROW_DIM,
    attention_with_lse, dcp_decode, dcp_merge, decode_bf16, decode_e4m3,
    decode_rows, e4m3_value, fetch_rows, local_positions, mla_decode_partial,
)
from .cache_write import (  # noqa: F401
    bf16_row, encode_e4m3, kv_append, quantize_fp8_row,
)
from .multi_query import dcp_decode_multi, mla_decode_partial_multi  # noqa: F401
from .pcp import (  # noqa: F401
    gather_prompt_rows, pcp_chunks, pcp_prefill, pcp_prefill_rank, pcp_rank_tokens,
)
