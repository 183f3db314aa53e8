"""ctypes binding of libdcpmla.so (argument marshalling only).

The functions keep the C names (``mla_decode_partial``, ``dcp_merge``,
``mla_decode_workspace_size``, ``dcpmla_error_string``); they take torch
tensors for device memory, pass raw pointers and sizes, and raise
:class:`DcpMlaError` on a negative return code.  All arithmetic happens in the
library's CUDA kernels.  :class:`DcpDecoder` strings the calls together for a
whole emulated DCP step (N shard partials, then the merge).
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdcpmla.so")

KV_DTYPES = {"bf16": 0, "fp8": 1}
IMPLS = {"auto": 0, "simt": 1, "tc": 2, "tc16": 3}
HEAD_DIM, V_DIM, BLOCK_SIZE, MAX_HEADS = 576, 512, 64, 64
FLAG_BAD_BLOCK, FLAG_BAD_LENGTH, FLAG_TIMEOUT, FLAG_RANGE = 1, 2, 4, 8

_lib = None


class DcpMlaError(RuntimeError):
    def __init__(self, code: int, where: str):
        super().__init__(f"{where} failed: {error_string(code)} (code {code})")
        self.code = code


def lib() -> ctypes.CDLL:
    """Load libdcpmla.so (once).  Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"{LIB_PATH} is missing: build it with `python -m long_context_decode_mla_b200.build`"
            " (the decode path has no fallback)")
    L = ctypes.CDLL(LIB_PATH)
    vp, i32, i64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
    f32, sz = ctypes.c_float, ctypes.c_size_t
    L.mla_decode_workspace_size.argtypes = [i32, i32, i32, i32, ctypes.POINTER(sz)]
    L.mla_decode_workspace_size.restype = i32
    L.mla_decode_partial.argtypes = [vp, vp, i32, i64, i32, vp, i32, vp, i32, i32, i32, i32, vp,
                                     i32, f32, vp, vp, vp, sz, i32, i32, vp]
    L.mla_decode_partial.restype = i32
    L.dcp_merge.argtypes = [vp, vp, i32, i32, i32, vp, vp, vp]
    L.dcp_merge.restype = i32
    L.dcpmla_error_string.argtypes = [i32]
    L.dcpmla_error_string.restype = ctypes.c_char_p
    L.dcpmla_device_sm_count.argtypes = [ctypes.POINTER(i32)]
    L.dcpmla_device_sm_count.restype = i32
    L.mla_decode_partial_multi.argtypes = [vp, vp, i32, i64, i32, vp, i32, vp, i32, i32, i32, i32,
                                           i32, f32, vp, vp, vp, sz, i32, i32, vp]
    L.mla_decode_partial_multi.restype = i32
    L.mla_decode_partial_noalloc.argtypes = [vp, vp, i32, i64, i32, vp, i32, vp, i32, i32, i32,
                                             i32, vp, i32, f32, vp, vp, vp, i32, i32, vp]
    L.mla_decode_partial_noalloc.restype = i32
    L.mla_kv_append.argtypes = [vp, vp, i32, vp, vp, vp, i32, i32, i32, i32, vp, i32, i64, i32,
                                vp, vp]
    L.mla_kv_append.restype = i32
    L.dcp_merge_heads.argtypes = [vp, vp, i32, i32, i32, i32, i32, vp, vp, vp]
    L.dcp_merge_heads.restype = i32
    L.dcp_exchange_alloc.argtypes = [sz, ctypes.POINTER(vp), vp]
    L.dcp_exchange_alloc.restype = i32
    L.dcp_exchange_open.argtypes = [vp, ctypes.POINTER(vp)]
    L.dcp_exchange_open.restype = i32
    L.dcp_exchange_close.argtypes = [vp]
    L.dcp_exchange_close.restype = i32
    L.dcp_exchange_free.argtypes = [vp]
    L.dcp_exchange_free.restype = i32
    L.pcp_rank_tokens.argtypes = [i32, i32, i32, vp, i32, ctypes.POINTER(i32)]
    L.pcp_rank_tokens.restype = i32
    L.pcp_gathered_bytes.argtypes = [i32, i32]
    L.pcp_gathered_bytes.restype = sz
    L.pcp_gather_rows.argtypes = [vp, i32, i64, i32, vp, i32, i32, i32, vp, sz, vp, vp]
    L.pcp_gather_rows.restype = i32
    L.pcp_prefill_attention.argtypes = [vp, vp, i32, i32, vp, i32, i64, f32, vp, vp, vp, sz, i32,
                                        i32, vp]
    L.pcp_prefill_attention.restype = i32
    _lib = L
    return L


def error_string(code: int) -> str:
    return lib().dcpmla_error_string(int(code)).decode()


dcpmla_error_string = error_string


def _check(code: int, where: str):
    if code != 0:
        raise DcpMlaError(code, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def padded_heads(num_heads: int) -> int:
    """Query-head envelope of the tensor-core kernel (heads padded to 64 rows).

    Mirrors the fp8 sparse-MLA head envelope ("GLM-5.2 vLLM Decode Context
    Parallelism", "Calculate the GLM-5.2 head envelope"): 8 local or up to 64
    gathered heads all land in the 64-row envelope; more than 64 would need
    the 128 envelope, which this library does not take.
    """
    if num_heads < 1:
        raise ValueError("num_heads must be >= 1")
    return 64 if num_heads <= 64 else 128


def device_sm_count() -> int:
    n = ctypes.c_int(0)
    _check(lib().dcpmla_device_sm_count(ctypes.byref(n)), "dcpmla_device_sm_count")
    return n.value


def mla_decode_workspace_size(batch: int, num_heads: int, num_splits: int = 0,
                              topk: int = 0) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().mla_decode_workspace_size(batch, num_heads, num_splits, topk, ctypes.byref(n)),
           "mla_decode_workspace_size")
    return n.value


def mla_decode_partial(q, kv_cache, kv_dtype, block_table, seq_lens, shard_id, num_shards,
                       sparse_idx, softmax_scale, out_partial, out_lse, workspace,
                       num_splits: int = 0, impl: str | int = "auto", stream=None,
                       block_size: int = BLOCK_SIZE, num_blocks: int | None = None):
    """One shard's partial attention + LSE (see include/dcpmla.h)."""
    B, H = q.shape[0], q.shape[1]
    kvd = KV_DTYPES[kv_dtype] if isinstance(kv_dtype, str) else int(kv_dtype)
    nb = kv_cache.shape[0] if num_blocks is None else num_blocks
    topk = 0 if sparse_idx is None else sparse_idx.shape[1]
    impl_code = IMPLS[impl] if isinstance(impl, str) else int(impl)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = lib().mla_decode_partial(
        _ptr(q), _ptr(kv_cache), kvd, nb, block_size, _ptr(block_table), block_table.shape[-1],
        _ptr(seq_lens), B, H, shard_id, num_shards, _ptr(sparse_idx), topk,
        float(softmax_scale), _ptr(out_partial), _ptr(out_lse), _ptr(workspace), ws_bytes,
        num_splits, impl_code, _stream(stream))
    _check(rc, "mla_decode_partial")


def mla_kv_append(latent, rope, positions, req_idx, block_table, shard_id, num_shards, kv_cache,
                  kv_dtype, flags=None, stream=None, block_size: int = BLOCK_SIZE,
                  num_blocks: int | None = None):
    """This shard's cache write of new tokens (see include/dcpmla.h).

    latent [T, 512] bf16, rope [T, 64] bf16, positions / req_idx [T] int32,
    block_table [B, stride] int32 (this shard's), kv_cache the raw pool;
    ``flags`` an optional one-element int32 device tensor.
    """
    T = latent.shape[0]
    kvd = KV_DTYPES[kv_dtype] if isinstance(kv_dtype, str) else int(kv_dtype)
    nb = kv_cache.shape[0] if num_blocks is None else num_blocks
    rc = lib().mla_kv_append(
        _ptr(latent), _ptr(rope), T, _ptr(positions), _ptr(req_idx), _ptr(block_table),
        block_table.shape[-1], block_table.shape[0], shard_id, num_shards, _ptr(kv_cache), kvd, nb,
        block_size, _ptr(flags), _stream(stream))
    _check(rc, "mla_kv_append")


NOALLOC_SCRATCH_BYTES = 32 << 20          # DCPMLA_NOALLOC_SCRATCH_BYTES


def mla_decode_partial_noalloc(q, kv_cache, kv_dtype, block_table, seq_lens, shard_id,
                               num_shards, sparse_idx, softmax_scale, out_partial, out_lse,
                               out_flags=None, num_splits: int = 0, impl: str | int = "auto",
                               stream=None, block_size: int = BLOCK_SIZE,
                               num_blocks: int | None = None):
    """mla_decode_partial on the library's built-in scratch (see include/dcpmla.h).

    For callers that cannot pass device memory for a workspace.  ``out_flags``
    is an optional one-element int32 device tensor that receives this call's
    flag bits.  Calls whose work overlaps on one device race on the shared
    scratch; the first call on a device does the setup and should come before
    any stream capture.
    """
    B, H = q.shape[0], q.shape[1]
    kvd = KV_DTYPES[kv_dtype] if isinstance(kv_dtype, str) else int(kv_dtype)
    nb = kv_cache.shape[0] if num_blocks is None else num_blocks
    topk = 0 if sparse_idx is None else sparse_idx.shape[1]
    impl_code = IMPLS[impl] if isinstance(impl, str) else int(impl)
    rc = lib().mla_decode_partial_noalloc(
        _ptr(q), _ptr(kv_cache), kvd, nb, block_size, _ptr(block_table), block_table.shape[-1],
        _ptr(seq_lens), B, H, shard_id, num_shards, _ptr(sparse_idx), topk,
        float(softmax_scale), _ptr(out_partial), _ptr(out_lse), _ptr(out_flags),
        num_splits, impl_code, _stream(stream))
    _check(rc, "mla_decode_partial_noalloc")


def mla_decode_partial_multi(q, kv_cache, kv_dtype, block_table, seq_lens, shard_id, num_shards,
                             softmax_scale, out_partial, out_lse, workspace, num_splits: int = 0,
                             impl: str | int = "auto", stream=None, block_size: int = BLOCK_SIZE,
                             num_blocks: int | None = None):
    """One shard's multi-query partials (see include/dcpmla.h): q [B, q_len, H, 576]."""
    B, q_len, H = q.shape[0], q.shape[1], q.shape[2]
    kvd = KV_DTYPES[kv_dtype] if isinstance(kv_dtype, str) else int(kv_dtype)
    nb = kv_cache.shape[0] if num_blocks is None else num_blocks
    impl_code = IMPLS[impl] if isinstance(impl, str) else int(impl)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = lib().mla_decode_partial_multi(
        _ptr(q), _ptr(kv_cache), kvd, nb, block_size, _ptr(block_table), block_table.shape[-1],
        _ptr(seq_lens), B, H, q_len, shard_id, num_shards, float(softmax_scale), _ptr(out_partial),
        _ptr(out_lse), _ptr(workspace), ws_bytes, num_splits, impl_code, _stream(stream))
    _check(rc, "mla_decode_partial_multi")


def dcp_merge(partials, lses, out, out_lse=None, stream=None):
    """LSE-weighted merge of [N, B, H, 512] partials (see include/dcpmla.h)."""
    N, B, H = partials.shape[0], partials.shape[1], partials.shape[2]
    rc = lib().dcp_merge(_ptr(partials), _ptr(lses), N, B, H, _ptr(out), _ptr(out_lse),
                         _stream(stream))
    _check(rc, "dcp_merge")


MAX_MERGE_SHARDS, IPC_HANDLE_BYTES = 64, 64   # DCPMLA_MAX_MERGE_SHARDS, DCPMLA_IPC_HANDLE_BYTES


def _addr(x) -> int:
    return x.data_ptr() if hasattr(x, "data_ptr") else int(x)


def dcp_merge_heads(partials, lses, batch, num_heads, head_begin, head_count, out,
                    out_lse=None, stream=None):
    """Merge of one slice of heads over per-shard buffers (see include/dcpmla.h).

    ``partials`` / ``lses``: one entry per shard, each a tensor or a raw device
    address of that shard's [batch, num_heads, 512] / [batch, num_heads] fp32
    buffer (another rank's, mapped with :func:`dcp_exchange_open`, included).
    ``out`` is [batch, head_count, 512], ``out_lse`` [batch, head_count].
    """
    n = len(partials)
    if len(lses) != n:
        raise ValueError("one LSE buffer per partial buffer")
    po = (ctypes.c_void_p * max(n, 1))(*[_addr(x) for x in partials])
    pl = (ctypes.c_void_p * max(n, 1))(*[_addr(x) for x in lses])
    rc = lib().dcp_merge_heads(po, pl, n, batch, num_heads, head_begin, head_count, _ptr(out),
                               _ptr(out_lse), _stream(stream))
    _check(rc, "dcp_merge_heads")


def dcp_exchange_alloc(nbytes: int) -> tuple[int, bytes]:
    """Device buffer other processes can map: returns (address, IPC handle bytes)."""
    ptr = ctypes.c_void_p(0)
    handle = ctypes.create_string_buffer(IPC_HANDLE_BYTES)
    _check(lib().dcp_exchange_alloc(nbytes, ctypes.byref(ptr), handle), "dcp_exchange_alloc")
    return int(ptr.value), handle.raw


def dcp_exchange_open(handle: bytes) -> int:
    """Map another process's exchange buffer into the current device: its address."""
    if len(handle) != IPC_HANDLE_BYTES:
        raise ValueError(f"an IPC handle has {IPC_HANDLE_BYTES} bytes, got {len(handle)}")
    ptr = ctypes.c_void_p(0)
    buf = ctypes.create_string_buffer(bytes(handle), IPC_HANDLE_BYTES)
    _check(lib().dcp_exchange_open(buf, ctypes.byref(ptr)), "dcp_exchange_open")
    return int(ptr.value)


def dcp_exchange_close(address: int) -> None:
    _check(lib().dcp_exchange_close(ctypes.c_void_p(address)), "dcp_exchange_close")


def dcp_exchange_free(address: int) -> None:
    _check(lib().dcp_exchange_free(ctypes.c_void_p(address)), "dcp_exchange_free")


def pcp_rank_tokens(num_tokens: int, pcp_size: int, rank: int) -> list[int]:
    """Prompt positions of PCP rank ``rank``'s query tokens (see include/dcpmla.h)."""
    n = ctypes.c_int(0)
    _check(lib().pcp_rank_tokens(num_tokens, pcp_size, rank, None, 0, ctypes.byref(n)),
           "pcp_rank_tokens")
    buf = (ctypes.c_int32 * max(1, n.value))()
    _check(lib().pcp_rank_tokens(num_tokens, pcp_size, rank, buf, n.value, ctypes.byref(n)),
           "pcp_rank_tokens")
    return list(buf)[:n.value]


def pcp_gathered_bytes(num_tokens: int, kv_dtype) -> int:
    kvd = KV_DTYPES[kv_dtype] if isinstance(kv_dtype, str) else int(kv_dtype)
    return int(lib().pcp_gathered_bytes(num_tokens, kvd))


def pcp_gather_rows(kv_cache, kv_dtype, block_tables, num_tokens, gathered, flags=None,
                    stream=None, block_size: int = BLOCK_SIZE, num_blocks: int | None = None):
    """One request's prompt rows in token order: block_tables [N, stride] (each shard's
    table row for the request) -> gathered (uint8, pcp_gathered_bytes)."""
    kvd = KV_DTYPES[kv_dtype] if isinstance(kv_dtype, str) else int(kv_dtype)
    nb = kv_cache.shape[0] if num_blocks is None else num_blocks
    nbytes = gathered.numel() * gathered.element_size()
    rc = lib().pcp_gather_rows(_ptr(kv_cache), kvd, nb, block_size, _ptr(block_tables),
                               block_tables.shape[-1], block_tables.shape[0], num_tokens,
                               _ptr(gathered), nbytes, None if flags is None else _ptr(flags),
                               _stream(stream))
    _check(rc, "pcp_gather_rows")


def pcp_prefill_attention(q, positions, gathered, kv_dtype, softmax_scale, out, out_lse,
                          workspace, num_splits: int = 0, impl: str | int = "auto", stream=None,
                          num_gathered_blocks: int | None = None):
    """Causal attention of query tokens q [n, H, 576] at ``positions`` [n] over a
    gathered prompt (see include/dcpmla.h)."""
    kvd = KV_DTYPES[kv_dtype] if isinstance(kv_dtype, str) else int(kv_dtype)
    rb = 656 if kvd == KV_DTYPES["fp8"] else 1152
    nblk = (gathered.numel() * gathered.element_size() // (BLOCK_SIZE * rb)
            if num_gathered_blocks is None else num_gathered_blocks)
    impl_code = IMPLS[impl] if isinstance(impl, str) else int(impl)
    ws_bytes = workspace.numel() * workspace.element_size()
    rc = lib().pcp_prefill_attention(_ptr(q), _ptr(positions), q.shape[0], q.shape[1],
                                     _ptr(gathered), kvd, nblk, float(softmax_scale), _ptr(out),
                                     _ptr(out_lse), _ptr(workspace), ws_bytes, num_splits,
                                     impl_code, _stream(stream))
    _check(rc, "pcp_prefill_attention")


class PcpPrefill:
    """One request's PCP prefill on one GPU: the gathered copy of its prompt
    rows and each rank's causal attention over it (the ranks of a real PCP
    group would each hold the gathered copy; here they run in turn)."""

    def __init__(self, num_tokens: int, num_heads: int, pcp_size: int, kv_dtype: str,
                 device="cuda", num_splits: int = 0, impl: str = "auto"):
        self.num_tokens, self.num_heads, self.pcp_size = num_tokens, num_heads, pcp_size
        self.kv_dtype, self.num_splits, self.impl = kv_dtype, num_splits, impl
        dev = torch.device(device)
        self.gathered = torch.empty(max(16, pcp_gathered_bytes(num_tokens, kv_dtype)),
                                    dtype=torch.uint8, device=dev)
        self.flags = torch.zeros(1, dtype=torch.int32, device=dev)
        self.tokens = [torch.tensor(pcp_rank_tokens(num_tokens, pcp_size, r), dtype=torch.int32,
                                    device=dev) for r in range(pcp_size)]
        most = max(int(t.numel()) for t in self.tokens)
        self.workspace = torch.zeros(mla_decode_workspace_size(max(1, most), num_heads,
                                                               num_splits), dtype=torch.uint8,
                                     device=dev)
        self.out = [torch.empty(int(t.numel()), num_heads, V_DIM, device=dev)
                    for t in self.tokens]
        self.out_lse = [torch.empty(int(t.numel()), num_heads, device=dev) for t in self.tokens]
        self._q = [None] * pcp_size

    def gather(self, kv_cache, block_tables, stream=None):
        """block_tables [N, stride]: each DCP shard's table row for the request."""
        pcp_gather_rows(kv_cache, self.kv_dtype, block_tables, self.num_tokens, self.gathered,
                        self.flags, stream)

    def attend(self, q_prompt, softmax_scale, stream=None):
        """q_prompt [T, H, 576] bf16 (every prompt token's query); every rank's
        share.  Results in ``out[r]`` / ``out_lse[r]``, rows in ``tokens[r]`` order."""
        for r in range(self.pcp_size):
            if self.tokens[r].numel() == 0:
                continue
            if self._q[r] is None or self._q[r].shape[1] != q_prompt.shape[1]:
                self._q[r] = torch.empty(self.tokens[r].numel(), q_prompt.shape[1], HEAD_DIM,
                                         dtype=torch.bfloat16, device=q_prompt.device)
            torch.index_select(q_prompt, 0, self.tokens[r].long(), out=self._q[r])
            pcp_prefill_attention(self._q[r], self.tokens[r], self.gathered, self.kv_dtype,
                                  softmax_scale, self.out[r], self.out_lse[r], self.workspace,
                                  self.num_splits, self.impl, stream)


def check_inputs(block_tables, seq_lens, num_blocks: int, num_shards: int,
                 sparse_idx=None, block_size: int = BLOCK_SIZE) -> None:
    """Debug-mode validation of device contents on the host side.

    The kernels never read outside the cache: an out-of-range table entry or
    length is skipped and reported through a flag bit.  This check finds such
    inputs before a call, with a precise message: block tables [N, B, stride]
    must map every block a shard's local rows use into [0, num_blocks);
    lengths must be >= 0 and fit the table rows; sparse indices must be -1
    (padding) or inside [0, L_b).  Raises ValueError on the first problem.
    """
    import torch
    bt = torch.as_tensor(block_tables)
    lens = torch.as_tensor(seq_lens).to(torch.int64)
    if bt.dim() != 3 or bt.shape[0] != num_shards:
        raise ValueError(f"block_tables must be [num_shards, batch, stride], got {tuple(bt.shape)}")
    N, B, stride = bt.shape
    if lens.shape != (B,):
        raise ValueError(f"seq_lens must be [{B}], got {tuple(lens.shape)}")
    if bool((lens < 0).any()):
        b = int(torch.nonzero(lens < 0)[0, 0])
        raise ValueError(f"seq_lens[{b}] = {int(lens[b])} is negative")
    for s in range(N):
        local = torch.where(lens > s, (lens - s - 1) // N + 1, torch.zeros_like(lens))
        need = (local + block_size - 1) // block_size
        if bool((need > stride).any()):
            b = int(torch.nonzero(need > stride)[0, 0])
            raise ValueError(f"shard {s}, request {b}: {int(local[b])} local rows need "
                             f"{int(need[b])} blocks, the table row has {stride}")
        used = torch.arange(stride, device=bt.device)[None, :] < need.to(bt.device)[:, None]
        bad = used & ((bt[s] < 0) | (bt[s] >= num_blocks))
        if bool(bad.any()):
            b, k = (int(v) for v in torch.nonzero(bad)[0])
            raise ValueError(f"shard {s}, request {b}: block_tables[{s}][{b}][{k}] = "
                             f"{int(bt[s, b, k])} is outside [0, {num_blocks})")
    if sparse_idx is not None:
        idx = torch.as_tensor(sparse_idx).to(torch.int64)
        lim = lens.to(idx.device)[:, None]
        bad = (idx != -1) & ((idx < 0) | (idx >= lim))
        if bool(bad.any()):
            b, i = (int(v) for v in torch.nonzero(bad)[0])
            raise ValueError(f"sparse_idx[{b}][{i}] = {int(idx[b, i])} is neither -1 nor in "
                             f"[0, {int(lens[b])})")


class DcpDecoder:
    """Buffers and calls for whole emulated DCP decode steps on one GPU.

    Holds the outputs ([N, B, H, 512] partials, [N, B, H] LSEs, merged
    [B, H, 512] and [B, H]) and one workspace per shard, so shards issued on
    different streams never share scratch memory.  With ``q_len`` > 1 the
    step is multi-query decode: ``prob.q`` holds [B, q_len * H, 576] rows
    ordered [q_len][H], and the outputs have q_len * H rows in that order.
    """

    def __init__(self, batch, heads, num_shards, topk=0, num_splits=0, device="cuda",
                 impl="auto", streams=None, q_len=1):
        self.batch, self.heads, self.num_shards = batch, heads, num_shards
        self.num_splits, self.impl, self.topk, self.q_len = num_splits, impl, topk, q_len
        rows = heads * q_len                 # multi-query: rows [q_len][heads]
        dev = torch.device(device)
        self.partials = torch.empty(num_shards, batch, rows, V_DIM, device=dev)
        self.lses = torch.empty(num_shards, batch, rows, device=dev)
        self.out = torch.empty(batch, rows, V_DIM, device=dev)
        self.out_lse = torch.empty(batch, rows, device=dev)
        nbytes = mla_decode_workspace_size(batch, rows, num_splits, topk)
        self.workspaces = [torch.zeros(nbytes, dtype=torch.uint8, device=dev)
                           for _ in range(num_shards)]
        self.streams = streams

    def flags(self) -> int:
        """OR of the device flag words of all shard workspaces (syncs)."""
        v = 0
        for w in self.workspaces:
            v |= int(w[:4].view(torch.int32).item())
        return v

    def step(self, prob, stream=None, merge=True):
        """All N shard partials, then the merge, for a DecodeProblem on the GPU."""
        base = torch.cuda.current_stream() if stream is None else stream
        streams = self.streams
        if streams:
            ev = torch.cuda.Event()
            ev.record(base)
        for s in range(self.num_shards):
            st = streams[s % len(streams)] if streams else base
            if streams:
                st.wait_event(ev)
            if self.q_len > 1:
                qv = prob.q.view(self.batch, self.q_len, self.heads, HEAD_DIM)
                mla_decode_partial_multi(qv, prob.kv_cache, prob.kv_dtype, prob.block_tables[s],
                                         prob.seq_lens, s, self.num_shards, prob.softmax_scale,
                                         self.partials[s], self.lses[s], self.workspaces[s],
                                         self.num_splits, self.impl, st, prob.block_size)
            else:
                mla_decode_partial(prob.q, prob.kv_cache, prob.kv_dtype, prob.block_tables[s],
                                   prob.seq_lens, s, self.num_shards, prob.sparse_idx,
                                   prob.softmax_scale, self.partials[s], self.lses[s],
                                   self.workspaces[s], self.num_splits, self.impl, st,
                                   prob.block_size)
        if streams:
            for st in streams:
                e2 = torch.cuda.Event()
                e2.record(st)
                base.wait_event(e2)
        if merge:
            dcp_merge(self.partials, self.lses, self.out, self.out_lse, base)
        return self.out, self.out_lse

    def capture(self, prob, merge=True):
        """Record one whole step (or only the shard partials) into a CUDA graph.

        The graph reads the problem's buffers in place: refill ``prob.q``,
        ``prob.seq_lens``, ``prob.block_tables`` (and ``prob.sparse_idx``) and
        call ``graph.replay()`` for the next step; results land in
        ``self.out`` / ``self.out_lse`` (and ``self.partials`` / ``self.lses``).
        """
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            self.step(prob, side, merge)         # resolve lazy state before capture
        torch.cuda.current_stream().wait_stream(side)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=side):
            self.step(prob, side, merge)
        return g


class _StepInputs:
    """Device copies of one step's inputs, in the attribute form DcpDecoder
    reads; the cache is shared resident state."""

    def __init__(self, prob):
        self.q = prob.q.clone()
        self.kv_cache = prob.kv_cache
        self.kv_dtype = prob.kv_dtype
        self.block_tables = prob.block_tables.clone()
        self.seq_lens = prob.seq_lens.clone()
        self.sparse_idx = None if prob.sparse_idx is None else prob.sparse_idx.clone()
        self.softmax_scale = prob.softmax_scale
        self.block_size = prob.block_size
        self.num_shards = prob.num_shards


class HostPipeline:
    """Whole decode steps fed from host memory, host copies overlapped with
    the compute of the neighbouring steps.

    Two slots, each a DcpDecoder with its own device inputs (q, lengths,
    block tables, sparse lists), outputs and captured step graph; the KV cache
    (``prob.kv_cache``) is shared, resident state.  Step k runs in slot k % 2:

    * its inputs are copied in on the copy-in stream, once the slot's previous
      graph has finished reading them;
    * its graph runs on the compute stream, after that copy and after the
      slot's previous results have been copied out;
    * its merged O and LSE are copied out on the copy-out stream.

    So step k + 1's inputs and step k − 1's results cross PCIe while step k
    computes.  Host buffers should be pinned (``tensor.pin_memory()``) for
    the copies to be asynchronous.  A step's host results are ready once
    ``done_event(k)`` has completed; the host input buffers of step k may be
    reused once ``inputs_copied_event(k)`` has.
    """

    def __init__(self, prob, num_shards=None, topk=0, num_splits=0, impl="auto", streams=None,
                 compute_stream=None):
        n = prob.num_shards if num_shards is None else num_shards
        if prob.q.dim() != 3 or prob.q.shape[1] > MAX_HEADS:
            raise ValueError("HostPipeline runs single-query steps: q must be [B, H <= 64, 576]")
        dev = prob.q.device
        self.compute = compute_stream or torch.cuda.current_stream(dev)
        self.copy_in = torch.cuda.Stream(device=dev)
        self.copy_out = torch.cuda.Stream(device=dev)
        self.slots = []
        for _ in range(2):
            inputs = _StepInputs(prob)
            dec = DcpDecoder(prob.q.shape[0], prob.q.shape[1], n, topk=topk,
                             num_splits=num_splits, device=dev, impl=impl, streams=streams)
            with torch.cuda.stream(self.compute):
                graph = dec.capture(inputs)
            self.slots.append((inputs, dec, graph))
        torch.cuda.synchronize(dev)
        self._in_copied = [None, None]      # per slot: inputs landed (copy-in stream)
        self._computed = [None, None]       # per slot: graph done (compute stream)
        self._out_copied = [None, None]     # per slot: results copied out
        self.k = 0

    def decoder(self, slot: int) -> DcpDecoder:
        return self.slots[slot][1]

    def submit(self, h_q, h_lens, h_tables, h_idx, h_out, h_lse) -> int:
        """Enqueue one step; returns its index k.  ``h_out`` [B, H, 512] and
        ``h_lse`` [B, H] receive the merged results."""
        x = self.k % 2
        inputs, dec, graph = self.slots[x]
        if self._computed[x] is not None:
            self.copy_in.wait_event(self._computed[x])
        with torch.cuda.stream(self.copy_in):
            inputs.q.copy_(h_q, non_blocking=True)
            inputs.seq_lens.copy_(h_lens, non_blocking=True)
            inputs.block_tables.copy_(h_tables, non_blocking=True)
            if h_idx is not None:
                inputs.sparse_idx.copy_(h_idx, non_blocking=True)
        e_in = torch.cuda.Event()
        e_in.record(self.copy_in)
        self._in_copied[x] = e_in
        self.compute.wait_event(e_in)
        if self._out_copied[x] is not None:
            self.compute.wait_event(self._out_copied[x])
        with torch.cuda.stream(self.compute):
            graph.replay()
        e_c = torch.cuda.Event()
        e_c.record(self.compute)
        self._computed[x] = e_c
        self.copy_out.wait_event(e_c)
        with torch.cuda.stream(self.copy_out):
            h_out.copy_(dec.out, non_blocking=True)
            h_lse.copy_(dec.out_lse, non_blocking=True)
        e_o = torch.cuda.Event()
        e_o.record(self.copy_out)
        self._out_copied[x] = e_o
        self.k += 1
        return self.k - 1

    def done_event(self, k: int):
        """Event completing when step k's results are on the host (valid
        until step k + 2 is submitted)."""
        assert k in (self.k - 1, self.k - 2), "only the last two steps are tracked"
        return self._out_copied[k % 2]

    def inputs_copied_event(self, k: int):
        assert k in (self.k - 1, self.k - 2), "only the last two steps are tracked"
        return self._in_copied[k % 2]

    def start_after(self, event) -> None:
        """Make the pipeline's next work (on all three streams) wait for
        ``event`` (e.g. the start event of a timed region)."""
        for s in (self.copy_in, self.compute, self.copy_out):
            s.wait_event(event)

    def join(self, stream=None) -> None:
        """Make ``stream`` (default: the compute stream) wait for every
        submitted step's copies."""
        s = self.compute if stream is None else stream
        for e in self._out_copied + self._in_copied:
            if e is not None:
                s.wait_event(e)

    def flags(self) -> int:
        return self.slots[0][1].flags() | self.slots[1][1].flags()
