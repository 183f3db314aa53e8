"""Real multi-GPU DCP decode: one process per GPU, cache shard r on rank r.

"GLM-5.2 vLLM Decode Context Parallelism", section "Keep the current-main
correctness blocker visible": pure DCP gathers the query heads before
attention and combines the partial output/LSE across ranks after it.  Section
"Separate the backend merge from stable": the combine takes the ag_rs path
(all-gather of the LSEs, reduce-scatter of the rescaled partials), so each
rank ends with the merged result of its own heads.  Section "Calculate the
GLM-5.2 head envelope": a rank holds heads / DCP-size local heads and attends
with all of them gathered (8 local x DCP8 = 64).

One step on rank r of N, in order on the caller's current stream:

1. query all-gather (NCCL): each rank holds its H/N local heads [B, H/N, 576];
   every rank gets the H gathered heads in rank order (gathered head
   r * H/N + i is local head i of rank r);
2. ``mla_decode_partial`` over this rank's shard (tokens t with t mod N == r)
   into this step's slot of the rank's exchange buffer, which the other
   ranks have mapped into their devices (CUDA IPC over NVLink / NVSwitch);
3. a one-integer NCCL all-reduce: a rank passes it only once every rank's
   partial of this step is complete;
4. ``dcp_merge_heads``: the rank reads its H/N heads' LSEs and partials from
   all N slots (its own, and its peers' over NVLink) and merges them -- the
   LSE all-gather, the rescale and the reduce-scatter of ag_rs in one kernel.

Two slots alternate.  A slot is written again two steps later, after the
next step's all-reduce, which no rank passes before every rank has finished
the merge that read the slot; so no buffer is rewritten while a peer reads
it, and no kernel ever waits on another GPU (the only cross-rank waits are
NCCL's).

Everything above the C ABI here is plumbing (collectives, buffer mapping);
the arithmetic runs in libdcpmla.so.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import dcpmla

SLOT_ALIGN = 256


def head_slice(rank: int, world: int, heads: int) -> tuple[int, int]:
    """First gathered head and head count of ``rank``'s local heads."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside a group of {world}")
    if heads < 1 or heads % world:
        raise ValueError(f"{heads} heads do not split evenly over {world} ranks")
    n = heads // world
    return rank * n, n


def slot_layout(batch: int, heads: int) -> tuple[int, int]:
    """(byte offset of the LSEs in a slot, bytes per slot): a slot holds the
    [batch, heads, 512] fp32 partial, then the [batch, heads] fp32 LSEs."""
    rows = batch * heads
    lse_off = rows * dcpmla.V_DIM * 4
    size = lse_off + rows * 4
    return lse_off, (size + SLOT_ALIGN - 1) // SLOT_ALIGN * SLOT_ALIGN


def gather_query_heads(q_local: torch.Tensor, group=None, out: torch.Tensor | None = None):
    """All-gather of the local query heads: [B, H/N, D] on each rank ->
    [B, H, D] on every rank, rank r's heads at [r * H/N, (r + 1) * H/N)."""
    world = dist.get_world_size(group)
    B, hn, D = q_local.shape
    flat = torch.empty(world * B, hn, D, dtype=q_local.dtype, device=q_local.device)
    dist.all_gather_into_tensor(flat, q_local.contiguous(), group=group)
    if out is None:
        out = torch.empty(B, world * hn, D, dtype=q_local.dtype, device=q_local.device)
    out.view(B, world, hn, D).copy_(flat.view(world, B, hn, D).transpose(0, 1))
    return out


def exchange_handles(handle: bytes, group=None) -> list[bytes]:
    """Every rank's exchange-buffer handle, in rank order (host all-gather)."""
    handles = [None] * dist.get_world_size(group)
    dist.all_gather_object(handles, handle, group=group)
    return handles


class _Address:
    """A raw device address where the binding expects a tensor."""

    def __init__(self, addr: int):
        self.addr = addr

    def data_ptr(self) -> int:
        return self.addr


class _ArrayView:
    """``__cuda_array_interface__`` over a raw fp32 device buffer (no copy)."""

    def __init__(self, addr: int, shape):
        self.__cuda_array_interface__ = {"shape": tuple(shape), "typestr": "<f4",
                                         "data": (addr, False), "strides": None, "version": 3}


def device_view(addr: int, shape) -> torch.Tensor:
    """An fp32 tensor of ``shape`` over raw device memory at ``addr`` (no copy;
    the memory must outlive the tensor)."""
    return torch.as_tensor(_ArrayView(addr, shape), device="cuda")


class DcpRankDecoder:
    """This rank's share of a real multi-GPU DCP decode step (see module doc).

    ``group``: the DCP process group (NCCL, one rank per GPU, the current
    device being this rank's, unless ``device`` names another).  ``batch``
    and ``heads`` (gathered heads, a multiple of the group size) fix the
    buffers; ``topk`` > 0 sizes the workspace for sparse decode.  Results of
    :meth:`step` land in ``out`` [batch, H/N, 512] and ``out_lse`` [batch, H/N]
    for this rank's heads.  Call :meth:`close` on every rank before the group
    is destroyed.
    """

    def __init__(self, batch: int, heads: int, group=None, topk: int = 0, num_splits: int = 0,
                 impl: str = "auto", device=None):
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)
        self.batch, self.heads, self.num_splits, self.impl = batch, heads, num_splits, impl
        self.head_begin, self.head_count = head_slice(self.rank, self.world, heads)
        dev = (torch.device("cuda", torch.cuda.current_device()) if device is None
               else torch.device(device))
        self._lse_off, self._slot_bytes = slot_layout(batch, heads)
        self._map_exchange_buffers()
        self.q = torch.empty(batch, heads, dcpmla.HEAD_DIM, dtype=torch.bfloat16, device=dev)
        self.out = torch.empty(batch, self.head_count, dcpmla.V_DIM, device=dev)
        self.out_lse = torch.empty(batch, self.head_count, device=dev)
        nbytes = dcpmla.mla_decode_workspace_size(batch, heads, num_splits, topk)
        self.workspace = torch.zeros(nbytes, dtype=torch.uint8, device=dev)
        self._tick = torch.zeros(1, dtype=torch.int32, device=dev)
        self.steps = 0

    def _map_exchange_buffers(self):
        """Allocate this rank's buffer and map every peer's.  All ranks agree
        on the outcome before returning: if any rank failed (allocation or a
        mapping), every rank unmaps, frees and raises, so none is left
        waiting in a later collective."""
        self._base, self._mapped, self._bases = None, [], []
        err = None
        handle = b""
        try:
            self._base, handle = dcpmla.dcp_exchange_alloc(2 * self._slot_bytes)
        except dcpmla.DcpMlaError as e:
            err = e
        handles = exchange_handles(handle, self.group)
        if err is None and all(handles):
            try:
                for r, h in enumerate(handles):
                    if r == self.rank:
                        self._bases.append(self._base)
                    else:
                        addr = dcpmla.dcp_exchange_open(h)
                        self._mapped.append(addr)
                        self._bases.append(addr)
            except dcpmla.DcpMlaError as e:
                err = e
        oks = [None] * self.world
        dist.all_gather_object(oks, err is None, group=self.group)
        if all(oks):
            return
        for addr in self._mapped:
            dcpmla.dcp_exchange_close(addr)
        self._mapped = []
        done = [None] * self.world
        dist.all_gather_object(done, True, group=self.group)   # every peer has unmapped
        if self._base is not None:
            dcpmla.dcp_exchange_free(self._base)
            self._base = None
        bad = [r for r, ok in enumerate(oks) if not ok]
        raise RuntimeError(f"rank {self.rank}: DCP exchange buffers failed on rank(s) {bad}"
                           + (f": {err}" if err is not None else "")) from err

    def slot(self, rank: int, parity: int) -> tuple[int, int]:
        """Device addresses (partial, LSEs) of ``rank``'s slot ``parity``."""
        o = self._bases[rank] + parity * self._slot_bytes
        return o, o + self._lse_off

    def partial(self, parity: int | None = None):
        """This rank's partial and LSEs of a slot (default: the last step's), as
        tensors viewing the exchange buffer."""
        if parity is None:
            parity = (self.steps - 1) & 1
        o, l = self.slot(self.rank, parity)
        B, H = self.batch, self.heads
        return device_view(o, (B, H, dcpmla.V_DIM)), device_view(l, (B, H))

    def flags(self) -> int:
        """The partial workspace's device flag word (syncs)."""
        return int(self.workspace[:4].view(torch.int32).item())

    def step(self, q_local, kv_cache, kv_dtype, block_table, seq_lens, softmax_scale,
             sparse_idx=None, block_size: int = dcpmla.BLOCK_SIZE):
        """One decode step: ``q_local`` [B, H/N, 576] bf16 (this rank's heads),
        ``kv_cache`` / ``block_table`` this rank's shard, ``seq_lens`` [B] and
        ``sparse_idx`` [B, topk] (global positions) the same on every rank."""
        gather_query_heads(q_local, self.group, out=self.q)
        parity = self.steps & 1
        o, l = self.slot(self.rank, parity)
        dcpmla.mla_decode_partial(self.q, kv_cache, kv_dtype, block_table, seq_lens, self.rank,
                                  self.world, sparse_idx, softmax_scale, _Address(o), _Address(l),
                                  self.workspace, self.num_splits, self.impl, None, block_size)
        dist.all_reduce(self._tick, group=self.group)
        slots = [self.slot(r, parity) for r in range(self.world)]
        dcpmla.dcp_merge_heads([s[0] for s in slots], [s[1] for s in slots], self.batch,
                               self.heads, self.head_begin, self.head_count, self.out,
                               self.out_lse)
        self.steps += 1
        return self.out, self.out_lse

    def _sync(self):
        if self.q.is_cuda:
            torch.cuda.synchronize(self.q.device)

    def close(self):
        """Unmap the peers' buffers and free this rank's, once no rank reads it."""
        if self._base is None:
            return
        self._sync()
        for addr in self._mapped:
            dcpmla.dcp_exchange_close(addr)
        self._mapped = []
        dist.all_reduce(self._tick, group=self.group)      # every rank is done reading
        self._sync()
        dcpmla.dcp_exchange_free(self._base)
        self._base = None
