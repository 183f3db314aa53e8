"""Seeded synthetic inputs for DCP MLA decode.

This module only draws random numbers and packs them into the byte layouts
the decode path reads.  It holds no attention arithmetic and is the one piece
of code shared by the tests, the smoke check and the benchmark (the CUDA path
and the CPU oracle each read what it produces, never each other's results).

Workloads (the shapes the pages' serving discussion implies; no public trace
or checkpoint is available, so every input is synthetic):

* ``tiny``     - batch 1, 8 heads, 1,024 cached bf16 tokens, 2 shards.
* ``dense``    - batch 32, 64 heads, 8,192 bf16 tokens each, 8 shards.
* ``agentic``  - batch 64, 64 heads, fp8 rows, lengths lognormal with median
  67,000 (sigma 1 in log space) clipped to [4,096, 200,000], 8 shards: the
  length mix of the agentic trace described in "The 3.3x Belongs to the
  Model, Not the Flag" (median input near 67K, sequences past 200K, 8K at the
  bottom of the distribution).
* ``million``  - batch 1, 64 heads, 1,048,576 fp8 tokens, 8 shards ("How vLLM
  Serves GLM-5.3 with Million-Token Contexts on 16 H200s", "The core design").
* ``sparse``   - batch 128, 64 heads, 131,072 fp8 tokens, a top-2,048 index
  list per request drawn uniformly without replacement, 8 shards (top-K 2,048
  from "GLM-5.2 vLLM Decode Context Parallelism", "Understand the cache-copy
  opportunity").

Cache layouts (the readings used throughout the package):

* bf16 row: 576 bf16 values (512 latent + 64 rope) = 1,152 bytes.
* fp8 row: 512 E4M3 codes, 4 little-endian fp32 scales (one per 128 latent
  values, scale = amax / 448, 1.0 for an all-zero group), 64 bf16 rope values
  = 656 bytes.
* Paged: a pool of blocks of 64 rows.  Every shard has its own block table
  over its local token index j; token t of a request lives on shard t mod N at
  local index t div N.  All shards' blocks sit disjoint in one pool, placed by
  a seeded random permutation.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

LATENT_DIM = 512
ROPE_DIM = 64
ROW_DIM = 576
BLOCK_SIZE = 64
ROW_BYTES = {"bf16": 1152, "fp8": 656}
SOFTMAX_SCALE = 192 ** -0.5
FP8_MAX = 448.0

CONFIGS = {
    "tiny": dict(batch=1, heads=8, seq_len=1024, kv_dtype="bf16", num_shards=2, seed=1001),
    "dense": dict(batch=32, heads=64, seq_len=8192, kv_dtype="bf16", num_shards=8, seed=1002),
    "agentic": dict(batch=64, heads=64, seq_len="lognormal", kv_dtype="fp8", num_shards=8,
                    seed=1003),
    "million": dict(batch=1, heads=64, seq_len=1 << 20, kv_dtype="fp8", num_shards=8, seed=1004),
    "sparse": dict(batch=128, heads=64, seq_len=131072, kv_dtype="fp8", num_shards=8,
                   topk=2048, seed=1005),
    # the agentic shape with every request at exactly 64K tokens ("steps/s at 64K")
    "agentic64k": dict(batch=64, heads=64, seq_len=65536, kv_dtype="fp8", num_shards=8,
                       seed=1006),
}

LOGNORMAL_MEDIAN = 67000
LOGNORMAL_SIGMA = 1.0
LOGNORMAL_CLIP = (4096, 200000)


@dataclass
class DecodeProblem:
    """One batch of decode inputs laid out for N shards."""
    q: torch.Tensor                 # [B, H, 576] bf16
    kv_cache: torch.Tensor          # uint8 [num_blocks, 64, row_bytes]
    kv_dtype: str                   # "bf16" | "fp8"
    block_tables: torch.Tensor      # int32 [N, B, max_blocks]
    seq_lens: torch.Tensor          # int32 [B] global lengths
    num_shards: int
    softmax_scale: float = SOFTMAX_SCALE
    sparse_idx: torch.Tensor | None = None   # int32 [B, topk] or None
    block_size: int = BLOCK_SIZE
    meta: dict = field(default_factory=dict)

    @property
    def batch(self) -> int:
        return self.q.shape[0]

    @property
    def heads(self) -> int:
        return self.q.shape[1]

    def to(self, device) -> "DecodeProblem":
        mv = lambda t: None if t is None else t.to(device)  # noqa: E731
        return DecodeProblem(mv(self.q), mv(self.kv_cache), self.kv_dtype, mv(self.block_tables),
                             mv(self.seq_lens), self.num_shards, self.softmax_scale,
                             mv(self.sparse_idx), self.block_size, dict(self.meta))

    def numpy_inputs(self) -> dict:
        """The same bytes as numpy arrays (bf16 as uint16 bit patterns)."""
        c = lambda t: None if t is None else t.detach().cpu()  # noqa: E731
        return dict(
            q=c(self.q).view(torch.int16).numpy().view("uint16"),
            kv_cache=c(self.kv_cache).numpy(),
            kv_dtype=self.kv_dtype,
            block_tables=c(self.block_tables).numpy(),
            seq_lens=c(self.seq_lens).numpy(),
            num_shards=self.num_shards,
            softmax_scale=self.softmax_scale,
            sparse_idx=None if self.sparse_idx is None else c(self.sparse_idx).numpy(),
            block_size=self.block_size,
        )


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def lognormal_lengths(batch: int, seed: int) -> torch.Tensor:
    """Lengths lognormal(ln 67,000, 1.0), rounded, clipped to [4,096, 200,000]."""
    g = _gen(seed, "cpu")
    z = torch.randn(batch, generator=g, dtype=torch.float64)
    L = torch.exp(math.log(LOGNORMAL_MEDIAN) + LOGNORMAL_SIGMA * z).round()
    return L.clamp(*LOGNORMAL_CLIP).to(torch.int32)


def blocks_per_shard(seq_len: int, num_shards: int, block_size: int = BLOCK_SIZE) -> int:
    """Blocks reserved for one request on every shard: room for ceil(L/N) rows."""
    return -(-(-(-seq_len // num_shards)) // block_size)


def shard_block_tables(seq_lens, num_shards: int, seed: int, block_size: int = BLOCK_SIZE):
    """Per-shard block tables over one pool, physical order a seeded permutation.

    Returns (tables int32 [N, B, max_blocks], num_blocks).  Unused entries are 0.
    """
    lens = [int(x) for x in seq_lens]
    per = [blocks_per_shard(L, num_shards, block_size) for L in lens]
    max_blocks = max(1, max(per) if per else 1)
    total = num_shards * sum(per)
    perm = torch.randperm(max(total, 1), generator=_gen(seed + 7, "cpu")).to(torch.int32)
    tables = torch.zeros(num_shards, len(lens), max_blocks, dtype=torch.int32)
    k = 0
    for s in range(num_shards):
        for b, nb in enumerate(per):
            tables[s, b, :nb] = perm[k:k + nb]
            k += nb
    return tables, max(total, 1)


def pack_fp8_rows(latent: torch.Tensor, rope: torch.Tensor) -> torch.Tensor:
    """Quantise latent fp32 [n, 512] per 128-value group and pack 656-byte rows."""
    n = latent.shape[0]
    grp = latent.view(n, 4, 128).float()
    amax = grp.abs().amax(dim=2)
    scale = torch.where(amax > 0, amax / FP8_MAX, torch.ones_like(amax))
    codes = (grp / scale[:, :, None]).clamp(-FP8_MAX, FP8_MAX).to(torch.float8_e4m3fn)
    out = torch.empty(n, ROW_BYTES["fp8"], dtype=torch.uint8, device=latent.device)
    out[:, :512] = codes.view(n, 512).view(torch.uint8)
    out[:, 512:528] = scale.contiguous().view(torch.uint8).view(n, 16)
    out[:, 528:] = rope.to(torch.bfloat16).contiguous().view(torch.uint8).view(n, 128)
    return out


def random_kv_pool(num_blocks: int, kv_dtype: str, seed: int, device="cpu",
                   block_size: int = BLOCK_SIZE, chunk_rows: int = 1 << 18,
                   out: torch.Tensor | None = None) -> torch.Tensor:
    """Pool of i.i.d. N(0,1) rows in the requested byte layout."""
    rows = num_blocks * block_size
    rb = ROW_BYTES[kv_dtype]
    if out is None:
        out = torch.empty(num_blocks, block_size, rb, dtype=torch.uint8, device=device)
    flat = out.view(rows, rb)
    g = _gen(seed, device)
    for r0 in range(0, rows, chunk_rows):
        n = min(chunk_rows, rows - r0)
        if kv_dtype == "bf16":
            x = torch.randn(n, ROW_DIM, generator=g, device=device).to(torch.bfloat16)
            flat[r0:r0 + n] = x.view(torch.uint8).view(n, rb)
        else:
            x = torch.randn(n, ROW_DIM, generator=g, device=device)
            flat[r0:r0 + n] = pack_fp8_rows(x[:, :512], x[:, 512:])
    return out


def random_q(batch: int, heads: int, seed: int, device="cpu") -> torch.Tensor:
    g = _gen(seed + 3, device)
    return torch.randn(batch, heads, ROW_DIM, generator=g, device=device).to(torch.bfloat16)


def sparse_indices(seq_lens, topk: int, seed: int) -> torch.Tensor:
    """Per request, ``topk`` distinct positions drawn uniformly from [0, L_b); -1 pads."""
    g = _gen(seed + 11, "cpu")
    lens = [int(x) for x in seq_lens]
    idx = torch.full((len(lens), topk), -1, dtype=torch.int32)
    for b, L in enumerate(lens):
        k = min(topk, L)
        idx[b, :k] = torch.randperm(L, generator=g)[:k].to(torch.int32)
    return idx


def make_problem(name: str, num_shards: int | None = None, device="cpu", kv_device=None,
                 **overrides) -> DecodeProblem:
    """Build the named workload (optionally overriding batch/heads/seq_len/...).

    ``kv_device`` is where the (possibly large) cache is drawn; it defaults to
    ``device``.  Everything small is drawn on the CPU so that it is identical
    wherever the cache lives.
    """
    cfg = dict(CONFIGS[name])
    cfg.update(overrides)
    if num_shards is not None:
        cfg["num_shards"] = num_shards
    B, H, N, seed = cfg["batch"], cfg["heads"], cfg["num_shards"], cfg["seed"]
    if cfg["seq_len"] == "lognormal":
        seq_lens = lognormal_lengths(B, seed)
    elif isinstance(cfg["seq_len"], (list, tuple, torch.Tensor)):
        seq_lens = torch.as_tensor(cfg["seq_len"], dtype=torch.int32)
    else:
        seq_lens = torch.full((B,), int(cfg["seq_len"]), dtype=torch.int32)
    tables, num_blocks = shard_block_tables(seq_lens, N, seed)
    kv_device = kv_device or device
    kv = random_kv_pool(num_blocks, cfg["kv_dtype"], seed, device=kv_device)
    q = random_q(B, H, seed)
    sp = sparse_indices(seq_lens, cfg["topk"], seed) if cfg.get("topk") else None
    prob = DecodeProblem(q, kv, cfg["kv_dtype"], tables, seq_lens, N, sparse_idx=sp,
                         meta=dict(name=name, seed=seed))
    return prob.to(device)


# ------------------------------------------------------- addressing inputs --

ID_BITS = 21


def place_rows(rows_per_request, num_shards: int, kv_dtype: str, seed: int = 0) -> tuple:
    """Write given logical rows into a paged per-shard cache.

    ``rows_per_request[b]`` is uint8 [L_b, row_bytes] in token order.  Token t
    goes to shard t mod N at local index t div N, through that shard's
    (randomly permuted) block table.  Returns (cache, tables, seq_lens).
    """
    seq_lens = torch.tensor([r.shape[0] for r in rows_per_request], dtype=torch.int32)
    tables, num_blocks = shard_block_tables(seq_lens, num_shards, seed + 101)
    rb = ROW_BYTES[kv_dtype]
    cache = torch.zeros(num_blocks, BLOCK_SIZE, rb, dtype=torch.uint8)
    for b, rows in enumerate(rows_per_request):
        L = rows.shape[0]
        if L == 0:
            continue
        t = torch.arange(L)
        s, j = t % num_shards, t // num_shards
        blk = tables[s, b, j // BLOCK_SIZE].long()
        cache[blk, (j % BLOCK_SIZE).long()] = rows
    return cache, tables, seq_lens


def random_logical_rows(seq_lens, kv_dtype: str, seed: int) -> list:
    """I.i.d. N(0,1) rows per request, in token order, packed in the row layout."""
    g = _gen(seed, "cpu")
    out = []
    for L in seq_lens:
        x = torch.randn(int(L), ROW_DIM, generator=g)
        if kv_dtype == "bf16":
            out.append(x.to(torch.bfloat16).view(torch.uint8).view(int(L), ROW_BYTES["bf16"]))
        else:
            out.append(pack_fp8_rows(x[:, :512], x[:, 512:]))
    return out


def logical_problem(seq_lens, num_shards: int, kv_dtype: str, heads: int, seed: int,
                    sparse_idx=None):
    """Random problem that also returns its logical rows: (problem, rows_per_request)."""
    rows = random_logical_rows(seq_lens, kv_dtype, seed)
    cache, tables, lens = place_rows(rows, num_shards, kv_dtype, seed)
    q = random_q(len(rows), heads, seed)
    sp = None if sparse_idx is None else torch.as_tensor(sparse_idx, dtype=torch.int32)
    prob = DecodeProblem(q, cache, kv_dtype, tables, lens, num_shards, sparse_idx=sp,
                         meta=dict(name="logical", seed=seed))
    return prob, rows


def id_coded_rows(seq_len: int, kv_dtype: str) -> torch.Tensor:
    """Rows whose latent value d < 21 is bit d of the token id; all else 0.

    fp8 scales are 1.0, so the code of 1.0 is stored where a bit is set.
    """
    rb = ROW_BYTES[kv_dtype]
    rows = torch.zeros(seq_len, rb, dtype=torch.uint8)
    t = torch.arange(seq_len)
    on = ((t[:, None] >> torch.arange(ID_BITS)[None, :]) & 1).bool()
    if kv_dtype == "bf16":
        one = torch.tensor([1.0], dtype=torch.bfloat16).view(torch.uint8)
        for d in range(ID_BITS):
            rows[on[:, d], 2 * d:2 * d + 2] = one
    else:
        one = torch.tensor([1.0]).to(torch.float8_e4m3fn).view(torch.uint8)[0]
        rows[:, 512:528] = torch.tensor([1.0] * 4, dtype=torch.float32).view(torch.uint8)
        for d in range(ID_BITS):
            rows[on[:, d], d] = one
    return rows


def id_coded_problem_device(seq_lens, num_shards: int, kv_dtype: str, heads: int = 64,
                            seed: int = 0, device="cuda") -> DecodeProblem:
    """id_coded_problem built directly on a device, for full-size caches.

    Same rows and placement as ``id_coded_problem`` (token t of request b at
    block tables[t mod N, b, (t div N) div 64], row (t div N) mod 64), made
    with vectorised tensor operations instead of per-request host copies.
    """
    lens = torch.as_tensor([int(x) for x in seq_lens], dtype=torch.int32)
    tables, num_blocks = shard_block_tables(lens, num_shards, seed + 101)
    rb = ROW_BYTES[kv_dtype]
    dev = torch.device(device)
    cache = torch.zeros(num_blocks, BLOCK_SIZE, rb, dtype=torch.uint8, device=dev)
    flat = cache.view(-1, rb)
    tab = tables.to(dev)
    bits = torch.arange(ID_BITS, device=dev)
    if kv_dtype == "bf16":
        one = torch.tensor([1.0], dtype=torch.bfloat16).view(torch.uint8).to(dev)
    else:
        one = torch.tensor([1.0]).to(torch.float8_e4m3fn).view(torch.uint8).to(dev)
        scales = torch.tensor([1.0] * 4, dtype=torch.float32).view(torch.uint8).to(dev)
    chunk = 1 << 20
    for b, L in enumerate(lens.tolist()):
        for t0 in range(0, L, chunk):
            t = torch.arange(t0, min(L, t0 + chunk), device=dev)
            s, j = t % num_shards, t // num_shards
            blk = tab[s, b, j // BLOCK_SIZE].long()
            dst = blk * BLOCK_SIZE + (j % BLOCK_SIZE)
            on = ((t[:, None] >> bits[None, :]) & 1).bool()
            rows = torch.zeros(t.numel(), rb, dtype=torch.uint8, device=dev)
            if kv_dtype == "bf16":
                for d in range(ID_BITS):
                    rows[on[:, d], 2 * d:2 * d + 2] = one
            else:
                rows[:, 512:528] = scales
                for d in range(ID_BITS):
                    rows[on[:, d], d] = one[0]
            flat[dst] = rows
    q = torch.zeros(len(lens), heads, ROW_DIM, dtype=torch.bfloat16, device=dev)
    return DecodeProblem(q, cache, kv_dtype, tab, lens.to(dev), num_shards,
                         meta=dict(name="id_coded"))


def id_coded_problem(seq_lens, num_shards: int, kv_dtype: str, heads: int = 8, seed: int = 0,
                     sparse_idx=None) -> DecodeProblem:
    """Cache whose row for global token t carries t in binary (exact addressing tests).

    The query is all zeros, so every selected row gets the same weight: the
    LSE of a shard is ln(count) and count * O[d] is the number of selected
    ids with bit d set.
    """
    rows = [id_coded_rows(int(L), kv_dtype) for L in seq_lens]
    cache, tables, lens = place_rows(rows, num_shards, kv_dtype, seed)
    q = torch.zeros(len(rows), heads, ROW_DIM, dtype=torch.bfloat16)
    sp = None if sparse_idx is None else torch.as_tensor(sparse_idx, dtype=torch.int32)
    return DecodeProblem(q, cache, kv_dtype, tables, lens, num_shards, sparse_idx=sp,
                         meta=dict(name="id_coded"))
