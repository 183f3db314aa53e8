// Shared device-side pieces of the DCP MLA decode kernels: parameters, the
// round-robin shard arithmetic, the split-KV work schedule and the workspace
// layout.  Everything here is plain integer bookkeeping; the attention math
// lives in the kernels themselves.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace dcpmla {

constexpr int kHeadDim = 576;     // 512 latent + 64 rope
constexpr int kVDim = 512;
constexpr int kRopeDim = 64;
constexpr int kBlock = 64;        // rows per cache block
constexpr int kMaxHeads = 64;
constexpr int kMaxRequestsPerCta = 32;   // request-aligned schedule: requests a CTA takes
constexpr int kMaxQueryLen = 64;   // query tokens per request of a multi-query call
constexpr int kRowBytesBf16 = 1152;
constexpr int kRowBytesFp8 = 656;
// Q operand image of one request for the e4m3 kernel: the e4m3 hi and lo
// codes of the latent (2 x 4 chunks of 64 rows x 128 B), the bf16 rope
// (64 rows x 128 B), each in the kernel's 128-byte-swizzled shared-memory
// order, then the 64 per-head frame factors 2^-a (fp32).
constexpr int kQImageBytes = 2 * 4 * 8192 + 8192 + 64 * 4;
constexpr int kWsHeader = 256;    // workspace header: flag word + reserved
constexpr int kMaxDevicesConfigured = 64;   // device ordinals the per-device caches cover

enum : int { kKvBf16 = 0, kKvFp8 = 1 };
enum : int { kFlagBadBlock = 1, kFlagBadLength = 2 };

// Everything one shard's partial-attention launch needs.
struct PartialParams {
  const __nv_bfloat16* q;     // [B][rows_q][576], the first `heads` rows of each request;
                              // multi-query: query-major rows (query i, head h)
  const uint8_t* kv;          // [num_blocks][64][row_bytes]
  long long num_blocks;
  const int* block_table;     // [B][bt_stride] this shard's table; nullptr: request b's
                              // tile k is block b * id_stride + k of the pool (rows that
                              // were gathered in order: a prompt, or sparse selections)
  int bt_stride;
  int id_stride;
  const int* seq_lens;        // [B] global lengths
  int batch;
  int heads;                  // rows per request in this pass: query heads x q_len (<= 64)
  int q_len;                  // query tokens per request (1 = plain decode); row r is
                              // query r / (heads / q_len), causal at L_b - q_len + that
  int shard;
  int nshards;
  const int* sparse_idx;      // [B][topk] or nullptr
  int topk;
  int sparse_parts;           // index-list chunks per request (sparse mode)
  float scale;                // softmax scale
  float* out;                 // [B][rows_o][512] (the first `heads` rows of each request)
  float* out_lse;             // [B][rows_o]
  int rows_q;                 // rows between consecutive requests in q (>= heads)
  int rows_o;                 // rows between consecutive requests in out / out_lse
  int len_delta;              // subtracted from every valid length: a multi-query pass
                              // that ends len_delta tokens before the request's end; -1
                              // for prefill queries, whose "length" is their position
  int* flags;                 // workspace flag word
  float* ws_o;                // [slots][H][512]
  float* ws_lse;              // [slots][H]
  int* ws_list;               // sparse mode: per-CTA lists of selected local rows
  int num_ctas;               // G: CTAs sharing the dense tile space
  uint8_t* q_image;           // e4m3 kernel: per-request Q operand images (workspace)
  int q_image_ready;          // 1: an earlier launch of the call built them
  const int* row_ids;         // e4m3 kernel, sparse: per-request flat cache rows (padded
                              // to whole tiles); tile k of request b is rows
                              // [b * row_stride + 64 k, + 64) of the list
  int row_stride;
  int request_aligned;        // 1: CTA c takes requests [c B / G, (c+1) B / G) whole (no splits)
  int test_withhold;          // test only: converters skip their first arrival (timeout path)
};

// Number of tokens t in [0, L) with t mod N == s (round-robin ownership).
__host__ __device__ __forceinline__ int local_len(int L, int s, int N) {
  return L > s ? (L - s - 1) / N + 1 : 0;
}

// Dense schedule.  The local tokens of all requests are cut into 64-row tiles
// (one cache block each) and laid end to end; CTA c owns the tiles
// [c * tpc, (c + 1) * tpc) with tpc = ceil(T / G).  A CTA that covers part of
// request b writes its partial result to workspace slot c + b: along the tile
// order both c and b never decrease and at least one grows from one segment
// to the next, so c + b is distinct for every (CTA, request) segment, and
// fewer than G + B slots are used.

// Tiles of request b on this shard, with the range checks on the length and
// on the block-table row; sets flag bits instead of reading out of range.
// Length request b is attended over: its cached length, less len_delta (a
// negative length stays negative: it is flagged by the callers).
__device__ __forceinline__ int seq_len_of(const PartialParams& p, int b) {
  const int L = __ldg(p.seq_lens + b);
  return L < 0 ? L : max(L - p.len_delta, 0);
}

__device__ __forceinline__ int request_tiles(const PartialParams& p, int b, int* n_rows) {
  int L = seq_len_of(p, b);
  if (L < 0) {
    if (p.flags) atomicOr(p.flags, kFlagBadLength);
    L = 0;
  }
  int n = local_len(L, p.shard, p.nshards);
  int nt = (n + kBlock - 1) / kBlock;
  if (nt > p.bt_stride) {
    if (p.flags) atomicOr(p.flags, kFlagBadLength);
    nt = p.bt_stride;
    n = nt * kBlock;
  }
  *n_rows = n;
  return nt;
}

// Block-wide exclusive scan of one int per thread (blockDim.x a multiple of
// 32, at most 1024).  `warp_sums` needs blockDim.x / 32 ints of shared memory.
__device__ __forceinline__ int block_exclusive_scan(int v, int* warp_sums, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nwarps = blockDim.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sums[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = lane < nwarps ? warp_sums[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    if (lane < nwarps) warp_sums[lane] = w;   // inclusive warp prefix
  }
  __syncthreads();
  int before = (warp > 0 ? warp_sums[warp - 1] : 0) + x - v;
  *total = warp_sums[nwarps - 1];
  __syncthreads();
  return before;
}

// Total number of dense tiles over all requests (every thread gets it).
__device__ __forceinline__ int total_tiles(const PartialParams& p, int* warp_sums) {
  int acc = 0;
  for (int base = 0; base < p.batch; base += blockDim.x) {
    int b = base + threadIdx.x;
    int n, nt = 0;
    if (b < p.batch) nt = request_tiles(p, b, &n);
    int tot;
    block_exclusive_scan(nt, warp_sums, &tot);
    acc += tot;
  }
  return acc;
}

// Request-aligned schedule: CTA c of G = num_ctas takes the whole requests
// [c B / G, (c+1) B / G) and covers their tiles [lo, hi) of the request-major
// tile order (all threads of the block call it).  Requests of the range with
// no tile on this shard are marked in *empty_mask (bit r - r0; at most 32
// requests a CTA).
__device__ __forceinline__ void request_range_tiles(const PartialParams& p, int* warp_sums,
                                                    int* r0_out, int* lo, int* hi,
                                                    uint32_t* empty_mask) {
  const int r0 = (int)(((long long)blockIdx.x * p.batch) / p.num_ctas);
  const int r1 = (int)(((long long)(blockIdx.x + 1) * p.batch) / p.num_ctas);
  __shared__ int range[2];
  __shared__ uint32_t empties;
  if (threadIdx.x == 0) empties = 0u;
  __syncthreads();
  int acc = 0;
  for (int base = 0; base < p.batch; base += blockDim.x) {
    const int b = base + threadIdx.x;
    int n, nt = 0;
    if (b < p.batch) nt = request_tiles(p, b, &n);
    int tot;
    const int pre = acc + block_exclusive_scan(nt, warp_sums, &tot);
    if (b == r0) range[0] = pre;
    if (b == r1 - 1) range[1] = pre + nt;
    if (b >= r0 && b < r1 && nt == 0) atomicOr(&empties, 1u << (b - r0));
    acc += tot;
  }
  __syncthreads();
  *r0_out = r0;
  *lo = r1 > r0 ? range[0] : 0;
  *hi = r1 > r0 ? range[1] : 0;
  *empty_mask = empties;
}

struct Segment {
  int b;          // request
  int t0, t1;     // tile range within the request
  int n_rows;     // local rows of the request
  int nt;         // tiles of the request
};

}  // namespace dcpmla

namespace dcpmla {

// Calls f(seg) for every request whose dense tiles meet [lo, hi), with the
// tile range clipped to it.  Requests are visited blockDim.x at a time; `list`
// needs blockDim.x Segments of shared memory, `list_n` one int, `warp_sums`
// blockDim.x / 32 ints.  All threads of the block must call it; f is called
// by all threads with the same argument and may synchronise.
template <class F>
__device__ __forceinline__ void for_each_dense_segment(const PartialParams& p, int lo, int hi,
                                                       int* warp_sums, Segment* list,
                                                       int* list_n, F&& f) {
  int off = 0;
  for (int base = 0; base < p.batch && off < hi; base += blockDim.x) {
    const int b = base + threadIdx.x;
    int n = 0, nt = 0;
    if (b < p.batch) nt = request_tiles(p, b, &n);
    int tot;
    const int start = off + block_exclusive_scan(nt, warp_sums, &tot);
    if (threadIdx.x == 0) *list_n = 0;
    __syncthreads();
    if (nt > 0 && start < hi && start + nt > lo) {
      int k = atomicAdd(list_n, 1);
      Segment s;
      s.b = b;
      s.t0 = max(lo, start) - start;
      s.t1 = min(hi, start + nt) - start;
      s.n_rows = n;
      s.nt = nt;
      list[k] = s;
    }
    __syncthreads();
    const int cnt = *list_n;
    for (int k = 0; k < cnt; ++k) {
      Segment s = list[k];
      f(s);
    }
    __syncthreads();
    off += tot;
  }
}

// Physical block of local tile `tile` of request b, or -1 (flagged) if the
// table entry is outside the pool.
__device__ __forceinline__ int tile_block(const PartialParams& p, int b, int tile) {
  int blk = p.block_table ? __ldg(p.block_table + (size_t)b * p.bt_stride + tile)
                          : b * p.id_stride + tile;
  if (blk < 0 || (long long)blk >= p.num_blocks) {
    if (p.flags) atomicOr(p.flags, kFlagBadBlock);
    return -1;
  }
  return blk;
}

// Slot arrays of the workspace for `slots` slots of H heads.
__host__ __device__ __forceinline__ size_t ws_o_offset() { return kWsHeader; }
__host__ __device__ __forceinline__ size_t ws_lse_offset(long long slots, int heads) {
  return kWsHeader + (size_t)slots * heads * kVDim * sizeof(float);
}
__host__ __device__ __forceinline__ size_t ws_list_offset(long long slots, int heads) {
  size_t lse_bytes = ((size_t)slots * heads * sizeof(float) + 255) & ~(size_t)255;
  return ws_lse_offset(slots, heads) + lse_bytes;
}
// `list_ints` = CTAs x index-list chunk for sparse mode, 0 for dense.
__host__ __device__ __forceinline__ size_t ws_total(long long slots, int heads,
                                                   long long list_ints = 0) {
  return ws_list_offset(slots, heads) + (((size_t)list_ints * sizeof(int) + 255) & ~(size_t)255);
}

}  // namespace dcpmla
