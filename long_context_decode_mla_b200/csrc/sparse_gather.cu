// Sparse decode on the tensor-core kernels: each request's index list is
// localised to this shard and compacted, in list order, into the selected
// rows of the cache.  Two outputs:
//  * rows: the flat cache row (block * 64 + row) of every selection, the
//    list padded to whole 64-row tiles with its last entry; the e4m3 kernel
//    fetches these rows itself (TMA gathers and cp.async).  The same launch
//    builds that kernel's Q operand images in CTAs of their own;
//  * gathered: the selected rows copied into a contiguous run of the
//    workspace (tile k of request b is gathered block b * maxblk + k), for
//    the kernels that read whole blocks.
//
// "GLM-5.2 vLLM Decode Context Parallelism", section "Separate the backend
// merge from stable": the global top-K indices are localised to the rank
// that owns each token (t mod N == shard, local row t div N).  Entries
// outside [0, L_b) are skipped, duplicates count as listed.
#include <cstdint>

#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"
#include "q_image.cuh"

namespace dcpmla {
namespace {

constexpr int kGatherThreads = 256;
constexpr int kPerThread = 8;                    // indices per thread and pass
constexpr int kPass = kGatherThreads * kPerThread;

// One CTA per request.  Each pass takes 2,048 indices, 8 consecutive ones per
// thread: their loads, then their table entries, are independent, so a pass
// costs two global round trips; a block scan of the per-thread counts places
// the selections in list order.  kCopy: the CTA's warps copy the selected
// rows, four rows in flight per warp; else the rows' flat indices are
// written to rows[b * maxblk * 64 + slot].
template <bool kCopy>
__global__ void __launch_bounds__(kGatherThreads) sparse_gather_kernel(
    const uint8_t* kv, long long num_blocks, int row_bytes, const int* block_table, int bt_stride,
    const int* seq_lens, const int* idx, int topk, int shard, int nshards, int maxblk,
    uint8_t* gathered, int* rows, int* counts, int* flags, const __nv_bfloat16* q, int rows_q,
    int heads, uint8_t* q_image) {
  __shared__ int warp_sums[kGatherThreads / 32];
  __shared__ long long sel_row[kCopy ? kPass : 1];
  // CTAs past the batch build the e4m3 kernel's Q operand images (two per
  // request, 32 head rows each) alongside the lists, in the same launch
  if (!kCopy && (int)blockIdx.x >= gridDim.x / 3) {
    const int k = blockIdx.x - gridDim.x / 3;
    qimg::build_q_image_row(q, rows_q, heads, k >> 1, (k & 1) * 32 + (threadIdx.x >> 3),
                            threadIdx.x & 7, q_image);
    return;
  }
  const int b = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int kWarps = kGatherThreads / 32;
  int L = __ldg(seq_lens + b);
  if (L < 0) {
    if (threadIdx.x == 0 && flags) atomicOr(flags, kFlagBadLength);
    L = 0;
  }
  const int units = row_bytes / 16;
  int count = 0;
  for (int base = 0; base < topk; base += kPass) {
    const int i0 = base + threadIdx.x * kPerThread;
    int t[kPerThread];
#pragma unroll
    for (int k = 0; k < kPerThread; ++k)
      t[k] = i0 + k < topk ? __ldg(idx + (size_t)b * topk + i0 + k) : -1;
    int blk[kPerThread];
    bool own[kPerThread];
#pragma unroll
    for (int k = 0; k < kPerThread; ++k) {
      own[k] = t[k] >= 0 && t[k] < L && t[k] % nshards == shard;
      const int j = own[k] ? t[k] / nshards : 0;
      if (own[k] && (j >> 6) >= bt_stride) {
        if (flags) atomicOr(flags, kFlagBadLength);
        own[k] = false;
      }
      blk[k] = own[k] ? __ldg(block_table + (size_t)b * bt_stride + (j >> 6)) : 0;
    }
    int n = 0;
#pragma unroll
    for (int k = 0; k < kPerThread; ++k) {
      if (own[k] && (blk[k] < 0 || (long long)blk[k] >= num_blocks)) {
        // flagged and left out: the row is absent, as a bad block's rows
        // are in dense decode
        if (flags) atomicOr(flags, kFlagBadBlock);
        own[k] = false;
      }
      n += own[k] ? 1 : 0;
    }
    int tot;
    int pos = block_exclusive_scan(n, warp_sums, &tot);
    if constexpr (!kCopy) {
      int* out = rows + (size_t)b * maxblk * kBlock + count;
#pragma unroll
      for (int k = 0; k < kPerThread; ++k)
        if (own[k]) out[pos++] = blk[k] * kBlock + ((t[k] / nshards) & 63);
      count += tot;                 // the scan's barriers order the passes
    } else {
#pragma unroll
      for (int k = 0; k < kPerThread; ++k)
        if (own[k]) sel_row[pos++] = (long long)blk[k] * kBlock + ((t[k] / nshards) & 63);
      __syncthreads();
      for (int k0 = warp * 4; k0 < tot; k0 += kWarps * 4) {
        uint4 v[4][2];
        const int nr = min(4, tot - k0);
        // a row is at most 72 units: each lane moves units lane and lane + 32
        // (and lane + 64 for bf16 rows, below)
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const uint4* src = reinterpret_cast<const uint4*>(kv + (size_t)sel_row[k0 + min(r, nr - 1)] * row_bytes);
          v[r][0] = lane < units ? __ldg(src + lane) : make_uint4(0, 0, 0, 0);
          v[r][1] = lane + 32 < units ? __ldg(src + lane + 32) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          if (r >= nr) break;
          const int slot = count + k0 + r;
          uint4* dst = reinterpret_cast<uint4*>(
              gathered + (((size_t)b * maxblk + slot / kBlock) * kBlock + slot % kBlock) * row_bytes);
          if (lane < units) dst[lane] = v[r][0];
          if (lane + 32 < units) dst[lane + 32] = v[r][1];
          if (lane + 64 < units) {
            const uint4* src = reinterpret_cast<const uint4*>(kv + (size_t)sel_row[k0 + r] * row_bytes);
            dst[lane + 64] = __ldg(src + lane + 64);
          }
        }
      }
      count += tot;
      __syncthreads();
    }
  }
  if constexpr (!kCopy) {
    // pad the last tile with the last selection (its rows past the count are
    // cleared and masked by the kernel)
    __syncthreads();
    int* out = rows + (size_t)b * maxblk * kBlock;
    const int pad = (kBlock - count % kBlock) % kBlock;
    if (count > 0 && (int)threadIdx.x < pad) out[count + threadIdx.x] = out[count - 1];
  }
  if (threadIdx.x == 0) counts[b] = count;
}

}  // namespace

cudaError_t launch_sparse_gather(const PartialParams& p, int row_bytes, int maxblk,
                                 uint8_t* gathered, int* counts, cudaStream_t st) {
  sparse_gather_kernel<true><<<p.batch, kGatherThreads, 0, st>>>(
      p.kv, p.num_blocks, row_bytes, p.block_table, p.bt_stride, p.seq_lens, p.sparse_idx,
      p.topk, p.shard, p.nshards, maxblk, gathered, nullptr, counts, p.flags, nullptr, 0, 0,
      nullptr);
  return cudaGetLastError();
}

cudaError_t launch_sparse_rows(const PartialParams& p, int maxblk, int* rows, int* counts,
                               uint8_t* q_image, cudaStream_t st) {
  // grid: batch list CTAs, then 2 x batch Q image CTAs
  sparse_gather_kernel<false><<<3 * p.batch, kGatherThreads, 0, st>>>(
      p.kv, p.num_blocks, 0, p.block_table, p.bt_stride, p.seq_lens, p.sparse_idx, p.topk,
      p.shard, p.nshards, maxblk, nullptr, rows, counts, p.flags, p.q, p.rows_q, p.heads,
      q_image);
  return cudaGetLastError();
}

}  // namespace dcpmla
