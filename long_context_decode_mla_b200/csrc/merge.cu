// LSE-weighted merges: the cross-shard DCP merge and the combine of split-KV
// pieces inside one shard (the formula of merge_rows.cuh applied one level
// down).
#include "common.cuh"
#include "kernels.h"
#include "merge_rows.cuh"

#include <math_constants.h>

namespace dcpmla {
namespace {

constexpr int kMergeWarps = 8;

__global__ void __launch_bounds__(kMergeWarps * 32) dcp_merge_kernel(
    const float* __restrict__ partials, const float* __restrict__ lses, int nshards, int rows,
    float* __restrict__ out, float* __restrict__ out_lse) {
  const int row = blockIdx.x * kMergeWarps + (threadIdx.x >> 5);
  if (row >= rows) return;
  merge_warp(StridedPieces{partials, lses, (size_t)row, (size_t)rows}, nshards,
             out + (size_t)row * kVDim, out_lse ? out_lse + row : nullptr);
}

// Combine of the split pieces of each request.  Grid: one CTA per
// (request, group of 8 heads), one warp per head.
__global__ void __launch_bounds__(256) split_combine_kernel(PartialParams p) {
  __shared__ int warp_sums[8];
  __shared__ int sh_start, sh_nt;
  const int hgroups = (p.heads + 7) / 8;
  const int b = blockIdx.x / hgroups;
  const int h = (blockIdx.x % hgroups) * 8 + (threadIdx.x >> 5);
  int first_slot, count;
  if (p.sparse_idx) {
    if (p.sparse_parts == 1) return;          // written directly by the partial kernel
    first_slot = b * p.sparse_parts;
    count = p.sparse_parts;
  } else {
    // start tile of request b and the total, with the partial kernel's schedule
    int T = 0;
    for (int base = 0; base < p.batch; base += blockDim.x) {
      const int r = base + threadIdx.x;
      int n = 0, nt = 0;
      if (r < p.batch) nt = request_tiles(p, r, &n);
      int tot;
      const int ex = block_exclusive_scan(nt, warp_sums, &tot);
      if (r == b) {
        sh_start = T + ex;
        sh_nt = nt;
      }
      T += tot;
    }
    __syncthreads();
    const int start = sh_start, nt_b = sh_nt;
    if (nt_b == 0) {
      if (h < p.heads) {
        float* o = p.out + ((size_t)b * p.rows_o + h) * kVDim;
        for (int i = threadIdx.x & 31; i < kVDim; i += 32) o[i] = 0.f;
        if ((threadIdx.x & 31) == 0) p.out_lse[(size_t)b * p.rows_o + h] = -CUDART_INF_F;
      }
      return;
    }
    const int tpc = (T + p.num_ctas - 1) / p.num_ctas;
    const int c_first = start / tpc, c_last = (start + nt_b - 1) / tpc;
    if (c_first == c_last) return;            // one piece, already final
    first_slot = c_first + b;
    count = c_last - c_first + 1;
  }
  if (h < p.heads)
    merge_warp(StridedPieces{p.ws_o, p.ws_lse, (size_t)first_slot * p.heads + h, (size_t)p.heads},
               count, p.out + ((size_t)b * p.rows_o + h) * kVDim,
               p.out_lse + (size_t)b * p.rows_o + h);
}

}  // namespace

cudaError_t launch_dcp_merge(const float* partials, const float* lses, int num_shards, int batch,
                             int heads, float* out, float* out_lse, cudaStream_t st) {
  const int rows = batch * heads;
  const int grid = (rows + kMergeWarps - 1) / kMergeWarps;
  dcp_merge_kernel<<<grid, kMergeWarps * 32, 0, st>>>(partials, lses, num_shards, rows, out,
                                                      out_lse);
  return cudaGetLastError();
}

cudaError_t launch_split_combine(const PartialParams& p, cudaStream_t st) {
  if ((p.sparse_idx && p.sparse_parts == 1) || p.request_aligned) return cudaSuccess;
  const int hgroups = (p.heads + 7) / 8;
  split_combine_kernel<<<p.batch * hgroups, 256, 0, st>>>(p);
  return cudaGetLastError();
}

}  // namespace dcpmla
