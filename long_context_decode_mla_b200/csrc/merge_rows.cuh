// The LSE-weighted merge of one (request, head) row, shared by the cross-shard
// DCP merges (stacked buffers or one pointer per shard) and the split-KV
// combine inside a shard.
//
// With M = max_i LSE_i and w_i = exp(LSE_i - M):
//   O = sum_i w_i O_i / sum_i w_i,   LSE = M + ln sum_i w_i,
// and pieces with LSE = -inf weigh exactly zero; if all are -inf the result
// is (0, -inf).  "GLM-5.2 vLLM Decode Context Parallelism", sections "See why
// vLLM 0.26.0 fails" (partials combined with the softmax normalisation via
// LSE) and "Separate the backend merge from stable" (the neutral (0, -inf)
// pair of an empty shard drops out of the merge).
#pragma once

#include <math_constants.h>

#include "common.cuh"

namespace dcpmla {

// Pieces laid out with a fixed stride: piece k of the row is entry
// first + k * stride of lse, with its 512 outputs at that entry of o.
struct StridedPieces {
  const float* __restrict__ o;
  const float* __restrict__ lse;
  size_t first, stride;
  __device__ __forceinline__ float lse_of(int k) const { return __ldg(lse + first + k * stride); }
  __device__ __forceinline__ const float4* row(int k) const {
    return reinterpret_cast<const float4*>(o + (first + k * stride) * kVDim);
  }
};

// One buffer per piece: piece k of the row is entry `entry` of lse[k], with
// its 512 outputs at that entry of o[k].  The pointer tables live in shared
// memory; the buffers may be another device's memory mapped into this one.
struct TablePieces {
  const float* const* o;
  const float* const* lse;
  size_t entry;
  __device__ __forceinline__ float lse_of(int k) const { return __ldg(lse[k] + entry); }
  __device__ __forceinline__ const float4* row(int k) const {
    return reinterpret_cast<const float4*>(o[k] + entry * kVDim);
  }
};

// One warp merges `count` pieces of one row into out_o (512 floats, 16-byte
// aligned) and *out_lse (if not null).
template <class Pieces>
__device__ __forceinline__ void merge_warp(const Pieces& pc, int count, float* __restrict__ out_o,
                                           float* __restrict__ out_lse) {
  const int lane = threadIdx.x & 31;
  float M = -CUDART_INF_F;
  for (int k = lane; k < count; k += 32) M = fmaxf(M, pc.lse_of(k));
#pragma unroll
  for (int s = 16; s > 0; s >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, s));
  float4 acc[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) acc[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  if (M == -CUDART_INF_F) {
#pragma unroll
    for (int i = 0; i < 4; ++i) reinterpret_cast<float4*>(out_o)[i * 32 + lane] = acc[i];
    if (lane == 0 && out_lse) *out_lse = -CUDART_INF_F;
    return;
  }
  float wsum = 0.f;
  for (int k = 0; k < count; ++k) {
    const float lk = pc.lse_of(k);
    if (lk == -CUDART_INF_F) continue;
    const float w = expf(lk - M);
    wsum += w;
    const float4* src = pc.row(k);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float4 v = __ldg(src + i * 32 + lane);
      acc[i].x = fmaf(w, v.x, acc[i].x);
      acc[i].y = fmaf(w, v.y, acc[i].y);
      acc[i].z = fmaf(w, v.z, acc[i].z);
      acc[i].w = fmaf(w, v.w, acc[i].w);
    }
  }
  const float inv = 1.f / wsum;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float4 v = acc[i];
    v.x *= inv; v.y *= inv; v.z *= inv; v.w *= inv;
    reinterpret_cast<float4*>(out_o)[i * 32 + lane] = v;
  }
  if (lane == 0 && out_lse) *out_lse = M + logf(wsum);
}

}  // namespace dcpmla
