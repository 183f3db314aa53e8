// Plain CUDA-core kernel for one shard's partial attention (any H <= 64).
//
// It is the simple, obviously-structured GPU path: rows are decoded to fp32
// in shared memory 16 at a time, every (head, token) score is a 576-long dot
// product, and an online softmax (running max m, running sum l, rescale by
// exp(m_old - m_new)) accumulates the 512-wide output in registers.  The
// tensor-core kernel computes the same thing; this one backs it up for head
// counts and shapes it does not take, and serves as a second GPU opinion in
// the tests.
//
// Method: partial attention per shard plus LSE ("GLM-5.2 vLLM Decode Context
// Parallelism", sections "See why vLLM 0.26.0 fails" and "Separate the
// backend merge from stable"); round-robin ownership ("How vLLM Serves
// GLM-5.3 with Million-Token Contexts on 16 H200s", "The core design").
#include "common.cuh"
#include "kernels.h"

#include <cuda_fp8.h>
#include <math_constants.h>

namespace dcpmla {
namespace {

constexpr int kThreads = 256;
constexpr int kSub = 16;           // rows decoded per step
constexpr int kQPad = 584;         // bf16 row pitch of q in shared memory
constexpr int kKPad = 580;         // fp32 row pitch of decoded rows
constexpr int kSparseChunkMax = 2048;

struct SimtSmem {
  __nv_bfloat16 q[kMaxHeads * kQPad];
  float k[kSub * kKPad];
  float s[kMaxHeads * (kSub + 1)];
  float alpha[kMaxHeads];
  float m[kMaxHeads];
  float l[kMaxHeads];
  const uint8_t* rows[kSub];
  int warp_sums[kThreads / 32];
  int list_n;
  Segment seg[kThreads];
  int sel[kSparseChunkMax];
};

// Decode 16-byte chunk c (0..71 for bf16, 0..39 for fp8) of a row into fp32.
template <int KV>
__device__ __forceinline__ void decode_chunk(const uint8_t* row, int c, float* dst) {
  if (KV == kKvBf16) {
    uint4 v = *reinterpret_cast<const uint4*>(row + 16 * c);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
    float* o = dst + 8 * c;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float2 f = __bfloat1622float2(h[i]);
      o[2 * i] = f.x;
      o[2 * i + 1] = f.y;
    }
  } else {
    if (c < 32) {   // 16 E4M3 codes of latent values [16c, 16c + 16)
      uint4 v = *reinterpret_cast<const uint4*>(row + 16 * c);
      float sc = reinterpret_cast<const float*>(row + 512)[c >> 3];
      const __nv_fp8x2_storage_t* pr = reinterpret_cast<const __nv_fp8x2_storage_t*>(&v);
      float* o = dst + 16 * c;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(pr[i], __NV_E4M3);
        float2 f = __half22float2(*reinterpret_cast<__half2*>(&hr));
        o[2 * i] = f.x * sc;
        o[2 * i + 1] = f.y * sc;
      }
    } else {        // 8 bf16 rope values
      const int r = c - 32;
      uint4 v = *reinterpret_cast<const uint4*>(row + 528 + 16 * r);
      const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
      float* o = dst + 512 + 8 * r;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float2 f = __bfloat1622float2(h[i]);
        o[2 * i] = f.x;
        o[2 * i + 1] = f.y;
      }
    }
  }
}

// Accumulates attention over `n` rows (row r's bytes from row_of(r)) into
// acc/m/l.  All threads call it.
template <int KV, class RowOf>
__device__ void attend_rows(const PartialParams& p, SimtSmem& sm, int n, RowOf row_of,
                            float (&acc)[32][4]) {
  constexpr int kChunks = KV == kKvBf16 ? 72 : 40;
  const int tid = threadIdx.x;
  const int h_s = tid >> 2, tq = tid & 3;         // score layout
  const int hg = tid >> 7, dq = tid & 127;        // output layout
  for (int r0 = 0; r0 < n; r0 += kSub) {
    const int cnt = min(kSub, n - r0);
    if (tid < kSub) sm.rows[tid] = tid < cnt ? row_of(r0 + tid) : nullptr;
    __syncthreads();
    for (int i = tid; i < kSub * kChunks; i += kThreads) {
      const int r = i / kChunks, c = i % kChunks;
      const uint8_t* row = sm.rows[r];
      float* dst = sm.k + r * kKPad;
      if (row) {
        decode_chunk<KV>(row, c, dst);
      } else {
        const int w = KV == kKvBf16 ? 8 : (c < 32 ? 16 : 8);
        const int o = KV == kKvBf16 ? 8 * c : (c < 32 ? 16 * c : 512 + 8 * (c - 32));
        for (int e = 0; e < w; ++e) dst[o + e] = 0.f;
      }
    }
    __syncthreads();
    // scores
    if (h_s < p.heads) {
      float a[4] = {0.f, 0.f, 0.f, 0.f};
      const __nv_bfloat162* qh = reinterpret_cast<const __nv_bfloat162*>(sm.q + h_s * kQPad);
      for (int d2 = 0; d2 < kHeadDim / 2; ++d2) {
        float2 qv = __bfloat1622float2(qh[d2]);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          float2 kv = reinterpret_cast<const float2*>(sm.k + (tq + 4 * i) * kKPad)[d2];
          a[i] = fmaf(qv.x, kv.x, a[i]);
          a[i] = fmaf(qv.y, kv.y, a[i]);
        }
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int t = tq + 4 * i;
        const bool ok = t < cnt && sm.rows[t] != nullptr;
        sm.s[h_s * (kSub + 1) + t] = ok ? a[i] * p.scale : -CUDART_INF_F;
      }
    }
    __syncthreads();
    // online softmax, one thread per head
    if (tid < p.heads) {
      float* srow = sm.s + tid * (kSub + 1);
      float mx = sm.m[tid];
      for (int t = 0; t < kSub; ++t) mx = fmaxf(mx, srow[t]);
      float alpha, sum = 0.f;
      if (mx == -CUDART_INF_F) {
        alpha = 1.f;
        for (int t = 0; t < kSub; ++t) srow[t] = 0.f;
      } else {
        alpha = expf(sm.m[tid] - mx);
        for (int t = 0; t < kSub; ++t) {
          float e = expf(srow[t] - mx);
          srow[t] = e;
          sum += e;
        }
      }
      sm.l[tid] = sm.l[tid] * alpha + sum;
      sm.m[tid] = mx;
      sm.alpha[tid] = alpha;
    }
    __syncthreads();
    // output update
#pragma unroll
    for (int hh = 0; hh < 32; ++hh) {
      const int h = hg * 32 + hh;
      if (h < p.heads) {
        const float al = sm.alpha[h];
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[hh][e] *= al;
      }
    }
    for (int t = 0; t < cnt; ++t) {
      const float4 v = reinterpret_cast<const float4*>(sm.k + t * kKPad)[dq];
#pragma unroll
      for (int hh = 0; hh < 32; ++hh) {
        const float pr = sm.s[(hg * 32 + hh) * (kSub + 1) + t];
        acc[hh][0] = fmaf(pr, v.x, acc[hh][0]);
        acc[hh][1] = fmaf(pr, v.y, acc[hh][1]);
        acc[hh][2] = fmaf(pr, v.z, acc[hh][2]);
        acc[hh][3] = fmaf(pr, v.w, acc[hh][3]);
      }
    }
    __syncthreads();
  }
}

__device__ void load_q(const PartialParams& p, SimtSmem& sm, int b) {
  const uint4* src = reinterpret_cast<const uint4*>(p.q + (size_t)b * p.rows_q * kHeadDim);
  for (int i = threadIdx.x; i < p.heads * 72; i += kThreads) {
    const int h = i / 72, c = i % 72;
    *reinterpret_cast<uint4*>(sm.q + h * kQPad + 8 * c) = src[i];
  }
  if (threadIdx.x < kMaxHeads) {
    sm.m[threadIdx.x] = -CUDART_INF_F;
    sm.l[threadIdx.x] = 0.f;
  }
  __syncthreads();
}

// Writes the normalised result (or the empty pair) to out/lse rows of stride H.
__device__ void store_result(const PartialParams& p, SimtSmem& sm, float (&acc)[32][4],
                             float* o_base, float* lse_base) {
  const int tid = threadIdx.x, hg = tid >> 7, dq = tid & 127;
#pragma unroll
  for (int hh = 0; hh < 32; ++hh) {
    const int h = hg * 32 + hh;
    if (h >= p.heads) continue;
    const float l = sm.l[h];
    const float inv = l > 0.f ? 1.f / l : 0.f;
    float4 v = make_float4(acc[hh][0] * inv, acc[hh][1] * inv, acc[hh][2] * inv, acc[hh][3] * inv);
    reinterpret_cast<float4*>(o_base + (size_t)h * kVDim)[dq] = v;
  }
  if (tid < p.heads) {
    const float l = sm.l[tid];
    lse_base[tid] = l > 0.f ? sm.m[tid] + logf(l) : -CUDART_INF_F;
  }
  __syncthreads();
}

template <int KV>
__global__ void __launch_bounds__(kThreads, 1) partial_simt_dense(PartialParams p) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  SimtSmem& sm = *reinterpret_cast<SimtSmem*>(smem_raw);
  const int T = total_tiles(p, sm.warp_sums);
  if (T == 0) return;
  const int tpc = (T + p.num_ctas - 1) / p.num_ctas;
  const int lo = blockIdx.x * tpc, hi = min(T, lo + tpc);
  if (lo >= hi) return;
  constexpr int kRowBytes = KV == kKvBf16 ? kRowBytesBf16 : kRowBytesFp8;
  for_each_dense_segment(p, lo, hi, sm.warp_sums, sm.seg, &sm.list_n, [&](const Segment& s) {
    float acc[32][4];
#pragma unroll
    for (int i = 0; i < 32; ++i)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[i][e] = 0.f;
    load_q(p, sm, s.b);
    const int r_begin = s.t0 * kBlock;
    const int n = min(s.n_rows, s.t1 * kBlock) - r_begin;
    attend_rows<KV>(p, sm, n, [&](int r) -> const uint8_t* {
      const int j = r_begin + r;
      const int blk = tile_block(p, s.b, j / kBlock);
      if (blk < 0) return nullptr;
      return p.kv + ((size_t)blk * kBlock + (j % kBlock)) * kRowBytes;
    }, acc);
    const bool whole = s.t0 == 0 && s.t1 == s.nt;
    const size_t slot = whole ? (size_t)s.b : (size_t)blockIdx.x + s.b;
    float* o_base = (whole ? p.out : p.ws_o) + slot * (whole ? p.rows_o : p.heads) * kVDim;
    float* l_base = (whole ? p.out_lse : p.ws_lse) + slot * (whole ? p.rows_o : p.heads);
    store_result(p, sm, acc, o_base, l_base);
  });
}

template <int KV>
__global__ void __launch_bounds__(kThreads, 1) partial_simt_sparse(PartialParams p) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  SimtSmem& sm = *reinterpret_cast<SimtSmem*>(smem_raw);
  constexpr int kRowBytes = KV == kKvBf16 ? kRowBytesBf16 : kRowBytesFp8;
  const int b = blockIdx.x / p.sparse_parts, part = blockIdx.x % p.sparse_parts;
  if (b >= p.batch) return;
  const int chunk = (p.topk + p.sparse_parts - 1) / p.sparse_parts;
  const int i0 = part * chunk, i1 = min(p.topk, i0 + chunk);
  int L = seq_len_of(p, b);
  if (L < 0) {
    if (p.flags) atomicOr(p.flags, kFlagBadLength);
    L = 0;
  }
  // select the listed positions this shard owns; keep their local index
  if (threadIdx.x == 0) sm.list_n = 0;
  __syncthreads();
  for (int i = i0 + threadIdx.x; i < i1; i += kThreads) {
    const int t = __ldg(p.sparse_idx + (size_t)b * p.topk + i);
    if (t >= 0 && t < L && t % p.nshards == p.shard) {
      const int j = t / p.nshards;
      if (j / kBlock < p.bt_stride) {
        sm.sel[atomicAdd(&sm.list_n, 1)] = j;
      } else if (p.flags) {
        atomicOr(p.flags, kFlagBadLength);
      }
    }
  }
  __syncthreads();
  const int n = sm.list_n;
  float acc[32][4];
#pragma unroll
  for (int i = 0; i < 32; ++i)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[i][e] = 0.f;
  load_q(p, sm, b);
  attend_rows<KV>(p, sm, n, [&](int r) -> const uint8_t* {
    const int j = sm.sel[r];
    const int blk = tile_block(p, b, j / kBlock);
    if (blk < 0) return nullptr;
    return p.kv + ((size_t)blk * kBlock + (j % kBlock)) * kRowBytes;
  }, acc);
  const bool whole = p.sparse_parts == 1;
  const size_t slot = whole ? (size_t)b : (size_t)blockIdx.x;
  float* o_base = (whole ? p.out : p.ws_o) + slot * (whole ? p.rows_o : p.heads) * kVDim;
  float* l_base = (whole ? p.out_lse : p.ws_lse) + slot * (whole ? p.rows_o : p.heads);
  store_result(p, sm, acc, o_base, l_base);
}

template <class K>
cudaError_t launch(K kernel, int slot, int grid, const PartialParams& p, cudaStream_t st) {
  const int smem = (int)sizeof(SimtSmem);
  // Raise the shared-memory limit once per kernel and device (graph-capture safe afterwards).
  static int configured[4][64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (!configured[slot][dev & 63]) {
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    configured[slot][dev & 63] = 1;
  }
  kernel<<<grid, kThreads, smem, st>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_partial_simt(const PartialParams& p, int kv_dtype, cudaStream_t st) {
  if (p.sparse_idx) {
    const int grid = p.batch * p.sparse_parts;
    return kv_dtype == kKvBf16 ? launch(partial_simt_sparse<kKvBf16>, 0, grid, p, st)
                               : launch(partial_simt_sparse<kKvFp8>, 1, grid, p, st);
  }
  return kv_dtype == kKvBf16 ? launch(partial_simt_dense<kKvBf16>, 2, p.num_ctas, p, st)
                             : launch(partial_simt_dense<kKvFp8>, 3, p.num_ctas, p, st);
}

int simt_sparse_chunk_max() { return kSparseChunkMax; }

}  // namespace dcpmla
