// mla_kv_append: the DCP cache write of new decode tokens.
//
// "GLM-5.2 vLLM Decode Context Parallelism", section "Keep the current-main
// correctness blocker visible" ("Query work is skipped with an owner-remote KV
// slot"): under DCP only the rank that owns a token's cache slot writes it;
// the others skip the write (their query work is unaffected).  Ownership is
// round-robin ("How vLLM Serves GLM-5.3 with Million-Token Contexts on 16
// H200s", "The core design"): token t belongs to shard t mod N, local row
// t div N.  The fp8 row is the DeepSeek sparse-MLA packed layout ("GLM-5.2
// vLLM Decode Context Parallelism", "Stable H200 control: no DCP candidate"):
// 512 E4M3 codes with one fp32 scale per 128 values, then 64 bf16 rope values.
#include "dcpmla.h"

#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include <cstdint>

namespace {

constexpr int kBlockRows = 64;
constexpr int kWarpsPerCta = 8;
constexpr int kFp8RowBytes = 656;
constexpr int kBf16RowBytes = 1152;
constexpr float kE4m3Max = 448.f;

struct AppendParams {
  const uint4* latent;     // [T][512] bf16 as 16-byte units (64 per token)
  const uint4* rope;       // [T][64] bf16 (8 units per token)
  const int32_t* positions;
  const int32_t* req_idx;
  const int32_t* block_table;
  int bt_stride, batch, shard, nshards, num_tokens;
  uint8_t* cache;
  int64_t num_blocks;
  int32_t* flags;
};

__device__ __forceinline__ void set_flag(const AppendParams& p, int bit) {
  if (p.flags) atomicOr(p.flags, bit);
}

// Physical row of token i on this shard, or nullptr when the shard does not
// write it (not the owner, padding, or a range check failed and was flagged).
__device__ __forceinline__ uint8_t* owned_row(const AppendParams& p, int i, int row_bytes,
                                              bool report) {
  const int t = __ldg(p.positions + i);
  if (t < 0 || t % p.nshards != p.shard) return nullptr;
  const int b = __ldg(p.req_idx + i);
  const int j = t / p.nshards;
  const int k = j / kBlockRows;
  if (b < 0 || b >= p.batch || k >= p.bt_stride) {
    if (report) set_flag(p, DCPMLA_FLAG_BAD_LENGTH);
    return nullptr;
  }
  const int blk = __ldg(p.block_table + (size_t)b * p.bt_stride + k);
  if (blk < 0 || (int64_t)blk >= p.num_blocks) {
    if (report) set_flag(p, DCPMLA_FLAG_BAD_BLOCK);
    return nullptr;
  }
  return p.cache + ((size_t)blk * kBlockRows + (j % kBlockRows)) * row_bytes;
}

// bf16 rows: a plain copy of 72 16-byte units per token.
__global__ void __launch_bounds__(32 * kWarpsPerCta) append_bf16_kernel(AppendParams p) {
  const int i = blockIdx.x * kWarpsPerCta + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (i >= p.num_tokens) return;
  uint8_t* row = owned_row(p, i, kBf16RowBytes, lane == 0);
  if (!row) return;
  uint4* dst = reinterpret_cast<uint4*>(row);
  for (int u = lane; u < 72; u += 32)
    dst[u] = u < 64 ? __ldg(p.latent + (size_t)i * 64 + u) : __ldg(p.rope + (size_t)i * 8 + (u - 64));
}

// fp8 rows: lane l quantises latent values [16 l, 16 l + 16); lanes 8g .. 8g+7
// form scale group g.  scale = amax / 448 (1 when amax = 0); code = E4M3 of
// x / scale, round to nearest even, saturated at 448.
__global__ void __launch_bounds__(32 * kWarpsPerCta) append_fp8_kernel(AppendParams p) {
  const int i = blockIdx.x * kWarpsPerCta + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (i >= p.num_tokens) return;
  uint8_t* row = owned_row(p, i, kFp8RowBytes, lane == 0);
  if (!row) return;                                   // warp-uniform: every lane sees the same row
  const uint4 a = __ldg(p.latent + (size_t)i * 64 + 2 * lane);
  const uint4 b = __ldg(p.latent + (size_t)i * 64 + 2 * lane + 1);
  const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
  float x[16];
  float amax = 0.f;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    x[2 * k] = __uint_as_float(w[k] << 16);
    x[2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
    amax = fmaxf(amax, fmaxf(fabsf(x[2 * k]), fabsf(x[2 * k + 1])));
  }
#pragma unroll
  for (int off = 1; off < 8; off <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  const float scale = amax > 0.f ? __fdiv_rn(amax, kE4m3Max) : 1.f;
  uint32_t codes[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const __nv_fp8x2_storage_t lo = __nv_cvt_float2_to_fp8x2(
        make_float2(__fdiv_rn(x[4 * k], scale), __fdiv_rn(x[4 * k + 1], scale)), __NV_SATFINITE,
        __NV_E4M3);
    const __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(
        make_float2(__fdiv_rn(x[4 * k + 2], scale), __fdiv_rn(x[4 * k + 3], scale)),
        __NV_SATFINITE, __NV_E4M3);
    codes[k] = (uint32_t)lo | ((uint32_t)hi << 16);
  }
  reinterpret_cast<uint4*>(row)[lane] = make_uint4(codes[0], codes[1], codes[2], codes[3]);
  if ((lane & 7) == 0) reinterpret_cast<float*>(row + 512)[lane >> 3] = scale;
  if (lane < 8) reinterpret_cast<uint4*>(row + 528)[lane] = __ldg(p.rope + (size_t)i * 8 + lane);
}

bool aligned16(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }

}  // namespace

extern "C" int mla_kv_append(const void* latent, const void* rope, int num_tokens,
                             const int32_t* positions, const int32_t* req_idx,
                             const int32_t* block_table, int block_table_stride, int batch,
                             int shard_id, int num_shards, void* kv_cache, int kv_dtype,
                             int64_t num_blocks, int block_size, int32_t* flags, void* stream) {
  if (num_tokens < 0 || batch < 1 || block_table_stride < 1 || num_shards < 1 || shard_id < 0 ||
      shard_id >= num_shards || num_blocks < 1)
    return DCPMLA_ERR_INVALID_ARGUMENT;
  if (kv_dtype != DCPMLA_KV_BF16 && kv_dtype != DCPMLA_KV_FP8) return DCPMLA_ERR_INVALID_ARGUMENT;
  if (block_size != kBlockRows) return DCPMLA_ERR_UNSUPPORTED;
  if (num_tokens == 0) return DCPMLA_OK;
  if (!latent || !rope || !positions || !req_idx || !block_table || !kv_cache)
    return DCPMLA_ERR_INVALID_ARGUMENT;
  if (!aligned16(latent) || !aligned16(rope) || !aligned16(kv_cache)) return DCPMLA_ERR_ALIGNMENT;
  AppendParams p;
  p.latent = static_cast<const uint4*>(latent);
  p.rope = static_cast<const uint4*>(rope);
  p.positions = positions;
  p.req_idx = req_idx;
  p.block_table = block_table;
  p.bt_stride = block_table_stride;
  p.batch = batch;
  p.shard = shard_id;
  p.nshards = num_shards;
  p.num_tokens = num_tokens;
  p.cache = static_cast<uint8_t*>(kv_cache);
  p.num_blocks = num_blocks;
  p.flags = flags;
  const int grid = (num_tokens + kWarpsPerCta - 1) / kWarpsPerCta;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (kv_dtype == DCPMLA_KV_FP8)
    append_fp8_kernel<<<grid, 32 * kWarpsPerCta, 0, st>>>(p);
  else
    append_bf16_kernel<<<grid, 32 * kWarpsPerCta, 0, st>>>(p);
  return cudaGetLastError() == cudaSuccess ? DCPMLA_OK : DCPMLA_ERR_CUDA;
}
