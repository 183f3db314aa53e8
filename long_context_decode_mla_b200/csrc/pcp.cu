// Prefill context parallelism (PCP) over a DCP-sharded cache: the chunk plan,
// the per-layer gather of a prompt's distributed rows, and (in dcpmla_api.cu)
// the causal attention of a rank's query tokens over the gathered rows.
//
// "How vLLM Serves GLM-5.3 with Million-Token Contexts on 16 H200s", section
// "The core design": PCP splits a prompt's queries by token over the ranks,
// each rank computing all heads of its tokens; the prompt is cut into twice
// as many chunks as ranks and rank r takes a front chunk and the matching
// back chunk (16 chunks for 8 ranks) so that causal work evens out; because
// the cache stays distributed round-robin (token t on DCP shard t mod N at
// local row t div N), prefill gathers the distributed cache of the layer,
// attends, and drops the gathered copy.
#include "dcpmla.h"

#include <cstdint>

#include <cuda_runtime.h>

#include "common.cuh"

namespace dcpmla {
namespace {

// One warp per prompt token: copy its row (16-byte units) from the shard
// that owns it into the gathered buffer, in token order.
__global__ void __launch_bounds__(256) pcp_gather_kernel(const uint8_t* kv, long long num_blocks,
                                                         int row_bytes, const int* tables,
                                                         int table_stride, int num_shards,
                                                         int num_tokens, uint8_t* gathered,
                                                         int* flags) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (warp >= num_tokens) return;
  const int t = warp, s = t % num_shards, j = t / num_shards;
  const int k = j / kBlock;
  uint4* dst = reinterpret_cast<uint4*>(gathered + (size_t)t * row_bytes);
  const int units = row_bytes / 16;
  int blk = -1;
  if (k < table_stride) blk = __ldg(tables + (size_t)s * table_stride + k);
  if (blk < 0 || (long long)blk >= num_blocks) {
    // out of range: flagged, and the row is written as zeros
    if (lane == 0 && flags) atomicOr(flags, k < table_stride ? kFlagBadBlock : kFlagBadLength);
    for (int u = lane; u < units; u += 32) dst[u] = make_uint4(0, 0, 0, 0);
    return;
  }
  const uint4* src =
      reinterpret_cast<const uint4*>(kv + ((size_t)blk * kBlock + (j % kBlock)) * row_bytes);
  for (int u = lane; u < units; u += 32) dst[u] = __ldg(src + u);
}

}  // namespace
}  // namespace dcpmla

using namespace dcpmla;

extern "C" {

int pcp_rank_tokens(int num_tokens, int pcp_size, int rank, int32_t* tokens, int capacity,
                    int* count) {
  if (num_tokens < 0 || pcp_size < 1 || rank < 0 || rank >= pcp_size || !count)
    return DCPMLA_ERR_INVALID_ARGUMENT;
  // 2P contiguous chunks in prompt order, the first T mod 2P one token longer
  const long long n = 2LL * pcp_size, base = num_tokens / n, extra = num_tokens % n;
  auto start = [&](long long c) { return c * base + (c < extra ? c : extra); };
  auto size = [&](long long c) { return base + (c < extra ? 1 : 0); };
  const long long front = rank, back = n - 1 - rank;
  const long long total = size(front) + size(back);
  *count = (int)total;
  if (!tokens) return DCPMLA_OK;
  if (capacity < total) return DCPMLA_ERR_INVALID_ARGUMENT;
  int w = 0;
  for (long long t = start(front); t < start(front) + size(front); ++t) tokens[w++] = (int32_t)t;
  for (long long t = start(back); t < start(back) + size(back); ++t) tokens[w++] = (int32_t)t;
  return DCPMLA_OK;
}

int pcp_gather_rows(const void* kv_cache, int kv_dtype, int64_t num_blocks, int block_size,
                    const int32_t* block_tables, int block_table_stride, int num_shards,
                    int num_tokens, void* gathered, size_t gathered_bytes, int32_t* flags,
                    void* stream) {
  if (kv_dtype != DCPMLA_KV_BF16 && kv_dtype != DCPMLA_KV_FP8) return DCPMLA_ERR_INVALID_ARGUMENT;
  if (num_blocks < 1 || block_table_stride < 1 || num_shards < 1 || num_tokens < 0)
    return DCPMLA_ERR_INVALID_ARGUMENT;
  if (block_size != kBlock) return DCPMLA_ERR_UNSUPPORTED;
  if (num_tokens == 0) return DCPMLA_OK;
  if (!kv_cache || !block_tables || !gathered) return DCPMLA_ERR_INVALID_ARGUMENT;
  const int rb = kv_dtype == DCPMLA_KV_BF16 ? kRowBytesBf16 : kRowBytesFp8;
  if (gathered_bytes < pcp_gathered_bytes(num_tokens, kv_dtype)) return DCPMLA_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(kv_cache) & 15) || (reinterpret_cast<uintptr_t>(gathered) & 15))
    return DCPMLA_ERR_ALIGNMENT;
  const long long threads = (long long)num_tokens * 32;
  const int grid = (int)((threads + 255) / 256);
  pcp_gather_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint8_t*>(kv_cache), num_blocks, rb, block_tables, block_table_stride,
      num_shards, num_tokens, static_cast<uint8_t*>(gathered), flags);
  return cudaGetLastError() == cudaSuccess ? DCPMLA_OK : DCPMLA_ERR_CUDA;
}

size_t pcp_gathered_bytes(int num_tokens, int kv_dtype) {
  if (num_tokens <= 0) return 0;
  const size_t rb = kv_dtype == DCPMLA_KV_BF16 ? kRowBytesBf16 : kRowBytesFp8;
  // whole 64-row blocks: the attention reads the gathered rows block by block
  return (size_t)((num_tokens + kBlock - 1) / kBlock) * kBlock * rb;
}

}  // extern "C"
