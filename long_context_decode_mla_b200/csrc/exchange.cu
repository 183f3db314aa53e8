// Cross-rank exchange of DCP partials: the head-sliced merge that pulls every
// shard's partial from its own buffer (local memory or a peer GPU's memory
// mapped over NVLink), and the exchange buffers those partials live in.
//
// "GLM-5.2 vLLM Decode Context Parallelism", section "Separate the backend
// merge from stable": the sparse DCP decode is combined across ranks over the
// ag_rs path (all-gather of the LSEs, then a reduce-scatter of the rescaled
// partial outputs).  Section "Keep the current-main correctness blocker
// visible": the query heads are gathered before attention and the partial
// output/LSE combined after it.  dcp_merge_heads does the ag_rs exchange as
// one pull: the rank that owns a slice of heads reads those heads' LSEs and
// partials from all N shards and merges them, which is the LSE all-gather,
// the rescale and the reduce-scatter sum of that slice at once.
#include "dcpmla.h"

#include <cstdint>
#include <cstring>

#include "common.cuh"
#include "merge_rows.cuh"

namespace dcpmla {
namespace {

static_assert(sizeof(cudaIpcMemHandle_t) == DCPMLA_IPC_HANDLE_BYTES, "IPC handle size");

constexpr int kHeadsMergeWarps = 8;

struct HeadsMergeParams {
  const float* o[DCPMLA_MAX_MERGE_SHARDS];
  const float* lse[DCPMLA_MAX_MERGE_SHARDS];
  int num_shards, num_heads, head_begin, head_count, rows;
  float* out;
  float* out_lse;
};

// One warp per output row r = b * head_count + i (head h = head_begin + i);
// the row reads entry b * num_heads + h of every shard's buffers.
__global__ void __launch_bounds__(kHeadsMergeWarps * 32) dcp_merge_heads_kernel(
    const __grid_constant__ HeadsMergeParams p) {
  __shared__ const float* s_o[DCPMLA_MAX_MERGE_SHARDS];
  __shared__ const float* s_lse[DCPMLA_MAX_MERGE_SHARDS];
  for (int k = threadIdx.x; k < p.num_shards; k += blockDim.x) {
    s_o[k] = p.o[k];
    s_lse[k] = p.lse[k];
  }
  __syncthreads();
  const int row = blockIdx.x * kHeadsMergeWarps + (threadIdx.x >> 5);
  if (row >= p.rows) return;
  const int b = row / p.head_count;
  const int h = p.head_begin + row % p.head_count;
  const size_t entry = (size_t)b * p.num_heads + h;
  merge_warp(TablePieces{s_o, s_lse, entry}, p.num_shards, p.out + (size_t)row * kVDim,
             p.out_lse ? p.out_lse + row : nullptr);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace dcpmla

using namespace dcpmla;

extern "C" {

int dcp_merge_heads(const float* const* partials, const float* const* lses, int num_shards,
                    int batch, int num_heads, int head_begin, int head_count, float* out,
                    float* out_lse, void* stream) {
  if (num_shards < 1 || num_shards > DCPMLA_MAX_MERGE_SHARDS || batch < 0 || num_heads < 1 ||
      head_begin < 0 || head_count < 1 || head_begin + head_count > num_heads)
    return DCPMLA_ERR_INVALID_ARGUMENT;
  if (batch == 0) return DCPMLA_OK;
  if (!partials || !lses || !out) return DCPMLA_ERR_INVALID_ARGUMENT;
  if ((long long)batch * num_heads > INT32_MAX / kVDim) return DCPMLA_ERR_UNSUPPORTED;
  HeadsMergeParams p{};
  for (int k = 0; k < num_shards; ++k) {
    if (!partials[k] || !lses[k]) return DCPMLA_ERR_INVALID_ARGUMENT;
    if (!aligned16(partials[k])) return DCPMLA_ERR_ALIGNMENT;
    p.o[k] = partials[k];
    p.lse[k] = lses[k];
  }
  if (!aligned16(out)) return DCPMLA_ERR_ALIGNMENT;
  p.num_shards = num_shards;
  p.num_heads = num_heads;
  p.head_begin = head_begin;
  p.head_count = head_count;
  p.rows = batch * head_count;
  p.out = out;
  p.out_lse = out_lse;
  const int grid = (p.rows + kHeadsMergeWarps - 1) / kHeadsMergeWarps;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  dcp_merge_heads_kernel<<<grid, kHeadsMergeWarps * 32, 0, st>>>(p);
  return cudaGetLastError() == cudaSuccess ? DCPMLA_OK : DCPMLA_ERR_CUDA;
}

int dcp_exchange_alloc(size_t bytes, void** dev_ptr, void* ipc_handle) {
  if (!dev_ptr || !ipc_handle || bytes == 0) return DCPMLA_ERR_INVALID_ARGUMENT;
  *dev_ptr = nullptr;
  void* p = nullptr;
  if (cudaMalloc(&p, bytes) != cudaSuccess) return DCPMLA_ERR_CUDA;
  cudaIpcMemHandle_t h;
  if (cudaIpcGetMemHandle(&h, p) != cudaSuccess) {
    cudaFree(p);
    return DCPMLA_ERR_CUDA;
  }
  memcpy(ipc_handle, &h, sizeof(h));
  *dev_ptr = p;
  return DCPMLA_OK;
}

int dcp_exchange_open(const void* ipc_handle, void** dev_ptr) {
  if (!ipc_handle || !dev_ptr) return DCPMLA_ERR_INVALID_ARGUMENT;
  *dev_ptr = nullptr;
  cudaIpcMemHandle_t h;
  memcpy(&h, ipc_handle, sizeof(h));
  void* p = nullptr;
  if (cudaIpcOpenMemHandle(&p, h, cudaIpcMemLazyEnablePeerAccess) != cudaSuccess)
    return DCPMLA_ERR_CUDA;
  *dev_ptr = p;
  return DCPMLA_OK;
}

int dcp_exchange_close(void* dev_ptr) {
  if (!dev_ptr) return DCPMLA_ERR_INVALID_ARGUMENT;
  return cudaIpcCloseMemHandle(dev_ptr) == cudaSuccess ? DCPMLA_OK : DCPMLA_ERR_CUDA;
}

int dcp_exchange_free(void* dev_ptr) {
  if (!dev_ptr) return DCPMLA_ERR_INVALID_ARGUMENT;
  return cudaFree(dev_ptr) == cudaSuccess ? DCPMLA_OK : DCPMLA_ERR_CUDA;
}

}  // extern "C"
