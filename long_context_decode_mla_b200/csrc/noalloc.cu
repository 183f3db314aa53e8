// mla_decode_partial_noalloc: mla_decode_partial with its workspace taken
// from a fixed scratch array inside this library instead of from the caller.
//
// Who needs it: callers that cannot hand the library device memory.  A host
// program written in C that links only this library and the CUDA runtime
// may have no device allocator of its own; a serving loop may be forbidden
// to call cudaMalloc / cudaFree between decode steps, because those calls
// synchronise the whole device and stall every other request's stream.
// This entry point calls no allocator at all (no cudaMalloc, cudaFree or
// allocating library): its scratch is the file-scope device array below,
// whose address is looked up once per device.
//
// Limits, stated in dcpmla.h as well: one scratch array per device, so calls
// whose work overlaps on a device (two streams, two host threads) race on it
// and must be serialised by the caller; the first call on each device does
// the setup (symbol lookup, which may load this module) and should come
// before any stream capture.
#include "dcpmla.h"

#include <mutex>

#include <cuda_runtime.h>

namespace {

constexpr int kMaxDevices = 64;
constexpr size_t kFlagBytes = 4;   // int32 flag word at byte 0 of the workspace

static __device__ __align__(256) unsigned char g_scratch[DCPMLA_NOALLOC_SCRATCH_BYTES];

std::mutex g_setup_mutex;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_scratch on the current device.  The first call per
// device looks it up and clears the flag word on `stream`; later calls
// only read the cached address.
int scratch_for_current_device(cudaStream_t stream, void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return DCPMLA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return DCPMLA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (!g_scratch_addr[dev]) {
    void* addr = nullptr;
    if (cudaGetSymbolAddress(&addr, g_scratch) != cudaSuccess || !addr) return DCPMLA_ERR_CUDA;
    if (cudaMemsetAsync(addr, 0, kFlagBytes, stream) != cudaSuccess) return DCPMLA_ERR_CUDA;
    g_scratch_addr[dev] = addr;
  }
  *out = g_scratch_addr[dev];
  return DCPMLA_OK;
}

}  // namespace

extern "C" int mla_decode_partial_noalloc(
    const void* q, const void* kv_cache, int kv_dtype, int64_t num_blocks, int block_size,
    const int32_t* block_table, int block_table_stride, const int32_t* seq_lens, int batch,
    int num_heads, int shard_id, int num_shards, const int32_t* sparse_idx, int topk,
    float softmax_scale, float* out_partial, float* out_lse, int32_t* out_flags,
    int num_splits, int impl, void* stream) {
  // Size check first: a request that does not fit is refused before any
  // work is enqueued.  (The size function also sizes multi-query rows; this
  // entry point takes query heads only.)
  if (num_heads > DCPMLA_MAX_HEADS) return DCPMLA_ERR_UNSUPPORTED;
  size_t need = 0;
  int rc = mla_decode_workspace_size(batch, num_heads, num_splits, sparse_idx ? topk : 0, &need);
  if (rc != DCPMLA_OK) return rc;
  if (need > (size_t)DCPMLA_NOALLOC_SCRATCH_BYTES) return DCPMLA_ERR_WORKSPACE;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  void* scratch = nullptr;
  rc = scratch_for_current_device(st, &scratch);
  if (rc != DCPMLA_OK) return rc;

  // The flag word is zero here: cleared at setup and after every call.  Once
  // setup succeeded, the clear is queued on every return path, errors
  // included (best effort), so a failed call leaves no bits for the next.
  rc = mla_decode_partial(q, kv_cache, kv_dtype, num_blocks, block_size, block_table,
                          block_table_stride, seq_lens, batch, num_heads, shard_id, num_shards,
                          sparse_idx, topk, softmax_scale, out_partial, out_lse, scratch,
                          (size_t)DCPMLA_NOALLOC_SCRATCH_BYTES, num_splits, impl, stream);
  if (rc == DCPMLA_OK && out_flags &&
      cudaMemcpyAsync(out_flags, scratch, kFlagBytes, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    rc = DCPMLA_ERR_CUDA;
  const bool cleared = cudaMemsetAsync(scratch, 0, kFlagBytes, st) == cudaSuccess;
  if (rc != DCPMLA_OK) return rc;
  return cleared ? DCPMLA_OK : DCPMLA_ERR_CUDA;
}
