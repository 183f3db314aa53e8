// Internal launch entry points shared between the kernel files and the C ABI.
#pragma once

#include <cuda_runtime.h>

#include "common.cuh"

namespace dcpmla {

cudaError_t launch_partial_simt(const PartialParams& p, int kv_dtype, cudaStream_t st);
cudaError_t launch_partial_tc(const PartialParams& p, int kv_dtype, cudaStream_t st);
bool tc_supports(const PartialParams& p, int kv_dtype);
cudaError_t launch_partial_f8(const PartialParams& p, cudaStream_t st);
bool f8_supports(const PartialParams& p, int kv_dtype);
cudaError_t launch_split_combine(const PartialParams& p, cudaStream_t st);
cudaError_t launch_dcp_merge(const float* partials, const float* lses, int num_shards, int batch,
                             int heads, float* out, float* out_lse, cudaStream_t st);
int simt_sparse_chunk_max();
cudaError_t launch_sparse_gather(const PartialParams& p, int row_bytes, int maxblk,
                                 uint8_t* gathered, int* counts, cudaStream_t st);
cudaError_t launch_sparse_rows(const PartialParams& p, int maxblk, int* rows, int* counts,
                               uint8_t* q_image, cudaStream_t st);

}  // namespace dcpmla
