// Tensor-core (tcgen05 / TMEM) kernel for one shard's partial attention.
#include "common.cuh"
#include "kernels.h"

namespace dcpmla {

bool tc_supports(const PartialParams&, int) { return false; }

cudaError_t launch_partial_tc(const PartialParams&, int, cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace dcpmla
