// Backward kernels (placeholder until the tensor-core backward lands).
#include "common.cuh"
#include "internal.h"

namespace ra {
int launch_bwd_tc(const AttnArgs&, const void*, const float*, const void*, void*, void*, void*, void*,
                  cudaStream_t) {
  return RA_ERR_UNSUPPORTED;
}
}  // namespace ra
