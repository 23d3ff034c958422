// Blockwise FFN kernels (placeholder until the tensor-core GEMMs land).
#include "common.cuh"
#include "internal.h"

namespace ra {
int launch_ffn_tc(const void*, const void*, const void*, const void*, void*, int64_t, int64_t, int64_t, int64_t,
                  void*, cudaStream_t) {
  return RA_ERR_UNSUPPORTED;
}
}  // namespace ra
