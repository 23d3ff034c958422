// ringattn_bwd_noalloc: the attention backward without a caller-supplied
// workspace and without any device allocation.
//
// The paper has no counterpart to this entry point; it exists for callers
// that cannot allocate device memory at the moment they need the gradient:
// code running under an allocator owned by another framework (a memory pool
// they must not grow, or a process whose device memory budget is fixed when
// it starts), and real-time or embedded callers that forbid allocation on
// their hot path because cudaMalloc can synchronise the device and stall
// other streams.  Such callers cannot hand ringattn_bwd its workspace.
//
// The backward's scratch (fp32 dQ accumulator plus the two fp32 row
// vectors) lives instead in one file-scope device array of fixed size,
// kNoallocScratchBytes.  Every GPU that loads this part of the library
// keeps that array until the process exits.
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace ra {
namespace {

constexpr size_t kNoallocScratchBytes = RINGATTN_NOALLOC_SCRATCH_BYTES;  // 64 MiB per device

// The scratch itself.  In host code this name is only a stand-in for the
// device symbol: its device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_bwd_scratch[kNoallocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device, looked up once
// per device with that device current.
int scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return RA_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_bwd_scratch) != cudaSuccess || ptr == nullptr) return RA_ERR_CUDA;
    g_scratch_ptr[dev] = ptr;
  }
  *out = g_scratch_ptr[dev];
  return RA_OK;
}

}  // namespace
}  // namespace ra

extern "C" {

int ringattn_bwd_noalloc(const void* q, const void* k, const void* v, const void* out, const float* lse,
                         const void* dout, void* dq, void* dk, void* dv, int64_t B, int64_t H, int64_t N,
                         int64_t D, int dtype, int S, int q_chunk, int k_chunk, int causal, float scale,
                         void* stream) {
  const size_t need = ringattn_bwd_workspace_size(B, H, N, D);
  if (need > ra::kNoallocScratchBytes) return RA_ERR_WORKSPACE;  // larger than the static scratch
  if (need == 0) {
    // empty or invalid extents: the regular entry point validates and answers
    return ringattn_bwd(q, k, v, out, lse, dout, dq, dk, dv, B, H, N, D, dtype, S, q_chunk, k_chunk, causal,
                        scale, nullptr, 0, stream);
  }
  void* scratch = nullptr;
  const int rc = ra::scratch_address(&scratch);
  if (rc != RA_OK) return rc;
  // The preprocess phase clears the dQ accumulator and overwrites both row
  // vectors, so nothing left in the array by an earlier call leaks in.
  return ringattn_bwd(q, k, v, out, lse, dout, dq, dk, dv, B, H, N, D, dtype, S, q_chunk, k_chunk, causal, scale,
                      scratch, ra::kNoallocScratchBytes, stream);
}

}  // extern "C"
