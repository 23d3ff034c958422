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
// It runs the deterministic two-pass backward (the key/value-stationary and
// query-stationary passes), whose only scratch is two fp32 row vectors
// [B*H*N] -- D_i = dO_i . O_i and lse_i * log2(e) -- rather than the fused
// pass's fp32 dQ accumulator.  Those vectors live in one file-scope device
// array of fixed size, kNoallocScratchBytes.  Every GPU that loads this
// library keeps that array until the process exits.
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
  RA_NVTX_RANGE();
  constexpr int kPhases = ra::kPhasePre | ra::kPhaseKV | ra::kPhaseQ;
  // the same argument checks, in the same order, as the workspace entry points
  const int rc = ra::check_bwd_args(q, k, v, out, lse, dout, dq, dk, dv, B, H, H, N, D, dtype, S, q_chunk, k_chunk,
                                    causal, kPhases);
  if (rc == ra::kBwdEmpty) return RA_OK;
  if (rc != RA_OK) return rc;
  const size_t need = ra::bwd_workspace_bytes(B, H, N, D, false);
  if (need > ra::kNoallocScratchBytes) return RA_ERR_WORKSPACE;  // larger than the static scratch
  void* scratch = nullptr;
  const int rs = ra::scratch_address(&scratch);
  if (rs != RA_OK) return rs;
  // The preprocess phase overwrites both row vectors in full before the two
  // passes read them, so nothing an earlier call left in the array leaks in.
  return ra::run_bwd(q, k, v, out, lse, dout, dq, dk, dv, B, H, H, N, D, S, q_chunk, k_chunk, causal, scale,
                     scratch, need, kPhases, stream);
}

}  // extern "C"
