// Blockwise SwiGLU feed-forward.
//
// "Ring Attention with Blockwise Transformers for Near-Infinite Context",
// abstract: the feed-forward is computed blockwise like the attention.  The
// token sequence is cut into chunks; for each chunk c
//   h_c = silu(x_c w1^T) * (x_c w3^T)      (gate/up GEMM, fused SwiGLU)
//   y_c = h_c w2^T  (+ residual_c)         (down GEMM)
// so only one chunk's hidden activation [chunk, d_ff] (the workspace) exists
// at a time.  silu(z) = z / (1 + e^-z).
//
// Both GEMMs run on the tcgen05 GEMM engine (csrc/gemm_tc.cu).  The gate/up
// GEMM stacks 128 rows of w1 over the same 128 rows of w3 into one 256-wide
// B tile, so one accumulator holds g | u for 128 hidden units and its
// epilogue writes h directly.
#include "common.cuh"
#include "internal.h"

namespace ra {

int launch_ffn_tc(const void* x, const void* w1, const void* w2, const void* w3, void* y, int64_t T,
                  int64_t d_model, int64_t d_ff, int64_t chunk, void* workspace, cudaStream_t stream,
                  const void* residual) {
  if (d_ff % 128 || d_model % 128 || chunk % 128 || T % chunk) return RA_ERR_SHAPE;
  if (T > INT32_MAX || d_ff > INT32_MAX) return RA_ERR_UNSUPPORTED;
  auto* h = static_cast<__nv_bfloat16*>(workspace);
  auto* yb = static_cast<__nv_bfloat16*>(y);
  const auto* rb = static_cast<const __nv_bfloat16*>(residual);
  for (int64_t c0 = 0; c0 < T; c0 += chunk) {
    const GemmOperand xc{x, T, d_model, 0, 0, 0, 0, c0, 0};  // rows c0.. of x
    GemmSeg up[2] = {{xc, GemmOperand{w1, d_ff, d_model, 0, 0, 0, 0, 0, 0}, d_model},
                     {xc, GemmOperand{w3, d_ff, d_model, 0, 0, 0, 0, 0, 0}, d_model}};
    GemmOut ho{h, kEpiSwiGLU, 0, 0, 0, 0, nullptr, nullptr, nullptr};
    int rc = launch_gemm_tc(up, 2, chunk, d_ff, ho, 1, stream);
    if (rc != RA_OK) return rc;
    GemmSeg down{GemmOperand{h, chunk, d_ff, 0, 0, 0, 0, 0, 0}, GemmOperand{w2, d_model, d_ff, 0, 0, 0, 0, 0, 0},
                 d_ff};
    GemmOut yo{yb + c0 * d_model, rb ? kEpiBf16Res : kEpiBf16, 0, 0, 0, 0, rb ? rb + c0 * d_model : nullptr,
               nullptr, nullptr};
    rc = launch_gemm_tc(&down, 1, chunk, d_model, yo, 1, stream);
    if (rc != RA_OK) return rc;
  }
  return RA_OK;
}

}  // namespace ra
