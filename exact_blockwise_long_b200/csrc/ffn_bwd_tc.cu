// Backward of the blockwise SwiGLU feed-forward.
//
// The paper abstract pairs blockwise attention with a blockwise feed-forward
// for training; this is the chain rule through
//   g = x w1^T,  u = x w3^T,  h = silu(g) * u,  y = h w2^T
// with silu(g) = g s, s = 1 / (1 + e^-g), silu'(g) = s (1 + g (1 - s)):
//   dh = dy w2,  du = dh * silu(g),  dg = dh * u * silu'(g)
//   dx = dg w1 + du w3,  dw1 = dg^T x,  dw3 = du^T x,  dw2 = dy^T h
// taken chunk by chunk: only one chunk's dh, dg, du, h exist at a time (the
// workspace), g and u are recomputed, and the fp32 weight gradients are
// stored on the first chunk and TMA-added on the later ones (one add per
// element per launch, in stream order, so the sums are deterministic).
//
// Six GEMMs per chunk on the tcgen05 GEMM engine (csrc/gemm_tc.cu):
//   dh = dy_c w2                (fp32, kept for the next epilogue)
//   g | u = x_c [w1 ; w3]^T     (stacked B) -> dg, du, h  (SwiGLU-backward epilogue)
//   dx_c = dg w1 + du w3        (two K segments, w MN-major)
//   dw1 (+)= dg^T x_c, dw3 (+)= du^T x_c, dw2 (+)= dy_c^T h   (MN-major operands)
#include "common.cuh"
#include "internal.h"

namespace ra {

size_t ffn_bwd_workspace_bytes(int64_t chunk, int64_t d_ff) { return (size_t)chunk * d_ff * (4 + 3 * 2); }

int launch_ffn_bwd_tc(const void* x, const void* w1, const void* w2, const void* w3, const void* dy, void* dx,
                      float* dw1, float* dw2, float* dw3, int64_t T, int64_t d_model, int64_t d_ff, int64_t chunk,
                      void* workspace, cudaStream_t stream) {
  if (d_ff % 128 || d_model % 128 || chunk % 128 || T % chunk) return RA_ERR_SHAPE;
  if (T > INT32_MAX || d_ff > INT32_MAX) return RA_ERR_UNSUPPORTED;
  float* dh = static_cast<float*>(workspace);
  auto* dg = reinterpret_cast<__nv_bfloat16*>(dh + chunk * d_ff);
  __nv_bfloat16* du = dg + chunk * d_ff;
  __nv_bfloat16* h = du + chunk * d_ff;
  auto op = [](const void* p, int64_t rows, int64_t cols, int mn, int64_t r0) {
    return GemmOperand{p, rows, cols, mn, 0, 0, 0, r0, 0};
  };
  auto f32 = [](float* p, bool add) { return GemmOut{p, kEpiF32, add ? 1 : 0, 0, 0, 0, nullptr, nullptr, nullptr}; };
  for (int64_t c0 = 0; c0 < T; c0 += chunk) {
    const bool add = c0 > 0;
    int rc;
    {  // dh = dy_c w2: B[n = hidden unit, k = feature] is w2 read MN-major
      GemmSeg g{op(dy, T, d_model, 0, c0), op(w2, d_model, d_ff, 1, 0), d_model};
      if ((rc = launch_gemm_tc(&g, 1, chunk, d_ff, f32(dh, false), 1, stream)) != RA_OK) return rc;
    }
    {  // g | u recomputed, SwiGLU backward -> dg, du, h
      GemmSeg g[2] = {{op(x, T, d_model, 0, c0), op(w1, d_ff, d_model, 0, 0), d_model},
                      {op(x, T, d_model, 0, c0), op(w3, d_ff, d_model, 0, 0), d_model}};
      GemmOut o{dg, kEpiSwiGLUBwd, 0, 0, 0, 0, dh, du, h};
      if ((rc = launch_gemm_tc(g, 2, chunk, d_ff, o, 1, stream)) != RA_OK) return rc;
    }
    {  // dx_c = dg w1 + du w3
      GemmSeg g[2] = {{op(dg, chunk, d_ff, 0, 0), op(w1, d_ff, d_model, 1, 0), d_ff},
                      {op(du, chunk, d_ff, 0, 0), op(w3, d_ff, d_model, 1, 0), d_ff}};
      GemmOut o{static_cast<__nv_bfloat16*>(dx) + c0 * d_model, kEpiBf16, 0, 0, 0, 0, nullptr, nullptr, nullptr};
      if ((rc = launch_gemm_tc(g, 2, chunk, d_model, o, 1, stream)) != RA_OK) return rc;
    }
    {  // dw1, dw3 (+)= dg^T x_c, du^T x_c
      GemmSeg g1{op(dg, chunk, d_ff, 1, 0), op(x, T, d_model, 1, c0), chunk};
      if ((rc = launch_gemm_tc(&g1, 1, d_ff, d_model, f32(dw1, add), 1, stream)) != RA_OK) return rc;
      GemmSeg g3{op(du, chunk, d_ff, 1, 0), op(x, T, d_model, 1, c0), chunk};
      if ((rc = launch_gemm_tc(&g3, 1, d_ff, d_model, f32(dw3, add), 1, stream)) != RA_OK) return rc;
    }
    {  // dw2 (+)= dy_c^T h
      GemmSeg g{op(dy, T, d_model, 1, c0), op(h, chunk, d_ff, 1, 0), chunk};
      if ((rc = launch_gemm_tc(&g, 1, d_model, d_ff, f32(dw2, add), 1, stream)) != RA_OK) return rc;
    }
  }
  return RA_OK;
}

}  // namespace ra
