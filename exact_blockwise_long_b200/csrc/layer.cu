// One blockwise transformer layer, forward and backward ("Ring Attention
// with Blockwise Transformers for Near-Infinite Context", abstract: the
// layer's self-attention and feed-forward are both computed blockwise; the
// attention shards the sequence and visits the key/value shards in ring
// order).  Pre-norm decoder layer with the 7B shape conventions:
//
//   xn = rmsnorm(x) * g_attn
//   q, k, v = xn Wq^T, xn Wk^T, xn Wv^T        (written head-split [B,H,N,D])
//   o = ring attention(q, k, v)                  (exact, causal or not)
//   x2 = x + o Wo^T
//   xn2 = rmsnorm(x2) * g_ffn
//   y = x2 + ((silu(xn2 W1^T) * (xn2 W3^T)) W2^T)  (blockwise, per chunk)
//
// The backward is the chain rule in reverse through the same steps.  Every
// step is one of this library's kernels; the launches here only carve the
// caller's buffers and sequence the steps on one stream.
#include <math.h>

#include "common.cuh"
#include "internal.h"

using namespace ra;

namespace {

size_t up256(size_t x) { return (x + 255) & ~(size_t)255; }

struct Carve {
  uint8_t* base;
  size_t off = 0;
  template <typename T>
  T* take(size_t bytes) {
    T* p = reinterpret_cast<T*>(base + off);
    off += up256(bytes);
    return p;
  }
};

// The activations the backward reads, in the order they are carved from
// `saved`.
struct Saved {
  __nv_bfloat16 *xn, *q, *k, *v, *o, *x2, *xn2;
  float *lse, *rstd1, *rstd2;
};

size_t saved_bytes(int64_t B, int64_t N, int64_t H, int64_t D) {
  const size_t T = (size_t)B * N, act = T * (size_t)(H * D) * 2;
  return 7 * up256(act) + up256((size_t)B * H * N * 4) + 2 * up256(T * 4);
}

Saved carve_saved(void* p, int64_t B, int64_t N, int64_t H, int64_t D) {
  Carve c{static_cast<uint8_t*>(p)};
  const size_t T = (size_t)B * N, act = T * (size_t)(H * D) * 2;
  Saved s;
  s.xn = c.take<__nv_bfloat16>(act);
  s.q = c.take<__nv_bfloat16>(act);
  s.k = c.take<__nv_bfloat16>(act);
  s.v = c.take<__nv_bfloat16>(act);
  s.o = c.take<__nv_bfloat16>(act);
  s.x2 = c.take<__nv_bfloat16>(act);
  s.xn2 = c.take<__nv_bfloat16>(act);
  s.lse = c.take<float>((size_t)B * H * N * 4);
  s.rstd1 = c.take<float>(T * 4);
  s.rstd2 = c.take<float>(T * 4);
  return s;
}

bool a16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// shape rules shared by forward and backward
// kNoTokens: a valid request with an empty batch (B == 0)
constexpr int kNoTokens = 1;

int check_layer(int64_t B, int64_t N, int64_t H, int64_t D, int64_t d_ff, int S, int q_chunk, int k_chunk,
                int ffn_chunk, int causal) {
  if (B < 0 || N <= 0 || H <= 0 || D <= 0 || d_ff <= 0 || S <= 0 || q_chunk <= 0 || k_chunk <= 0 ||
      ffn_chunk <= 0)
    return RA_ERR_ARG;
  if (causal != 0 && causal != 1) return RA_ERR_ARG;
  if (D != 64 && D != 128) return RA_ERR_UNSUPPORTED;
  const int64_t dm = H * D;
  if (dm != 256 && dm != 512 && dm != 1024 && dm != 2048 && dm != 4096) return RA_ERR_UNSUPPORTED;
  if (N % S || N % 128) return RA_ERR_SHAPE;
  const int64_t L = N / S;
  if (L % q_chunk || L % k_chunk || q_chunk % 128 || k_chunk % 128) return RA_ERR_SHAPE;
  const int64_t T = B * N;
  if (T % ffn_chunk || ffn_chunk % 128 || d_ff % 128) return RA_ERR_SHAPE;
  if (B * H * N > (int64_t)INT32_MAX / 2 || d_ff > INT32_MAX / 4) return RA_ERR_UNSUPPORTED;
  return B == 0 ? kNoTokens : RA_OK;
}

GemmOperand plain(const void* p, int64_t rows, int64_t cols, int mn) {
  return GemmOperand{p, rows, cols, mn, 0, 0, 0, 0, 0};
}
GemmOperand split(const void* p, int64_t rows, int64_t cols, int mn, int64_t N, int64_t H, int64_t D) {
  return GemmOperand{p, rows, cols, mn, N, H, D, 0, 0};
}
GemmOut bf16_out(void* p, const void* residual = nullptr) {
  return GemmOut{p, residual ? kEpiBf16Res : kEpiBf16, 0, 0, 0, 0, residual, nullptr, nullptr};
}
GemmOut bf16_split_out(void* p, int64_t N, int64_t H, int64_t D) {
  return GemmOut{p, kEpiBf16, 0, N, H, D, nullptr, nullptr, nullptr};
}
GemmOut f32_out(float* p) { return GemmOut{p, kEpiF32, 0, 0, 0, 0, nullptr, nullptr, nullptr}; }

// Weight gradients [dm, dm] have few output tiles and a long K (all tokens):
// split K in two (two fp32 adds onto a zeroed output commute exactly) when
// the tiles alone would leave SMs idle in the last wave.
int wgrad_splits(int64_t dm, int64_t T) {
  const int64_t tiles = (dm / 128) * (dm / 256);
  return (tiles < 4 * 148 && T >= 1024) ? 2 : 1;
}

// Optional per-step timing marks: event i is recorded on the stream after
// step i (null array or null entries are skipped).
int mark(void* const* marks, int i, cudaStream_t st) {
  if (!marks || !marks[i]) return RA_OK;
  return cudaEventRecord(static_cast<cudaEvent_t>(marks[i]), st) == cudaSuccess ? RA_OK : RA_ERR_CUDA;
}

size_t bwd_ws_bytes(int64_t B, int64_t N, int64_t H, int64_t D, int64_t d_ff, int64_t ffn_chunk) {
  const size_t T = (size_t)B * N, dm = (size_t)(H * D), act = T * dm * 2;
  const size_t attn = bwd_workspace_bytes(B, H, N, D, bwd_fused_supported(D));
  return 7 * up256(act) + up256(attn) + up256(ffn_bwd_workspace_bytes(ffn_chunk, d_ff)) +
         up256(rmsnorm_dg_partial_floats((int64_t)T, (int64_t)dm) * 4);
}

}  // namespace

extern "C" {

size_t blockwise_layer_saved_size(int64_t B, int64_t N, int64_t H, int64_t D) {
  if (B <= 0 || N <= 0 || H <= 0 || D <= 0) return 0;
  return saved_bytes(B, N, H, D);
}

size_t blockwise_layer_fwd_workspace_size(int64_t ffn_chunk, int64_t d_ff) {
  if (ffn_chunk <= 0 || d_ff <= 0) return 0;
  return (size_t)ffn_chunk * d_ff * 2;
}

size_t blockwise_layer_bwd_workspace_size(int64_t B, int64_t N, int64_t H, int64_t D, int64_t d_ff,
                                          int64_t ffn_chunk) {
  if (B <= 0 || N <= 0 || H <= 0 || D <= 0 || d_ff <= 0 || ffn_chunk <= 0) return 0;
  return bwd_ws_bytes(B, N, H, D, d_ff, ffn_chunk);
}

int blockwise_layer_fwd(const void* x, const void* g_attn, const void* wq, const void* wk, const void* wv,
                        const void* wo, const void* g_ffn, const void* w1, const void* w2, const void* w3, void* y,
                        void* saved, size_t saved_size, int64_t B, int64_t N, int64_t H, int64_t D, int64_t d_ff,
                        int S, int q_chunk, int k_chunk, int causal, int ffn_chunk, float eps, void* workspace,
                        size_t workspace_bytes, void* const* marks, void* stream) {
  RA_NVTX_RANGE();
  int rc = check_layer(B, N, H, D, d_ff, S, q_chunk, k_chunk, ffn_chunk, causal);
  if (rc == kNoTokens) return RA_OK;  // no tokens: nothing to compute
  if (rc != RA_OK) return rc;
  if (!(eps > 0.f)) return RA_ERR_ARG;
  const void* ptrs[] = {x, g_attn, wq, wk, wv, wo, g_ffn, w1, w2, w3, y, saved, workspace};
  for (const void* p : ptrs)
    if (!p) return RA_ERR_ARG;
  for (const void* p : ptrs)
    if (!a16(p)) return RA_ERR_ALIGN;
  if (saved_size < saved_bytes(B, N, H, D)) return RA_ERR_WORKSPACE;
  if (workspace_bytes < blockwise_layer_fwd_workspace_size(ffn_chunk, d_ff)) return RA_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t T = B * N, dm = H * D;
  Saved s = carve_saved(saved, B, N, H, D);

  // steps (marks): 0 norm, 1 q/k/v projections, 2 attention, 3 output projection, 4 norm, 5 feed-forward
  if ((rc = launch_rmsnorm_fwd(x, g_attn, s.xn, s.rstd1, T, dm, eps, st)) != RA_OK) return rc;
  if ((rc = mark(marks, 0, st)) != RA_OK) return rc;
  const void* w_qkv[3] = {wq, wk, wv};
  __nv_bfloat16* d_qkv[3] = {s.q, s.k, s.v};
  for (int i = 0; i < 3; ++i) {
    GemmSeg g{plain(s.xn, T, dm, 0), plain(w_qkv[i], dm, dm, 0), dm};
    if ((rc = launch_gemm_tc(&g, 1, T, dm, bf16_split_out(d_qkv[i], N, H, D), 1, st)) != RA_OK) return rc;
  }
  if ((rc = mark(marks, 1, st)) != RA_OK) return rc;
  AttnArgs a{s.q, s.k, s.v, B, H, N, D, RA_BF16, S, q_chunk, k_chunk, causal, 1.0f / sqrtf((float)D), H};
  if ((rc = launch_fwd_tc(a, s.o, s.lse, nullptr, nullptr, -1, st)) != RA_OK) return rc;
  if ((rc = mark(marks, 2, st)) != RA_OK) return rc;
  {
    GemmSeg g{split(s.o, T, dm, 0, N, H, D), plain(wo, dm, dm, 0), dm};
    if ((rc = launch_gemm_tc(&g, 1, T, dm, bf16_out(s.x2, x), 1, st)) != RA_OK) return rc;
  }
  if ((rc = mark(marks, 3, st)) != RA_OK) return rc;
  if ((rc = launch_rmsnorm_fwd(s.x2, g_ffn, s.xn2, s.rstd2, T, dm, eps, st)) != RA_OK) return rc;
  if ((rc = mark(marks, 4, st)) != RA_OK) return rc;
  if ((rc = launch_ffn_tc(s.xn2, w1, w2, w3, y, T, dm, d_ff, ffn_chunk, workspace, st, s.x2)) != RA_OK) return rc;
  return mark(marks, 5, st);
}

int blockwise_layer_bwd(const void* x, const void* g_attn, const void* wq, const void* wk, const void* wv,
                        const void* wo, const void* g_ffn, const void* w1, const void* w2, const void* w3,
                        const void* saved, size_t saved_size, const void* dy, void* dx, float* dg_attn, float* dwq,
                        float* dwk, float* dwv, float* dwo, float* dg_ffn, float* dw1, float* dw2, float* dw3,
                        int64_t B, int64_t N, int64_t H, int64_t D, int64_t d_ff, int S, int q_chunk, int k_chunk,
                        int causal, int ffn_chunk, void* workspace, size_t workspace_bytes, void* const* marks,
                        void* stream) {
  RA_NVTX_RANGE();
  int rc = check_layer(B, N, H, D, d_ff, S, q_chunk, k_chunk, ffn_chunk, causal);
  if (rc == kNoTokens) {  // no tokens: every parameter gradient is zero
    const size_t dm = (size_t)(H * D), ff = (size_t)d_ff;
    float* grads[] = {dg_attn, dwq, dwk, dwv, dwo, dg_ffn, dw1, dw2, dw3};
    const size_t n[] = {dm, dm * dm, dm * dm, dm * dm, dm * dm, dm, ff * dm, dm * ff, ff * dm};
    for (int i = 0; i < 9; ++i) {
      if (!grads[i]) return RA_ERR_ARG;
      if (!a16(grads[i])) return RA_ERR_ALIGN;
    }
    for (int i = 0; i < 9; ++i)
      if (cudaMemsetAsync(grads[i], 0, n[i] * 4, static_cast<cudaStream_t>(stream)) != cudaSuccess) return RA_ERR_CUDA;
    return RA_OK;
  }
  if (rc != RA_OK) return rc;
  const void* ptrs[] = {x,   g_attn, wq,  wk,  wv,     wo,  g_ffn, w1,  w2,  w3,       saved,
                        dy,  dx,     dg_attn, dwq, dwk, dwv, dwo, dg_ffn, dw1, dw2, dw3, workspace};
  for (const void* p : ptrs)
    if (!p) return RA_ERR_ARG;
  for (const void* p : ptrs)
    if (!a16(p)) return RA_ERR_ALIGN;
  if (saved_size < saved_bytes(B, N, H, D)) return RA_ERR_WORKSPACE;
  if (workspace_bytes < bwd_ws_bytes(B, N, H, D, d_ff, ffn_chunk)) return RA_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t T = B * N, dm = H * D;
  const Saved s = carve_saved(const_cast<void*>(saved), B, N, H, D);
  Carve c{static_cast<uint8_t*>(workspace)};
  const size_t act = (size_t)T * dm * 2;
  auto* dxn2 = c.take<__nv_bfloat16>(act);
  auto* dx2 = c.take<__nv_bfloat16>(act);
  auto* dO = c.take<__nv_bfloat16>(act);
  auto* dq = c.take<__nv_bfloat16>(act);
  auto* dk = c.take<__nv_bfloat16>(act);
  auto* dv = c.take<__nv_bfloat16>(act);
  auto* dxn = c.take<__nv_bfloat16>(act);
  const size_t ws_attn_bytes = bwd_workspace_bytes(B, H, N, D, bwd_fused_supported(D));
  void* ws_attn = c.take<uint8_t>(ws_attn_bytes);
  void* ws_ffn = c.take<uint8_t>(ffn_bwd_workspace_bytes(ffn_chunk, d_ff));
  float* partial = c.take<float>(rmsnorm_dg_partial_floats(T, dm) * 4);

  // steps (marks): 0 feed-forward, 1 norm, 2 dO, 3 dWo, 4-6 attention (preprocess; main pass or passes;
  // dQ conversion or the query-stationary pass), 7 dxn, 8 dWq/dWk/dWv, 9 norm
  // feed-forward half: y = x2 + ffn(xn2)
  if ((rc = launch_ffn_bwd_tc(s.xn2, w1, w2, w3, dy, dxn2, dw1, dw2, dw3, T, dm, d_ff, ffn_chunk, ws_ffn, st)) !=
      RA_OK)
    return rc;
  if ((rc = mark(marks, 0, st)) != RA_OK) return rc;
  if ((rc = launch_rmsnorm_bwd(s.x2, g_ffn, s.rstd2, dxn2, dy, dx2, dg_ffn, partial, T, dm, st)) != RA_OK) return rc;
  if ((rc = mark(marks, 1, st)) != RA_OK) return rc;
  // attention half: x2 = x + o Wo^T
  {
    GemmSeg g{plain(dx2, T, dm, 0), plain(wo, dm, dm, 1), dm};  // dO = dx2 Wo
    if ((rc = launch_gemm_tc(&g, 1, T, dm, bf16_split_out(dO, N, H, D), 1, st)) != RA_OK) return rc;
  }
  if ((rc = mark(marks, 2, st)) != RA_OK) return rc;
  {
    GemmSeg g{plain(dx2, T, dm, 1), split(s.o, T, dm, 1, N, H, D), T};  // dWo = dx2^T o
    if ((rc = launch_gemm_tc(&g, 1, dm, dm, f32_out(dwo), wgrad_splits(dm, T), st)) != RA_OK) return rc;
  }
  if ((rc = mark(marks, 3, st)) != RA_OK) return rc;
  AttnArgs a{s.q, s.k, s.v, B, H, N, D, RA_BF16, S, q_chunk, k_chunk, causal, 1.0f / sqrtf((float)D), H};
  {
    // the default backward's phases, one mark after each
    const int all = bwd_default_phases(D);
    const int phases[3] = {kPhasePre, all & (kPhaseKV | kPhaseFused), all & (kPhaseQ | kPhaseConvert)};
    for (int i = 0; i < 3; ++i) {
      if ((rc = launch_bwd_tc(a, s.o, s.lse, dO, dq, dk, dv, ws_attn, ws_attn_bytes, phases[i], st)) != RA_OK)
        return rc;
      if ((rc = mark(marks, 4 + i, st)) != RA_OK) return rc;
    }
  }
  {
    // dxn = dq Wq + dk Wk + dv Wv (one accumulation over three K ranges)
    GemmSeg g[3] = {{split(dq, T, dm, 0, N, H, D), plain(wq, dm, dm, 1), dm},
                    {split(dk, T, dm, 0, N, H, D), plain(wk, dm, dm, 1), dm},
                    {split(dv, T, dm, 0, N, H, D), plain(wv, dm, dm, 1), dm}};
    if ((rc = launch_gemm_tc(g, 3, T, dm, bf16_out(dxn), 1, st)) != RA_OK) return rc;
  }
  if ((rc = mark(marks, 7, st)) != RA_OK) return rc;
  const __nv_bfloat16* gq[3] = {dq, dk, dv};
  float* gw[3] = {dwq, dwk, dwv};
  for (int i = 0; i < 3; ++i) {
    GemmSeg g{split(gq[i], T, dm, 1, N, H, D), plain(s.xn, T, dm, 1), T};  // dW = d(q|k|v)^T xn
    if ((rc = launch_gemm_tc(&g, 1, dm, dm, f32_out(gw[i]), wgrad_splits(dm, T), st)) != RA_OK) return rc;
  }
  if ((rc = mark(marks, 8, st)) != RA_OK) return rc;
  if ((rc = launch_rmsnorm_bwd(x, g_attn, s.rstd1, dxn, dx2, dx, dg_attn, partial, T, dm, st)) != RA_OK) return rc;
  return mark(marks, 9, st);
}

}  // extern "C"
