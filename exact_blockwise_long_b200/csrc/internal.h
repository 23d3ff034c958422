// Internal launch interface between the C ABI (abi.cu) and the kernel files.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <nvtx3/nvToolsExt.h>

#include "ringattn.h"

namespace ra {

// An NVTX range over one ABI call's host-side work (argument checks and the
// enqueue of its kernels), named after the call; visible in profilers that
// attach an NVTX collector, free otherwise.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};
#define RA_NVTX_RANGE() const ::ra::NvtxRange ra_nvtx_range_(__func__)

struct DevStatus;

// Status word of the current device plus the bounded-wait limit.  Returns
// RA_OK or RA_ERR_CUDA.
int current_status(DevStatus* out);

struct AttnArgs {
  const void* q;
  const void* k;
  const void* v;
  int64_t B, H, N, D;
  int dtype;
  int S, q_chunk, k_chunk, causal;
  float scale;  // already resolved (> 0)
  int64_t Hkv;  // key/value heads; query head h reads key/value head h / (H / Hkv)
};

// Exact fp32 CUDA-core ring forward (whole ring, or one step merged into
// fp32 accumulators when step >= 0).  Inputs fp32 or bf16.
int launch_fwd_simt(const AttnArgs& a, void* out, float* lse, float* o_acc, float* lse_acc, int step,
                    cudaStream_t stream);

// tcgen05 ring forward, bf16 inputs (whole ring, or one step merged into
// fp32 accumulators when step >= 0).
int launch_fwd_tc(const AttnArgs& a, void* out, float* lse, float* o_acc, float* lse_acc, int step,
                  cudaStream_t stream);

// Name of the forward kernel launch_fwd_tc runs for shard length L and
// head dimension D on the current device (nullptr for an unsupported D).
const char* fwd_tc_kernel_name(int64_t L, int64_t D);

// Names of the kernels the default backward (ringattn_bwd) launches for
// head dimension D, joined by '+' (nullptr for an unsupported D).
const char* bwd_tc_kernel_names(int64_t D);

int launch_merge(float* o_a, float* lse_a, const float* o_b, const float* lse_b, int64_t rows, int64_t D,
                 cudaStream_t stream);

// Backward phases (bits of phase_mask):
//   kPhasePre      D_i, lse_i*log2e into the workspace; zeroes the fp32 dQ
//                  accumulator when the workspace holds one
//   kPhaseKV       key/value-stationary pass writing dk, dv    } deterministic
//   kPhaseQ        query-stationary pass writing dq            } split backward
//   kPhaseFused    one key/value-stationary pass writing dk, dv and adding
//                  dQ into the fp32 accumulator (D = 128)
//   kPhaseConvert  dq = bf16(scale * accumulator)
enum BwdPhase { kPhasePre = 1, kPhaseKV = 2, kPhaseQ = 4, kPhaseFused = 8, kPhaseConvert = 16, kPhaseAll = 31 };
bool bwd_fused_supported(int64_t D);
// Workspace bytes: two fp32 row vectors [B*H*N], each 256-byte aligned, then
// (fused) the fp32 dQ accumulator [B*H*N, D].
size_t bwd_workspace_bytes(int64_t B, int64_t H, int64_t N, int64_t D, bool fused);
// Phases of the default backward for head dimension D.
int bwd_default_phases(int64_t D);
int launch_bwd_tc(const AttnArgs& a, const void* out, const float* lse, const void* dout, void* dq, void* dk,
                  void* dv, void* workspace, size_t workspace_bytes, int phase_mask, cudaStream_t stream);

// One shard pair's gradient into fp32 accumulators (ringattn_bwd_pair):
// a.N is the pair's block length, a.S = 1, a.causal the diagonal mask; prep
// holds the query block's two row vectors (kPhasePre output).
int launch_bwd_pair(const AttnArgs& a, const void* dout, const void* prep, float* dq_acc, float* dk_acc,
                    float* dv_acc, int kv_add, cudaStream_t stream);

// Argument checks of the backward entry points (abi.cu), everything but the
// workspace: RA_OK, kBwdEmpty (a valid empty problem: nothing to launch) or
// a negative ra_status.  run_bwd launches the phases after the checks.
constexpr int kBwdEmpty = 1;
int check_bwd_args(const void* q, const void* k, const void* v, const void* out, const float* lse, const void* dout,
                   const void* dq, const void* dk, const void* dv, int64_t B, int64_t H, int64_t Hkv, int64_t N,
                   int64_t D, int dtype, int S, int q_chunk, int k_chunk, int causal, int phase_mask);
int run_bwd(const void* q, const void* k, const void* v, const void* out, const float* lse, const void* dout,
            void* dq, void* dk, void* dv, int64_t B, int64_t H, int64_t Hkv, int64_t N, int64_t D, int S,
            int q_chunk, int k_chunk, int causal, float scale, void* workspace, size_t workspace_bytes,
            int phase_mask, void* stream);

// Blockwise SwiGLU FFN on the tensor cores.
// residual: optional bf16 [T, d_model] added to y before its rounding.
int launch_ffn_tc(const void* x, const void* w1, const void* w2, const void* w3, void* y, int64_t T,
                  int64_t d_model, int64_t d_ff, int64_t chunk, void* workspace, cudaStream_t stream,
                  const void* residual = nullptr);

// Decode: splits of the key/value cache (S shards of ceil(N/S) keys, each
// cut into pieces of at most k_chunk keys) and the launch.
int decode_splits(int64_t N, int S, int k_chunk);
int launch_decode(const void* q, const void* k, const void* v, void* out, float* lse, int64_t B, int64_t H,
                  int64_t Hkv, int64_t N, int64_t D, int S, int k_chunk, float scale, void* workspace,
                  cudaStream_t stream);

// Blockwise SwiGLU FFN backward: workspace (dg, du, h of one chunk) and launch.
size_t ffn_bwd_workspace_bytes(int64_t chunk, int64_t d_ff);
int launch_ffn_bwd_tc(const void* x, const void* w1, const void* w2, const void* w3, const void* dy, void* dx,
                      float* dw1, float* dw2, float* dw3, int64_t T, int64_t d_model, int64_t d_ff, int64_t chunk,
                      void* workspace, cudaStream_t stream);

// Generic bf16 GEMM (csrc/gemm_tc.cu): D[M,N] = sum_s A_s[M,K_s] B_s[N,K_s]^T.
// An operand is a logical row-major bf16 matrix [rows, cols]: K-major
// (rows index M or N, cols index K) or MN-major (rows index K, cols index M
// or N).  With hs_ntok > 0 the logical [batch*hs_ntok, hs_heads*hs_d] matrix
// is stored head-split as [batch, hs_heads, hs_ntok, hs_d].  (r0, c0) is the
// operand's origin inside the logical matrix.
struct GemmOperand {
  const void* ptr;
  int64_t rows, cols;
  int mn_major;
  int64_t hs_ntok, hs_heads, hs_d;
  int64_t r0, c0;
};
struct GemmSeg {
  GemmOperand a, b;
  int64_t K;
};
// Epilogues of launch_gemm_tc (see csrc/gemm_tc.cu).
enum GemmEpi { kEpiBf16 = 0, kEpiBf16Res = 1, kEpiF32 = 2, kEpiSwiGLU = 3, kEpiSwiGLUBwd = 4 };
struct GemmOut {
  void* ptr;                        // [M, N] (bf16: plain or head-split; fp32: plain)
  int epi;                          // GemmEpi
  int add;                          // kEpiF32: add into the existing values
  int64_t hs_ntok, hs_heads, hs_d;  // bf16 head-split output
  const void* aux;                  // kEpiBf16Res: bf16 residual [M, N]; kEpiSwiGLUBwd: fp32 dh [M, N]
  void* ptr2;                       // kEpiSwiGLUBwd: du (ptr: dg)
  void* ptr3;                       // kEpiSwiGLUBwd: h
};
// M % 128 == 0, K_s % 64 == 0, N % 128 == 0 (N % 256 == 0 with head-split
// output or B); the last N tile may be half full (TMA fills and clips).
// kEpiSwiGLU / kEpiSwiGLUBwd: two segments with the same A and K, B_0 = w1,
// B_1 = w3 (K-major), N = d_ff (output width).  splits 1 or 2 (2: kEpiF32
// only, K split across two CTAs that each add onto a zeroed output).
int launch_gemm_tc(const GemmSeg* segs, int nseg, int64_t M, int64_t N, const GemmOut& out, int splits,
                   cudaStream_t stream);

// RMS normalisation (csrc/rmsnorm.cu) of rows of d_model bf16 values
// (d_model = 256 * {1,2,4,8,16}): out = x * rstd * g, rstd = (mean(x^2) + eps)^-1/2.
int launch_rmsnorm_fwd(const void* x, const void* g, void* out, float* rstd, int64_t T, int64_t d_model, float eps,
                       cudaStream_t stream);
// dx = dres + rstd (g*dxn - xhat mean(g*dxn*xhat)), xhat = x rstd (dres may be null);
// dg = sum over rows of dxn * xhat (fp32), through `partial` scratch of
// rmsnorm_dg_partial_floats(T, d_model) floats.
int launch_rmsnorm_bwd(const void* x, const void* g, const float* rstd, const void* dxn, const void* dres, void* dx,
                       float* dg, float* partial, int64_t T, int64_t d_model, cudaStream_t stream);
size_t rmsnorm_dg_partial_floats(int64_t T, int64_t d_model);

// acc[i] += x[i] (x of dtype RA_BF16 or RA_F32); out[i] = x[i] rounded to dtype (csrc/elementwise.cu).
int launch_accumulate(float* acc, const void* x, int64_t n, int dtype, cudaStream_t stream);
int launch_cast(const float* x, void* out, int64_t n, int dtype, cudaStream_t stream);

int launch_selftest_timeout(int timeout_us, cudaStream_t stream);

// cuTensorMapEncodeTiled through the runtime's driver entry point.
// 2-D bf16 map over a row-major [rows, inner] matrix with the given row
// pitch, box [box_rows, box_inner], 128-byte swizzle.
int make_tmap_bf16_2d(void* tmap /* CUtensorMap* */, const void* base, uint64_t inner, uint64_t rows,
                      uint64_t row_pitch_bytes, uint32_t box_inner, uint32_t box_rows);

// The same for a 2-D fp32 map (box inner extent at most 32 elements).
// 3-D map over a [rows x D] bf16 tensor whose box is one row-tile of box_rows
// rows with all D / 64 slabs (for tma_load_tile).
int make_tmap_bf16_tile(void* tmap /* CUtensorMap* */, const void* base, uint64_t D, uint64_t rows,
                        uint32_t box_rows);
int make_tmap_f32_2d(void* tmap /* CUtensorMap* */, const void* base, uint64_t inner, uint64_t rows,
                     uint64_t row_pitch_bytes, uint32_t box_inner, uint32_t box_rows);

// Head-group size for grouped_order: as many heads as keep their working
// set (bytes_per_head) within budget_bytes of the 126 MB L2, but enough that
// a group holds two waves of work items; at least one, at most `heads`.
int head_group(int per_head, int heads, double bytes_per_head, double budget_bytes);

// Opt a kernel into more than 48 KB of dynamic shared memory.
int set_smem_attr(const void* func, int bytes);

}  // namespace ra
