// Blockwise SwiGLU feed-forward on the sm_100a tensor cores.
//
// "Ring Attention with Blockwise Transformers for Near-Infinite Context",
// abstract: the feed-forward is computed blockwise like the attention.  The
// token sequence is cut into chunks; for each chunk c
//   h_c = silu(x_c w1^T) * (x_c w3^T)      (gate/up GEMM, fused SwiGLU)
//   y_c = h_c w2^T                         (down GEMM)
// so only one chunk's hidden activation [chunk, d_ff] (the workspace) exists
// at a time.  silu(z) = z / (1 + e^-z).
//
// One tcgen05 GEMM kernel, C[M,N] = A[M,K] B[N,K]^T with both operands
// K-major (row-major activations, [out,in] weights), 128-row output tiles
// accumulated in tensor memory:
//   kGateUp: two B operands (w1 and w3 tiles of the same rows), two TMEM
//            accumulators, epilogue silu(g) * u -> bf16 h
//   kDown:   one B operand, epilogue -> bf16 y
// Warp roles: warp 0 TMA producer (4-stage ring of 64-wide K slabs), warp 1
// MMA issuer, warp 2 TMEM allocator, warps 4-7 epilogue (one thread per
// output row = TMEM lane).
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace ra {
namespace {

constexpr int kBM = 128;
constexpr int kBK = 64;       // one 128-byte swizzle slab of bf16
constexpr int kStages = 4;
constexpr int kThreads = 256;

enum Mode { kGateUp = 0, kDown = 1 };

template <int MODE, int BN>
struct GLayout {
  static constexpr int kNumB = (MODE == kGateUp) ? 2 : 1;
  static constexpr int kABytes = kBM * kBK * 2;   // 16 KB
  static constexpr int kBBytes = BN * kBK * 2;
  static constexpr int kStageBytes = kABytes + kNumB * kBBytes;
  static constexpr int kBar = kStages * kStageBytes;
  static constexpr int kNumBars = 2 * kStages + 1;
  static constexpr int kTmemSlot = kBar + kNumBars * 8;
  static constexpr int kAbort = kTmemSlot + 4;
  static constexpr int kBytes = kAbort + 4;
  static constexpr uint32_t kTmemCols = (kNumB * BN <= 256) ? 256 : 512;
};

struct GParams {
  __nv_bfloat16* out;   // [M rows of this launch, ldo]
  const __nv_bfloat16* res;  // kDown: residual added to y (same layout as out), or null
  int a_row0;           // first row of A in its tensor map
  int ldo;              // output row pitch (elements)
  int K;                // reduction length
  int m_tiles;
  DevStatus st;
};

__device__ __forceinline__ float silu_f(float z) { return z / (1.f + __expf(-z)); }

template <int MODE, int BN>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
                   const __grid_constant__ CUtensorMap tmB1, const GParams p) {
  using LY = GLayout<MODE, BN>;
  extern __shared__ __align__(1024) uint8_t smem[];
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (smem_u32(smem) & 1023) {
    if (threadIdx.x == 0) atomicExch(p.st.word, (int)RA_ERR_ALIGN);
    return;
  }
  // Output tile: m fastest, so CTAs that run together share weight tiles in L2.
  const int mt = (int)(blockIdx.x % p.m_tiles);
  const int nt = (int)(blockIdx.x / p.m_tiles);
  const int kblocks = p.K / kBK;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + LY::kBar);
  uint64_t* bar_full = bars;
  uint64_t* bar_empty = bars + kStages;
  uint64_t* bar_done = bars + 2 * kStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + LY::kTmemSlot);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + LY::kAbort);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bar_full[s], 1);
      mbar_init(&bar_empty[s], 1);
    }
    mbar_init(bar_done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 2) {
    tmem_alloc(tmem_slot, LY::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tmA);
      tma_prefetch_desc(&tmB0);
      if (MODE == kGateUp) tma_prefetch_desc(&tmB1);
      for (int kb = 0; kb < kblocks; ++kb) {
        const int s = kb % kStages;
        if (!mbar_wait(&bar_empty[s], ((kb / kStages) & 1) ^ 1, p.st, abort_flag)) break;
        uint8_t* st = smem + s * LY::kStageBytes;
        mbar_arrive_expect_tx(&bar_full[s], LY::kStageBytes);
        tma_load_2d(st, &tmA, &bar_full[s], kb * kBK, p.a_row0 + mt * kBM);
        tma_load_2d(st + LY::kABytes, &tmB0, &bar_full[s], kb * kBK, nt * BN);
        if (MODE == kGateUp) tma_load_2d(st + LY::kABytes + LY::kBBytes, &tmB1, &bar_full[s], kb * kBK, nt * BN);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(kBM, BN, false, false);
      const uint32_t base = smem_u32(smem);
      for (int kb = 0; kb < kblocks; ++kb) {
        const int s = kb % kStages;
        if (!mbar_wait(&bar_full[s], (kb / kStages) & 1, p.st, abort_flag)) break;
        tc_fence_after();
        const uint32_t a = base + s * LY::kStageBytes;
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk) {
          const uint64_t ad = sdesc_sw128(a + kk * 32, 16, 1024);
#pragma unroll
          for (int b = 0; b < LY::kNumB; ++b) {
            const uint64_t bd = sdesc_sw128(a + LY::kABytes + b * LY::kBBytes + kk * 32, 16, 1024);
            mma_bf16_ss(tmem + b * BN, ad, bd, idesc, (kb > 0 || kk > 0) ? 1u : 0u);
          }
        }
        mma_commit(&bar_empty[s]);
      }
      mma_commit(bar_done);
    }
  } else if (warp >= 4) {
    const int r = (warp - 4) * 32 + lane;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    if (__all_sync(0xffffffffu, mbar_wait(bar_done, 0, p.st, abort_flag))) {
      tc_fence_after();
      __nv_bfloat16* orow = p.out + (size_t)(mt * kBM + r) * p.ldo + (size_t)nt * BN;
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t g[32];
        tmem_ld32(tmem + lane_off + c * 32, g);
        uint32_t pk[16];
        if (MODE == kGateUp) {
          uint32_t u[32];
          tmem_ld32(tmem + lane_off + BN + c * 32, u);
          tmem_ld_wait();
#pragma unroll
          for (int x = 0; x < 16; ++x) {
            const float h0 = silu_f(__uint_as_float(g[2 * x])) * __uint_as_float(u[2 * x]);
            const float h1 = silu_f(__uint_as_float(g[2 * x + 1])) * __uint_as_float(u[2 * x + 1]);
            pk[x] = pack_bf16x2(h0, h1);
          }
        } else {
          tmem_ld_wait();
          if (p.res) {  // y = residual + h w2^T, rounded once
            const uint4* rr = reinterpret_cast<const uint4*>(p.res + (size_t)(mt * kBM + r) * p.ldo +
                                                             (size_t)nt * BN + c * 32);
#pragma unroll
            for (int x = 0; x < 4; ++x) {
              const uint4 q = rr[x];
              const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int i = 8 * x + 2 * e;
                pk[4 * x + e] = pack_bf16x2(__uint_as_float(g[i]) + __uint_as_float(w[e] << 16),
                                            __uint_as_float(g[i + 1]) + __uint_as_float(w[e] & 0xffff0000u));
              }
            }
          } else {
#pragma unroll
            for (int x = 0; x < 16; ++x)
              pk[x] = pack_bf16x2(__uint_as_float(g[2 * x]), __uint_as_float(g[2 * x + 1]));
          }
        }
        uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
        for (int x = 0; x < 4; ++x) dst[x] = make_uint4(pk[4 * x], pk[4 * x + 1], pk[4 * x + 2], pk[4 * x + 3]);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, LY::kTmemCols);
  }
}

template <int MODE, int BN>
int launch_gemm(const CUtensorMap& ta, const CUtensorMap& tb0, const CUtensorMap& tb1, __nv_bfloat16* out,
                int a_row0, int ldo, int M, int N, int K, const DevStatus& st, cudaStream_t stream,
                const __nv_bfloat16* res = nullptr) {
  using LY = GLayout<MODE, BN>;
  static_assert(LY::kBytes <= 232448, "GEMM stages exceed shared memory");
  GParams p{};
  p.out = out;
  p.res = res;
  p.a_row0 = a_row0;
  p.ldo = ldo;
  p.K = K;
  p.m_tiles = M / kBM;
  p.st = st;
  auto kern = gemm_tc_kernel<MODE, BN>;
  if (set_smem_attr((const void*)kern, LY::kBytes) != RA_OK) return RA_ERR_CUDA;
  const unsigned grid = (unsigned)((M / kBM) * (N / BN));
  kern<<<grid, kThreads, LY::kBytes, stream>>>(ta, tb0, tb1, p);
  return cudaGetLastError() == cudaSuccess ? RA_OK : RA_ERR_CUDA;
}

}  // namespace

int launch_ffn_tc(const void* x, const void* w1, const void* w2, const void* w3, void* y, int64_t T,
                  int64_t d_model, int64_t d_ff, int64_t chunk, void* workspace, cudaStream_t stream,
                  const void* residual) {
  constexpr int kBNUp = 128;    // per weight: two 128-column accumulators
  constexpr int kBNDown = 128;
  if (d_ff % kBNUp || d_model % kBNDown || d_model % kBK || d_ff % kBK || chunk % kBM) return RA_ERR_SHAPE;
  if (T > INT32_MAX || d_ff > INT32_MAX) return RA_ERR_UNSUPPORTED;
  DevStatus st;
  int rc = current_status(&st);
  if (rc != RA_OK) return rc;
  __nv_bfloat16* h = static_cast<__nv_bfloat16*>(workspace);
  alignas(64) CUtensorMap tx, tw1, tw3, th, tw2;
  if (make_tmap_bf16_2d(&tx, x, d_model, T, d_model * 2, kBK, kBM) != RA_OK) return RA_ERR_CUDA;
  if (make_tmap_bf16_2d(&tw1, w1, d_model, d_ff, d_model * 2, kBK, kBNUp) != RA_OK) return RA_ERR_CUDA;
  if (make_tmap_bf16_2d(&tw3, w3, d_model, d_ff, d_model * 2, kBK, kBNUp) != RA_OK) return RA_ERR_CUDA;
  if (make_tmap_bf16_2d(&th, h, d_ff, chunk, d_ff * 2, kBK, kBM) != RA_OK) return RA_ERR_CUDA;
  if (make_tmap_bf16_2d(&tw2, w2, d_ff, d_model, d_ff * 2, kBK, kBNDown) != RA_OK) return RA_ERR_CUDA;
  __nv_bfloat16* yb = static_cast<__nv_bfloat16*>(y);
  for (int64_t c0 = 0; c0 < T; c0 += chunk) {
    rc = launch_gemm<kGateUp, kBNUp>(tx, tw1, tw3, h, (int)c0, (int)d_ff, (int)chunk, (int)d_ff, (int)d_model, st,
                                     stream);
    if (rc != RA_OK) return rc;
    const __nv_bfloat16* res =
        residual ? static_cast<const __nv_bfloat16*>(residual) + c0 * d_model : nullptr;
    rc = launch_gemm<kDown, kBNDown>(th, tw2, tw2, yb + c0 * d_model, 0, (int)d_model, (int)chunk, (int)d_model,
                                     (int)d_ff, st, stream, res);
    if (rc != RA_OK) return rc;
  }
  return RA_OK;
}

}  // namespace ra
