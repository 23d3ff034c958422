// Backward of the blockwise SwiGLU feed-forward on the sm_100a tensor cores.
//
// The paper abstract pairs blockwise attention with a blockwise feed-forward
// for training; this is the chain rule through
//   g = x w1^T,  u = x w3^T,  h = silu(g) * u,  y = h w2^T
// with silu(g) = g s, s = 1 / (1 + e^-g), silu'(g) = s (1 + g (1 - s)):
//   dh = dy w2,  du = dh * silu(g),  dg = dh * u * silu'(g)
//   dx = dg w1 + du w3,  dw1 = dg^T x,  dw3 = du^T x,  dw2 = dy^T h
// taken chunk by chunk (only one chunk's g, u, dh, dg, du, h exist at a time;
// g and u are recomputed), the weight gradients summed over the chunks in
// fp32.
//
// Four launches per chunk, one tcgen05 GEMM kernel with 128 x 128 output
// tiles and 64-deep K steps, in four modes:
//   kSwiGLUBwd  g, u (x . w1^T, x . w3^T) and dh (dy . w2) in three TMEM
//               accumulators; epilogue writes dg, du and h (bf16)
//   kDx         dx = dg w1 + du w3: one accumulator over both K halves
//   kDw13       dw1, dw3 = dg^T x, du^T x: two accumulators sharing x
//   kDw2        dw2 = dy^T h
// Operands are K-major (rows of the activations, [out, in] weight rows) or
// MN-major (an operand used transposed); both come in by TMA with the
// 128-byte swizzle, 16 KB per 128 x 64 tile.  Results leave by TMA too:
// bf16 tiles as stores, fp32 weight gradients as a store on the first chunk
// and an element-wise TMA add on the later ones (one add per element per
// launch, in stream order, so the sums are deterministic).
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace ra {
namespace {

constexpr int kBM = 128, kBN = 128, kBK = 64;
constexpr int kThreads = 256;
constexpr int kTile = 16384;  // one 128 x 64 bf16 operand tile (either major)

enum BMode { kSwiGLUBwd = 0, kDx = 1, kDw13 = 2, kDw2 = 3 };

template <int MODE>
struct BCfg;
template <>
struct BCfg<kSwiGLUBwd> {
  static constexpr int nA = 2, nB = 3, nAcc = 3, stages = 2;
  static constexpr bool a_mn = false;
  static constexpr bool b_mn(int b) { return b == 2; }
};
template <>
struct BCfg<kDx> {
  static constexpr int nA = 1, nB = 1, nAcc = 1, stages = 6;
  static constexpr bool a_mn = false;
  static constexpr bool b_mn(int) { return true; }
};
template <>
struct BCfg<kDw13> {
  static constexpr int nA = 2, nB = 1, nAcc = 2, stages = 4;
  static constexpr bool a_mn = true;
  static constexpr bool b_mn(int) { return true; }
};
template <>
struct BCfg<kDw2> {
  static constexpr int nA = 1, nB = 1, nAcc = 1, stages = 6;
  static constexpr bool a_mn = true;
  static constexpr bool b_mn(int) { return true; }
};

template <int MODE>
struct BLay {
  using C = BCfg<MODE>;
  static constexpr int kStage = (C::nA + C::nB) * kTile;
  static constexpr int kBar = C::stages * kStage;
  static constexpr int kTmemSlot = kBar + (2 * C::stages + 1) * 8;
  static constexpr int kAbort = kTmemSlot + 4;
  static constexpr int kBytes = kAbort + 4;
  static constexpr int kAlloc = kBytes + 1024;
  static constexpr uint32_t kTmemCols = C::nAcc * kBN <= 256 ? 256 : 512;
};

struct BGParams {
  int out_row;            // first output row of this launch (dx: the chunk's first token)
  int accumulate;         // weight gradients: add into the fp32 output (0 on the first chunk)
  int a_off[2], b_off[3]; // K-major: first row; MN-major: first K index
  int kblocks;            // 64-deep K steps
  int kb_split;           // kDx: K step where (dg, w1) hand over to (du, w3)
  int m_tiles;
  DevStatus st;
};

// one 16 KB operand tile for K step kb: K-major -> one box of 64 K x 128
// rows; MN-major -> two boxes of 64 MN x 64 K rows (slabs of 8 KB)
template <bool MN>
__device__ __forceinline__ void load_operand(uint8_t* dst, const CUtensorMap* map, uint64_t* bar, int tile_mn,
                                             int off, int kb) {
  if (MN) {
    tma_load_2d(dst, map, bar, tile_mn * 128, off + kb * kBK);
    tma_load_2d(dst + 8192, map, bar, tile_mn * 128 + 64, off + kb * kBK);
  } else {
    tma_load_2d(dst, map, bar, kb * kBK, off + tile_mn * 128);
  }
}

template <bool MN>
__device__ __forceinline__ uint64_t operand_desc(uint32_t tile, int kk) {
  return MN ? sdesc_sw128(tile + kk * 2048, 8192, 1024) : sdesc_sw128(tile + kk * 32, 16, 1024);
}

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    ffn_bwd_gemm_kernel(const __grid_constant__ CUtensorMap tA0, const __grid_constant__ CUtensorMap tA1,
                        const __grid_constant__ CUtensorMap tB0, const __grid_constant__ CUtensorMap tB1,
                        const __grid_constant__ CUtensorMap tB2, const __grid_constant__ CUtensorMap tO0,
                        const __grid_constant__ CUtensorMap tO1, const __grid_constant__ CUtensorMap tO2,
                        const BGParams p) {
  using C = BCfg<MODE>;
  using LY = BLay<MODE>;
  extern __shared__ uint8_t smem_fb[];
  uint8_t* smem = smem_fb + ((1024 - (smem_u32(smem_fb) & 1023)) & 1023);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int mt = (int)(blockIdx.x % p.m_tiles);
  const int nt = (int)(blockIdx.x / p.m_tiles);

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + LY::kBar);
  uint64_t* bar_full = bars;
  uint64_t* bar_empty = bars + C::stages;
  uint64_t* bar_done = bars + 2 * C::stages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + LY::kTmemSlot);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + LY::kAbort);

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::stages; ++s) {
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
      for (int kb = 0; kb < p.kblocks; ++kb) {
        const int s = kb % C::stages;
        if (!mbar_wait(&bar_empty[s], ((kb / C::stages) & 1) ^ 1, p.st, abort_flag)) break;
        uint8_t* st = smem + s * LY::kStage;
        mbar_arrive_expect_tx(&bar_full[s], LY::kStage);
        if constexpr (MODE == kDx) {
          const bool hi = kb >= p.kb_split;
          const int k = hi ? kb - p.kb_split : kb;
          load_operand<false>(st, hi ? &tA1 : &tA0, &bar_full[s], mt, p.a_off[0], k);
          load_operand<true>(st + kTile, hi ? &tB1 : &tB0, &bar_full[s], nt, 0, k);
        } else {
          load_operand<C::a_mn>(st, &tA0, &bar_full[s], mt, p.a_off[0], kb);
          if (C::nA > 1) load_operand<C::a_mn>(st + kTile, &tA1, &bar_full[s], mt, p.a_off[1], kb);
          uint8_t* bt = st + C::nA * kTile;
          load_operand<C::b_mn(0)>(bt, &tB0, &bar_full[s], nt, p.b_off[0], kb);
          if (C::nB > 1) load_operand<C::b_mn(1)>(bt + kTile, &tB1, &bar_full[s], nt, p.b_off[1], kb);
          if (C::nB > 2) load_operand<C::b_mn(2)>(bt + 2 * kTile, &tB2, &bar_full[s], nt, p.b_off[2], kb);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t base = smem_u32(smem);
      for (int kb = 0; kb < p.kblocks; ++kb) {
        const int s = kb % C::stages;
        if (!mbar_wait(&bar_full[s], (kb / C::stages) & 1, p.st, abort_flag)) break;
        tc_fence_after();
        const uint32_t a0 = base + s * LY::kStage, b0 = a0 + C::nA * kTile;
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk) {
          const uint32_t acc = (kb > 0 || kk > 0) ? 1u : 0u;
          if constexpr (MODE == kSwiGLUBwd) {
            constexpr uint32_t idK = idesc_bf16_f32(kBM, kBN, false, false);
            constexpr uint32_t idM = idesc_bf16_f32(kBM, kBN, false, true);
            const uint64_t ax = operand_desc<false>(a0, kk), ady = operand_desc<false>(a0 + kTile, kk);
            mma_bf16_ss(tmem, ax, operand_desc<false>(b0, kk), idK, acc);                 // g
            mma_bf16_ss(tmem + kBN, ax, operand_desc<false>(b0 + kTile, kk), idK, acc);   // u
            mma_bf16_ss(tmem + 2 * kBN, ady, operand_desc<true>(b0 + 2 * kTile, kk), idM, acc);  // dh
          } else if constexpr (MODE == kDx) {
            constexpr uint32_t id = idesc_bf16_f32(kBM, kBN, false, true);
            mma_bf16_ss(tmem, operand_desc<false>(a0, kk), operand_desc<true>(b0, kk), id, acc);
          } else if constexpr (MODE == kDw13) {
            constexpr uint32_t id = idesc_bf16_f32(kBM, kBN, true, true);
            const uint64_t bx = operand_desc<true>(b0, kk);
            mma_bf16_ss(tmem, operand_desc<true>(a0, kk), bx, id, acc);                  // dw1
            mma_bf16_ss(tmem + kBN, operand_desc<true>(a0 + kTile, kk), bx, id, acc);    // dw3
          } else {
            constexpr uint32_t id = idesc_bf16_f32(kBM, kBN, true, true);
            mma_bf16_ss(tmem, operand_desc<true>(a0, kk), operand_desc<true>(b0, kk), id, acc);
          }
        }
        mma_commit(&bar_empty[s]);
      }
      mma_commit(bar_done);
    }
  } else if (warp >= 4) {
    // Epilogue: accumulator rows -> 128-byte-swizzled staging boxes in the
    // (now idle) pipeline buffers -> TMA stores (or TMA adds for the fp32
    // weight gradients after the first chunk).  One 16 KB box holds 128 rows
    // x 128 bytes: 64 bf16 or 32 fp32 columns.
    const int r = (warp - 4) * 32 + lane;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const bool ok = __all_sync(0xffffffffu, mbar_wait(bar_done, 0, p.st, abort_flag));
    if (ok) {
      tc_fence_after();
      const uint32_t row_base = smem_u32(smem) + (uint32_t)r * 128;
      const uint32_t sw = (uint32_t)(r & 7);
#pragma unroll 1
      for (int c = 0; c < kBN / 32; ++c) {
        if constexpr (MODE == kSwiGLUBwd) {
          uint32_t g[32], u[32], dh[32];
          tmem_ld32(tmem + lane_off + c * 32, g);
          tmem_ld32(tmem + lane_off + kBN + c * 32, u);
          tmem_ld32(tmem + lane_off + 2 * kBN + c * 32, dh);
          tmem_ld_wait();
          uint32_t pg[16], pu[16], ph[16];
#pragma unroll
          for (int x = 0; x < 16; ++x) {
            float dgv[2], duv[2], hv[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const float gg = __uint_as_float(g[2 * x + e]), uu = __uint_as_float(u[2 * x + e]);
              const float d = __uint_as_float(dh[2 * x + e]);
              const float sg = 1.f / (1.f + __expf(-gg));
              const float si = gg * sg;
              hv[e] = si * uu;
              duv[e] = d * si;
              dgv[e] = d * uu * (sg * (1.f + gg * (1.f - sg)));
            }
            pg[x] = pack_bf16x2(dgv[0], dgv[1]);
            pu[x] = pack_bf16x2(duv[0], duv[1]);
            ph[x] = pack_bf16x2(hv[0], hv[1]);
          }
#pragma unroll
          for (int o = 0; o < 3; ++o) {
            const uint32_t* src = o == 0 ? pg : (o == 1 ? pu : ph);
            const uint32_t box = row_base + (uint32_t)(o * 2 + (c >> 1)) * kTile;
#pragma unroll
            for (int x = 0; x < 4; ++x) {
              const uint32_t unit = (uint32_t)((c & 1) * 4 + x);
              st_shared_v4(box + ((unit ^ sw) << 4), src[4 * x], src[4 * x + 1], src[4 * x + 2], src[4 * x + 3]);
            }
          }
        } else if constexpr (MODE == kDx) {
          uint32_t a[32];
          tmem_ld32(tmem + lane_off + c * 32, a);
          tmem_ld_wait();
          uint32_t pk[16];
#pragma unroll
          for (int x = 0; x < 16; ++x) pk[x] = pack_bf16x2(__uint_as_float(a[2 * x]), __uint_as_float(a[2 * x + 1]));
          const uint32_t box = row_base + (uint32_t)(c >> 1) * kTile;
#pragma unroll
          for (int x = 0; x < 4; ++x) {
            const uint32_t unit = (uint32_t)((c & 1) * 4 + x);
            st_shared_v4(box + ((unit ^ sw) << 4), pk[4 * x], pk[4 * x + 1], pk[4 * x + 2], pk[4 * x + 3]);
          }
        } else {
#pragma unroll
          for (int o = 0; o < C::nAcc; ++o) {
            uint32_t a[32];
            tmem_ld32(tmem + lane_off + o * kBN + c * 32, a);
            tmem_ld_wait();
            const uint32_t box = row_base + (uint32_t)(o * 4 + c) * kTile;
#pragma unroll
            for (int x = 0; x < 8; ++x)
              st_shared_v4(box + (((uint32_t)x ^ sw) << 4), a[4 * x], a[4 * x + 1], a[4 * x + 2], a[4 * x + 3]);
          }
        }
      }
      fence_proxy_async_smem();
    }
    named_bar_sync(1, 128);
    if (threadIdx.x == 128 && ok) {
      const uint8_t* stage = smem;
      const int y = p.out_row + mt * kBM;
      if constexpr (MODE == kSwiGLUBwd || MODE == kDx) {
        constexpr int nOut = MODE == kSwiGLUBwd ? 3 : 1;
#pragma unroll
        for (int o = 0; o < nOut; ++o) {
          const CUtensorMap* m = o == 0 ? &tO0 : (o == 1 ? &tO1 : &tO2);
          tma_store_2d(m, stage + (o * 2) * kTile, nt * kBN, y);
          tma_store_2d(m, stage + (o * 2 + 1) * kTile, nt * kBN + 64, y);
        }
      } else {
#pragma unroll
        for (int o = 0; o < C::nAcc; ++o) {
          const CUtensorMap* m = o == 0 ? &tO0 : &tO1;
#pragma unroll
          for (int c = 0; c < kBN / 32; ++c) {
            if (p.accumulate)
              tma_add_2d(m, stage + (o * 4 + c) * kTile, nt * kBN + c * 32, y);
            else
              tma_store_2d(m, stage + (o * 4 + c) * kTile, nt * kBN + c * 32, y);
          }
        }
      }
      bulk_commit_group();
      bulk_wait_read_all();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, LY::kTmemCols);
  }
}

template <int MODE>
int launch_mode(const CUtensorMap* maps[8], const BGParams& p, int grid, cudaStream_t stream) {
  static_assert(BLay<MODE>::kAlloc <= 232448, "FFN backward stages exceed shared memory");
  // the epilogue's staging boxes live in the pipeline buffers
  constexpr int kStaging = MODE == kSwiGLUBwd ? 6 : (MODE == kDx ? 2 : 4 * BCfg<MODE>::nAcc);
  static_assert(kStaging * kTile <= BLay<MODE>::kBar, "epilogue staging exceeds the pipeline buffers");
  auto kern = ffn_bwd_gemm_kernel<MODE>;
  if (set_smem_attr((const void*)kern, BLay<MODE>::kAlloc) != RA_OK) return RA_ERR_CUDA;
  kern<<<grid, kThreads, BLay<MODE>::kAlloc, stream>>>(*maps[0], *maps[1], *maps[2], *maps[3], *maps[4], *maps[5],
                                                       *maps[6], *maps[7], p);
  return cudaGetLastError() == cudaSuccess ? RA_OK : RA_ERR_CUDA;
}

}  // namespace

size_t ffn_bwd_workspace_bytes(int64_t chunk, int64_t d_ff) { return (size_t)3 * chunk * d_ff * 2; }

int launch_ffn_bwd_tc(const void* x, const void* w1, const void* w2, const void* w3, const void* dy, void* dx,
                      float* dw1, float* dw2, float* dw3, int64_t T, int64_t d_model, int64_t d_ff, int64_t chunk,
                      void* workspace, cudaStream_t stream) {
  if (d_ff % 128 || d_model % 128 || chunk % 128 || T % chunk) return RA_ERR_SHAPE;
  if (T > INT32_MAX || d_ff > INT32_MAX) return RA_ERR_UNSUPPORTED;
  DevStatus st;
  int rc = current_status(&st);
  if (rc != RA_OK) return rc;
  __nv_bfloat16* dg = static_cast<__nv_bfloat16*>(workspace);
  __nv_bfloat16* du = dg + chunk * d_ff;
  __nv_bfloat16* h = du + chunk * d_ff;
  // K-major maps (box 64 K x 128 rows) and MN-major maps (box 64 MN x 64 K)
  alignas(64) CUtensorMap x_k, dy_k, w1_k, w3_k, dg_k, du_k;       // K-major
  alignas(64) CUtensorMap w2_m, w1_m, w3_m, x_m, dg_m, du_m, dy_m, h_m;  // MN-major
  alignas(64) CUtensorMap h_o, dx_o, dw1_o, dw3_o, dw2_o;               // output boxes
  int ok = RA_OK;
  ok |= make_tmap_bf16_2d(&h_o, h, d_ff, chunk, d_ff * 2, 64, 128);
  ok |= make_tmap_bf16_2d(&dx_o, dx, d_model, T, d_model * 2, 64, 128);
  ok |= make_tmap_f32_2d(&dw1_o, dw1, d_model, d_ff, d_model * 4, 32, 128);
  ok |= make_tmap_f32_2d(&dw3_o, dw3, d_model, d_ff, d_model * 4, 32, 128);
  ok |= make_tmap_f32_2d(&dw2_o, dw2, d_ff, d_model, d_ff * 4, 32, 128);
  ok |= make_tmap_bf16_2d(&x_k, x, d_model, T, d_model * 2, 64, 128);
  ok |= make_tmap_bf16_2d(&dy_k, dy, d_model, T, d_model * 2, 64, 128);
  ok |= make_tmap_bf16_2d(&w1_k, w1, d_model, d_ff, d_model * 2, 64, 128);
  ok |= make_tmap_bf16_2d(&w3_k, w3, d_model, d_ff, d_model * 2, 64, 128);
  ok |= make_tmap_bf16_2d(&dg_k, dg, d_ff, chunk, d_ff * 2, 64, 128);
  ok |= make_tmap_bf16_2d(&du_k, du, d_ff, chunk, d_ff * 2, 64, 128);
  ok |= make_tmap_bf16_2d(&w2_m, w2, d_ff, d_model, d_ff * 2, 64, 64);
  ok |= make_tmap_bf16_2d(&w1_m, w1, d_model, d_ff, d_model * 2, 64, 64);
  ok |= make_tmap_bf16_2d(&w3_m, w3, d_model, d_ff, d_model * 2, 64, 64);
  ok |= make_tmap_bf16_2d(&x_m, x, d_model, T, d_model * 2, 64, 64);
  ok |= make_tmap_bf16_2d(&dg_m, dg, d_ff, chunk, d_ff * 2, 64, 64);
  ok |= make_tmap_bf16_2d(&du_m, du, d_ff, chunk, d_ff * 2, 64, 64);
  ok |= make_tmap_bf16_2d(&dy_m, dy, d_model, T, d_model * 2, 64, 64);
  ok |= make_tmap_bf16_2d(&h_m, h, d_ff, chunk, d_ff * 2, 64, 64);
  if (ok != RA_OK) return RA_ERR_CUDA;
  const int ch = (int)chunk, dm = (int)d_model, df = (int)d_ff;
  for (int64_t c0 = 0; c0 < T; c0 += chunk) {
    const int c = (int)c0;
    {  // g, u, dh -> dg, du, h
      BGParams p{};
      p.a_off[0] = c;
      p.a_off[1] = c;
      p.kblocks = dm / kBK;
      p.m_tiles = ch / kBM;
      p.st = st;
      const CUtensorMap* maps[8] = {&x_k, &dy_k, &w1_k, &w3_k, &w2_m, &dg_k, &du_k, &h_o};
      if ((rc = launch_mode<kSwiGLUBwd>(maps, p, (ch / kBM) * (df / kBN), stream)) != RA_OK) return rc;
    }
    {  // dx = dg w1 + du w3
      BGParams p{};
      p.out_row = c;
      p.kblocks = 2 * (df / kBK);
      p.kb_split = df / kBK;
      p.m_tiles = ch / kBM;
      p.st = st;
      const CUtensorMap* maps[8] = {&dg_k, &du_k, &w1_m, &w3_m, &w3_m, &dx_o, &dx_o, &dx_o};
      if ((rc = launch_mode<kDx>(maps, p, (ch / kBM) * (dm / kBN), stream)) != RA_OK) return rc;
    }
    {  // dw1, dw3 (+)= dg^T x, du^T x
      BGParams p{};
      p.accumulate = c0 > 0;
      p.b_off[0] = c;
      p.kblocks = ch / kBK;
      p.m_tiles = df / kBM;
      p.st = st;
      const CUtensorMap* maps[8] = {&dg_m, &du_m, &x_m, &x_m, &x_m, &dw1_o, &dw3_o, &dw3_o};
      if ((rc = launch_mode<kDw13>(maps, p, (df / kBM) * (dm / kBN), stream)) != RA_OK) return rc;
    }
    {  // dw2 (+)= dy^T h
      BGParams p{};
      p.accumulate = c0 > 0;
      p.a_off[0] = c;
      p.kblocks = ch / kBK;
      p.m_tiles = dm / kBM;
      p.st = st;
      const CUtensorMap* maps[8] = {&dy_m, &dy_m, &h_m, &h_m, &h_m, &dw2_o, &dw2_o, &dw2_o};
      if ((rc = launch_mode<kDw2>(maps, p, (dm / kBM) * (df / kBN), stream)) != RA_OK) return rc;
    }
  }
  return RA_OK;
}

}  // namespace ra
