// bf16 GEMM engine on the sm_100a tensor cores for the blockwise transformer
// layer ("Ring Attention with Blockwise Transformers", abstract: the layer --
// attention and feed-forward -- is computed blockwise; the projections around
// the attention and the feed-forward's matmuls are plain per-token GEMMs).
//
//   D[M, N] = sum over up to three segments s of A_s[M, K_s] . B_s[N, K_s]^T
//
// Each operand is a logical row-major matrix seen through a 2-D TMA map,
// either K-major (logical rows index M or N, columns index K) or MN-major
// (logical rows index K, columns index M or N: an operand used transposed).
// A logical [tokens, heads*d] matrix may be stored head-split as
// [batch, heads, tokens per sequence, d] (the attention layout): the load
// and store coordinates are remapped per box, so no transpose kernel exists.
//
// One CTA computes one 128 x 256 accumulator tile (tcgen05 M=128, N=256,
// fp32 in 256 TMEM columns) over a 4-stage TMA ring of 64-deep K slabs; the
// residual or dh rows an epilogue needs are loaded into the epilogue warps'
// registers while the main loop runs.  Epilogues
// (results leave through 128-byte-swizzled staging boxes and TMA stores):
//   kEpiBf16       bf16 tile
//   kEpiBf16Res    bf16 tile + a bf16 residual tile
//   kEpiF32        fp32 tile, stored or element-wise TMA-added (the K range
//                  may be split across two CTAs adding onto a zeroed output:
//                  two addends onto zero commute exactly, so it stays
//                  deterministic)
//   kEpiSwiGLU     B is stacked: rows 0-127 from w1, 128-255 from w3 (the same
//                  hidden units), so the accumulator holds g | u and the tile
//                  leaves as h = silu(g) * u  [128 x 128]
//   kEpiSwiGLUBwd  the same g | u, plus an fp32 dh tile:
//                  dg = dh u s (1 + g (1 - s)), du = dh g s, h = g s u,
//                  s = 1 / (1 + e^-g)  (three bf16 tiles)
// Warp roles: 0 TMA producer, 1 MMA issuer, 2 TMEM allocator, 4-7 epilogue.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace ra {
namespace {

constexpr int kBM = 128, kBN = 256, kBK = 64;
constexpr int kThreads = 256;
constexpr int kATile = kBM * kBK * 2;  // 16 KB
constexpr int kBTile = kBN * kBK * 2;  // 32 KB
constexpr int kStage = kATile + kBTile;
constexpr int kBox = 16384;  // one staging box: 128 rows x 128 bytes

// Shared memory: a 4-stage ring, reused as the epilogue's staging boxes once
// the main loop has drained.  The epilogues' auxiliary inputs (residual, dh)
// are read into the epilogue warps' registers while the main loop runs.
template <int EPI>
struct GLay {
  static constexpr int kStages = 4;
  static constexpr int kBarOff = kStages * kStage;
  static constexpr int kTmemSlot = kBarOff + (2 * kStages + 1) * 8;
  static constexpr int kAbortOff = kTmemSlot + 4;
  static constexpr int kSmemBytes = kAbortOff + 4 + 1024;
  static_assert(kSmemBytes <= 232448, "GEMM stages exceed shared memory");
  static_assert(EPI != kEpiF32 || 8 * kBox <= kBarOff, "fp32 staging exceeds the pipeline buffers");
  static_assert(EPI != kEpiSwiGLUBwd || 6 * kBox <= kBarOff, "staging exceeds the pipeline buffers");
};

struct OpGeo {
  int hs;                  // head-split storage
  int ntok, heads, d;      // [batch, heads, ntok, d] when hs
  int r0, c0;              // origin of the operand in its logical matrix
};

struct GemmMaps {
  CUtensorMap a[3], b[3];  // per segment (b[1] is the stacked half for the SwiGLU epilogues)
  CUtensorMap out[3];      // outputs
};

struct GemmParams {
  OpGeo a[3], b[3];
  int seg_end[3];          // cumulative K steps at the end of each segment
  OpGeo out;               // output geometry (bf16 only may be head-split)
  int m_tiles, n_tiles;
  int n_fast;              // raster: consecutive CTAs share the A tile (n fastest) or the B tile
  int kb_per_split;        // K steps per blockIdx.y
  int kb_total;
  int f32_add;             // fp32 output: TMA add instead of store
  const void* aux;         // kEpiBf16Res: bf16 residual [M, N]; kEpiSwiGLUBwd: fp32 dh [M, N]
  int aux_ld;              // its row pitch (elements)
  int n_valid;             // output columns; boxes of a half-full last tile past it are not stored
  DevStatus st;
};

__device__ __forceinline__ void op_coord(const OpGeo& g, int r, int c, int& x, int& y) {
  r += g.r0;
  c += g.c0;
  if (g.hs) {
    const int b = r / g.ntok, n = r - b * g.ntok, h = c / g.d;
    x = c - h * g.d;
    y = (b * g.heads + h) * g.ntok + n;
  } else {
    x = c;
    y = r;
  }
}

// operand tile for K step k: K-major -> boxes of 64 K x 128 rows stacked;
// MN-major -> slabs of 64 MN x 64 K side by side (8 KB each)
template <bool MN, int ROWS>
__device__ __forceinline__ void load_tile(uint8_t* dst, const CUtensorMap* map, uint64_t* bar, const OpGeo& g,
                                          int mn0, int k) {
  int x, y;
  if (MN) {
#pragma unroll
    for (int j = 0; j < ROWS / 64; ++j) {
      op_coord(g, k * kBK, mn0 + j * 64, x, y);
      tma_load_2d(dst + j * 8192, map, bar, x, y);
    }
  } else {
#pragma unroll
    for (int i = 0; i < ROWS / 128; ++i) {
      op_coord(g, mn0 + i * 128, k * kBK, x, y);
      tma_load_2d(dst + i * 16384, map, bar, x, y);
    }
  }
}

template <bool MN>
__device__ __forceinline__ uint64_t tile_desc(uint32_t tile, int kk) {
  return MN ? sdesc_sw128(tile + kk * 2048, 8192, 1024) : sdesc_sw128(tile + kk * 32, 16, 1024);
}

// eight floats -> four packed bf16 pairs -> one swizzled 16-byte unit
__device__ __forceinline__ void st_unit_bf16(uint32_t row_base_box, uint32_t unit, uint32_t sw, const float* v) {
  st_shared_v4(row_base_box + ((unit ^ sw) << 4), pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]),
               pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7]));
}

template <bool A_MN, bool B_MN, int EPI>
__global__ void __launch_bounds__(kThreads, 1) gemm_kernel(const __grid_constant__ GemmMaps maps, const GemmParams p) {
  using LY = GLay<EPI>;
  constexpr int kStages = LY::kStages;
  constexpr bool kSwi = EPI == kEpiSwiGLU || EPI == kEpiSwiGLUBwd;
  extern __shared__ uint8_t smem_g[];
  uint8_t* smem = smem_g + ((1024 - (smem_u32(smem_g) & 1023)) & 1023);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int mt = p.n_fast ? (int)(blockIdx.x / p.n_tiles) : (int)(blockIdx.x % p.m_tiles);
  const int nt = p.n_fast ? (int)(blockIdx.x % p.n_tiles) : (int)(blockIdx.x / p.m_tiles);
  const int kb0 = (int)blockIdx.y * p.kb_per_split;
  const int kb1 = min(p.kb_total, kb0 + p.kb_per_split);
  // output columns per tile: 128 for the SwiGLU epilogues (g | u halves), else 256
  constexpr int kOutN = kSwi ? 128 : kBN;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + LY::kBarOff);
  uint64_t* bar_full = bars;
  uint64_t* bar_empty = bars + kStages;
  uint64_t* bar_done = bars + 2 * kStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + LY::kTmemSlot);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + LY::kAbortOff);

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
    tmem_alloc(tmem_slot, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      for (int kb = kb0; kb < kb1; ++kb) {
        const int i = kb - kb0;
        const int s = i % kStages;
        if (!mbar_wait(&bar_empty[s], ((i / kStages) & 1) ^ 1, p.st, abort_flag)) break;
        const int seg = (kb >= p.seg_end[0]) + (kb >= p.seg_end[1]);
        const int k = kb - (seg ? p.seg_end[seg - 1] : 0);
        uint8_t* st = smem + s * kStage;
        mbar_arrive_expect_tx(&bar_full[s], kStage);
        load_tile<A_MN, kBM>(st, &maps.a[seg], &bar_full[s], p.a[seg], mt * kBM, k);
        if constexpr (kSwi) {  // 128 rows of w1, then the same 128 rows of w3
          load_tile<false, 128>(st + kATile, &maps.b[0], &bar_full[s], p.b[0], nt * 128, k);
          load_tile<false, 128>(st + kATile + 16384, &maps.b[1], &bar_full[s], p.b[1], nt * 128, k);
        } else {
          load_tile<B_MN, kBN>(st + kATile, &maps.b[seg], &bar_full[s], p.b[seg], nt * kBN, k);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(kBM, kBN, A_MN, B_MN);
      const uint32_t base = smem_u32(smem);
      for (int kb = kb0; kb < kb1; ++kb) {
        const int i = kb - kb0;
        const int s = i % kStages;
        if (!mbar_wait(&bar_full[s], (i / kStages) & 1, p.st, abort_flag)) break;
        tc_fence_after();
        const uint32_t a = base + s * kStage, b = a + kATile;
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk)
          mma_bf16_ss(tmem, tile_desc<A_MN>(a, kk), tile_desc<B_MN>(b, kk), idesc, (i > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&bar_empty[s]);
      }
      mma_commit(bar_done);
    }
  } else if (warp >= 4) {
    // accumulator rows -> swizzled staging boxes in the drained pipeline
    // buffers -> TMA stores / adds
    const int r = (warp - 4) * 32 + lane;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t row_base = smem_u32(smem) + (uint32_t)r * 128;
    const uint32_t sw = (uint32_t)(r & 7);
    // the auxiliary row slice of this thread (residual: 256 bf16; dh: 128
    // fp32), loaded while the main loop runs
    constexpr bool kAux = EPI == kEpiBf16Res || EPI == kEpiSwiGLUBwd;
    uint4 auxv[kAux ? 32 : 1];
    if constexpr (kAux) {
      const size_t row = (size_t)(mt * kBM + r);
      if constexpr (EPI == kEpiBf16Res) {
        const uint4* src = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.aux) +
                                                          row * p.aux_ld + (size_t)nt * kBN);
#pragma unroll
        for (int j = 0; j < 32; ++j)
          auxv[j] = (nt * kBN + j * 8 < p.n_valid) ? __ldg(src + j) : make_uint4(0, 0, 0, 0);
      } else {
        const uint4* src = reinterpret_cast<const uint4*>(static_cast<const float*>(p.aux) + row * p.aux_ld +
                                                          (size_t)nt * 128);
#pragma unroll
        for (int j = 0; j < 32; ++j) auxv[j] = __ldg(src + j);
      }
    }
    const bool ok = __all_sync(0xffffffffu, mbar_wait(bar_done, 0, p.st, abort_flag));
    if (ok) {
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < kOutN / 32; ++c) {
        if constexpr (EPI == kEpiF32) {
          uint32_t a[32];
          tmem_ld32(tmem + lane_off + c * 32, a);
          tmem_ld_wait();
          const uint32_t box = row_base + (uint32_t)c * kBox;
#pragma unroll
          for (int x = 0; x < 8; ++x)
            st_shared_v4(box + (((uint32_t)x ^ sw) << 4), a[4 * x], a[4 * x + 1], a[4 * x + 2], a[4 * x + 3]);
        } else if constexpr (EPI == kEpiBf16 || EPI == kEpiBf16Res) {
          uint32_t a[32];
          tmem_ld32(tmem + lane_off + c * 32, a);
          tmem_ld_wait();
          const uint32_t box = row_base + (uint32_t)(c >> 1) * kBox;
          float v[32];
#pragma unroll
          for (int x = 0; x < 32; ++x) v[x] = __uint_as_float(a[x]);
          if constexpr (EPI == kEpiBf16Res) {
#pragma unroll
            for (int x = 0; x < 4; ++x) {
              const uint4 q = auxv[c * 4 + x];
              const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                v[8 * x + 2 * e] += __uint_as_float(w[e] << 16);
                v[8 * x + 2 * e + 1] += __uint_as_float(w[e] & 0xffff0000u);
              }
            }
          }
#pragma unroll
          for (int x = 0; x < 4; ++x) st_unit_bf16(box, (uint32_t)((c & 1) * 4 + x), sw, v + 8 * x);
        } else {
          uint32_t g[32], u[32];
          tmem_ld32(tmem + lane_off + c * 32, g);
          tmem_ld32(tmem + lane_off + 128 + c * 32, u);
          tmem_ld_wait();
          if constexpr (EPI == kEpiSwiGLU) {
            float h[32];
#pragma unroll
            for (int x = 0; x < 32; ++x) {
              const float gg = __uint_as_float(g[x]);
              h[x] = gg / (1.f + __expf(-gg)) * __uint_as_float(u[x]);
            }
            const uint32_t box = row_base + (uint32_t)(c >> 1) * kBox;
#pragma unroll
            for (int x = 0; x < 4; ++x) st_unit_bf16(box, (uint32_t)((c & 1) * 4 + x), sw, h + 8 * x);
          } else {
            // eight columns at a time: dh from the registers, dg, du, h to staging
#pragma unroll
            for (int x = 0; x < 4; ++x) {
              float dg[8], du[8], h[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                const int i = 8 * x + e;
                const uint4 q = auxv[c * 8 + i / 4];
                const uint32_t w = (i & 3) == 0 ? q.x : ((i & 3) == 1 ? q.y : ((i & 3) == 2 ? q.z : q.w));
                const float gg = __uint_as_float(g[i]), uu = __uint_as_float(u[i]), d = __uint_as_float(w);
                const float sg = 1.f / (1.f + __expf(-gg));
                const float si = gg * sg;
                h[e] = si * uu;
                du[e] = d * si;
                dg[e] = d * uu * (sg * (1.f + gg * (1.f - sg)));
              }
              const uint32_t unit = (uint32_t)((c & 1) * 4 + x);
              st_unit_bf16(row_base + (uint32_t)(0 * 2 + (c >> 1)) * kBox, unit, sw, dg);
              st_unit_bf16(row_base + (uint32_t)(1 * 2 + (c >> 1)) * kBox, unit, sw, du);
              st_unit_bf16(row_base + (uint32_t)(2 * 2 + (c >> 1)) * kBox, unit, sw, h);
            }
          }
        }
      }
      fence_proxy_async_smem();
    }
    named_bar_sync(1, 128);
    if (threadIdx.x == 128 && ok) {
      const uint8_t* stage = smem;
      int ox, oy;
      if constexpr (EPI == kEpiF32) {
        for (int c = 0; c < kBN / 32; ++c) {
          if (nt * kBN + c * 32 >= p.n_valid) break;
          op_coord(p.out, mt * kBM, nt * kBN + c * 32, ox, oy);
          if (p.f32_add)
            tma_add_2d(&maps.out[0], stage + c * kBox, ox, oy);
          else
            tma_store_2d(&maps.out[0], stage + c * kBox, ox, oy);
        }
      } else {
        constexpr int kOuts = EPI == kEpiSwiGLUBwd ? 3 : 1;
        for (int o = 0; o < kOuts; ++o)
          for (int j = 0; j < kOutN / 64; ++j) {
            if (nt * kOutN + j * 64 >= p.n_valid) break;
            op_coord(p.out, mt * kBM, nt * kOutN + j * 64, ox, oy);
            tma_store_2d(&maps.out[o], stage + (o * (kOutN / 64) + j) * kBox, ox, oy);
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
    tmem_dealloc(tmem, 256);
  }
}

OpGeo geo_of(const GemmOperand& o) {
  OpGeo g{};
  g.hs = o.hs_ntok > 0;
  g.ntok = (int)o.hs_ntok;
  g.heads = (int)o.hs_heads;
  g.d = (int)o.hs_d;
  g.r0 = (int)o.r0;
  g.c0 = (int)o.c0;
  return g;
}

// 2-D map over the operand's physical storage with the box of its major-ness
int operand_map(CUtensorMap* m, const GemmOperand& o, bool mn_major) {
  const uint32_t box_rows = mn_major ? 64 : 128;
  if (o.hs_ntok > 0) {
    const uint64_t rows = (uint64_t)(o.rows / o.hs_ntok) * (uint64_t)o.hs_heads * (uint64_t)o.hs_ntok;
    return make_tmap_bf16_2d(m, o.ptr, (uint64_t)o.hs_d, rows, (uint64_t)o.hs_d * 2, 64, box_rows);
  }
  return make_tmap_bf16_2d(m, o.ptr, (uint64_t)o.cols, (uint64_t)o.rows, (uint64_t)o.cols * 2, 64, box_rows);
}

template <bool A_MN, bool B_MN, int EPI>
int launch_typed(const GemmMaps& maps, const GemmParams& p, dim3 grid, cudaStream_t stream) {
  constexpr int kSmemBytes = GLay<EPI>::kSmemBytes;
  auto kern = gemm_kernel<A_MN, B_MN, EPI>;
  if (set_smem_attr((const void*)kern, kSmemBytes) != RA_OK) return RA_ERR_CUDA;
  kern<<<grid, kThreads, kSmemBytes, stream>>>(maps, p);
  return cudaGetLastError() == cudaSuccess ? RA_OK : RA_ERR_CUDA;
}

}  // namespace

int launch_gemm_tc(const GemmSeg* segs, int nseg, int64_t M, int64_t N, const GemmOut& out, int splits,
                   cudaStream_t stream) {
  const int epi = out.epi;
  const bool swi = epi == kEpiSwiGLU || epi == kEpiSwiGLUBwd;
  const int tile_n = swi ? 128 : kBN;
  if (epi < kEpiBf16 || epi > kEpiSwiGLUBwd) return RA_ERR_ARG;
  if (nseg < 1 || nseg > 3 || (swi && nseg != 2) || M <= 0 || N <= 0 || M % kBM || N % 128) return RA_ERR_SHAPE;
  // a half-full last N tile relies on TMA zero fill and clipping, which a
  // head-split (remapped) box does not have
  if (!swi && N % kBN && (out.hs_ntok > 0 || segs[0].b.hs_ntok > 0)) return RA_ERR_SHAPE;
  if (splits < 1 || splits > 2 || (splits > 1 && (epi != kEpiF32 || out.add))) return RA_ERR_ARG;
  if ((epi == kEpiBf16Res || epi == kEpiSwiGLUBwd) && !out.aux) return RA_ERR_ARG;
  if (epi == kEpiSwiGLUBwd && (!out.ptr2 || !out.ptr3)) return RA_ERR_ARG;
  const bool a_mn = segs[0].a.mn_major != 0, b_mn = segs[0].b.mn_major != 0;
  if (M > INT32_MAX / 2 || N > INT32_MAX / 2) return RA_ERR_UNSUPPORTED;
  GemmParams p{};
  int kb = 0;
  for (int s = 0; s < 3; ++s) {
    if (s < nseg) {
      const GemmSeg& g = segs[s];
      if ((g.a.mn_major != 0) != a_mn || (g.b.mn_major != 0) != b_mn) return RA_ERR_ARG;
      if (g.K <= 0 || g.K % kBK) return RA_ERR_SHAPE;
      for (const GemmOperand* o : {&g.a, &g.b})
        if (o->hs_ntok > 0 && (o->hs_ntok % 128 || o->hs_d % 64 || o->rows % o->hs_ntok)) return RA_ERR_SHAPE;
      p.a[s] = geo_of(g.a);
      p.b[s] = geo_of(g.b);
      // the SwiGLU epilogues stack segment 1's B under segment 0's; K runs once
      if (!(swi && s == 1)) kb += (int)(g.K / kBK);
    }
    p.seg_end[s] = kb;
  }
  if (swi && (b_mn || a_mn || segs[1].K != segs[0].K)) return RA_ERR_ARG;
  if (epi == kEpiF32 && out.hs_ntok > 0) return RA_ERR_UNSUPPORTED;
  p.out = geo_of(GemmOperand{out.ptr, M, N, 0, out.hs_ntok, out.hs_heads, out.hs_d, 0, 0});
  p.m_tiles = (int)(M / kBM);
  p.n_tiles = (int)((N + tile_n - 1) / tile_n);
  // Concurrent CTAs should share the larger operand's tiles: with M >= N the
  // A rows (activations) are re-read from L2 by the n tiles running together
  // and the smaller B stays L2-resident.
  p.n_fast = M >= N;
  p.kb_total = kb;
  if (kb < splits) return RA_ERR_SHAPE;  // every split needs at least one K step
  p.kb_per_split = (kb + splits - 1) / splits;
  p.f32_add = epi == kEpiF32 && (out.add || splits > 1);
  p.aux = out.aux;
  p.aux_ld = (int)N;
  p.n_valid = (int)N;
  int rc = current_status(&p.st);
  if (rc != RA_OK) return rc;

  alignas(64) GemmMaps maps;
  int ok = RA_OK;
  for (int s = 0; s < 3; ++s) {
    const GemmSeg& g = segs[s < nseg ? s : 0];
    ok |= operand_map(&maps.a[s], g.a, a_mn);
    ok |= operand_map(&maps.b[s], g.b, b_mn);
  }
  void* outs[3] = {out.ptr, out.ptr2 ? out.ptr2 : out.ptr, out.ptr3 ? out.ptr3 : out.ptr};
  for (int o = 0; o < 3; ++o) {
    if (epi == kEpiF32) {
      ok |= make_tmap_f32_2d(&maps.out[o], outs[o], (uint64_t)N, (uint64_t)M, (uint64_t)N * 4, 32, 128);
    } else {
      GemmOperand og{outs[o], M, N, 0, out.hs_ntok, out.hs_heads, out.hs_d, 0, 0};
      ok |= operand_map(&maps.out[o], og, false);
    }
  }
  if (ok != RA_OK) return RA_ERR_CUDA;
  if (epi == kEpiF32 && splits > 1) {
    if (cudaMemsetAsync(out.ptr, 0, (size_t)M * N * 4, stream) != cudaSuccess) return RA_ERR_CUDA;
  }
  const dim3 grid((unsigned)(p.m_tiles * p.n_tiles), (unsigned)splits);
  switch (epi) {
    case kEpiF32:
      if (a_mn && b_mn) return launch_typed<true, true, kEpiF32>(maps, p, grid, stream);
      if (!a_mn && b_mn) return launch_typed<false, true, kEpiF32>(maps, p, grid, stream);
      return RA_ERR_UNSUPPORTED;
    case kEpiBf16Res:
      if (!a_mn && !b_mn) return launch_typed<false, false, kEpiBf16Res>(maps, p, grid, stream);
      return RA_ERR_UNSUPPORTED;
    case kEpiSwiGLU:
      return launch_typed<false, false, kEpiSwiGLU>(maps, p, grid, stream);
    case kEpiSwiGLUBwd:
      return launch_typed<false, false, kEpiSwiGLUBwd>(maps, p, grid, stream);
    default:
      if (!a_mn && !b_mn) return launch_typed<false, false, kEpiBf16>(maps, p, grid, stream);
      if (!a_mn && b_mn) return launch_typed<false, true, kEpiBf16>(maps, p, grid, stream);
      return RA_ERR_UNSUPPORTED;
  }
}

}  // namespace ra
