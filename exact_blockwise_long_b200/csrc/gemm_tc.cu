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
// Persistent CTAs, one per SM, stride over 128 x 256 accumulator tiles
// (tcgen05 M=128, N=256, fp32) fed by a TMA ring of 64-deep K slabs.  The
// accumulator is double-buffered in TMEM (2 x 256 columns) and the epilogue
// stages through its own shared-memory slots, so a tile's epilogue runs
// while the next tile's main loop fills the other buffer.  The residual or
// dh rows an epilogue needs are loaded into the epilogue warps' registers
// while that tile's main loop runs.  Epilogues
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

#include <algorithm>

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

// Shared memory: the TMA ring (4 stages; 3 for the three-output SwiGLU
// backward) and a ring of epilogue staging slots separate from it, so one
// tile's epilogue overlaps the next tile's main loop.  A slot is one 16 KB
// box (128 rows x 128 bytes: 64 bf16 or 32 fp32 columns), three for the
// SwiGLU backward (dg, du, h).
template <int EPI>
struct GLay {
  static constexpr int kStages = EPI == kEpiSwiGLUBwd ? 3 : 4;
  static constexpr int kSlotBoxes = EPI == kEpiSwiGLUBwd ? 3 : 1;
  static constexpr int kSlots = EPI == kEpiSwiGLUBwd ? 1 : 2;
  static constexpr int kStagingOff = kStages * kStage;
  static constexpr int kBarOff = kStagingOff + kSlots * kSlotBoxes * kBox;
  static constexpr int kTmemSlot = kBarOff + (2 * kStages + 4) * 8;
  static constexpr int kAbortOff = kTmemSlot + 4;
  static constexpr int kEpiAbortOff = kAbortOff + 4;  // written by the epilogue warps only
  static constexpr int kSmemBytes = kEpiAbortOff + 4 + 1024;
  static_assert(kSmemBytes <= 232448, "GEMM stages exceed shared memory");
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
  int m_tiles, n_tiles, num_tiles;  // num_tiles counts the K splits too
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
  // output columns per tile: 128 for the SwiGLU epilogues (g | u halves), else 256
  constexpr int kOutN = kSwi ? 128 : kBN;
  // epilogue groups per tile: one staging slot each (32 fp32 or 64 bf16 columns)
  constexpr int kChunksPerGroup = EPI == kEpiF32 ? 1 : 2;
  constexpr int kGroups = kOutN / 32 / kChunksPerGroup;
  extern __shared__ uint8_t smem_g[];
  uint8_t* smem = smem_g + ((1024 - (smem_u32(smem_g) & 1023)) & 1023);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int tiles_mn = p.m_tiles * p.n_tiles;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + LY::kBarOff);
  uint64_t* bar_full = bars;
  uint64_t* bar_empty = bars + kStages;
  uint64_t* acc_full = bars + 2 * kStages;       // [2] accumulator buffer holds a finished tile
  uint64_t* acc_empty = bars + 2 * kStages + 2;  // [2] accumulator buffer read out by the epilogue
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + LY::kTmemSlot);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + LY::kAbortOff);
  volatile int* epi_abort = reinterpret_cast<volatile int*>(smem + LY::kEpiAbortOff);

  if (threadIdx.x == 0) {
    *epi_abort = 0;
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bar_full[s], 1);
      mbar_init(&bar_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 128);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 2) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // tile -> (split, m tile, n tile); consecutive tiles share the A tile (n
  // fastest) or the B tile (m fastest)
  auto coords = [&](int tile, int& mt, int& nt, int& kb0, int& kb1) {
    const int split = tile / tiles_mn, t2 = tile - split * tiles_mn;
    mt = p.n_fast ? t2 / p.n_tiles : t2 % p.m_tiles;
    nt = p.n_fast ? t2 % p.n_tiles : t2 / p.m_tiles;
    kb0 = split * p.kb_per_split;
    kb1 = min(p.kb_total, kb0 + p.kb_per_split);
  };

  if (warp == 0) {
    if (lane == 0) {
      int g = 0;  // K steps loaded by this CTA so far (the ring runs on across tiles)
      bool ok = true;
      for (int tile = (int)blockIdx.x; ok && tile < p.num_tiles; tile += (int)gridDim.x) {
        int mt, nt, kb0, kb1;
        coords(tile, mt, nt, kb0, kb1);
        for (int kb = kb0; kb < kb1; ++kb, ++g) {
          const int s = g % kStages;
          if (!(ok = mbar_wait(&bar_empty[s], ((g / kStages) & 1) ^ 1, p.st, abort_flag))) break;
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
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(kBM, kBN, A_MN, B_MN);
      const uint32_t base = smem_u32(smem);
      int g = 0, li = 0;
      bool ok = true;
      for (int tile = (int)blockIdx.x; ok && tile < p.num_tiles; tile += (int)gridDim.x, ++li) {
        int mt, nt, kb0, kb1;
        coords(tile, mt, nt, kb0, kb1);
        const int buf = li & 1;
        // the epilogue has read this buffer's previous tile out
        if (!(ok = mbar_wait(&acc_empty[buf], ((li >> 1) & 1) ^ 1, p.st, abort_flag))) break;
        tc_fence_after();
        const uint32_t acc = tmem + (uint32_t)buf * 256;
        for (int kb = kb0; kb < kb1; ++kb, ++g) {
          const int s = g % kStages;
          if (!(ok = mbar_wait(&bar_full[s], (g / kStages) & 1, p.st, abort_flag))) break;
          tc_fence_after();
          const uint32_t a = base + s * kStage, b = a + kATile;
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            mma_bf16_ss(acc, tile_desc<A_MN>(a, kk), tile_desc<B_MN>(b, kk), idesc, (kb > kb0 || kk > 0) ? 1u : 0u);
          mma_commit(&bar_empty[s]);
        }
        if (ok) mma_commit(&acc_full[buf]);
      }
    }
  } else if (warp >= 4) {
    // accumulator rows -> swizzled staging slots -> TMA stores / adds
    const int r = (warp - 4) * 32 + lane;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t sw = (uint32_t)(r & 7);
    const uint32_t staging = smem_u32(smem) + LY::kStagingOff;
    const uint8_t* staging_gen = smem + LY::kStagingOff;
    constexpr bool kAux = EPI == kEpiBf16Res || EPI == kEpiSwiGLUBwd;
    int gcount = 0, li = 0;
    for (int tile = (int)blockIdx.x; tile < p.num_tiles; tile += (int)gridDim.x, ++li) {
      int mt, nt, kb0, kb1;
      coords(tile, mt, nt, kb0, kb1);
      const int buf = li & 1;
      // the auxiliary row slice of this thread (residual: 256 bf16; dh: 128
      // fp32), loaded while this tile's main loop runs
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
      // one decision for all four epilogue warps, which meet at named
      // barriers: a flag only they write, read by all after the barrier
      const bool mine = __all_sync(0xffffffffu, mbar_wait(&acc_full[buf], (li >> 1) & 1, p.st, abort_flag));
      if (!mine && lane == 0) *epi_abort = 1;
      named_bar_sync(1, 128);
      if (*epi_abort) break;
      tc_fence_after();
      const uint32_t acc = tmem + (uint32_t)buf * 256 + lane_off;
#pragma unroll
      for (int grp = 0; grp < kGroups; ++grp, ++gcount) {
        const uint32_t slot = staging + (uint32_t)((gcount % LY::kSlots) * LY::kSlotBoxes) * kBox;
        const uint32_t row_base = slot + (uint32_t)r * 128;
        // the slot's previous TMA store has finished reading it
        if (gcount >= LY::kSlots) {
          if (threadIdx.x == 128) bulk_wait_read<LY::kSlots - 1>();
          named_bar_sync(1, 128);
        }
#pragma unroll
        for (int ch = 0; ch < kChunksPerGroup; ++ch) {
          const int c = grp * kChunksPerGroup + ch;  // 32-column chunk of the tile
          const bool last = c == kOutN / 32 - 1;
          if constexpr (EPI == kEpiF32) {
            uint32_t a[32];
            tmem_ld32(acc + c * 32, a);
            tmem_ld_wait();
            if (last) {
              tc_fence_before();
              mbar_arrive(&acc_empty[buf]);
            }
#pragma unroll
            for (int x = 0; x < 8; ++x)
              st_shared_v4(row_base + (((uint32_t)x ^ sw) << 4), a[4 * x], a[4 * x + 1], a[4 * x + 2], a[4 * x + 3]);
          } else if constexpr (EPI == kEpiBf16 || EPI == kEpiBf16Res) {
            uint32_t a[32];
            tmem_ld32(acc + c * 32, a);
            tmem_ld_wait();
            if (last) {
              tc_fence_before();
              mbar_arrive(&acc_empty[buf]);
            }
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
            for (int x = 0; x < 4; ++x) st_unit_bf16(row_base, (uint32_t)(ch * 4 + x), sw, v + 8 * x);
          } else {
            uint32_t g[32], u[32];
            tmem_ld32(acc + c * 32, g);
            tmem_ld32(acc + 128 + c * 32, u);
            tmem_ld_wait();
            if (last) {
              tc_fence_before();
              mbar_arrive(&acc_empty[buf]);
            }
            if constexpr (EPI == kEpiSwiGLU) {
              float h[32];
#pragma unroll
              for (int x = 0; x < 32; ++x) {
                const float gg = __uint_as_float(g[x]);
                h[x] = gg / (1.f + __expf(-gg)) * __uint_as_float(u[x]);
              }
#pragma unroll
              for (int x = 0; x < 4; ++x) st_unit_bf16(row_base, (uint32_t)(ch * 4 + x), sw, h + 8 * x);
            } else {
              // eight columns at a time: dh from the registers, dg, du, h to the slot's three boxes
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
                const uint32_t unit = (uint32_t)(ch * 4 + x);
                st_unit_bf16(row_base, unit, sw, dg);
                st_unit_bf16(row_base + kBox, unit, sw, du);
                st_unit_bf16(row_base + 2 * kBox, unit, sw, h);
              }
            }
          }
        }
        fence_proxy_async_smem();
        named_bar_sync(1, 128);
        if (threadIdx.x == 128) {
          const uint8_t* src = staging_gen + (size_t)((gcount % LY::kSlots) * LY::kSlotBoxes) * kBox;
          const int col = nt * kOutN + grp * kChunksPerGroup * 32;  // first output column of the group
          if (col < p.n_valid) {
            int ox, oy;
            op_coord(p.out, mt * kBM, col, ox, oy);
            if constexpr (EPI == kEpiF32) {
              if (p.f32_add)
                tma_add_2d(&maps.out[0], src, ox, oy);
              else
                tma_store_2d(&maps.out[0], src, ox, oy);
            } else {
#pragma unroll
              for (int o = 0; o < LY::kSlotBoxes; ++o) tma_store_2d(&maps.out[o], src + o * kBox, ox, oy);
            }
          }
          bulk_commit_group();
        }
      }
    }
    if (threadIdx.x == 128) bulk_wait_read_all();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
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
  p.num_tiles = p.m_tiles * p.n_tiles * splits;
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
  // persistent CTAs, one per SM, striding over the tiles
  static int sms = 0;
  if (sms == 0) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) !=
                                                  cudaSuccess || sms <= 0)
      sms = 148;
  }
  const dim3 grid((unsigned)std::min(p.num_tiles, sms));
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
