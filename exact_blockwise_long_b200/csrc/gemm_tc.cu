// bf16 GEMM on the sm_100a tensor cores for the projections of the blockwise
// transformer layer ("Ring Attention with Blockwise Transformers", abstract:
// the layer -- attention and feed-forward -- is computed blockwise; the
// query/key/value and output projections around the attention are plain
// per-token matmuls).
//
//   D[M, N] = sum over up to three segments s of A_s[M, K_s] . B_s[N, K_s]^T
//
// Each operand is a logical row-major matrix seen through a 2-D TMA map,
// either K-major (logical rows index M or N, columns index K) or MN-major
// (logical rows index K, columns index M or N: an operand used transposed).
// A logical [tokens, heads*d] matrix may be stored head-split as
// [batch, heads, tokens per sequence, d] (the attention layout): the load
// coordinates are remapped per box, so no transpose kernel exists.
//
// One CTA computes one 128 x 256 output tile (tcgen05 M=128, N=256, fp32 in
// 256 TMEM columns) over a 4-stage TMA ring of 64-deep K slabs (3 stages
// when a residual tile is prefetched).  Epilogues:
// bf16 (optionally + a bf16 residual tile) or fp32 (store, or element-wise
// TMA add onto a zeroed output when the K range is split across two CTAs;
// two addends onto zero commute exactly, so the result is deterministic).
// Warp roles: 0 TMA producer, 1 MMA issuer, 2 TMEM allocator, 4-7 epilogue.
#include "common.cuh"
#include "internal.h"

namespace ra {
namespace {

constexpr int kBM = 128, kBN = 256, kBK = 64;
constexpr int kThreads = 256;
constexpr int kATile = kBM * kBK * 2;  // 16 KB
constexpr int kBTile = kBN * kBK * 2;  // 32 KB
constexpr int kStage = kATile + kBTile;
constexpr int kBox = 16384;  // one epilogue staging box: 128 rows x 128 bytes

// Shared-memory layout per epilogue: a 4-stage ring; with a residual, a
// 3-stage ring plus the residual tile (prefetched at the start, then
// overwritten in place by the output tile).
template <int EPI>
struct GLay {
  static constexpr int kStages = EPI == 1 ? 3 : 4;
  static constexpr int kResOff = kStages * kStage;
  static constexpr int kBarOff = kResOff + (EPI == 1 ? 4 * kBox : 0);
  static constexpr int kTmemSlot = kBarOff + (2 * kStages + 2) * 8;
  static constexpr int kAbortOff = kTmemSlot + 4;
  static constexpr int kSmemBytes = kAbortOff + 4 + 1024;
  static_assert(kSmemBytes <= 232448, "GEMM stages exceed shared memory");
  static_assert(EPI != 2 || 8 * kBox <= kResOff, "fp32 staging exceeds the pipeline buffers");
};

struct OpGeo {
  int hs;                  // head-split storage
  int ntok, heads, d;      // [batch, heads, ntok, d] when hs
  int r0, c0;              // origin of the operand in its logical matrix
};

struct GemmParams {
  OpGeo a[3], b[3];
  int seg_end[3];          // cumulative K steps at the end of each segment
  OpGeo out;               // output (bf16 only may be head-split)
  int m_tiles, n_tiles;
  int n_fast;              // raster: consecutive CTAs share the A tile (n fastest) or the B tile
  int kb_per_split;        // K steps per blockIdx.y
  int kb_total;
  int f32_add;             // fp32 output: TMA add instead of store
  int has_residual;
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

template <bool A_MN, bool B_MN, int EPI>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tA0, const __grid_constant__ CUtensorMap tA1,
                const __grid_constant__ CUtensorMap tA2, const __grid_constant__ CUtensorMap tB0,
                const __grid_constant__ CUtensorMap tB1, const __grid_constant__ CUtensorMap tB2,
                const __grid_constant__ CUtensorMap tOut, const __grid_constant__ CUtensorMap tRes,
                const GemmParams p) {
  using LY = GLay<EPI>;
  constexpr int kStages = LY::kStages;
  extern __shared__ uint8_t smem_g[];
  uint8_t* smem = smem_g + ((1024 - (smem_u32(smem_g) & 1023)) & 1023);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int mt = p.n_fast ? (int)(blockIdx.x / p.n_tiles) : (int)(blockIdx.x % p.m_tiles);
  const int nt = p.n_fast ? (int)(blockIdx.x % p.n_tiles) : (int)(blockIdx.x / p.m_tiles);
  const int kb0 = (int)blockIdx.y * p.kb_per_split;
  const int kb1 = min(p.kb_total, kb0 + p.kb_per_split);

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + LY::kBarOff);
  uint64_t* bar_full = bars;
  uint64_t* bar_empty = bars + kStages;
  uint64_t* bar_done = bars + 2 * kStages;
  uint64_t* bar_res = bars + 2 * kStages + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + LY::kTmemSlot);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + LY::kAbortOff);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bar_full[s], 1);
      mbar_init(&bar_empty[s], 1);
    }
    mbar_init(bar_done, 1);
    mbar_init(bar_res, 1);
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
      if (EPI == 1 && p.has_residual) {  // residual tile [128 rows x 256 cols], needed only by the epilogue
        mbar_arrive_expect_tx(bar_res, 4 * kBox);
        for (int j = 0; j < 4; ++j)
          tma_load_2d(smem + LY::kResOff + j * kBox, &tRes, bar_res, nt * kBN + j * 64, mt * kBM);
      }
      for (int kb = kb0; kb < kb1; ++kb) {
        const int i = kb - kb0;
        const int s = i % kStages;
        if (!mbar_wait(&bar_empty[s], ((i / kStages) & 1) ^ 1, p.st, abort_flag)) break;
        const int seg = (kb >= p.seg_end[0]) + (kb >= p.seg_end[1]);
        const int k = kb - (seg ? p.seg_end[seg - 1] : 0);
        const CUtensorMap* ma = seg == 0 ? &tA0 : (seg == 1 ? &tA1 : &tA2);
        const CUtensorMap* mb = seg == 0 ? &tB0 : (seg == 1 ? &tB1 : &tB2);
        uint8_t* st = smem + s * kStage;
        mbar_arrive_expect_tx(&bar_full[s], kStage);
        load_tile<A_MN, kBM>(st, ma, &bar_full[s], p.a[seg], mt * kBM, k);
        load_tile<B_MN, kBN>(st + kATile, mb, &bar_full[s], p.b[seg], nt * kBN, k);
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
    // accumulator rows -> swizzled 16 KB staging boxes in the idle pipeline
    // buffers -> TMA store / add
    const int r = (warp - 4) * 32 + lane;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    // output boxes: the drained pipeline buffers, or the residual tile in place
    const uint32_t stage_base = smem_u32(smem) + (EPI == 1 ? LY::kResOff : 0);
    const uint32_t row_base = stage_base + (uint32_t)r * 128;
    const uint32_t sw = (uint32_t)(r & 7);
    int ox, oy;
    bool ok = __all_sync(0xffffffffu, mbar_wait(bar_done, 0, p.st, abort_flag));
    if (EPI == 1 && p.has_residual) ok = __all_sync(0xffffffffu, ok && mbar_wait(bar_res, 0, p.st, abort_flag));
    if (ok) {
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < kBN / 32; ++c) {
        uint32_t a[32];
        tmem_ld32(tmem + lane_off + c * 32, a);
        tmem_ld_wait();
        if constexpr (EPI == 2) {
          const uint32_t box = row_base + (uint32_t)c * kBox;
#pragma unroll
          for (int x = 0; x < 8; ++x)
            st_shared_v4(box + (((uint32_t)x ^ sw) << 4), a[4 * x], a[4 * x + 1], a[4 * x + 2], a[4 * x + 3]);
        } else {
          const uint32_t box = row_base + (uint32_t)(c >> 1) * kBox;
          float v[32];
#pragma unroll
          for (int x = 0; x < 32; ++x) v[x] = __uint_as_float(a[x]);
          if (EPI == 1 && p.has_residual) {
#pragma unroll
            for (int x = 0; x < 4; ++x) {
              const uint32_t unit = (uint32_t)((c & 1) * 4 + x);
              uint4 q;
              asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                           : "=r"(q.x), "=r"(q.y), "=r"(q.z), "=r"(q.w)
                           : "r"(box + ((unit ^ sw) << 4)));
              const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                v[8 * x + 2 * e] += __uint_as_float(w[e] << 16);
                v[8 * x + 2 * e + 1] += __uint_as_float(w[e] & 0xffff0000u);
              }
            }
          }
#pragma unroll
          for (int x = 0; x < 4; ++x) {
            const uint32_t unit = (uint32_t)((c & 1) * 4 + x);
            st_shared_v4(box + ((unit ^ sw) << 4), pack_bf16x2(v[8 * x], v[8 * x + 1]),
                         pack_bf16x2(v[8 * x + 2], v[8 * x + 3]), pack_bf16x2(v[8 * x + 4], v[8 * x + 5]),
                         pack_bf16x2(v[8 * x + 6], v[8 * x + 7]));
          }
        }
      }
      fence_proxy_async_smem();
    }
    named_bar_sync(1, 128);
    if (threadIdx.x == 128 && ok) {
      const uint8_t* stage = smem + (EPI == 1 ? LY::kResOff : 0);
      if constexpr (EPI == 2) {
        for (int c = 0; c < kBN / 32; ++c) {
          op_coord(p.out, mt * kBM, nt * kBN + c * 32, ox, oy);
          if (p.f32_add)
            tma_add_2d(&tOut, stage + c * kBox, ox, oy);
          else
            tma_store_2d(&tOut, stage + c * kBox, ox, oy);
        }
      } else {
        for (int j = 0; j < 4; ++j) {
          op_coord(p.out, mt * kBM, nt * kBN + j * 64, ox, oy);
          tma_store_2d(&tOut, stage + j * kBox, ox, oy);
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
int launch_typed(const CUtensorMap* maps, const GemmParams& p, dim3 grid, cudaStream_t stream) {
  constexpr int kSmemBytes = GLay<EPI>::kSmemBytes;
  auto kern = gemm_kernel<A_MN, B_MN, EPI>;
  if (set_smem_attr((const void*)kern, kSmemBytes) != RA_OK) return RA_ERR_CUDA;
  kern<<<grid, kThreads, kSmemBytes, stream>>>(maps[0], maps[1], maps[2], maps[3], maps[4], maps[5], maps[6],
                                               maps[7], p);
  return cudaGetLastError() == cudaSuccess ? RA_OK : RA_ERR_CUDA;
}


}  // namespace

int launch_gemm_tc(const GemmSeg* segs, int nseg, int64_t M, int64_t N, const GemmOut& out, int splits,
                   cudaStream_t stream) {
  if (nseg < 1 || nseg > 3 || M <= 0 || N <= 0 || M % kBM || N % kBN) return RA_ERR_SHAPE;
  if (splits < 1 || splits > 2 || (splits > 1 && (!out.f32 || out.add))) return RA_ERR_ARG;
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
      kb += (int)(g.K / kBK);
    }
    p.seg_end[s] = kb;
  }
  if (out.f32 && out.hs_ntok > 0) return RA_ERR_UNSUPPORTED;
  p.out = geo_of(GemmOperand{out.ptr, M, N, 0, out.hs_ntok, out.hs_heads, out.hs_d, 0, 0});
  p.m_tiles = (int)(M / kBM);
  p.n_tiles = (int)(N / kBN);
  // Concurrent CTAs should share the larger operand's tiles: with M >= N the
  // A rows (activations) are re-read from L2 by the n tiles running together
  // and the smaller B stays L2-resident.
  p.n_fast = M >= N;
  p.kb_total = kb;
  if (kb < splits) return RA_ERR_SHAPE;  // every split needs at least one K step
  p.kb_per_split = (kb + splits - 1) / splits;
  p.f32_add = out.f32 && (out.add || splits > 1);
  p.has_residual = out.residual != nullptr;
  int rc = current_status(&p.st);
  if (rc != RA_OK) return rc;

  alignas(64) CUtensorMap maps[8];
  int ok = RA_OK;
  for (int s = 0; s < 3; ++s) {
    const GemmSeg& g = segs[s < nseg ? s : 0];
    ok |= operand_map(&maps[s], g.a, a_mn);
    ok |= operand_map(&maps[3 + s], g.b, b_mn);
  }
  if (out.f32) {
    ok |= make_tmap_f32_2d(&maps[6], out.ptr, (uint64_t)N, (uint64_t)M, (uint64_t)N * 4, 32, 128);
  } else {
    GemmOperand o{out.ptr, M, N, 0, out.hs_ntok, out.hs_heads, out.hs_d, 0, 0};
    ok |= operand_map(&maps[6], o, false);
  }
  if (out.residual)
    ok |= make_tmap_bf16_2d(&maps[7], out.residual, (uint64_t)N, (uint64_t)M, (uint64_t)N * 2, 64, 128);
  else
    maps[7] = maps[6];
  if (ok != RA_OK) return RA_ERR_CUDA;
  if (out.f32 && splits > 1 && !out.add) {
    if (cudaMemsetAsync(out.ptr, 0, (size_t)M * N * 4, stream) != cudaSuccess) return RA_ERR_CUDA;
  }
  const dim3 grid((unsigned)((M / kBM) * (N / kBN)), (unsigned)splits);
  if (out.f32) {
    if (a_mn && b_mn) return launch_typed<true, true, 2>(maps, p, grid, stream);
    return RA_ERR_UNSUPPORTED;
  }
  if (!a_mn && !b_mn) {
    if (out.residual) return launch_typed<false, false, 1>(maps, p, grid, stream);
    return launch_typed<false, false, 0>(maps, p, grid, stream);
  }
  if (!a_mn && b_mn) return launch_typed<false, true, 0>(maps, p, grid, stream);
  return RA_ERR_UNSUPPORTED;
}

}  // namespace ra
