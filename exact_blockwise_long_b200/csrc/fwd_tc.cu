// Ring blockwise attention forward on the sm_100a tensor cores (bf16 in,
// fp32 accumulate).
//
// Method (sources by page and section):
//  - chapterpal "Ring Attention", definition: each query block stays put
//    while key/value blocks circulate; here query shard i visits KV shard
//    j = (i - t) mod S at ring step t, the shards being slices of HBM.
//  - paper abstract: blockwise, exact attention.
//  - darcstar note, DarcStar commentary, paragraphs one and two: the partial
//    softmax states combine exactly; the causal mask and the denominator are
//    combined across chunks exactly (causal pairs j > i skipped, the diagonal
//    pair masked inside its tiles).
//
// One CTA owns one 128-row query tile of one (batch, head) and walks the key
// tiles of the visited shards in ring order.  The running state (row max m,
// denominator l, unnormalised O) is folded with each key tile's partial state
// by the exact log-sum-exp merge: O and l are rescaled by 2^(m_old - m_new)
// whenever the max moves up by more than 2^8 (a stale max is exact because
// the final normalisation uses the same max), and O += P V accumulates in
// tensor memory.  Hardware tiles of 128 x 128 are exact sub-blocks of the
// query_chunk x key_chunk blocks, so the chunk sizes only fix the merge
// boundaries, which do not change the value.
//
// Warp roles (256 threads):
//   warp 0      TMA producer: Q once, then K and V tiles into a 2-stage ring
//   warp 1      MMA issuer (one thread): S = Q K^T into TMEM (two S buffers),
//               O += P V with P read from TMEM
//   warp 2      TMEM allocator
//   warps 4-7   softmax: one thread per query row (TMEM lane), the row max
//               and row sum stay inside the thread; P written back to TMEM
//               as bf16 over the S buffer; final O / l and LSE epilogue
// Tensor memory (512 columns): S0 [0,128), S1 [128,256), O [256, 256+D).
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace ra {
namespace {

constexpr int kBM = 128;    // query rows per tile (TMEM lanes)
constexpr int kBN = 128;    // keys per tile
constexpr int kKSt = 2;     // K stages
constexpr int kVSt = 2;     // V stages
constexpr int kThreads = 256;
constexpr float kRescaleLog2 = 8.0f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr uint32_t kTmemCols = 512;

template <int D>
struct Layout {
  static constexpr int kTileBytes = kBM * D * 2;  // D/64 slabs of [128 rows x 128 B]
  static constexpr int kSlabBytes = kBM * 128;    // 16 KB
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + kTileBytes;
  static constexpr int kV = kK + kKSt * kTileBytes;
  static constexpr int kBar = kV + kVSt * kTileBytes;
  static constexpr int kNumBars = 1 + 2 * kKSt + 2 * kVSt + 2 + 2 + 1;
  static constexpr int kTmemSlot = kBar + kNumBars * 8;
  static constexpr int kAbort = kTmemSlot + 4;
  static constexpr int kBytes = kAbort + 4;
  static constexpr int kAlloc = kBytes + 1024;  // slack for aligning the base to 1024
};

struct Params {
  __nv_bfloat16* out;
  float* lse;
  float* o_acc;     // step mode: fp32 running output
  float* lse_acc;   // step mode: fp32 running lse
  int BH, N, S, L, causal, step;
  int num_qtiles;
  float scale_log2;
  DevStatus st;
};

// Enumerates the key tiles a query tile visits, in ring order.
struct RingWalk {
  int ishard, S, tps, qt, causal, step;
  template <typename F>
  __device__ __forceinline__ bool run(F&& body) const {
    for (int t = 0; t < S; ++t) {
      if (step >= 0 && t != step) continue;
      int j = ishard - t;
      if (j < 0) j += S;
      if (causal && j > ishard) continue;
      const int kt0 = j * tps;
      const int kt1 = (causal && j == ishard) ? qt + 1 : kt0 + tps;
      for (int kt = kt0; kt < kt1; ++kt)
        if (!body(kt, causal && kt == qt)) return false;
    }
    return true;
  }
  __device__ __forceinline__ int count() const {
    int n = 0;
    for (int t = 0; t < S; ++t) {
      if (step >= 0 && t != step) continue;
      int j = ishard - t;
      if (j < 0) j += S;
      if (causal && j > ishard) continue;
      n += (causal && j == ishard) ? (qt + 1 - j * tps) : tps;
    }
    return n;
  }
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const Params p) {
  using LY = Layout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // Work item: heaviest causal query tiles are scheduled first.
  const int qt = p.num_qtiles - 1 - (int)(blockIdx.x / p.BH);
  const int bh = (int)(blockIdx.x % p.BH);
  const int q0 = qt * kBM;
  const int qrow0 = bh * p.N + q0;
  RingWalk walk{q0 / p.L, p.S, p.L / kBN, qt, p.causal, p.step};
  const int n_total = walk.count();
  if (n_total == 0) return;  // step mode, causal pair skipped: accumulators unchanged

  uint8_t* sQ = smem + LY::kQ;
  uint8_t* sK = smem + LY::kK;
  uint8_t* sV = smem + LY::kV;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + LY::kBar);
  uint64_t* bar_q = bars;
  uint64_t* bar_kf = bar_q + 1;
  uint64_t* bar_ke = bar_kf + kKSt;
  uint64_t* bar_vf = bar_ke + kKSt;
  uint64_t* bar_ve = bar_vf + kVSt;
  uint64_t* bar_sf = bar_ve + kVSt;
  uint64_t* bar_pf = bar_sf + 2;
  uint64_t* bar_od = bar_pf + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + LY::kTmemSlot);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + LY::kAbort);

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int s = 0; s < kKSt; ++s) {
      mbar_init(&bar_kf[s], 1);
      mbar_init(&bar_ke[s], 1);
    }
    for (int s = 0; s < kVSt; ++s) {
      mbar_init(&bar_vf[s], 1);
      mbar_init(&bar_ve[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar_sf[s], 1);
      mbar_init(&bar_pf[s], 128);
    }
    mbar_init(bar_od, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 2) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS0 = tmem, tS1 = tmem + 128, tO = tmem + 256;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer ----------------
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      mbar_arrive_expect_tx(bar_q, LY::kTileBytes);
#pragma unroll
      for (int s = 0; s < D / 64; ++s) tma_load_2d(sQ + s * LY::kSlabBytes, &tmQ, bar_q, s * 64, qrow0);
      int n = 0;
      walk.run([&](int kt, bool) {
        const int krow = bh * p.N + kt * kBN;
        const int ks = n % kKSt, vs = n % kVSt;
        if (!mbar_wait(&bar_ke[ks], ((n / kKSt) & 1) ^ 1, p.st, abort_flag)) return false;
        mbar_arrive_expect_tx(&bar_kf[ks], LY::kTileBytes);
#pragma unroll
        for (int s = 0; s < D / 64; ++s)
          tma_load_2d(sK + ks * LY::kTileBytes + s * LY::kSlabBytes, &tmK, &bar_kf[ks], s * 64, krow);
        if (!mbar_wait(&bar_ve[vs], ((n / kVSt) & 1) ^ 1, p.st, abort_flag)) return false;
        mbar_arrive_expect_tx(&bar_vf[vs], LY::kTileBytes);
#pragma unroll
        for (int s = 0; s < D / 64; ++s)
          tma_load_2d(sV + vs * LY::kTileBytes + s * LY::kSlabBytes, &tmV, &bar_vf[vs], s * 64, krow);
        ++n;
        return true;
      });
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      constexpr uint32_t idS = idesc_bf16_f32(kBM, kBN, false, false);  // Q, K both K-major
      constexpr uint32_t idPV = idesc_bf16_f32(kBM, D, false, true);    // V is MN-major (d contiguous)
      const uint32_t q_base = smem_u32(sQ), k_base = smem_u32(sK), v_base = smem_u32(sV);
      bool ok = mbar_wait(bar_q, 0, p.st, abort_flag);
      int n = 0;
      auto issue_pv = [&](int m) -> bool {
        const int pb = m & 1, vs = m % kVSt;
        if (!mbar_wait(&bar_pf[pb], (m >> 1) & 1, p.st, abort_flag)) return false;
        if (!mbar_wait(&bar_vf[vs], (m / kVSt) & 1, p.st, abort_flag)) return false;
        tc_fence_after();
        const uint32_t tP = pb ? tS1 : tS0;
        const uint32_t vb = v_base + vs * LY::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk) {
          const uint64_t bdesc = sdesc_sw128(vb + kk * 16 * 128, LY::kSlabBytes, 1024);
          mma_bf16_ts(tO, tP + kk * 8, bdesc, idPV, (m > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(bar_od);
        mma_commit(&bar_ve[vs]);
        return true;
      };
      if (ok) {
        ok = walk.run([&](int, bool) {
          const int ks = n % kKSt, sb = n & 1;
          if (!mbar_wait(&bar_kf[ks], (n / kKSt) & 1, p.st, abort_flag)) return false;
          tc_fence_after();
          const uint32_t kb = k_base + ks * LY::kTileBytes;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * LY::kSlabBytes + (kk & 3) * 32;
            const uint64_t adesc = sdesc_sw128(q_base + off, 16, 1024);
            const uint64_t bdesc = sdesc_sw128(kb + off, 16, 1024);
            mma_bf16_ss(sb ? tS1 : tS0, adesc, bdesc, idS, kk > 0 ? 1u : 0u);
          }
          mma_commit(&bar_sf[sb]);
          mma_commit(&bar_ke[ks]);
          if (n > 0 && !issue_pv(n - 1)) return false;
          ++n;
          return true;
        });
        if (ok && n > 0) issue_pv(n - 1);
      }
    }
  } else if (warp >= 4) {
    // ---------------- softmax / correction / epilogue ----------------
    const int r = (warp - 4) * 32 + lane;                 // row of the tile = TMEM lane
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const float sl2 = p.scale_log2;
    float m_run = -INFINITY, l_run = 0.f;
    int n = 0;
    const bool ok = walk.run([&](int, bool diag) {
      const int sb = n & 1;
      const uint32_t tS = (sb ? tS1 : tS0) + lane_off;
      // tcgen05.ld/st are warp-collective: every branch below that reaches
      // them is taken by the whole warp.
      if (!__all_sync(0xffffffffu, mbar_wait(&bar_sf[sb], (n >> 1) & 1, p.st, abort_flag))) return false;
      tc_fence_after();
      float s[kBN];
#pragma unroll
      for (int c = 0; c < kBN / 32; ++c) {
        uint32_t reg[32];
        tmem_ld32(tS + c * 32, reg);
        tmem_ld_wait();
#pragma unroll
        for (int x = 0; x < 32; ++x) s[c * 32 + x] = __uint_as_float(reg[x]);
      }
      if (diag) {
#pragma unroll
        for (int c = 0; c < kBN; ++c)
          if (c > r) s[c] = -INFINITY;
      }
      float mx = s[0];
#pragma unroll
      for (int c = 1; c < kBN; ++c) mx = fmaxf(mx, s[c]);
      const float m_new = fmaxf(m_run, mx * sl2);
      if (n == 0) {
        m_run = m_new;
      } else if (__any_sync(0xffffffffu, m_new > m_run + kRescaleLog2)) {
        // Some row of this warp saw its max grow by more than 2^8: the whole
        // warp moves to its new maxima (exact for every row).  O holds P V of
        // every earlier tile once the last one has landed.
        if (!__all_sync(0xffffffffu, mbar_wait(bar_od, (n - 1) & 1, p.st, abort_flag))) return false;
        tc_fence_after();
        const float alpha = ex2_approx(m_run - m_new);
        l_run *= alpha;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t reg[32];
          tmem_ld32(tO + lane_off + c * 32, reg);
          tmem_ld_wait();
#pragma unroll
          for (int x = 0; x < 32; ++x) reg[x] = __float_as_uint(__uint_as_float(reg[x]) * alpha);
          tmem_st32(tO + lane_off + c * 32, reg);
        }
        m_run = m_new;
      }
      const float neg_m = -m_run;
      float rowsum = 0.f;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t pk[32];
#pragma unroll
        for (int x = 0; x < 32; ++x) {
          const float p0 = ex2_approx(fmaf(s[h * 64 + 2 * x], sl2, neg_m));
          const float p1 = ex2_approx(fmaf(s[h * 64 + 2 * x + 1], sl2, neg_m));
          rowsum += p0 + p1;
          pk[x] = pack_bf16x2(p0, p1);
        }
        tmem_st32(tS + h * 32, pk);
      }
      tmem_st_wait();
      l_run += rowsum;
      tc_fence_before();
      mbar_arrive(&bar_pf[sb]);
      ++n;
      return true;
    });
    if (ok && __all_sync(0xffffffffu, mbar_wait(bar_od, (n - 1) & 1, p.st, abort_flag))) {
      tc_fence_after();
      const int grow = qrow0 + r;  // row of the [BH*N, D] view
      const float lse_t = (m_run + __log2f(l_run)) * kLn2;
      const float inv = 1.f / l_run;
      if (p.step < 0) {
        __nv_bfloat16* orow = p.out + (size_t)grow * D;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t reg[32];
          tmem_ld32(tO + lane_off + c * 32, reg);
          tmem_ld_wait();
          uint32_t pk[16];
#pragma unroll
          for (int x = 0; x < 16; ++x)
            pk[x] = pack_bf16x2(__uint_as_float(reg[2 * x]) * inv, __uint_as_float(reg[2 * x + 1]) * inv);
          uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
          for (int x = 0; x < 4; ++x) dst[x] = make_uint4(pk[4 * x], pk[4 * x + 1], pk[4 * x + 2], pk[4 * x + 3]);
        }
        p.lse[grow] = lse_t;
      } else {
        // fused exact merge into the running fp32 accumulators in HBM
        const float lse_a = p.lse_acc[grow];
        float wa = 0.f, wb = 1.f, lse_new = lse_t;
        if (lse_a != -INFINITY) {
          const float mx2 = fmaxf(lse_a, lse_t);
          const float ea = expf(lse_a - mx2), eb = expf(lse_t - mx2);
          const float tot = ea + eb;
          lse_new = mx2 + logf(tot);
          wa = ea / tot;
          wb = eb / tot;
        }
        float* arow = p.o_acc + (size_t)grow * D;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t reg[32];
          tmem_ld32(tO + lane_off + c * 32, reg);
          tmem_ld_wait();
          float4* dst = reinterpret_cast<float4*>(arow + c * 32);
#pragma unroll
          for (int x = 0; x < 8; ++x) {
            float4 o4;
            o4.x = __uint_as_float(reg[4 * x + 0]) * inv * wb;
            o4.y = __uint_as_float(reg[4 * x + 1]) * inv * wb;
            o4.z = __uint_as_float(reg[4 * x + 2]) * inv * wb;
            o4.w = __uint_as_float(reg[4 * x + 3]) * inv * wb;
            if (wa != 0.f) {
              const float4 a4 = dst[x];
              o4.x = fmaf(wa, a4.x, o4.x);
              o4.y = fmaf(wa, a4.y, o4.y);
              o4.z = fmaf(wa, a4.z, o4.z);
              o4.w = fmaf(wa, a4.w, o4.w);
            }
            dst[x] = o4;
          }
        }
        p.lse_acc[grow] = lse_new;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D>
int launch_d(const AttnArgs& a, void* out, float* lse, float* o_acc, float* lse_acc, int step,
             cudaStream_t stream) {
  alignas(64) CUtensorMap tq, tk, tv;
  const uint64_t rows = (uint64_t)(a.B * a.H * a.N);
  if (make_tmap_bf16_2d(&tq, a.q, D, rows, D * 2, 64, kBM) != RA_OK) return RA_ERR_CUDA;
  if (make_tmap_bf16_2d(&tk, a.k, D, rows, D * 2, 64, kBN) != RA_OK) return RA_ERR_CUDA;
  if (make_tmap_bf16_2d(&tv, a.v, D, rows, D * 2, 64, kBN) != RA_OK) return RA_ERR_CUDA;
  Params p{};
  p.out = (__nv_bfloat16*)out;
  p.lse = lse;
  p.o_acc = o_acc;
  p.lse_acc = lse_acc;
  p.BH = (int)(a.B * a.H);
  p.N = (int)a.N;
  p.S = a.S;
  p.L = (int)(a.N / a.S);
  p.causal = a.causal;
  p.step = step;
  p.num_qtiles = (int)(a.N / kBM);
  p.scale_log2 = a.scale * 1.4426950408889634f;
  int rc = current_status(&p.st);
  if (rc != RA_OK) return rc;
  auto kern = fwd_tc_kernel<D>;
  if (set_smem_attr((const void*)kern, Layout<D>::kAlloc) != RA_OK) return RA_ERR_CUDA;
  const unsigned grid = (unsigned)(p.BH * p.num_qtiles);
  kern<<<grid, kThreads, Layout<D>::kAlloc, stream>>>(tq, tk, tv, p);
  return cudaGetLastError() == cudaSuccess ? RA_OK : RA_ERR_CUDA;
}

}  // namespace

int launch_fwd_tc(const AttnArgs& a, void* out, float* lse, float* o_acc, float* lse_acc, int step,
                  cudaStream_t stream) {
  if (a.D == 64) return launch_d<64>(a, out, lse, o_acc, lse_acc, step, stream);
  if (a.D == 128) return launch_d<128>(a, out, lse, o_acc, lse_acc, step, stream);
  return RA_ERR_UNSUPPORTED;
}

}  // namespace ra
