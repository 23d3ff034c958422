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

#include <mutex>

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
  int H, G;  // query heads; query heads per key/value head
  int num_qtiles;
  int group;  // heads per scheduling group
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

// ---------------------------------------------------------------------------
// Softmax pieces shared by both kernels.  One thread owns one query row
// (one TMEM lane) of a 128 x 128 score tile, so the row max and the row sum
// never leave the thread; they are reduced over several independent partial
// accumulators to keep the dependency chains short.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void load_scores(uint32_t tS, float (&s)[kBN]) {
  uint32_t a[32], b[32], c[32], d[32];
  tmem_ld32(tS, a);
  tmem_ld32(tS + 32, b);
  tmem_ld32(tS + 64, c);
  tmem_ld32(tS + 96, d);
  tmem_ld_wait();
#pragma unroll
  for (int x = 0; x < 32; ++x) {
    s[x] = __uint_as_float(a[x]);
    s[32 + x] = __uint_as_float(b[x]);
    s[64 + x] = __uint_as_float(c[x]);
    s[96 + x] = __uint_as_float(d[x]);
  }
}

// Causal mask inside the diagonal tile: key c is in the future of row r.
__device__ __forceinline__ void mask_future(float (&s)[kBN], int r) {
#pragma unroll
  for (int c = 0; c < kBN; ++c)
    if (c > r) s[c] = -INFINITY;
}

__device__ __forceinline__ float row_max(const float (&s)[kBN]) {
  float m[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) m[k] = max3f(s[k], s[k + 8], s[k + 16]);
#pragma unroll
  for (int x = 24; x < 120; x += 16)
#pragma unroll
    for (int k = 0; k < 8; ++k) m[k] = max3f(m[k], s[x + k], s[x + 8 + k]);
#pragma unroll
  for (int k = 0; k < 8; ++k) m[k] = fmaxf(m[k], s[120 + k]);
  return max3f(max3f(m[0], m[1], m[2]), max3f(m[3], m[4], m[5]), fmaxf(m[6], m[7]));
}

// P = 2^(s * scale * log2(e) - m) as bf16 pairs over the first 64 columns of
// the tile's TMEM (P of keys 2c, 2c+1 in column c); returns the row sum of
// the fp32 probabilities.  Masked scores are -inf and give exactly 0.
// One pair in PolyEvery is computed by ex2_poly2 on the FMA/integer pipes,
// the rest by the MUFU: each 128 x 128 tile needs as many MUFU cycles for its
// exponentials as tensor cycles for its two matmuls, so moving part of them
// off the MUFU shortens the softmax's critical path.  Measured best: one pair
// in four at d = 128, one in three at d = 64 (whose matmuls take half as
// long); one in two is slower at both.
// With bar_half, the first half of P (keys 0-63) is published on it as soon
// as it is in TMEM, so the P V matmul over those keys can start while the
// second half is computed.
template <int D>
constexpr int kEx2PolyEvery = D == 64 ? 3 : 4;
template <int PolyEvery>
__device__ __forceinline__ float exp_store(const float (&s)[kBN], uint32_t tS, float sl2, float m,
                                           uint64_t* bar_half = nullptr) {
  const float2 k2 = make_float2(sl2, sl2), nm2 = make_float2(-m, -m);
  float2 acc[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) acc[k] = make_float2(0.f, 0.f);
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    uint32_t pk[32];
#pragma unroll
    for (int x = 0; x < 32; ++x) {
      const float2 t = fma2(make_float2(s[h * 64 + 2 * x], s[h * 64 + 2 * x + 1]), k2, nm2);
      const float2 pr = (x % PolyEvery == PolyEvery - 1) ? ex2_poly2(t)
                                                                : make_float2(ex2_approx(t.x), ex2_approx(t.y));
      acc[x & 3] = add2(acc[x & 3], pr);
      pk[x] = pack_bf16x2(pr.x, pr.y);
    }
    tmem_st32(tS + h * 32, pk);
    if (h == 0 && bar_half) {
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar_half);
    }
  }
  const float2 a01 = add2(acc[0], acc[1]), a23 = add2(acc[2], acc[3]);
  const float2 t = add2(a01, a23);
  return t.x + t.y;
}

// Multiply this row of O (D fp32 columns in TMEM) by alpha.
template <int D>
__device__ __forceinline__ void rescale_o(uint32_t tO, float alpha) {
#pragma unroll
  for (int cc = 0; cc < D / 32; ++cc) {
    uint32_t reg[32];
    tmem_ld32(tO + cc * 32, reg);
    tmem_ld_wait();
#pragma unroll
    for (int x = 0; x < 32; ++x) reg[x] = __float_as_uint(__uint_as_float(reg[x]) * alpha);
    tmem_st32(tO + cc * 32, reg);
  }
}

// Final O / l and LSE of one query row held by this thread (TMEM lane), or,
// in ring-step mode, the exact merge of that row's normalised partial into
// the fp32 running accumulators in HBM.  tO: TMEM address of the row's O.
template <int D>
__device__ __forceinline__ void store_row(uint32_t tO, float m_run, float l_run, int grow, const Params& p) {
  const float lse_t = (m_run + __log2f(l_run)) * kLn2;
  const float inv = 1.f / l_run;
  if (p.step < 0) {
    __nv_bfloat16* orow = p.out + (size_t)grow * D;
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
      uint32_t reg[32];
      tmem_ld32(tO + c * 32, reg);
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
      tmem_ld32(tO + c * 32, reg);
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

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const Params p) {
  using LY = Layout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // Work item: heads in small groups, heaviest causal query tiles first.
  int bh, rank;
  grouped_order((int)blockIdx.x, p.num_qtiles, p.BH, p.group, bh, rank);
  const int qt = p.num_qtiles - 1 - rank;
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
      if (in_bounds(qrow0 + kBM <= p.BH * p.N, p.st, abort_flag)) tma_load_tile(sQ, &tmQ, bar_q, qrow0);
      int n = 0;
      walk.run([&](int kt, bool) {
        const int krow = kv_head_of(bh, p.H, p.G) * p.N + kt * kBN;
        const int ks = n % kKSt, vs = n % kVSt;
        if (!in_bounds(krow + kBN <= (p.BH / p.G) * p.N, p.st, abort_flag)) return false;
        if (!mbar_wait(&bar_ke[ks], ((n / kKSt) & 1) ^ 1, p.st, abort_flag)) return false;
        mbar_arrive_expect_tx(&bar_kf[ks], LY::kTileBytes);
        tma_load_tile(sK + ks * LY::kTileBytes, &tmK, &bar_kf[ks], krow);
        if (!mbar_wait(&bar_ve[vs], ((n / kVSt) & 1) ^ 1, p.st, abort_flag)) return false;
        mbar_arrive_expect_tx(&bar_vf[vs], LY::kTileBytes);
        tma_load_tile(sV + vs * LY::kTileBytes, &tmV, &bar_vf[vs], krow);
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
      load_scores(tS, s);
      if (diag) mask_future(s, r);
      const float m_new = fmaxf(m_run, row_max(s) * sl2);
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
        rescale_o<D>(tO + lane_off, alpha);
        m_run = m_new;
      }
      const float rowsum = exp_store<kEx2PolyEvery<D>>(s, tS, sl2, m_run);
      tmem_st_wait();
      l_run += rowsum;
      tc_fence_before();
      mbar_arrive(&bar_pf[sb]);
      ++n;
      return true;
    });
    if (ok && __all_sync(0xffffffffu, mbar_wait(bar_od, (n - 1) & 1, p.st, abort_flag))) {
      tc_fence_after();
      if (in_bounds(qrow0 + r < p.BH * p.N, p.st, abort_flag)) store_row<D>(tO + lane_off, m_run, l_run, qrow0 + r, p);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// Two query tiles per CTA (256 rows), used when the shard length is a
// multiple of 256.  Two softmax warpgroups, one per 128-row tile, take turns
// with the tensor core: while one warpgroup turns its scores into
// probabilities the MMA warp runs the other tile's P V and Q K^T, so the
// exponentials of one tile overlap the MMAs of the other.
//   warps 0-3  softmax + epilogue of tile 0 (TMEM lanes 0-127)
//   warps 4-7  softmax + epilogue of tile 1
//   warp 8     TMEM allocator, then (one lane) TMA producer
//   warp 9     MMA issuer (one lane); warps 10-11 idle
// The softmax warpgroups take registers from the third warpgroup so each
// softmax thread holds its row of 128 scores in registers.
// Tensor memory: S0 [0,128), S1 [128,256), O0 [256,256+D), O1 [384,384+D);
// P of each tile is written as bf16 over the first 64 columns of its S.
// MMA issue order per key tile n: S0_n, PV1_{n-1}, S1_n, PV0_n.  A tile's
// S_n is issued after its PV_{n-1}, so once a softmax warp sees S_n complete
// the O it may rescale holds every earlier tile's P V already.
// ---------------------------------------------------------------------------
constexpr int kThreads2 = 384;
// Register split: launched at kLaunchRegs per thread (384 x 168 = 64512);
// the softmax warpgroups rise to kSoftmaxRegs, the producer/MMA warpgroup
// drops to kOtherRegs: 256 x 208 + 128 x 88 = 64512.  Per sub-partition:
// 2 x 32 x 208 + 32 x 88 = 16128 of 16384.  The host launches this kernel
// only when the compiled register count equals kLaunchRegs (tc2_usable).
constexpr int kLaunchRegs = 168;
constexpr uint32_t kSoftmaxRegs = 208;
constexpr uint32_t kOtherRegs = 88;
static_assert(256 * kSoftmaxRegs + 128 * kOtherRegs <= kThreads2 * kLaunchRegs, "register split exceeds launch");

template <int D>
struct Layout2 {
  static constexpr int kTileBytes = kBM * D * 2;
  static constexpr int kSlabBytes = kBM * 128;
  static constexpr int kQ = 0;  // Q0, Q1
  static constexpr int kK = 2 * kTileBytes;
  static constexpr int kV = kK + kKSt * kTileBytes;
  static constexpr int kBar = kV + kVSt * kTileBytes;
  static constexpr int kNumBars = 1 + 2 * kKSt + 2 * kVSt + 2 + 2 + 2 + 1;
  static constexpr int kTmemSlot = kBar + kNumBars * 8;
  static constexpr int kAbort = kTmemSlot + 4;
  static constexpr int kBytes = kAbort + 4;
  static constexpr int kAlloc = kBytes + 1024;  // slack for aligning the base to 1024
};
static_assert(Layout2<128>::kAlloc <= 232448, "forward tile set exceeds shared memory");

// Key tiles met by a pair of query tiles (qt0, qt0 + 1) of one shard, in
// ring order.  Under the causal mask the last key tile of the diagonal shard
// (qt0 + 1) lies entirely in the future of tile 0, which skips it.
struct PairWalk {
  int ishard, S, tps, qt0, causal, step;
  template <typename F>
  __device__ __forceinline__ bool run(F&& body) const {
    for (int t = 0; t < S; ++t) {
      if (step >= 0 && t != step) continue;
      int j = ishard - t;
      if (j < 0) j += S;
      if (causal && j > ishard) continue;
      const int kt0 = j * tps;
      const int kt1 = (causal && j == ishard) ? qt0 + 2 : kt0 + tps;
      for (int kt = kt0; kt < kt1; ++kt)
        if (!body(kt, !(causal && kt > qt0), causal && kt == qt0, causal && kt == qt0 + 1)) return false;
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
      n += (causal && j == ishard) ? (qt0 + 2 - j * tps) : tps;
    }
    return n;
  }
};

template <int D>
__global__ void __launch_bounds__(kThreads2, 1)
    fwd_tc2_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const Params p) {
  using LY = Layout2<D>;
  extern __shared__ uint8_t smem_raw2[];
  uint8_t* smem = smem_raw2 + ((1024 - (smem_u32(smem_raw2) & 1023)) & 1023);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // Heads in small groups (their K and V stay in L2), heaviest causal query
  // pairs first.
  const int num_pairs = p.num_qtiles / 2;
  int bh, rank;
  grouped_order((int)blockIdx.x, num_pairs, p.BH, p.group, bh, rank);
  const int pair = num_pairs - 1 - rank;
  const int qt0 = 2 * pair;
  const int qrow0 = bh * p.N + qt0 * kBM;
  PairWalk walk{(qt0 * kBM) / p.L, p.S, p.L / kBN, qt0, p.causal, p.step};
  if (walk.count() == 0) return;  // step mode, causal pair skipped

  uint8_t* sQ = smem + LY::kQ;
  uint8_t* sK = smem + LY::kK;
  uint8_t* sV = smem + LY::kV;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + LY::kBar);
  uint64_t* bar_q = bars;
  uint64_t* bar_kf = bar_q + 1;
  uint64_t* bar_ke = bar_kf + kKSt;
  uint64_t* bar_vf = bar_ke + kKSt;
  uint64_t* bar_ve = bar_vf + kVSt;
  uint64_t* bar_sf = bar_ve + kVSt;  // [2] S of tile t computed
  uint64_t* bar_pf = bar_sf + 2;     // [2] P of tile t written
  uint64_t* bar_ph = bar_pf + 2;     // [2] first half of P (keys 0-63) of tile t written
  uint64_t* bar_done = bar_ph + 2;   // every MMA finished
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
    for (int t = 0; t < 2; ++t) {
      mbar_init(&bar_sf[t], 1);
      mbar_init(&bar_pf[t], 128);
      mbar_init(&bar_ph[t], 128);
    }
    mbar_init(bar_done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 8) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp >= 8) {
   regs_dec<kOtherRegs>();
   if (warp == 8) {
    if (lane == 0) {
      // ---------------- TMA producer ----------------
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      mbar_arrive_expect_tx(bar_q, 2 * LY::kTileBytes);
#pragma unroll
      for (int t = 0; t < 2; ++t)
        if (in_bounds(qrow0 + (t + 1) * kBM <= p.BH * p.N, p.st, abort_flag))
          tma_load_tile(sQ + t * LY::kTileBytes, &tmQ, bar_q, qrow0 + t * kBM);
      int n = 0;
      walk.run([&](int kt, bool, bool, bool) {
        const int krow = kv_head_of(bh, p.H, p.G) * p.N + kt * kBN;
        const int ks = n % kKSt, vs = n % kVSt;
        if (!in_bounds(krow + kBN <= (p.BH / p.G) * p.N, p.st, abort_flag)) return false;
        if (!mbar_wait(&bar_ke[ks], ((n / kKSt) & 1) ^ 1, p.st, abort_flag)) return false;
        mbar_arrive_expect_tx(&bar_kf[ks], LY::kTileBytes);
        tma_load_tile(sK + ks * LY::kTileBytes, &tmK, &bar_kf[ks], krow);
        if (!mbar_wait(&bar_ve[vs], ((n / kVSt) & 1) ^ 1, p.st, abort_flag)) return false;
        mbar_arrive_expect_tx(&bar_vf[vs], LY::kTileBytes);
        tma_load_tile(sV + vs * LY::kTileBytes, &tmV, &bar_vf[vs], krow);
        ++n;
        return true;
      });
    }
  } else if (warp == 9) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      constexpr uint32_t idS = idesc_bf16_f32(kBM, kBN, false, false);
      constexpr uint32_t idPV = idesc_bf16_f32(kBM, D, false, true);
      const uint32_t q_base = smem_u32(sQ), k_base = smem_u32(sK), v_base = smem_u32(sV);
      int n = 0, prev_vs = 0;
      int pv_cnt[2] = {0, 0};
      auto issue_s = [&](int t, uint32_t kb) {
        const uint32_t qb = q_base + t * LY::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * LY::kSlabBytes + (kk & 3) * 32;
          mma_bf16_ss(tmem + t * 128, sdesc_sw128(qb + off, 16, 1024), sdesc_sw128(kb + off, 16, 1024), idS,
                      kk > 0 ? 1u : 0u);
        }
        mma_commit(&bar_sf[t]);
      };
      auto issue_pv = [&](int t, int vs) -> bool {
        const uint32_t vb = v_base + vs * LY::kTileBytes;
#pragma unroll
        for (int half = 0; half < 2; ++half) {  // keys 0-63 as soon as their P is in TMEM, then 64-127
          if (!mbar_wait(half ? &bar_pf[t] : &bar_ph[t], pv_cnt[t] & 1, p.st, abort_flag)) return false;
          tc_fence_after();
#pragma unroll
          for (int kk = half * (kBN / 32); kk < (half + 1) * (kBN / 32); ++kk)
            mma_bf16_ts(tmem + 256 + t * 128, tmem + t * 128 + kk * 8,
                        sdesc_sw128(vb + kk * 16 * 128, LY::kSlabBytes, 1024), idPV,
                        (pv_cnt[t] > 0 || kk > 0) ? 1u : 0u);
        }
        ++pv_cnt[t];
        return true;
      };
      bool ok = mbar_wait(bar_q, 0, p.st, abort_flag);
      if (ok) {
        ok = walk.run([&](int, bool do0, bool, bool) {
          const int ks = n % kKSt, vs = n % kVSt;
          if (!mbar_wait(&bar_kf[ks], (n / kKSt) & 1, p.st, abort_flag)) return false;
          tc_fence_after();
          const uint32_t kb = k_base + ks * LY::kTileBytes;
          if (do0) issue_s(0, kb);
          if (n > 0) {
            if (!issue_pv(1, prev_vs)) return false;
            mma_commit(&bar_ve[prev_vs]);
          }
          issue_s(1, kb);
          mma_commit(&bar_ke[ks]);
          if (!mbar_wait(&bar_vf[vs], (n / kVSt) & 1, p.st, abort_flag)) return false;
          if (do0 && !issue_pv(0, vs)) return false;
          prev_vs = vs;
          ++n;
          return true;
        });
        if (ok && n > 0 && issue_pv(1, prev_vs)) mma_commit(&bar_ve[prev_vs]);
      }
      mma_commit(bar_done);
    }
   }
  } else {
    regs_inc<kSoftmaxRegs>();
    // ---------------- softmax / correction / epilogue of one tile ----------------
    constexpr uint32_t FULL = 0xffffffffu;
    const int tile = warp >> 2;
    const int r = (warp & 3) * 32 + lane;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + tile * 128 + lane_off;
    const uint32_t tO = tmem + 256 + tile * 128 + lane_off;
    const float sl2 = p.scale_log2;
    float m_run = -INFINITY, l_run = 0.f;
    int c = 0;
    const bool ok = walk.run([&](int, bool do0, bool diag0, bool diag1) {
      if (tile == 0 && !do0) return true;
      const bool diag = tile ? diag1 : diag0;
      if (!__all_sync(FULL, mbar_wait(&bar_sf[tile], c & 1, p.st, abort_flag))) return false;
      tc_fence_after();
      float s[kBN];
      load_scores(tS, s);
      if (diag) mask_future(s, r);
      const float m_new = fmaxf(m_run, row_max(s) * sl2);
      if (c == 0) {
        m_run = m_new;
      } else if (__any_sync(FULL, m_new > m_run + kRescaleLog2)) {
        // this tile's S is complete, hence so is its previous P V: rescale O
        const float alpha = ex2_approx(m_run - m_new);
        l_run *= alpha;
        rescale_o<D>(tO, alpha);
        m_run = m_new;
      }
      const float rowsum = exp_store<kEx2PolyEvery<D>>(s, tS, sl2, m_run, &bar_ph[tile]);
      tmem_st_wait();
      l_run += rowsum;
      tc_fence_before();
      mbar_arrive(&bar_pf[tile]);
      ++c;
      return true;
    });
    if (ok && __all_sync(FULL, mbar_wait(bar_done, 0, p.st, abort_flag))) {
      tc_fence_after();
      if (in_bounds(qrow0 + tile * kBM + r < p.BH * p.N, p.st, abort_flag))
        store_row<D>(tO, m_run, l_run, qrow0 + tile * kBM + r, p);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// Whether fwd_tc2_kernel<D> may run on the current device: its register
// split (setmaxnreg) is sized for exactly kLaunchRegs registers per thread at
// launch, so a build that compiled it to another count must not launch it
// (a split larger than the launch's registers would wait forever).  Decided
// once per device and cached; ringattn_kernel_plan reports the outcome.
// Without a device nothing launches; the answer is then the build's (its
// register count is checked when the library is built).
template <int D>
bool tc2_usable() {
  constexpr int kMaxDev = 64;
  static std::mutex mu;
  static signed char known[kMaxDev] = {};  // 0 unknown, 1 usable, -1 not
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {  // no device: nothing launches; the build checked the count
    cudaGetLastError();
    return true;
  }
  if (dev < 0 || dev >= kMaxDev) return false;
  std::lock_guard<std::mutex> lk(mu);
  if (known[dev] == 0) {
    cudaFuncAttributes fa;
    const bool ok = cudaFuncGetAttributes(&fa, (const void*)fwd_tc2_kernel<D>) == cudaSuccess &&
                    fa.numRegs == kLaunchRegs;
    known[dev] = ok ? 1 : -1;
  }
  return known[dev] > 0;
}

template <int D>
int launch_d(const AttnArgs& a, void* out, float* lse, float* o_acc, float* lse_acc, int step,
             cudaStream_t stream) {
  alignas(64) CUtensorMap tq, tk, tv;
  const uint64_t rows = (uint64_t)(a.B * a.H * a.N);
  const uint64_t kv_rows = (uint64_t)(a.B * a.Hkv * a.N);
  if (make_tmap_bf16_tile(&tq, a.q, D, rows, kBM) != RA_OK) return RA_ERR_CUDA;
  if (make_tmap_bf16_tile(&tk, a.k, D, kv_rows, kBN) != RA_OK) return RA_ERR_CUDA;
  if (make_tmap_bf16_tile(&tv, a.v, D, kv_rows, kBN) != RA_OK) return RA_ERR_CUDA;
  Params p{};
  p.out = (__nv_bfloat16*)out;
  p.lse = lse;
  p.o_acc = o_acc;
  p.lse_acc = lse_acc;
  p.BH = (int)(a.B * a.H);
  p.H = (int)a.H;
  p.G = (int)(a.H / a.Hkv);
  p.N = (int)a.N;
  p.S = a.S;
  p.L = (int)(a.N / a.S);
  p.causal = a.causal;
  p.step = step;
  p.num_qtiles = (int)(a.N / kBM);
  p.scale_log2 = a.scale * 1.4426950408889634f;
  int rc = current_status(&p.st);
  if (rc != RA_OK) return rc;
  const bool two_tiles = (p.L % (2 * kBM) == 0) && tc2_usable<D>();
  // per head the key/value tiles every query tile streams through
  p.group = head_group(two_tiles ? p.num_qtiles / 2 : p.num_qtiles, p.BH, 2.0 * a.N * D * 2, 60.0e6);
  if (two_tiles) {
    auto kern = fwd_tc2_kernel<D>;
    if (set_smem_attr((const void*)kern, Layout2<D>::kAlloc) != RA_OK) return RA_ERR_CUDA;
    const unsigned grid = (unsigned)(p.BH * (p.num_qtiles / 2));
    kern<<<grid, kThreads2, Layout2<D>::kAlloc, stream>>>(tq, tk, tv, p);
  } else {
    auto kern = fwd_tc_kernel<D>;
    if (set_smem_attr((const void*)kern, Layout<D>::kAlloc) != RA_OK) return RA_ERR_CUDA;
    const unsigned grid = (unsigned)(p.BH * p.num_qtiles);
    kern<<<grid, kThreads, Layout<D>::kAlloc, stream>>>(tq, tk, tv, p);
  }
  return cudaGetLastError() == cudaSuccess ? RA_OK : RA_ERR_CUDA;
}

}  // namespace

const char* fwd_tc_kernel_name(int64_t L, int64_t D) {
  const bool pair = L % (2 * kBM) == 0;
  if (D == 64) return pair && tc2_usable<64>() ? "fwd_tc2_kernel" : "fwd_tc_kernel";
  if (D == 128) return pair && tc2_usable<128>() ? "fwd_tc2_kernel" : "fwd_tc_kernel";
  return nullptr;
}

int launch_fwd_tc(const AttnArgs& a, void* out, float* lse, float* o_acc, float* lse_acc, int step,
                  cudaStream_t stream) {
  if (a.D == 64) return launch_d<64>(a, out, lse, o_acc, lse_acc, step, stream);
  if (a.D == 128) return launch_d<128>(a, out, lse, o_acc, lse_acc, step, stream);
  return RA_ERR_UNSUPPORTED;
}

}  // namespace ra
