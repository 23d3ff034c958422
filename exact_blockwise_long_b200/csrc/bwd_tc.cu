// Backward of exact ring blockwise attention on the sm_100a tensor cores.
//
// The pages use the method for training ("training and inference", paper
// abstract) but print no backward algorithm; this is the plain chain rule
// through the softmax, recomputing P from the forward's log-sum-exp:
//   P_ij = exp(s_ij - lse_i) on visible pairs,  D_i = dO_i . O_i
//   dV_j = sum_i P_ij dO_i            dS_ij = P_ij (dO_i . V_j - D_i)
//   dK_j = scale sum_i dS_ij Q_i      dQ_i = scale sum_j dS_ij K_j
//
// The default backward (ringattn_bwd) is three launches:
//   preprocess  D_i = dO_i . O_i and lse_i * log2(e); zeroes the fp32 dQ
//               accumulator                                         (HBM-bound)
//   fused pass  a key/value tile stays on chip while the query shards pass
//               by in ring order i = (j + t) mod S (the forward's pairs, loop
//               nest turned around; under the causal mask pairs of shards in
//               the future are skipped and the diagonal pair is masked inside
//               its tiles).  Per (key tile, query tile) 5 tcgen05 MMAs:
//                 S^T  = K Q^T, dP^T = V dO^T       (into TMEM)
//                 dV  += P^T dO, dK += dS^T Q       (A operands from TMEM)
//                 dQ^T = K^T dS^T (d = 128) or dQ = dS K (d = 64), added in
//                 fp32 into the accumulator by a drain warpgroup
//               dK and dV are written once per key tile; dQ sums over key
//               tiles in arrival order (reproducible up to fp32 order).
//   conversion  dq = bf16(accumulator)                               (HBM-bound)
//
// The deterministic backward (ringattn_bwd_phase mask 7, ringattn_bwd_noalloc)
// splits the work in two passes, each gradient accumulated in tensor memory
// and written once (no additions in memory, every output bit-reproducible):
//   dK/dV       per (key tile, query tile) 4 tcgen05 MMAs:
//                 S^T  = K Q^T    (TMEM [0,128))
//                 dP^T = V dO^T   (TMEM [128,256))
//                 dV  += P^T dO   (P^T bf16 over S^T, A operand from TMEM)
//                 dK  += dS^T Q   (dS^T bf16 over dP^T, A operand from TMEM)
//   dQ          the query tile stationary, the KV shards visited in ring
//               order j = (i - t) mod S exactly like the forward; per
//               (query tile, key tile) 3 tcgen05 MMAs, Q and dO held in TMEM
//               as their A operands:
//                 S    = Q K^T    (TMEM [0,128))
//                 dP   = dO V^T   (TMEM [128,256))
//                 dQ  += dS K     (dS bf16 over dP, A operand from TMEM)
#include <math.h>

#include <mutex>
#include <type_traits>

#include "common.cuh"
#include "internal.h"

namespace ra {

bool fused_usable(int64_t D);  // below: the fused pass's register split fits this build on this device

namespace {

constexpr int kT = 128;        // rows per tile (TMEM lanes)
constexpr int kSt = 2;         // streamed-tile stages
constexpr int kThreads = 384;   // 4 role warps + two element-wise warpgroups
constexpr int kHalf = 64;      // score columns per element-wise warpgroup
// At d = 64 the four matmuls of a dK/dV step take half as long as at
// d = 128 while the exponentials do not, so the MUFU would bound that pass:
// there every second exponential pair is computed by ex2_poly2 on the
// FMA/integer pipes (0.76 -> 0.72 ms on the causal 8k workload).  Everywhere
// else all stay on the MUFU: moving some was measured no faster at d = 128
// and slower in the dQ pass.
constexpr float kLog2e = 1.4426950408889634f;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t FULL = 0xffffffffu;
constexpr int kMaxDynSmem = 232448;  // 227 KB: the most dynamic shared memory one CTA may use

struct BParams {
  const __nv_bfloat16* q;     // [BH*N, D]
  const __nv_bfloat16* dout;  // [BH*N, D]
  const float* lse2;   // lse * log2(e)    [BH*N]
  const float* dvec;   // D_i = dO_i . O_i  [BH*N]
  __nv_bfloat16* dq;
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  float* dqacc;        // fused pass: fp32 dQ accumulator [BH*N, D] (scaled dQ added into it)
  float* dq32;         // query-stationary pass: fp32 dq accumulator to add into instead of writing dq
  float* dk32;         // key/value passes: fp32 dk, dv outputs instead of bf16 dk, dv
  float* dv32;
  int kv_add;          // with dk32, dv32: add into them (1) or overwrite them (0)
  int smem_alloc;      // fused pass: dynamic shared memory bytes of the launch
  int BH, N, S, L, causal, num_tiles;
  int H, G;            // query heads; query heads per key/value head
  int BHkv;            // batch x key/value heads
  int group;           // heads per scheduling group
  float scale, scale_log2;
  DevStatus st;
};

// Query tiles a stationary key tile meets, in ring order (j + t) mod S, for
// each of the G query heads (flat indices qbh0 .. qbh0 + G - 1) that share
// its key/value head.
struct RingWalkKV {
  int jshard, S, tps, kt, causal, qbh0, G;
  template <typename F>
  __device__ __forceinline__ bool run(F&& body) const {
    for (int g = 0; g < G; ++g) {
      for (int t = 0; t < S; ++t) {
        int i = jshard + t;
        if (i >= S) i -= S;
        if (causal && i < jshard) continue;
        const int qt0 = (causal && i == jshard) ? kt : i * tps;
        for (int qt = qt0; qt < i * tps + tps; ++qt)
          if (!body(qbh0 + g, qt, causal && qt == kt)) return false;
      }
    }
    return true;
  }
  __device__ __forceinline__ int count() const {
    int n = 0;
    for (int t = 0; t < S; ++t) {
      int i = jshard + t;
      if (i >= S) i -= S;
      if (causal && i < jshard) continue;
      n += (causal && i == jshard) ? (i * tps + tps - kt) : tps;
    }
    return n * G;
  }
};

// Key tiles a stationary query tile meets, in ring order (i - t) mod S.
struct RingWalkQ {
  int ishard, S, tps, qt, causal;
  template <typename F>
  __device__ __forceinline__ bool run(F&& body) const {
    for (int t = 0; t < S; ++t) {
      int j = ishard - t;
      if (j < 0) j += S;
      if (causal && j > ishard) continue;
      const int kt1 = (causal && j == ishard) ? qt + 1 : j * tps + tps;
      for (int kt = j * tps; kt < kt1; ++kt)
        if (!body(kt, causal && kt == qt)) return false;
    }
    return true;
  }
  __device__ __forceinline__ int count() const {
    int n = 0;
    for (int t = 0; t < S; ++t) {
      int j = ishard - t;
      if (j < 0) j += S;
      if (causal && j > ishard) continue;
      n += (causal && j == ishard) ? (qt + 1 - j * tps) : tps;
    }
    return n;
  }
};

__device__ __forceinline__ void load_row64(uint32_t taddr, float (&s)[kHalf]) {
  uint32_t a[32], b[32];
  tmem_ld32(taddr, a);
  tmem_ld32(taddr + 32, b);
  tmem_ld_wait();
#pragma unroll
  for (int x = 0; x < 32; ++x) {
    s[x] = __uint_as_float(a[x]);
    s[32 + x] = __uint_as_float(b[x]);
  }
}

template <int W>
__device__ __forceinline__ void store_acc_row(uint32_t taddr, float mul, __nv_bfloat16* dst_row);

// Store W fp32 columns of one TMEM row, times `mul`, as fp32 to global, or
// add them to what is there (add != 0).
template <int W>
__device__ __forceinline__ void store_acc_row_f32(uint32_t taddr, float mul, float* dst_row, int add) {
#pragma unroll
  for (int c = 0; c < W / 32; ++c) {
    uint32_t reg[32];
    tmem_ld32(taddr + c * 32, reg);
    tmem_ld_wait();
    float4* dst = reinterpret_cast<float4*>(dst_row + c * 32);
#pragma unroll
    for (int x = 0; x < 8; ++x) {
      float4 o = make_float4(__uint_as_float(reg[4 * x]) * mul, __uint_as_float(reg[4 * x + 1]) * mul,
                             __uint_as_float(reg[4 * x + 2]) * mul, __uint_as_float(reg[4 * x + 3]) * mul);
      if (add) {
        const float4 a = dst[x];
        o.x += a.x;
        o.y += a.y;
        o.z += a.z;
        o.w += a.w;
      }
      dst[x] = o;
    }
  }
}

// The dK and dV rows of one thread (key row `row`, half h of the d columns):
// bf16 dk, dv, or fp32 dk32, dv32 (written or added) when those are given.
template <int D>
__device__ __forceinline__ void store_dkdv(uint32_t tDK, uint32_t tDV, size_t row, int h, const BParams& p) {
  if (p.dk32) {
    store_acc_row_f32<D / 2>(tDK, p.scale, p.dk32 + row * D + h * (D / 2), p.kv_add);
    store_acc_row_f32<D / 2>(tDV, 1.f, p.dv32 + row * D + h * (D / 2), p.kv_add);
  } else {
    store_acc_row<D / 2>(tDK, p.scale, p.dk + row * D + h * (D / 2));
    store_acc_row<D / 2>(tDV, 1.f, p.dv + row * D + h * (D / 2));
  }
}

// Store W fp32 columns of one TMEM row, times `mul`, as bf16 to global.
template <int W>
__device__ __forceinline__ void store_acc_row(uint32_t taddr, float mul, __nv_bfloat16* dst_row) {
#pragma unroll
  for (int c = 0; c < W / 32; ++c) {
    uint32_t reg[32];
    tmem_ld32(taddr + c * 32, reg);
    tmem_ld_wait();
    uint32_t pk[16];
#pragma unroll
    for (int x = 0; x < 16; ++x)
      pk[x] = pack_bf16x2(__uint_as_float(reg[2 * x]) * mul, __uint_as_float(reg[2 * x + 1]) * mul);
    uint4* dst = reinterpret_cast<uint4*>(dst_row + c * 32);
#pragma unroll
    for (int x = 0; x < 4; ++x) dst[x] = make_uint4(pk[4 * x], pk[4 * x + 1], pk[4 * x + 2], pk[4 * x + 3]);
  }
}

// ===========================================================================
// dK, dV: key/value tile stationary
// ===========================================================================
template <int D>
struct KVLayout {
  static constexpr int kTile = kT * D * 2;  // 128 rows x D bf16 (D/64 slabs)
  static constexpr int kSlab = kT * 128;
  static constexpr int kK = 0;
  static constexpr int kV = kK + kTile;
  static constexpr int kQ = kV + kTile;
  static constexpr int kDO = kQ + kSt * kTile;
  static constexpr int kVec = kDO + kSt * kTile;  // per stage: lse*log2e [128], D [128]
  static constexpr int kBar = kVec + kSt * 1024;
  static constexpr int kNumBars = 1 + 2 * kSt + 6;
  static constexpr int kTmemSlot = kBar + kNumBars * 8;
  static constexpr int kAbort = kTmemSlot + 4;
  static constexpr int kBytes = kAbort + 4;
  static constexpr int kAlloc = kBytes + 1024;
};
static_assert(KVLayout<128>::kAlloc <= kMaxDynSmem, "dK/dV tile set exceeds shared memory");

// Warp roles: warp 0 TMA producer (K, V once; Q, dO, lse, D per step),
// warp 1 MMA issuer, warp 2 TMEM allocator, warps 4-7 and 8-11 one thread
// per key row each, the first warpgroup on query columns [0,64), the second
// on [64,128): P^T, dS^T and half of the dK/dV epilogue.  Each warpgroup
// writes its bf16 P^T (dS^T) over the first 32 of the S^T (dP^T) columns it
// has itself read, so the A operand of dV (dK) sits in columns [0,32) and
// [64,96).
// MMA order per step n: dP_n, dV_n, S_{n+1}, dK_n (S_0 first); S_{n+1} is
// issued as soon as dV_n has read P_n out of the S columns.  P^T is
// published in two halves (queries {0-31, 64-95}, then {32-63, 96-127}), so
// the first half of dV runs while the second half of the exponentials is
// computed.
template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_kv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                  const BParams p) {
  using LY = KVLayout<D>;
  extern __shared__ uint8_t smem_kv[];
  uint8_t* smem = smem_kv + ((1024 - (smem_u32(smem_kv) & 1023)) & 1023);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // key/value heads in small groups; the heaviest causal key tiles (smallest
  // index) first
  int kvbh, kt;
  grouped_order((int)blockIdx.x, p.num_tiles, p.BHkv, p.group, kvbh, kt);
  const int krow0 = kvbh * p.N + kt * kT;
  const int tps = p.L / kT;
  const int Hkv = p.H / p.G;
  const int qbh0 = (kvbh / Hkv) * p.H + (kvbh % Hkv) * p.G;  // first query head of the group
  const RingWalkKV walk{(kt * kT) / p.L, p.S, tps, kt, p.causal, qbh0, p.G};
  const int n_total = walk.count();

  uint8_t* sK = smem + LY::kK;
  uint8_t* sV = smem + LY::kV;
  uint8_t* sQ = smem + LY::kQ;
  uint8_t* sDO = smem + LY::kDO;
  float* sVec = reinterpret_cast<float*>(smem + LY::kVec);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + LY::kBar);
  uint64_t* bar_kv = bars;
  uint64_t* bar_qf = bar_kv + 1;
  uint64_t* bar_qe = bar_qf + kSt;
  uint64_t* bar_sf = bar_qe + kSt;   // S^T computed
  uint64_t* bar_dpf = bar_sf + 1;    // dP^T computed
  uint64_t* bar_ph = bar_dpf + 1;    // first half of P^T (queries [0,32) and [64,96)) written to TMEM
  uint64_t* bar_pr = bar_ph + 1;     // all of P^T written to TMEM
  uint64_t* bar_dsr = bar_pr + 1;    // dS^T written to TMEM
  uint64_t* bar_done = bar_dsr + 1;  // dK, dV final
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + LY::kTmemSlot);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + LY::kAbort);

  if (threadIdx.x == 0) {
    mbar_init(bar_kv, 1);
    for (int s = 0; s < kSt; ++s) {
      mbar_init(&bar_qf[s], 1);
      mbar_init(&bar_qe[s], 1);
    }
    mbar_init(bar_sf, 1);
    mbar_init(bar_dpf, 1);
    mbar_init(bar_ph, 2 * 128);
    mbar_init(bar_pr, 2 * 128);
    mbar_init(bar_dsr, 2 * 128);
    mbar_init(bar_done, 1);
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
  const uint32_t tS = tmem, tDP = tmem + 128, tDK = tmem + 256, tDV = tmem + 384;

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmDO);
      mbar_arrive_expect_tx(bar_kv, 2 * LY::kTile);
      if (in_bounds(krow0 + kT <= p.BHkv * p.N, p.st, abort_flag)) {
        tma_load_tile(sK, &tmK, bar_kv, krow0);
        tma_load_tile(sV, &tmV, bar_kv, krow0);
      }
      int n = 0;
      walk.run([&](int qbh, int qt, bool) {
        const int st = n % kSt;
        const int qrow = qbh * p.N + qt * kT;
        if (!in_bounds(qrow + kT <= p.BH * p.N, p.st, abort_flag)) return false;
        if (!mbar_wait(&bar_qe[st], ((n / kSt) & 1) ^ 1, p.st, abort_flag)) return false;
        mbar_arrive_expect_tx(&bar_qf[st], 2 * LY::kTile + 1024);
        tma_load_tile(sQ + st * LY::kTile, &tmQ, &bar_qf[st], qrow);
        tma_load_tile(sDO + st * LY::kTile, &tmDO, &bar_qf[st], qrow);
        bulk_load(sVec + st * 256, p.lse2 + qrow, 512, &bar_qf[st]);
        bulk_load(sVec + st * 256 + 128, p.dvec + qrow, 512, &bar_qf[st]);
        ++n;
        return true;
      });
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idSS = idesc_bf16_f32(kT, kT, false, false);  // K-major x K-major
      constexpr uint32_t idTS = idesc_bf16_f32(kT, D, false, true);    // TMEM A x MN-major B
      const uint32_t k_base = smem_u32(sK), v_base = smem_u32(sV);
      const uint32_t q_base = smem_u32(sQ), do_base = smem_u32(sDO);
      // TMEM column of the bf16 A operand for queries [16 kk, 16 kk + 16)
      auto a_col = [](int kk) -> uint32_t { return kk < 4 ? kk * 8 : 64 + (kk - 4) * 8; };
      auto issue_s = [&](int st) {
        const uint32_t qb = q_base + st * LY::kTile;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * LY::kSlab + (kk & 3) * 32;
          mma_bf16_ss(tS, sdesc_sw128(k_base + off, 16, 1024), sdesc_sw128(qb + off, 16, 1024), idSS,
                      kk > 0 ? 1u : 0u);
        }
        mma_commit(bar_sf);
      };
      bool ok = mbar_wait(bar_kv, 0, p.st, abort_flag) && mbar_wait(&bar_qf[0], 0, p.st, abort_flag);
      if (ok) {
        tc_fence_after();
        issue_s(0);
      }
      for (int n = 0; ok && n < n_total; ++n) {
        const int st = n % kSt;
        const uint32_t qb = q_base + st * LY::kTile, dob = do_base + st * LY::kTile;
        // dP^T = V dO^T (its columns were last read by dK of the previous step)
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * LY::kSlab + (kk & 3) * 32;
          mma_bf16_ss(tDP, sdesc_sw128(v_base + off, 16, 1024), sdesc_sw128(dob + off, 16, 1024), idSS,
                      kk > 0 ? 1u : 0u);
        }
        mma_commit(bar_dpf);
        // dV += P^T dO in two halves: queries {0-31, 64-95} as soon as the
        // element-wise warps have published them, then {32-63, 96-127}
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          if (!(ok = mbar_wait(half ? bar_pr : bar_ph, n & 1, p.st, abort_flag))) break;
          tc_fence_after();
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int kk = (j >> 1) * 4 + half * 2 + (j & 1);
            mma_bf16_ts(tDV, tS + a_col(kk), sdesc_sw128(dob + kk * 2048, LY::kSlab, 1024), idTS,
                        (n > 0 || half > 0 || j > 0) ? 1u : 0u);
          }
        }
        if (!ok) break;
        // S^T of the next query tile into the columns dV has just read
        if (n + 1 < n_total) {
          const int st1 = (n + 1) % kSt;
          if (!(ok = mbar_wait(&bar_qf[st1], ((n + 1) / kSt) & 1, p.st, abort_flag))) break;
          tc_fence_after();
          issue_s(st1);
        }
        // dK += dS^T Q
        if (!(ok = mbar_wait(bar_dsr, n & 1, p.st, abort_flag))) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kT / 16; ++kk)
          mma_bf16_ts(tDK, tDP + a_col(kk), sdesc_sw128(qb + kk * 2048, LY::kSlab, 1024), idTS,
                      (n > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&bar_qe[st]);
      }
      mma_commit(bar_done);
    }
  } else if (warp >= 4) {
    const int h = (warp >> 2) - 1;          // query columns [64 h, 64 h + 64)
    const int r = (warp & 3) * 32 + lane;   // key row = TMEM lane
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t cS = tS + lane_off + h * kHalf, cDP = tDP + lane_off + h * kHalf;
    const float2 sl22 = make_float2(p.scale_log2, p.scale_log2);
    int n = 0;
    const bool ok = walk.run([&](int, int, bool diag) {
      const int st = n % kSt;
      if (!__all_sync(FULL, mbar_wait(&bar_qf[st], (n / kSt) & 1, p.st, abort_flag))) return false;
      if (!__all_sync(FULL, mbar_wait(bar_sf, n & 1, p.st, abort_flag))) return false;
      tc_fence_after();
      const float* lse2 = sVec + st * 256 + h * kHalf;
      const float* dvec = lse2 + 128;
      float P[kHalf];
      load_row64(cS, P);
      // P^T (bf16) over the first 32 columns this group read, formed and
      // published in two halves of 32 queries so that dV starts on the first
#pragma unroll
      for (int half = 0; half < 2; ++half) {
#pragma unroll
        for (int c = 32 * half; c < 32 * half + 32; c += 2) {
          const float2 t = fma2(make_float2(P[c], P[c + 1]), sl22, make_float2(-lse2[c], -lse2[c + 1]));
          const float2 e = (D == 64 && (c / 2) % 2 == 1) ? ex2_poly2(t) : make_float2(ex2_approx(t.x), ex2_approx(t.y));
          P[c] = e.x;
          P[c + 1] = e.y;
        }
        if (diag) {
#pragma unroll
          for (int c = 32 * half; c < 32 * half + 32; ++c)
            if (r > h * kHalf + c) P[c] = 0.f;  // key r is in the future of the query
        }
        uint32_t pk[16];
#pragma unroll
        for (int x = 0; x < 16; ++x) pk[x] = pack_bf16x2(P[32 * half + 2 * x], P[32 * half + 2 * x + 1]);
        tmem_st16(cS + 16 * half, pk);
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(half ? bar_pr : bar_ph);
      }

      if (!__all_sync(FULL, mbar_wait(bar_dpf, n & 1, p.st, abort_flag))) return false;
      tc_fence_after();
      // dS^T = P^T (dP^T - D) as bf16 over the first half of this group's dP^T columns
      {
        uint32_t a[32], b[32];
        tmem_ld32(cDP, a);
        tmem_ld32(cDP + 32, b);
        tmem_ld_wait();
        uint32_t pk[32];
#pragma unroll
        for (int x = 0; x < 16; ++x) {
          const int q = 2 * x;
          pk[x] = pack_bf16x2(P[q] * (__uint_as_float(a[2 * x]) - dvec[q]),
                              P[q + 1] * (__uint_as_float(a[2 * x + 1]) - dvec[q + 1]));
          pk[16 + x] = pack_bf16x2(P[32 + q] * (__uint_as_float(b[2 * x]) - dvec[32 + q]),
                                   P[33 + q] * (__uint_as_float(b[2 * x + 1]) - dvec[33 + q]));
        }
        tmem_st32(cDP, pk);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar_dsr);
      ++n;
      return true;
    });
    if (ok && __all_sync(FULL, mbar_wait(bar_done, 0, p.st, abort_flag))) {
      tc_fence_after();
      if (in_bounds(krow0 + r < p.BHkv * p.N, p.st, abort_flag))
        store_dkdv<D>(tDK + lane_off + h * (D / 2), tDV + lane_off + h * (D / 2), (size_t)krow0 + r, h, p);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ===========================================================================
// dK, dV and dQ in one pass: key/value tile stationary, dQ reduced in fp32
// ===========================================================================
// The dK/dV loop above plus a fifth matmul per tile pair,
//   dQ^T_n = K^T dS^T_n   (M = d, N = 128 queries, K = 128 keys),
// whose 128 x 128 fp32 result is added into an fp32 dQ accumulator in HBM
// (L2-resident for the head group in flight).  It replaces the
// query-stationary pass, which recomputes S and dP (two of its three
// matmuls) to avoid those additions.  The sum over key tiles runs in
// whatever order the CTAs reach L2, so dQ is reproducible only up to fp32
// summation order; dK and dV are still written once per key tile.
//
// The additions are this pass's limiter: an SM moves fp32 reductions to L2
// at about 22 bytes per clock, whichever instruction carries them (scalar
// or vector reductions, or bulk reductions from shared memory, measured
// with all SMs busy), and each tile pair adds 64 KB -- about 3000 clocks,
// more than the pair's 2560 clocks of matmuls.  So a warpgroup of its own
// (the drain warps) keeps that path busy without pause, and the element-wise
// warps never wait on it.
//
// Both operands of dQ^T come from shared memory: K (stationary, read as an
// MN-major A operand) and dS^T (MN-major B), which the element-wise warps
// write beside their TMEM copy (the A operand of dK).  Tensor memory holds
// S^T [0,128), dP^T [128,256), dK [256,384), dV [384,512): dQ^T has no
// columns of its own and lands in the dP^T columns after dK has read dS^T
// from them.  The drain warps load all of it into registers and free the
// columns at once (dP^T of the next tile goes there), then add it into HBM
// while the next tile is computed: the additions stay off the chain
// dP -> dS -> dK, dQ^T -> next dP that sets the step time.  (Reading dK's
// dS^T from shared memory as well, so that dQ^T could go first, was slower:
// 32 KB more shared-memory reads per tile pair.)
//
// d = 64 (TMEM has room): dQ = dS K in its own columns (M = 128 queries,
// N = 64), double-buffered, so dP^T never waits for the drain.  The drain
// warps (TMEM lane = query row) stage each dQ tile into shared memory, 128-byte
// swizzled, and one thread adds it into the accumulator with two TMA tensor
// reductions (boxes of 32 fp32 columns x 128 rows).
//
// Warp roles (512 threads): warps 0-3 drain dQ^T (TMEM lane = d index),
// warps 4-11 element-wise (as in the dK/dV pass), warp 12 TMA producer,
// warp 13 MMA issuer, warp 14 TMEM allocator.
// MMA order per step n: dP_n and the two halves of dV_n in the order their
// inputs become ready (dP_n first when both are), S_{n+1}, dK_n, dQ^T_n.
constexpr int kThreadsF = 512;
// Register split: launched at kLaunchRegsF per thread (512 x 128 = 65536);
// the element-wise warpgroups rise to kEwRegsF and the drain warpgroup (128
// dQ^T values per thread) to kDrainRegsF, the producer/MMA warpgroup drops
// to kRoleRegsF: 256 x 144 + 128 x 144 + 128 x 80 = 65536.  The host
// launches this kernel only when the compiled register count equals
// kLaunchRegsF.
constexpr int kLaunchRegsF = 128;
constexpr uint32_t kEwRegsF = 144;
constexpr uint32_t kDrainRegsF = 144;
constexpr uint32_t kRoleRegsF = 80;
static_assert(256 * kEwRegsF + 128 * kDrainRegsF + 128 * kRoleRegsF <= kThreadsF * kLaunchRegsF,
              "register split exceeds launch");

template <int D>
struct FusedLayout {
  static constexpr int kStF = D == 64 ? 3 : 2;  // Q/dO stages
  static constexpr int kTile = kT * D * 2;
  static constexpr int kSlab = kT * 128;
  static constexpr int kK = 0;
  static constexpr int kV = kK + kTile;
  static constexpr int kQ = kV + kTile;
  static constexpr int kDO = kQ + kStF * kTile;
  static constexpr int kDS = kDO + kStF * kTile;  // dS^T bf16 [128 keys x 128 queries], two 64-query slabs
  // d = 64: the dQ tile staged for its TMA reduction, fp32 [128 rows x 64]
  // as two 128-byte swizzled boxes of 32 columns
  static constexpr int kStage = kDS + kT * kT * 2;
  static constexpr int kVec = kStage + (D == 64 ? kT * D * 4 : 0);  // per stage: lse*log2e [128], D [128]
  static constexpr int kBar = kVec + kStF * 1024;
  static constexpr int kNumBars = 1 + 2 * kStF + 10;
  static constexpr int kTmemSlot = kBar + kNumBars * 8;
  static constexpr int kAbort = kTmemSlot + 4;
  static constexpr int kBytes = kAbort + 4;
  // The tiles need a 1024-byte aligned base.  At d = 128 the layout leaves
  // less than 1024 bytes of the 227 KB a CTA may hold for aligning it, so
  // the launch asks for the maximum and the kernel checks its base.
  static constexpr int kAlloc = kBytes + 1024 <= kMaxDynSmem ? kBytes + 1024 : kMaxDynSmem;
};
static_assert(FusedLayout<128>::kBytes <= kMaxDynSmem, "fused backward tile set exceeds shared memory");
static_assert(FusedLayout<64>::kBytes <= kMaxDynSmem, "fused backward tile set exceeds shared memory");

template <int D>
__global__ void __launch_bounds__(kThreadsF, 1)
    bwd_fused_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                     const __grid_constant__ CUtensorMap tmDQ, const BParams p) {
  static_assert(D == 128 || D == 64, "head dimension 64 or 128");
  using LY = FusedLayout<D>;
  constexpr int kSt = LY::kStF;
  constexpr bool kD64 = D == 64;
  extern __shared__ uint8_t smem_fu[];
  const uint32_t pad = (1024 - (smem_u32(smem_fu) & 1023)) & 1023;
  if (pad + LY::kBytes > (uint32_t)p.smem_alloc) {
    // the shared-memory window cannot hold the aligned tile set: report, do nothing
    if (threadIdx.x == 0) atomicExch(p.st.word, (int)RA_ERR_UNSUPPORTED);
    return;
  }
  uint8_t* smem = smem_fu + pad;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  int kvbh, kt;
  grouped_order((int)blockIdx.x, p.num_tiles, p.BHkv, p.group, kvbh, kt);
  const int krow0 = kvbh * p.N + kt * kT;
  const int tps = p.L / kT;
  const int Hkv = p.H / p.G;
  const int qbh0 = (kvbh / Hkv) * p.H + (kvbh % Hkv) * p.G;
  const RingWalkKV walk{(kt * kT) / p.L, p.S, tps, kt, p.causal, qbh0, p.G};
  const int n_total = walk.count();

  uint8_t* sK = smem + LY::kK;
  uint8_t* sV = smem + LY::kV;
  uint8_t* sQ = smem + LY::kQ;
  uint8_t* sDO = smem + LY::kDO;
  uint8_t* sDS = smem + LY::kDS;
  float* sVec = reinterpret_cast<float*>(smem + LY::kVec);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + LY::kBar);
  uint64_t* bar_kv = bars;
  uint64_t* bar_qf = bar_kv + 1;
  uint64_t* bar_qe = bar_qf + kSt;
  uint64_t* bar_sf = bar_qe + kSt;    // S^T computed
  uint64_t* bar_dpf = bar_sf + 1;     // dP^T computed
  uint64_t* bar_ph = bar_dpf + 1;     // first half of P^T written to TMEM
  uint64_t* bar_pr = bar_ph + 1;      // all of P^T written to TMEM
  uint64_t* bar_dsr = bar_pr + 1;     // dS^T written to TMEM and shared memory
  uint64_t* bar_dqf = bar_dsr + 1;    // [2] dQ^T (d = 128: in the dP^T columns) / dQ buffer b computed
  uint64_t* bar_dqe = bar_dqf + 2;    // [2] ... loaded out: its columns free again
  uint64_t* bar_done = bar_dqe + 2;   // dK, dV final
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + LY::kTmemSlot);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + LY::kAbort);

  if (threadIdx.x == 0) {
    mbar_init(bar_kv, 1);
    for (int s = 0; s < kSt; ++s) {
      mbar_init(&bar_qf[s], 1);
      mbar_init(&bar_qe[s], 1);
    }
    mbar_init(bar_sf, 1);
    mbar_init(bar_dpf, 1);
    mbar_init(bar_ph, 2 * 128);
    mbar_init(bar_pr, 2 * 128);
    mbar_init(bar_dsr, 2 * 128);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bar_dqf[b], 1);
      mbar_init(&bar_dqe[b], 128);
    }
    mbar_init(bar_done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 14) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // d = 128: S^T, dP^T (shared with dQ^T), dK, dV, 128 columns each;
  // d = 64: S^T, dP^T, dK, dV (64), dQ buffers 0, 1 (64 each)
  const uint32_t tS = tmem, tDP = tmem + 128, tDK = tmem + 256, tDV = tmem + 256 + D;
  const uint32_t tDQ = tmem + 384;

  if (warp >= 12) {
    regs_dec<kRoleRegsF>();
    if (warp == 12 && lane == 0) {
      // ---------------- TMA producer ----------------
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmDO);
      mbar_arrive_expect_tx(bar_kv, 2 * LY::kTile);
      if (in_bounds(krow0 + kT <= p.BHkv * p.N, p.st, abort_flag)) {
        tma_load_tile(sK, &tmK, bar_kv, krow0);
        tma_load_tile(sV, &tmV, bar_kv, krow0);
      }
      int n = 0;
      walk.run([&](int qbh, int qt, bool) {
        const int st = n % kSt;
        const int qrow = qbh * p.N + qt * kT;
        if (!in_bounds(qrow + kT <= p.BH * p.N, p.st, abort_flag)) return false;
        if (!mbar_wait(&bar_qe[st], ((n / kSt) & 1) ^ 1, p.st, abort_flag)) return false;
        mbar_arrive_expect_tx(&bar_qf[st], 2 * LY::kTile + 1024);
        tma_load_tile(sQ + st * LY::kTile, &tmQ, &bar_qf[st], qrow);
        tma_load_tile(sDO + st * LY::kTile, &tmDO, &bar_qf[st], qrow);
        bulk_load(sVec + st * 256, p.lse2 + qrow, 512, &bar_qf[st]);
        bulk_load(sVec + st * 256 + 128, p.dvec + qrow, 512, &bar_qf[st]);
        ++n;
        return true;
      });
    } else if (warp == 13 && lane == 0) {
      // ---------------- MMA issuer ----------------
      constexpr uint32_t idSS = idesc_bf16_f32(kT, kT, false, false);  // K-major x K-major
      constexpr uint32_t idTS = idesc_bf16_f32(kT, D, false, true);    // TMEM A x MN-major B
      constexpr uint32_t idDQ = kD64 ? idesc_bf16_f32(kT, D, true, true)   // MN-major dS x MN-major K
                                     : idesc_bf16_f32(D, kT, true, true);  // MN-major K^T x MN-major dS^T
      const uint32_t k_base = smem_u32(sK), v_base = smem_u32(sV);
      const uint32_t q_base = smem_u32(sQ), do_base = smem_u32(sDO), ds_base = smem_u32(sDS);
      // P^T (dS^T) bf16 columns of K step kk: [0,32) and [64,96) of S^T (dP^T)
      constexpr auto a_col = [](int kk) constexpr -> uint32_t { return kk < 4 ? kk * 8 : 64 + (kk - 4) * 8; };
      // d = 64: each group builds its operand descriptors once and its K steps
      // add compile-time offsets inside the MMA instructions, which shortens
      // the single issuing thread's chain of dependent instructions between
      // MMAs (the d = 64 matmuls are short enough for it to matter: 1.078 ->
      // 1.024 ms on the 8k causal workload).  At d = 128 the same issue path
      // measured 2% slower, so the descriptors are built per step there.
      auto issue_s = [&](int st) {
        const uint32_t qb = q_base + st * LY::kTile;
        if constexpr (kD64) {
          const uint64_t a0 = sdesc_sw128(k_base, 16, 1024), b0 = sdesc_sw128(qb, 16, 1024);
          static_for<D / 16>([&](auto kc) {
            constexpr int kk = decltype(kc)::value;
            constexpr uint32_t off = kmajor_step(kk, LY::kSlab);
            mma_bf16_ss_at<off, off>(tS, a0, b0, idSS, kk > 0 ? 1u : 0u);
          });
        } else {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = kmajor_step(kk, LY::kSlab);
            mma_bf16_ss(tS, sdesc_sw128(k_base + off, 16, 1024), sdesc_sw128(qb + off, 16, 1024), idSS,
                        kk > 0 ? 1u : 0u);
          }
        }
        mma_commit(bar_sf);
      };
      bool ok = mbar_wait(bar_kv, 0, p.st, abort_flag) && mbar_wait(&bar_qf[0], 0, p.st, abort_flag);
      if (ok) {
        tc_fence_after();
        issue_s(0);
      }
      for (int n = 0; ok && n < n_total; ++n) {
        const int st = n % kSt;
        const uint32_t qb = q_base + st * LY::kTile, dob = do_base + st * LY::kTile;
        // dP^T = V dO^T (into the dP^T columns once the drain warps have loaded
        // dQ^T_{n-1} out of them) and dV += P^T dO in two halves (as the
        // element-wise warps publish P^T), each as soon as its input is ready;
        // dP^T, on the step's critical chain, goes first when both are
        auto issue_dp = [&]() {
          if constexpr (kD64) {
            const uint64_t a0 = sdesc_sw128(v_base, 16, 1024), b0 = sdesc_sw128(dob, 16, 1024);
            static_for<D / 16>([&](auto kc) {
              constexpr int kk = decltype(kc)::value;
              constexpr uint32_t off = kmajor_step(kk, LY::kSlab);
              mma_bf16_ss_at<off, off>(tDP, a0, b0, idSS, kk > 0 ? 1u : 0u);
            });
          } else {
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t off = kmajor_step(kk, LY::kSlab);
              mma_bf16_ss(tDP, sdesc_sw128(v_base + off, 16, 1024), sdesc_sw128(dob + off, 16, 1024), idSS,
                          kk > 0 ? 1u : 0u);
            }
          }
          mma_commit(bar_dpf);
        };
        // dV half `half`: queries {32 half .. +31, 64 + 32 half .. +31}, i.e.
        // K steps 2 half, 2 half + 1, 4 + 2 half, 5 + 2 half
        auto issue_dv = [&](int half) {
          if constexpr (kD64) {
            const uint64_t b0 = sdesc_sw128(dob, LY::kSlab, 1024);
            const uint32_t acc0 = (n > 0 || half > 0) ? 1u : 0u;
            auto group = [&](auto half_c) {
              constexpr int hf = decltype(half_c)::value;
              static_for<4>([&](auto jc) {
                constexpr int j = decltype(jc)::value;
                constexpr int kk = (j >> 1) * 4 + hf * 2 + (j & 1);
                mma_bf16_ts_at<mnmajor_step(kk)>(tDV, tS + a_col(kk), b0, idTS, j > 0 ? 1u : acc0);
              });
            };
            if (half == 0)
              group(std::integral_constant<int, 0>{});
            else
              group(std::integral_constant<int, 1>{});
          } else {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const int kk = (j >> 1) * 4 + half * 2 + (j & 1);
              mma_bf16_ts(tDV, tS + a_col(kk), sdesc_sw128(dob + mnmajor_step(kk), LY::kSlab, 1024), idTS,
                          (n > 0 || half > 0 || j > 0) ? 1u : 0u);
            }
          }
        };
        bool dp = false;
        int dv = 0;
        const unsigned long long t0 = globaltimer_ns();
        while (!dp || dv < 2) {
          if (!dp && (kD64 || n == 0 || mbar_try_wait(&bar_dqe[0], (n - 1) & 1))) {
            tc_fence_after();
            issue_dp();
            dp = true;
          } else if (dv < 2 && mbar_try_wait(dv ? bar_pr : bar_ph, n & 1)) {
            tc_fence_after();
            issue_dv(dv);
            ++dv;
          } else if (*abort_flag) {
            ok = false;
            break;
          } else if (globaltimer_ns() - t0 > p.st.timeout_ns) {
            atomicExch(p.st.word, (int)RA_ERR_TIMEOUT);
            *abort_flag = 1;
            ok = false;
            break;
          }
        }
        if (!ok) break;
        // S^T of the next query tile into the columns dV has read
        if (n + 1 < n_total) {
          const int st1 = (n + 1) % kSt;
          if (!(ok = mbar_wait(&bar_qf[st1], ((n + 1) / kSt) & 1, p.st, abort_flag))) break;
          tc_fence_after();
          issue_s(st1);
        }
        if (!(ok = mbar_wait(bar_dsr, n & 1, p.st, abort_flag))) break;
        tc_fence_after();
        // dK += dS^T Q (dS^T from the dP^T columns)
        if constexpr (kD64) {
          const uint64_t b0 = sdesc_sw128(qb, LY::kSlab, 1024);
          const uint32_t acc0 = n > 0 ? 1u : 0u;
          static_for<kT / 16>([&](auto kc) {
            constexpr int kk = decltype(kc)::value;
            mma_bf16_ts_at<mnmajor_step(kk)>(tDK, tDP + a_col(kk), b0, idTS, kk > 0 ? 1u : acc0);
          });
        } else {
#pragma unroll
          for (int kk = 0; kk < kT / 16; ++kk)
            mma_bf16_ts(tDK, tDP + a_col(kk), sdesc_sw128(qb + mnmajor_step(kk), LY::kSlab, 1024), idTS,
                        (n > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&bar_qe[st]);  // Q_n and dO_n are no longer read
        if constexpr (kD64) {
          // dQ = dS K into buffer n % 2 once the drain has loaded step n - 2 out of it
          const int b = n & 1;
          if (n >= 2 && !(ok = mbar_wait(&bar_dqe[b], ((n - 2) >> 1) & 1, p.st, abort_flag))) break;
          tc_fence_after();
          const uint64_t a0 = sdesc_sw128(ds_base, LY::kSlab, 1024), b0 = sdesc_sw128(k_base, LY::kSlab, 1024);
          const uint32_t tq = tDQ + b * D;
          static_for<kT / 16>([&](auto kc) {
            constexpr int kk = decltype(kc)::value;
            mma_bf16_ss_at<mnmajor_step(kk), mnmajor_step(kk)>(tq, a0, b0, idDQ, kk > 0 ? 1u : 0u);
          });
          mma_commit(&bar_dqf[b]);
        } else {
          // dQ^T = K^T dS^T over the dP^T columns (dK has been issued before it)
#pragma unroll
          for (int kk = 0; kk < kT / 16; ++kk)
            mma_bf16_ss(tDP, sdesc_sw128(k_base + kk * 2048, LY::kSlab, 1024),
                        sdesc_sw128(ds_base + kk * 2048, LY::kSlab, 1024), idDQ, kk > 0 ? 1u : 0u);
          mma_commit(&bar_dqf[0]);
        }
      }
      mma_commit(bar_done);
    }
  } else if (warp < 4 && kD64) {
    regs_inc<kDrainRegsF>();
    // ---------------- dQ drain, d = 64: one query row (TMEM lane) per thread ----------------
    const int r = warp * 32 + lane;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    // this thread's row of the two staging boxes (columns [0,32), [32,64)):
    // 128-byte row r, 16-byte chunk j at chunk j ^ (r % 8)
    const uint32_t stage_row = smem_u32(smem + LY::kStage) + r * 128;
    int m = 0;
    walk.run([&](int qbh, int qt, bool) {
      const int b = m & 1;
      if (!__all_sync(FULL, mbar_wait(&bar_dqf[b], (m >> 1) & 1, p.st, abort_flag))) return false;
      tc_fence_after();
      uint32_t a[2][32];
      tmem_ld32(tDQ + b * D + lane_off, a[0]);
      tmem_ld32(tDQ + b * D + lane_off + 32, a[1]);
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(&bar_dqe[b]);
      const int qrow = qbh * p.N + qt * kT;
      if (!in_bounds(qrow + kT <= p.BH * p.N, p.st, abort_flag)) return false;
      // the previous tile's reductions have read the staging boxes
      if (threadIdx.x == 0) bulk_wait_read_all();
      named_bar_sync(1, 128);
#pragma unroll
      for (int bx = 0; bx < 2; ++bx)
#pragma unroll
        for (int j = 0; j < 8; ++j)
          st_shared_v4(stage_row + bx * kT * 128 + ((j ^ (r & 7)) << 4),
                       __float_as_uint(__uint_as_float(a[bx][4 * j]) * p.scale),
                       __float_as_uint(__uint_as_float(a[bx][4 * j + 1]) * p.scale),
                       __float_as_uint(__uint_as_float(a[bx][4 * j + 2]) * p.scale),
                       __float_as_uint(__uint_as_float(a[bx][4 * j + 3]) * p.scale));
      fence_proxy_async_smem();
      named_bar_sync(1, 128);
      if (threadIdx.x == 0) {
        tma_add_2d(&tmDQ, smem + LY::kStage, 0, qrow);
        tma_add_2d(&tmDQ, smem + LY::kStage + kT * 128, 32, qrow);
        bulk_commit_group();
      }
      ++m;
      return true;
    });
    if (threadIdx.x == 0) bulk_wait_all();  // the staging boxes stay in use until the reductions are done
  } else if (warp < 4) {
    regs_inc<kDrainRegsF>();
    // ---------------- dQ drain: one d index (TMEM lane) per thread ----------------
    const int r = warp * 32 + lane;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    int m = 0;
    walk.run([&](int qbh, int qt, bool) {
      if (!__all_sync(FULL, mbar_wait(&bar_dqf[0], m & 1, p.st, abort_flag))) return false;
      tc_fence_after();
      // all 128 query columns of this d index: load, free the columns, add
      uint32_t a[4][32];
#pragma unroll
      for (int i = 0; i < 4; ++i) tmem_ld32(tDP + lane_off + 32 * i, a[i]);
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(&bar_dqe[0]);
      if (!in_bounds((qbh * p.N + qt * kT) + kT <= p.BH * p.N, p.st, abort_flag)) return false;
      float* dst = p.dqacc + ((size_t)qbh * p.N + qt * kT) * D + r;
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int c = 0; c < 32; ++c) red_add_f32(dst + (size_t)(32 * i + c) * D, __uint_as_float(a[i][c]) * p.scale);
      ++m;
      return true;
    });
  } else {
    regs_inc<kEwRegsF>();
    // ---------------- element-wise: P^T, dS^T; dK, dV epilogue ----------------
    const int h = (warp >> 2) - 1;          // query columns [64 h, 64 h + 64)
    const int r = (warp & 3) * 32 + lane;   // key row = TMEM lane
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t cS = tS + lane_off + h * kHalf, cDP = tDP + lane_off + h * kHalf;
    const float2 sl22 = make_float2(p.scale_log2, p.scale_log2);
    // this thread's row of the dS^T tile in shared memory: slab h, 128-byte
    // swizzled row r (16-byte chunk j stored at chunk j ^ (r % 8))
    const uint32_t ds_row = smem_u32(sDS) + h * LY::kSlab + r * 128;
    int n = 0;
    const bool ok = walk.run([&](int, int, bool diag) {
      const int st = n % kSt;
      if (!__all_sync(FULL, mbar_wait(&bar_qf[st], (n / kSt) & 1, p.st, abort_flag))) return false;
      if (!__all_sync(FULL, mbar_wait(bar_sf, n & 1, p.st, abort_flag))) return false;
      tc_fence_after();
      const float* lse2 = sVec + st * 256 + h * kHalf;
      const float* dvec = lse2 + 128;
      float P[kHalf];
      load_row64(cS, P);
#pragma unroll
      for (int half = 0; half < 2; ++half) {
#pragma unroll
        for (int c = 32 * half; c < 32 * half + 32; c += 2) {
          const float2 t = fma2(make_float2(P[c], P[c + 1]), sl22, make_float2(-lse2[c], -lse2[c + 1]));
          const float2 e = (kD64 && (c / 2) % 2 == 1) ? ex2_poly2(t) : make_float2(ex2_approx(t.x), ex2_approx(t.y));
          P[c] = e.x;
          P[c + 1] = e.y;
        }
        if (diag) {
#pragma unroll
          for (int c = 32 * half; c < 32 * half + 32; ++c)
            if (r > h * kHalf + c) P[c] = 0.f;  // key r is in the future of the query
        }
        uint32_t pk[16];
#pragma unroll
        for (int x = 0; x < 16; ++x) pk[x] = pack_bf16x2(P[32 * half + 2 * x], P[32 * half + 2 * x + 1]);
        tmem_st16(cS + 16 * half, pk);
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(half ? bar_pr : bar_ph);
      }
      // dP^T_n completes after dQ^T_{n-1} (in issue order), which was the
      // last reader of the shared-memory dS^T tile written below
      if (!__all_sync(FULL, mbar_wait(bar_dpf, n & 1, p.st, abort_flag))) return false;
      tc_fence_after();
      // dP^T columns of this group in; bf16 dS^T out over the first 32 of them
      // (the A operand of dK) and to row r of slab h of the shared-memory tile
      // (16-byte chunk j of the row at chunk j ^ (r % 8))
      {
        uint32_t a[32], b[32];
        tmem_ld32(cDP, a);
        tmem_ld32(cDP + 32, b);
        tmem_ld_wait();
#pragma unroll
        for (int g = 0; g < 2; ++g) {
          uint32_t pk[16];
#pragma unroll
          for (int x = 0; x < 16; ++x) {
            const int q = 32 * g + 2 * x;
            const uint32_t d0 = g ? b[2 * x] : a[2 * x], d1 = g ? b[2 * x + 1] : a[2 * x + 1];
            pk[x] = pack_bf16x2(P[q] * (__uint_as_float(d0) - dvec[q]), P[q + 1] * (__uint_as_float(d1) - dvec[q + 1]));
          }
          tmem_st16(cDP + 16 * g, pk);
#pragma unroll
          for (int j = 0; j < 4; ++j)
            st_shared_v4(ds_row + (((4 * g + j) ^ (r & 7)) << 4), pk[4 * j], pk[4 * j + 1], pk[4 * j + 2],
                         pk[4 * j + 3]);
        }
      }
      tmem_st_wait();
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bar_dsr);
      ++n;
      return true;
    });
    if (ok && __all_sync(FULL, mbar_wait(bar_done, 0, p.st, abort_flag))) {
      tc_fence_after();
      if (in_bounds(krow0 + r < p.BHkv * p.N, p.st, abort_flag))
        store_dkdv<D>(tDK + lane_off + h * (D / 2), tDV + lane_off + h * (D / 2), (size_t)krow0 + r, h, p);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 14) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// dq = bf16(dQ accumulator) (the accumulator holds scaled sums), four
// elements per thread per step; HBM-bound (reads 4 B, writes 2 B per element).
__global__ void __launch_bounds__(256) bwd_dq_convert_kernel(const float4* __restrict__ acc,
                                                             uint2* __restrict__ dq, int64_t n4) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += stride) {
    const float4 a = acc[i];
    dq[i] = make_uint2(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w));
  }
}

// ===========================================================================
// dQ: query tile stationary
// ===========================================================================
template <int D>
struct QLayout {
  static constexpr int kTile = kT * D * 2;
  static constexpr int kSlab = kT * 128;
  static constexpr int kKSt = D == 64 ? 6 : 4;  // K held from S until dQ
  static constexpr int kVSt = D == 64 ? 6 : 3;  // V held for dP
  static constexpr int kK = 0;
  static constexpr int kV = kK + kKSt * kTile;
  static constexpr int kBar = kV + kVSt * kTile;
  static constexpr int kNumBars = 1 + 2 * kKSt + 2 * kVSt + 5;
  static constexpr int kTmemSlot = kBar + kNumBars * 8;
  static constexpr int kAbort = kTmemSlot + 4;
  static constexpr int kBytes = kAbort + 4;
  static constexpr int kAlloc = kBytes + 1024;
};
static_assert(QLayout<128>::kAlloc <= kMaxDynSmem, "dQ tile set exceeds shared memory");

// Warp roles: warp 0 TMA producer (K, V per step), warp 1 MMA issuer,
// warp 2 TMEM allocator, warps 4-7 and 8-11 one thread per query row each,
// the first warpgroup on key columns [0,64), the second on [64,128): P, dS
// and half of the dQ epilogue.  The stationary Q and dO tiles live in tensor
// memory (written once by the element-wise warps), so all three matmuls take
// their A operand from TMEM and shared memory holds only the K, V ring:
// operand reads per step drop from 160 KB to 96 KB at d = 128 and the ring
// is 4 + 3 tiles deep.  TMEM: S [0,128), dP [128,256), dQ [256,256+D),
// Q [384,384+D/2), dO [448,448+D/2).  Each warpgroup writes its bf16 dS
// over the first 32 of the dP columns it has itself read (A operand of dQ in
// columns [0,32) and [64,96) of dP).
// MMA order per step n: dP_n, S_{n+1} (as soon as both warpgroups have
// loaded S_n), dQ_n; S_0 first.
template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_q_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                 const BParams p) {
  using LY = QLayout<D>;
  extern __shared__ uint8_t smem_q[];
  uint8_t* smem = smem_q + ((1024 - (smem_u32(smem_q) & 1023)) & 1023);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // heads in small groups; the heaviest causal query tiles (largest index) first
  int bh, rank;
  grouped_order((int)blockIdx.x, p.num_tiles, p.BH, p.group, bh, rank);
  const int qt = p.num_tiles - 1 - rank;
  const int qrow0 = bh * p.N + qt * kT;
  const int tps = p.L / kT;
  const RingWalkQ walk{(qt * kT) / p.L, p.S, tps, qt, p.causal};
  const int n_total = walk.count();

  uint8_t* sK = smem + LY::kK;
  uint8_t* sV = smem + LY::kV;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + LY::kBar);
  uint64_t* bar_qd = bars;                 // Q and dO written to TMEM
  uint64_t* bar_kf = bar_qd + 1;
  uint64_t* bar_ke = bar_kf + LY::kKSt;
  uint64_t* bar_vf = bar_ke + LY::kKSt;
  uint64_t* bar_ve = bar_vf + LY::kVSt;
  uint64_t* bar_sf = bar_ve + LY::kVSt;    // S computed
  uint64_t* bar_sfree = bar_sf + 1;        // S loaded by both warpgroups
  uint64_t* bar_dpf = bar_sfree + 1;       // dP computed
  uint64_t* bar_dsr = bar_dpf + 1;         // dS written to TMEM
  uint64_t* bar_done = bar_dsr + 1;        // dQ final
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + LY::kTmemSlot);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + LY::kAbort);

  if (threadIdx.x == 0) {
    mbar_init(bar_qd, 2 * 128);
    for (int s = 0; s < LY::kKSt; ++s) {
      mbar_init(&bar_kf[s], 1);
      mbar_init(&bar_ke[s], 1);
    }
    for (int s = 0; s < LY::kVSt; ++s) {
      mbar_init(&bar_vf[s], 1);
      mbar_init(&bar_ve[s], 1);
    }
    mbar_init(bar_sf, 1);
    mbar_init(bar_sfree, 2 * 128);
    mbar_init(bar_dpf, 1);
    mbar_init(bar_dsr, 2 * 128);
    mbar_init(bar_done, 1);
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
  const uint32_t tS = tmem, tDP = tmem + 128, tDQ = tmem + 256, tQ = tmem + 384, tDO = tmem + 448;

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      int n = 0;
      walk.run([&](int kt, bool) {
        const int ks = n % LY::kKSt, vs = n % LY::kVSt;
        const int krow = kv_head_of(bh, p.H, p.G) * p.N + kt * kT;
        if (!in_bounds(krow + kT <= p.BHkv * p.N, p.st, abort_flag)) return false;
        if (!mbar_wait(&bar_ke[ks], ((n / LY::kKSt) & 1) ^ 1, p.st, abort_flag)) return false;
        mbar_arrive_expect_tx(&bar_kf[ks], LY::kTile);
        tma_load_tile(sK + ks * LY::kTile, &tmK, &bar_kf[ks], krow);
        if (!mbar_wait(&bar_ve[vs], ((n / LY::kVSt) & 1) ^ 1, p.st, abort_flag)) return false;
        mbar_arrive_expect_tx(&bar_vf[vs], LY::kTile);
        tma_load_tile(sV + vs * LY::kTile, &tmV, &bar_vf[vs], krow);
        ++n;
        return true;
      });
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16_f32(kT, kT, false, false);  // TMEM A x K-major B
      constexpr uint32_t idDQ = idesc_bf16_f32(kT, D, false, true);   // TMEM dS x MN-major K
      const uint32_t k_base = smem_u32(sK), v_base = smem_u32(sV);
      auto a_col = [](int kk) -> uint32_t { return kk < 4 ? kk * 8 : 64 + (kk - 4) * 8; };
      // S_n = Q K_n^T, Q from TMEM (columns 8 kk hold d elements [16 kk, 16 kk + 16))
      auto issue_s = [&](int n) -> bool {
        const int ks = n % LY::kKSt;
        if (!mbar_wait(&bar_kf[ks], (n / LY::kKSt) & 1, p.st, abort_flag)) return false;
        tc_fence_after();
        const uint32_t kb = k_base + ks * LY::kTile;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * LY::kSlab + (kk & 3) * 32;
          mma_bf16_ts(tS, tQ + kk * 8, sdesc_sw128(kb + off, 16, 1024), idS, kk > 0 ? 1u : 0u);
        }
        mma_commit(bar_sf);
        return true;
      };
      bool ok = mbar_wait(bar_qd, 0, p.st, abort_flag);
      if (ok) tc_fence_after();
      ok = ok && issue_s(0);
      for (int n = 0; ok && n < n_total; ++n) {
        const int ks = n % LY::kKSt, vs = n % LY::kVSt;
        // dP = dO V^T, dO from TMEM; its columns were last read by dQ of the previous step
        if (!(ok = mbar_wait(&bar_vf[vs], (n / LY::kVSt) & 1, p.st, abort_flag))) break;
        tc_fence_after();
        const uint32_t vb = v_base + vs * LY::kTile;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * LY::kSlab + (kk & 3) * 32;
          mma_bf16_ts(tDP, tDO + kk * 8, sdesc_sw128(vb + off, 16, 1024), idS, kk > 0 ? 1u : 0u);
        }
        mma_commit(bar_dpf);
        mma_commit(&bar_ve[vs]);
        // scores of the next key tile once both warpgroups have read this one's
        if (n + 1 < n_total) {
          if (!(ok = mbar_wait(bar_sfree, n & 1, p.st, abort_flag))) break;
          if (!(ok = issue_s(n + 1))) break;
        }
        // dQ += dS K, dS read from the dP columns
        if (!(ok = mbar_wait(bar_dsr, n & 1, p.st, abort_flag))) break;
        tc_fence_after();
        const uint32_t kb = k_base + ks * LY::kTile;
#pragma unroll
        for (int kk = 0; kk < kT / 16; ++kk)
          mma_bf16_ts(tDQ, tDP + a_col(kk), sdesc_sw128(kb + kk * 2048, LY::kSlab, 1024), idDQ,
                      (n > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&bar_ke[ks]);
      }
      mma_commit(bar_done);
    }
  } else if (warp >= 4) {
    const int h = (warp >> 2) - 1;          // key columns [64 h, 64 h + 64)
    const int r = (warp & 3) * 32 + lane;   // query row = TMEM lane
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const bool row_ok = in_bounds(qrow0 + r < p.BH * p.N, p.st, abort_flag);
    const float nl2 = row_ok ? -p.lse2[qrow0 + r] : 0.f;
    const float Dr = row_ok ? p.dvec[qrow0 + r] : 0.f;
    const float2 sl22 = make_float2(p.scale_log2, p.scale_log2), nl22 = make_float2(nl2, nl2);
    // this row's Q and dO, d elements [D/2 h, D/2 h + D/2), into TMEM as bf16
    // pairs (column 8 kk + j holds elements 16 kk + 2 j, 16 kk + 2 j + 1)
    {
      const uint4* gq = reinterpret_cast<const uint4*>(p.q + ((size_t)qrow0 + r) * D + h * (D / 2));
      const uint4* gd = reinterpret_cast<const uint4*>(p.dout + ((size_t)qrow0 + r) * D + h * (D / 2));
      uint32_t wq[D / 4], wd[D / 4];
#pragma unroll
      for (int x = 0; x < D / 16; ++x) {
        const uint4 a = row_ok ? __ldg(gq + x) : make_uint4(0, 0, 0, 0);
        const uint4 b = row_ok ? __ldg(gd + x) : make_uint4(0, 0, 0, 0);
        wq[4 * x] = a.x; wq[4 * x + 1] = a.y; wq[4 * x + 2] = a.z; wq[4 * x + 3] = a.w;
        wd[4 * x] = b.x; wd[4 * x + 1] = b.y; wd[4 * x + 2] = b.z; wd[4 * x + 3] = b.w;
      }
      if constexpr (D == 128) {
        tmem_st32(tQ + lane_off + h * 32, wq);
        tmem_st32(tDO + lane_off + h * 32, wd);
      } else {
        tmem_st16(tQ + lane_off + h * 16, wq);
        tmem_st16(tDO + lane_off + h * 16, wd);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar_qd);
    }
    const uint32_t cS = tS + lane_off + h * kHalf, cDP = tDP + lane_off + h * kHalf;
    int n = 0;
    const bool ok = walk.run([&](int, bool diag) {
      if (!__all_sync(FULL, mbar_wait(bar_sf, n & 1, p.st, abort_flag))) return false;
      tc_fence_after();
      float P[kHalf];
      load_row64(cS, P);
      tc_fence_before();
      mbar_arrive(bar_sfree);  // the S columns may take the next tile's scores
#pragma unroll
      for (int c = 0; c < kHalf; c += 2) {
        const float2 t = fma2(make_float2(P[c], P[c + 1]), sl22, nl22);
        P[c] = ex2_approx(t.x);
        P[c + 1] = ex2_approx(t.y);
      }
      if (diag) {
#pragma unroll
        for (int c = 0; c < kHalf; ++c)
          if (h * kHalf + c > r) P[c] = 0.f;  // key in the future of query r
      }
      if (!__all_sync(FULL, mbar_wait(bar_dpf, n & 1, p.st, abort_flag))) return false;
      tc_fence_after();
      {
        uint32_t a[32], b[32];
        tmem_ld32(cDP, a);
        tmem_ld32(cDP + 32, b);
        tmem_ld_wait();
        uint32_t pk[32];
#pragma unroll
        for (int x = 0; x < 16; ++x) {
          pk[x] = pack_bf16x2(P[2 * x] * (__uint_as_float(a[2 * x]) - Dr),
                              P[2 * x + 1] * (__uint_as_float(a[2 * x + 1]) - Dr));
          pk[16 + x] = pack_bf16x2(P[32 + 2 * x] * (__uint_as_float(b[2 * x]) - Dr),
                                   P[33 + 2 * x] * (__uint_as_float(b[2 * x + 1]) - Dr));
        }
        tmem_st32(cDP, pk);  // bf16 dS over this group's first 32 dP columns (already read)
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar_dsr);
      ++n;
      return true;
    });
    if (ok && __all_sync(FULL, mbar_wait(bar_done, 0, p.st, abort_flag))) {
      tc_fence_after();
      const size_t qrow = (size_t)qrow0 + r;
      if (!row_ok) {
      } else if (p.dq32)
        store_acc_row_f32<D / 2>(tDQ + lane_off + h * (D / 2), p.scale, p.dq32 + qrow * D + h * (D / 2), 1);
      else
        store_acc_row<D / 2>(tDQ + lane_off + h * (D / 2), p.scale, p.dq + qrow * D + h * (D / 2));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// D_i = dO_i . O_i and lse_i * log2(e); with dqacc, also zeroes row i of
// the fp32 dQ accumulator.  One warp per row; HBM-bound.
template <int D>
__global__ void __launch_bounds__(256) bwd_preprocess_kernel(const __nv_bfloat16* __restrict__ out,
                                                             const __nv_bfloat16* __restrict__ dout,
                                                             const float* __restrict__ lse, float* __restrict__ dvec,
                                                             float* __restrict__ lse2, float* __restrict__ dqacc,
                                                             int64_t rows) {
  constexpr int E = D / 32;  // elements per lane (2 or 4)
  const int lane = threadIdx.x & 31;
  const int64_t w0 = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int64_t nw = (int64_t)gridDim.x * 8;
  for (int64_t row = w0; row < rows; row += nw) {
    const __nv_bfloat16* o = out + row * D + lane * E;
    const __nv_bfloat16* g = dout + row * D + lane * E;
    float acc = 0.f;
    if constexpr (E == 4) {
      const uint2 a = *reinterpret_cast<const uint2*>(o);
      const uint2 b = *reinterpret_cast<const uint2*>(g);
      const __nv_bfloat162* pa = reinterpret_cast<const __nv_bfloat162*>(&a);
      const __nv_bfloat162* pb = reinterpret_cast<const __nv_bfloat162*>(&b);
#pragma unroll
      for (int x = 0; x < 2; ++x) {
        const float2 fa = __bfloat1622float2(pa[x]), fb = __bfloat1622float2(pb[x]);
        acc = fmaf(fa.x, fb.x, acc);
        acc = fmaf(fa.y, fb.y, acc);
      }
    } else {
      const float2 fa = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(o));
      const float2 fb = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(g));
      acc = fmaf(fa.x, fb.x, fa.y * fb.y);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (lane == 0) {
      dvec[row] = acc;
      lse2[row] = lse[row] * kLog2e;
    }
    if (dqacc) {
      float4* z = reinterpret_cast<float4*>(dqacc + row * D);
#pragma unroll
      for (int c = lane; c < D / 4; c += 32) z[c] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
}

int sm_count() {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms;
}

// fp32 outputs of one shard pair's gradient (ringattn_bwd_pair).
struct PairOut {
  float* dq;   // added into
  float* dk;   // written, or added into with kv_add
  float* dv;
  int kv_add;
};

template <int D>
int launch_passes(const AttnArgs& a, const void* dout, void* dq, void* dk, void* dv, const float* dvec,
                  const float* lse2, float* dqacc, int phase_mask, cudaStream_t stream,
                  const PairOut* pair = nullptr);

template <int D>
int launch_d(const AttnArgs& a, const void* out, const float* lse, const void* dout, void* dq, void* dk, void* dv,
             void* workspace, size_t workspace_bytes, int phase_mask, cudaStream_t stream) {
  const int64_t rows = a.B * a.H * a.N;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const size_t vec_bytes = ((size_t)rows * 4 + 255) & ~(size_t)255;
  float* dvec = reinterpret_cast<float*>(ws);
  float* lse2 = reinterpret_cast<float*>(ws + vec_bytes);
  // the fused pass's fp32 dQ accumulator follows the two row vectors
  float* dqacc = (bwd_fused_supported(D) && workspace_bytes >= bwd_workspace_bytes(a.B, a.H, a.N, D, true))
                     ? reinterpret_cast<float*>(ws + 2 * vec_bytes)
                     : nullptr;
  if ((phase_mask & (kPhaseFused | kPhaseConvert)) && !dqacc) return RA_ERR_WORKSPACE;

  if (phase_mask & kPhasePre) {
    const int64_t want = (rows + 7) / 8;
    const int64_t cap = (int64_t)sm_count() * 16;
    const unsigned grid = (unsigned)(want < cap ? want : cap);
    bwd_preprocess_kernel<D><<<grid, 256, 0, stream>>>((const __nv_bfloat16*)out, (const __nv_bfloat16*)dout, lse,
                                                       dvec, lse2, dqacc, rows);
    if (cudaGetLastError() != cudaSuccess) return RA_ERR_CUDA;
  }
  if (phase_mask & (kPhaseKV | kPhaseQ | kPhaseFused)) {
    const int rc = launch_passes<D>(a, dout, dq, dk, dv, dvec, lse2, dqacc, phase_mask, stream);
    if (rc != RA_OK) return rc;
  }
  if (phase_mask & kPhaseConvert) {
    const int64_t n4 = rows * D / 4;
    const int64_t want = (n4 + 255) / 256, cap = (int64_t)sm_count() * 8;
    bwd_dq_convert_kernel<<<(unsigned)(want < cap ? want : cap), 256, 0, stream>>>(
        reinterpret_cast<const float4*>(dqacc), reinterpret_cast<uint2*>(dq), n4);
    if (cudaGetLastError() != cudaSuccess) return RA_ERR_CUDA;
  }
  return RA_OK;
}

// The tensor-core passes selected by phase_mask (kPhaseKV, kPhaseQ, kPhaseFused).
template <int D>
int launch_passes(const AttnArgs& a, const void* dout, void* dq, void* dk, void* dv, const float* dvec,
                  const float* lse2, float* dqacc, int phase_mask, cudaStream_t stream, const PairOut* pair) {
  const int64_t rows = a.B * a.H * a.N;

  alignas(64) CUtensorMap tq, tk, tv, tdo;
  const int64_t kv_rows = a.B * a.Hkv * a.N;
  if (make_tmap_bf16_tile(&tq, a.q, D, rows, kT) != RA_OK) return RA_ERR_CUDA;
  if (make_tmap_bf16_tile(&tk, a.k, D, kv_rows, kT) != RA_OK) return RA_ERR_CUDA;
  if (make_tmap_bf16_tile(&tv, a.v, D, kv_rows, kT) != RA_OK) return RA_ERR_CUDA;
  if (make_tmap_bf16_tile(&tdo, dout, D, rows, kT) != RA_OK) return RA_ERR_CUDA;
  BParams p{};
  p.q = (const __nv_bfloat16*)a.q;
  p.dout = (const __nv_bfloat16*)dout;
  p.lse2 = lse2;
  p.dvec = dvec;
  p.dq = (__nv_bfloat16*)dq;
  p.dk = (__nv_bfloat16*)dk;
  p.dv = (__nv_bfloat16*)dv;
  p.BH = (int)(a.B * a.H);
  p.H = (int)a.H;
  p.G = (int)(a.H / a.Hkv);
  p.BHkv = (int)(a.B * a.Hkv);
  p.N = (int)a.N;
  p.S = a.S;
  p.L = (int)(a.N / a.S);
  p.causal = a.causal;
  p.num_tiles = (int)(a.N / kT);
  p.scale = a.scale;
  p.scale_log2 = a.scale * kLog2e;
  int rc = current_status(&p.st);
  if (rc != RA_OK) return rc;
  p.dqacc = dqacc;
  if (pair) {
    p.dq32 = pair->dq;
    p.dk32 = pair->dk;
    p.dv32 = pair->dv;
    p.kv_add = pair->kv_add;
  }
  if (phase_mask & kPhaseKV) {
    // per key/value head: K, V and its query heads' Q, dO stream through L2
    p.group = head_group(p.num_tiles, p.BHkv, (double)a.N * D * 2 * (2 + 2 * p.G), 100.0e6);
    auto kern = bwd_kv_kernel<D>;
    if (set_smem_attr((const void*)kern, KVLayout<D>::kAlloc) != RA_OK) return RA_ERR_CUDA;
    kern<<<(unsigned)(p.BHkv * p.num_tiles), kThreads, KVLayout<D>::kAlloc, stream>>>(tq, tk, tv, tdo, p);
    if (cudaGetLastError() != cudaSuccess) return RA_ERR_CUDA;
  }
  if (phase_mask & kPhaseQ) {
    // per query head: Q, dO, K, V (bf16) stream through L2
    p.group = head_group(p.num_tiles, p.BH, (double)a.N * D * 4 * 2, 100.0e6);
    auto kern = bwd_q_kernel<D>;
    if (set_smem_attr((const void*)kern, QLayout<D>::kAlloc) != RA_OK) return RA_ERR_CUDA;
    kern<<<(unsigned)(p.BH * p.num_tiles), kThreads, QLayout<D>::kAlloc, stream>>>(tk, tv, p);
    if (cudaGetLastError() != cudaSuccess) return RA_ERR_CUDA;
  }
  if (phase_mask & kPhaseFused) {
    if (!fused_usable(D)) return RA_ERR_UNSUPPORTED;
    // d = 64: the dQ tiles reach the accumulator by TMA tensor reductions
    // (boxes of 32 fp32 columns x 128 rows); d = 128 adds with scalar
    // reductions and takes no map (tq stands in for it)
    alignas(64) CUtensorMap tdq = tq;
    if (D == 64 && make_tmap_f32_2d(&tdq, dqacc, D, rows, D * 4, 32, kT) != RA_OK) return RA_ERR_CUDA;
    // per key/value head: K, V, its query heads' Q, dO (bf16) and their
    // fp32 dQ accumulator rows stay in L2 while the head group is in flight
    p.group = head_group(p.num_tiles, p.BHkv, (double)a.N * D * (2.0 * (2 + 2 * p.G) + 4.0 * p.G), 100.0e6);
    p.smem_alloc = FusedLayout<D>::kAlloc;
    auto kern = bwd_fused_kernel<D>;
    if (set_smem_attr((const void*)kern, FusedLayout<D>::kAlloc) != RA_OK) return RA_ERR_CUDA;
    kern<<<(unsigned)(p.BHkv * p.num_tiles), kThreadsF, FusedLayout<D>::kAlloc, stream>>>(tq, tk, tv, tdo, tdq, p);
    if (cudaGetLastError() != cudaSuccess) return RA_ERR_CUDA;
  }
  return RA_OK;
}

}  // namespace

bool bwd_fused_supported(int64_t D) { return D == 128 || D == 64; }

// Whether bwd_fused_kernel may run on the current device: its register split
// (setmaxnreg) is sized for exactly kLaunchRegsF registers per thread at
// launch, so a build that compiled it to another count must not launch it
// (the split would then wait for registers that were never allocated).
// Decided once per device and cached.  Without a device nothing launches;
// the answer is then the build's (its register count is checked when the
// library is built).
bool fused_usable(int64_t D) {
  constexpr int kMaxDev = 64;
  static std::mutex mu;
  static signed char known[kMaxDev][2] = {};  // [device][d = 64, 128]: 0 unknown, 1 usable, -1 not
  if (D != 64 && D != 128) return false;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return true;
  }
  if (dev < 0 || dev >= kMaxDev) return false;
  const int i = D == 128;
  std::lock_guard<std::mutex> lk(mu);
  if (known[dev][i] == 0) {
    cudaFuncAttributes fa;
    const void* f = D == 128 ? (const void*)bwd_fused_kernel<128> : (const void*)bwd_fused_kernel<64>;
    const bool ok = cudaFuncGetAttributes(&fa, f) == cudaSuccess && fa.numRegs == kLaunchRegsF;
    known[dev][i] = ok ? 1 : -1;
  }
  return known[dev][i] > 0;
}

size_t bwd_workspace_bytes(int64_t B, int64_t H, int64_t N, int64_t D, bool fused) {
  if (B <= 0 || H <= 0 || N <= 0 || D <= 0) return 0;
  const size_t rows = (size_t)B * H * N;
  const size_t vec = (rows * 4 + 255) & ~(size_t)255;
  return 2 * vec + (fused ? rows * (size_t)D * 4 : 0);
}

int bwd_default_phases(int64_t D) {
  return bwd_fused_supported(D) && fused_usable(D) ? (kPhasePre | kPhaseFused | kPhaseConvert)
                                                   : (kPhasePre | kPhaseKV | kPhaseQ);
}

const char* bwd_tc_kernel_names(int64_t D) {
  if (D != 64 && D != 128) return nullptr;
  return (bwd_default_phases(D) & kPhaseFused) ? "bwd_preprocess_kernel+bwd_fused_kernel+bwd_dq_convert_kernel"
                                               : "bwd_preprocess_kernel+bwd_kv_kernel+bwd_q_kernel";
}

int launch_bwd_pair(const AttnArgs& a, const void* dout, const void* prep, float* dq_acc, float* dk_acc,
                    float* dv_acc, int kv_add, cudaStream_t stream) {
  const size_t vec_bytes = ((size_t)(a.B * a.H * a.N) * 4 + 255) & ~(size_t)255;
  const float* dvec = static_cast<const float*>(prep);
  const float* lse2 = reinterpret_cast<const float*>(static_cast<const uint8_t*>(prep) + vec_bytes);
  const PairOut po{dq_acc, dk_acc, dv_acc, kv_add};
  // the fused pass adds the scaled dQ into dq_acc itself; the split passes
  // add it in the query-stationary pass's epilogue
  const int phases = fused_usable(a.D) ? kPhaseFused : (kPhaseKV | kPhaseQ);
  float* acc = (phases & kPhaseFused) ? dq_acc : nullptr;
  if (a.D == 128)
    return launch_passes<128>(a, dout, nullptr, nullptr, nullptr, dvec, lse2, acc, phases, stream, &po);
  if (a.D == 64)
    return launch_passes<64>(a, dout, nullptr, nullptr, nullptr, dvec, lse2, acc, phases, stream, &po);
  return RA_ERR_UNSUPPORTED;
}

int launch_bwd_tc(const AttnArgs& a, const void* out, const float* lse, const void* dout, void* dq, void* dk,
                  void* dv, void* workspace, size_t workspace_bytes, int phase_mask, cudaStream_t stream) {
  if (a.D == 64)
    return launch_d<64>(a, out, lse, dout, dq, dk, dv, workspace, workspace_bytes, phase_mask, stream);
  if (a.D == 128)
    return launch_d<128>(a, out, lse, dout, dq, dk, dv, workspace, workspace_bytes, phase_mask, stream);
  return RA_ERR_UNSUPPORTED;
}

}  // namespace ra
