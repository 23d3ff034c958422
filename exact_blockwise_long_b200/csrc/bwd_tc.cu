// Backward of exact ring blockwise attention on the sm_100a tensor cores.
//
// The pages use the method for training ("training and inference", paper
// abstract) but print no backward algorithm; this is the plain chain rule
// through the softmax, recomputing P from the forward's log-sum-exp:
//   P_ij = exp(s_ij - lse_i) on visible pairs,  D_i = dO_i . O_i
//   dV_j += sum_i P_ij dO_i           dS_ij = P_ij (dO_i . V_j - D_i)
//   dK_j += scale sum_i dS_ij Q_i     dQ_i += scale sum_j dS_ij K_j
//
// Ring order, turned around for the key side: each CTA keeps one 128-key
// tile of KV shard j stationary (its dK, dV accumulate in tensor memory) and
// the query shards pass by in ring order i = (j + t) mod S; under the causal
// mask pairs i < j are skipped and the diagonal pair is masked in its tiles.
// The pairs visited are exactly the forward's pairs.
//
// Three launches:
//   preprocess  D_i = dO_i . O_i, lse_i * log2(e), dQ accumulator <- 0
//   main loop   per (key tile, query tile): 5 tcgen05 MMAs
//                 S^T  = K Q^T        (TMEM cols [0,128))
//                 dP^T = V dO^T       (TMEM cols [128,256))
//                 dV  += P^T dO       (P^T bf16 in TMEM over S^T)
//                 dK  += dS^T Q       (dS^T bf16 in TMEM over dP^T)
//                 dQ   = dS K         (dS from shared memory, result over dP^T)
//               dQ is drained from TMEM with fp32 vector reductions into the
//               dQ accumulator in HBM.
//   convert     dq = bf16(scale * dQ accumulator)
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace ra {
namespace {

constexpr int kT = 128;        // keys per CTA (TMEM lanes) and queries per step
constexpr int kQSt = 2;        // Q / dO stages
constexpr int kThreads = 256;
constexpr float kLog2e = 1.4426950408889634f;
constexpr uint32_t kTmemCols = 512;

template <int D>
struct BLayout {
  static constexpr int kTile = kT * D * 2;   // 128 rows x D bf16 (D/64 slabs of 16 KB)
  static constexpr int kSlab = kT * 128;
  static constexpr int kK = 0;
  static constexpr int kV = kK + kTile;
  static constexpr int kDS = kV + kTile;          // dS as an MN-major operand: 2 slabs [128 keys][64 queries]
  static constexpr int kQ = kDS + kT * kT * 2;
  static constexpr int kDO = kQ + kQSt * kTile;
  static constexpr int kVec = kDO + kQSt * kTile;  // per stage: lse*log2e [128] and D [128] (fp32)
  static constexpr int kBar = kVec + kQSt * 1024;
  static constexpr int kNumBars = 1 + 2 * kQSt + 7;
  static constexpr int kTmemSlot = kBar + kNumBars * 8;
  static constexpr int kAbort = kTmemSlot + 4;
  static constexpr int kBytes = kAbort + 4;
};
static_assert(BLayout<128>::kBytes <= 232448, "backward tile set exceeds shared memory");

struct BParams {
  const float* lse2;   // lse * log2(e)   [BH*N]
  const float* dvec;   // D_i = dO_i . O_i [BH*N]
  float* dq_acc;       // [BH*N, D] fp32
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  int BH, N, S, L, causal, num_tiles;
  int group;  // heads per scheduling group
  float scale, scale_log2;
  DevStatus st;
};

// Query tiles a key tile meets, in ring order.
struct RingWalkKV {
  int jshard, S, tps, kt, causal;
  template <typename F>
  __device__ __forceinline__ bool run(F&& body) const {
    for (int t = 0; t < S; ++t) {
      int i = jshard + t;
      if (i >= S) i -= S;
      if (causal && i < jshard) continue;
      const int qt0 = (causal && i == jshard) ? kt : i * tps;
      const int qt1 = i * tps + tps;
      for (int qt = qt0; qt < qt1; ++qt)
        if (!body(qt, causal && qt == kt)) return false;
    }
    return true;
  }
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                  const BParams p) {
  using LY = BLayout<D>;
  extern __shared__ __align__(1024) uint8_t smem[];
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (smem_u32(smem) & 1023) {  // the swizzled tiles need a 1024-byte aligned base
    if (threadIdx.x == 0) atomicExch(p.st.word, (int)RA_ERR_ALIGN);
    return;
  }

  // Work item: heads in small groups, so the CTAs in flight share a few
  // heads' Q, dO and dQ accumulator in L2; the heaviest causal key tiles
  // (smallest index) come first.
  int bh, kt;
  grouped_order((int)blockIdx.x, p.num_tiles, p.BH, p.group, bh, kt);
  const int krow0 = bh * p.N + kt * kT;
  const int tps = p.L / kT;
  RingWalkKV walk{(kt * kT) / p.L, p.S, tps, kt, p.causal};

  uint8_t* sK = smem + LY::kK;
  uint8_t* sV = smem + LY::kV;
  uint8_t* sDS = smem + LY::kDS;
  uint8_t* sQ = smem + LY::kQ;
  uint8_t* sDO = smem + LY::kDO;
  float* sVec = reinterpret_cast<float*>(smem + LY::kVec);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + LY::kBar);
  uint64_t* bar_kv = bars;
  uint64_t* bar_qf = bar_kv + 1;
  uint64_t* bar_qe = bar_qf + kQSt;
  uint64_t* bar_sf = bar_qe + kQSt;   // S^T computed
  uint64_t* bar_dpf = bar_sf + 1;     // dP^T computed
  uint64_t* bar_pr = bar_dpf + 1;     // P^T written to TMEM
  uint64_t* bar_dsr = bar_pr + 1;     // dS^T written to TMEM and shared memory
  uint64_t* bar_dqf = bar_dsr + 1;    // dQ computed
  uint64_t* bar_dqe = bar_dqf + 1;    // dQ drained
  uint64_t* bar_acc = bar_dqe + 1;    // dK, dV final
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + LY::kTmemSlot);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + LY::kAbort);

  if (threadIdx.x == 0) {
    mbar_init(bar_kv, 1);
    for (int s = 0; s < kQSt; ++s) {
      mbar_init(&bar_qf[s], 1);
      mbar_init(&bar_qe[s], 1);
    }
    mbar_init(bar_sf, 1);
    mbar_init(bar_dpf, 1);
    mbar_init(bar_pr, 128);
    mbar_init(bar_dsr, 128);
    mbar_init(bar_dqf, 1);
    mbar_init(bar_dqe, 128);
    mbar_init(bar_acc, 1);
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
      // ---------------- TMA producer ----------------
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmDO);
      mbar_arrive_expect_tx(bar_kv, 2 * LY::kTile);
#pragma unroll
      for (int s = 0; s < D / 64; ++s) {
        tma_load_2d(sK + s * LY::kSlab, &tmK, bar_kv, s * 64, krow0);
        tma_load_2d(sV + s * LY::kSlab, &tmV, bar_kv, s * 64, krow0);
      }
      int n = 0;
      walk.run([&](int qt, bool) {
        const int st = n % kQSt;
        const int qrow = bh * p.N + qt * kT;
        if (!mbar_wait(&bar_qe[st], ((n / kQSt) & 1) ^ 1, p.st, abort_flag)) return false;
        mbar_arrive_expect_tx(&bar_qf[st], 2 * LY::kTile + 1024);
#pragma unroll
        for (int s = 0; s < D / 64; ++s) {
          tma_load_2d(sQ + st * LY::kTile + s * LY::kSlab, &tmQ, &bar_qf[st], s * 64, qrow);
          tma_load_2d(sDO + st * LY::kTile + s * LY::kSlab, &tmDO, &bar_qf[st], s * 64, qrow);
        }
        bulk_load(sVec + st * 256, p.lse2 + qrow, 512, &bar_qf[st]);
        bulk_load(sVec + st * 256 + 128, p.dvec + qrow, 512, &bar_qf[st]);
        ++n;
        return true;
      });
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      constexpr uint32_t idSS = idesc_bf16_f32(kT, kT, false, false);  // K-major x K-major
      constexpr uint32_t idTS = idesc_bf16_f32(kT, D, false, true);    // TMEM A x MN-major B
      constexpr uint32_t idDQ = idesc_bf16_f32(kT, D, true, true);     // MN-major A x MN-major B
      const uint32_t k_base = smem_u32(sK), v_base = smem_u32(sV), ds_base = smem_u32(sDS);
      const uint32_t q_base = smem_u32(sQ), do_base = smem_u32(sDO);
      int n = 0;
      bool ok = mbar_wait(bar_kv, 0, p.st, abort_flag);
      if (ok) {
        ok = walk.run([&](int, bool) {
          const int st = n % kQSt;
          if (!mbar_wait(&bar_qf[st], (n / kQSt) & 1, p.st, abort_flag)) return false;
          tc_fence_after();
          const uint32_t qb = q_base + st * LY::kTile, dob = do_base + st * LY::kTile;
          // S^T = K Q^T  (the S^T / P^T region was last read by dV of the previous step)
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * LY::kSlab + (kk & 3) * 32;
            mma_bf16_ss(tS, sdesc_sw128(k_base + off, 16, 1024), sdesc_sw128(qb + off, 16, 1024), idSS,
                        kk > 0 ? 1u : 0u);
          }
          mma_commit(bar_sf);
          // dP^T = V dO^T, once the previous dQ has been drained from the same columns
          if (n > 0 && !mbar_wait(bar_dqe, (n - 1) & 1, p.st, abort_flag)) return false;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * LY::kSlab + (kk & 3) * 32;
            mma_bf16_ss(tDP, sdesc_sw128(v_base + off, 16, 1024), sdesc_sw128(dob + off, 16, 1024), idSS,
                        kk > 0 ? 1u : 0u);
          }
          mma_commit(bar_dpf);
          // dV += P^T dO
          if (!mbar_wait(bar_pr, n & 1, p.st, abort_flag)) return false;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < kT / 16; ++kk)
            mma_bf16_ts(tDV, tS + kk * 8, sdesc_sw128(dob + kk * 2048, LY::kSlab, 1024), idTS,
                        (n > 0 || kk > 0) ? 1u : 0u);
          // dK += dS^T Q ; dQ = dS K
          if (!mbar_wait(bar_dsr, n & 1, p.st, abort_flag)) return false;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < kT / 16; ++kk)
            mma_bf16_ts(tDK, tDP + kk * 8, sdesc_sw128(qb + kk * 2048, LY::kSlab, 1024), idTS,
                        (n > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
          for (int kk = 0; kk < kT / 16; ++kk)
            mma_bf16_ss(tDP, sdesc_sw128(ds_base + kk * 2048, LY::kSlab, 1024),
                        sdesc_sw128(k_base + kk * 2048, LY::kSlab, 1024), idDQ, kk > 0 ? 1u : 0u);
          mma_commit(bar_dqf);
          mma_commit(&bar_qe[st]);
          ++n;
          return true;
        });
      }
      mma_commit(bar_acc);
    }
  } else if (warp >= 4) {
    // ------- P^T, dS^T, dQ drain, dK/dV epilogue: one thread per key row -------
    const int r = (warp - 4) * 32 + lane;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const float sl2 = p.scale_log2;
    constexpr uint32_t FULL = 0xffffffffu;
    int n = 0;
    const bool ok = walk.run([&](int qt, bool diag) {
      const int st = n % kQSt;
      if (!__all_sync(FULL, mbar_wait(&bar_qf[st], (n / kQSt) & 1, p.st, abort_flag))) return false;
      if (!__all_sync(FULL, mbar_wait(bar_sf, n & 1, p.st, abort_flag))) return false;
      tc_fence_after();
      const float* lse2 = sVec + st * 256;
      const float* dvec = lse2 + 128;
      float P[kT];
#pragma unroll
      for (int c = 0; c < kT / 32; ++c) {
        uint32_t reg[32];
        tmem_ld32(tS + lane_off + c * 32, reg);
        tmem_ld_wait();
#pragma unroll
        for (int x = 0; x < 32; ++x) P[c * 32 + x] = __uint_as_float(reg[x]);
      }
#pragma unroll
      for (int c = 0; c < kT; ++c) {
        const float pv = ex2_approx(fmaf(P[c], sl2, -lse2[c]));
        P[c] = (diag && r > c) ? 0.f : pv;  // key r is in the future of query c
      }
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t pk[32];
#pragma unroll
        for (int x = 0; x < 32; ++x) pk[x] = pack_bf16x2(P[h * 64 + 2 * x], P[h * 64 + 2 * x + 1]);
        tmem_st32(tS + lane_off + h * 32, pk);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar_pr);

      if (!__all_sync(FULL, mbar_wait(bar_dpf, n & 1, p.st, abort_flag))) return false;
      tc_fence_after();
      // dS^T = P^T (dP^T - D), 32 query columns at a time; bf16 to TMEM (over
      // the dP^T columns already read) and to the MN-major shared operand.
      const uint32_t row_sw = (uint32_t)(r & 7);
      uint8_t* ds_row = sDS + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
      for (int c = 0; c < kT / 32; ++c) {
        uint32_t reg[32];
        tmem_ld32(tDP + lane_off + c * 32, reg);
        tmem_ld_wait();
        uint32_t pk[16];
#pragma unroll
        for (int x = 0; x < 16; ++x) {
          const int q0 = c * 32 + 2 * x;
          const float d0 = P[q0] * (__uint_as_float(reg[2 * x]) - dvec[q0]);
          const float d1 = P[q0 + 1] * (__uint_as_float(reg[2 * x + 1]) - dvec[q0 + 1]);
          pk[x] = pack_bf16x2(d0, d1);
        }
        tmem_st16(tDP + lane_off + c * 16, pk);
        // queries [32c, 32c+32) -> slab c/2, 16-byte chunks (c%2)*4 .. +4
        uint8_t* slab = ds_row + (c >> 1) * LY::kSlab;
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          const uint32_t chunk = (uint32_t)((c & 1) * 4 + x);
          *reinterpret_cast<uint4*>(slab + ((chunk ^ row_sw) << 4)) =
              make_uint4(pk[4 * x], pk[4 * x + 1], pk[4 * x + 2], pk[4 * x + 3]);
        }
      }
      tmem_st_wait();
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bar_dsr);

      // drain dQ (row r of this step's query tile) into the fp32 accumulator
      if (!__all_sync(FULL, mbar_wait(bar_dqf, n & 1, p.st, abort_flag))) return false;
      tc_fence_after();
      float* dq_row = p.dq_acc + ((size_t)bh * p.N + (size_t)qt * kT + r) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t reg[32];
        tmem_ld32(tDP + lane_off + c * 32, reg);
        tmem_ld_wait();
#pragma unroll
        for (int x = 0; x < 8; ++x)
          red_add_v4(dq_row + c * 32 + 4 * x, __uint_as_float(reg[4 * x]), __uint_as_float(reg[4 * x + 1]),
                     __uint_as_float(reg[4 * x + 2]), __uint_as_float(reg[4 * x + 3]));
      }
      tc_fence_before();
      mbar_arrive(bar_dqe);
      ++n;
      return true;
    });
    if (ok && __all_sync(FULL, mbar_wait(bar_acc, 0, p.st, abort_flag))) {
      tc_fence_after();
      const size_t grow = (size_t)krow0 + r;
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        const uint32_t tacc = which ? tDV : tDK;
        const float mul = which ? 1.f : p.scale;
        __nv_bfloat16* dst_row = (which ? p.dv : p.dk) + grow * D;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t reg[32];
          tmem_ld32(tacc + lane_off + c * 32, reg);
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
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// D_i = dO_i . O_i, lse_i * log2(e), and zero the dQ accumulator row.
// One warp per row; HBM-bound.
template <int D>
__global__ void __launch_bounds__(256) bwd_preprocess_kernel(const __nv_bfloat16* __restrict__ out,
                                                             const __nv_bfloat16* __restrict__ dout,
                                                             const float* __restrict__ lse, float* __restrict__ dvec,
                                                             float* __restrict__ lse2, float* __restrict__ dq_acc,
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
      *reinterpret_cast<float4*>(dq_acc + row * D + lane * E) = make_float4(0.f, 0.f, 0.f, 0.f);
    } else {
      const float2 fa = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(o));
      const float2 fb = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(g));
      acc = fmaf(fa.x, fb.x, fa.y * fb.y);
      *reinterpret_cast<float2*>(dq_acc + row * D + lane * E) = make_float2(0.f, 0.f);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (lane == 0) {
      dvec[row] = acc;
      lse2[row] = lse[row] * kLog2e;
    }
  }
}

// dq = bf16(scale * dq_acc), 8 elements per thread per step.
__global__ void __launch_bounds__(256) bwd_convert_kernel(const float* __restrict__ acc,
                                                          __nv_bfloat16* __restrict__ dq, float scale, int64_t n8) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n8; i += stride) {
    const float4 a = reinterpret_cast<const float4*>(acc)[2 * i];
    const float4 b = reinterpret_cast<const float4*>(acc)[2 * i + 1];
    uint4 o;
    o.x = pack_bf16x2(a.x * scale, a.y * scale);
    o.y = pack_bf16x2(a.z * scale, a.w * scale);
    o.z = pack_bf16x2(b.x * scale, b.y * scale);
    o.w = pack_bf16x2(b.z * scale, b.w * scale);
    reinterpret_cast<uint4*>(dq)[i] = o;
  }
}

int sm_count() {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms;
}

template <int D>
int launch_d(const AttnArgs& a, const void* out, const float* lse, const void* dout, void* dq, void* dk, void* dv,
             void* workspace, int phase_mask, cudaStream_t stream) {
  const int64_t rows = a.B * a.H * a.N;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* dq_acc = reinterpret_cast<float*>(ws);
  const size_t dq_bytes = ((size_t)rows * D * 4 + 255) & ~(size_t)255;
  const size_t vec_bytes = ((size_t)rows * 4 + 255) & ~(size_t)255;
  float* dvec = reinterpret_cast<float*>(ws + dq_bytes);
  float* lse2 = reinterpret_cast<float*>(ws + dq_bytes + vec_bytes);
  const int sms = sm_count();

  if (phase_mask & 1) {
    const int64_t want = (rows + 7) / 8;
    const unsigned grid = (unsigned)(want < (int64_t)sms * 16 ? want : (int64_t)sms * 16);
    bwd_preprocess_kernel<D><<<grid, 256, 0, stream>>>((const __nv_bfloat16*)out, (const __nv_bfloat16*)dout, lse,
                                                       dvec, lse2, dq_acc, rows);
    if (cudaGetLastError() != cudaSuccess) return RA_ERR_CUDA;
  }

  if (phase_mask & 2) {
  alignas(64) CUtensorMap tq, tk, tv, tdo;
  if (make_tmap_bf16_2d(&tq, a.q, D, rows, D * 2, 64, kT) != RA_OK) return RA_ERR_CUDA;
  if (make_tmap_bf16_2d(&tk, a.k, D, rows, D * 2, 64, kT) != RA_OK) return RA_ERR_CUDA;
  if (make_tmap_bf16_2d(&tv, a.v, D, rows, D * 2, 64, kT) != RA_OK) return RA_ERR_CUDA;
  if (make_tmap_bf16_2d(&tdo, dout, D, rows, D * 2, 64, kT) != RA_OK) return RA_ERR_CUDA;
  BParams p{};
  p.lse2 = lse2;
  p.dvec = dvec;
  p.dq_acc = dq_acc;
  p.dk = (__nv_bfloat16*)dk;
  p.dv = (__nv_bfloat16*)dv;
  p.BH = (int)(a.B * a.H);
  p.N = (int)a.N;
  p.S = a.S;
  p.L = (int)(a.N / a.S);
  p.causal = a.causal;
  p.num_tiles = (int)(a.N / kT);
  // per head: Q, dO, K, V (bf16) and the fp32 dQ accumulator
  p.group = head_group(p.num_tiles, p.BH, (double)a.N * D * (4 * 2 + 4), 100.0e6);
  p.scale = a.scale;
  p.scale_log2 = a.scale * kLog2e;
  int rc = current_status(&p.st);
  if (rc != RA_OK) return rc;
  auto kern = bwd_tc_kernel<D>;
  if (set_smem_attr((const void*)kern, BLayout<D>::kBytes) != RA_OK) return RA_ERR_CUDA;
  kern<<<(unsigned)(p.BH * p.num_tiles), kThreads, BLayout<D>::kBytes, stream>>>(tq, tk, tv, tdo, p);
  if (cudaGetLastError() != cudaSuccess) return RA_ERR_CUDA;
  }

  if (phase_mask & 4) {
    const int64_t n8 = rows * D / 8;
    const int64_t want = (n8 + 255) / 256;
    const unsigned grid = (unsigned)(want < (int64_t)sms * 16 ? want : (int64_t)sms * 16);
    bwd_convert_kernel<<<grid, 256, 0, stream>>>(dq_acc, (__nv_bfloat16*)dq, a.scale, n8);
    if (cudaGetLastError() != cudaSuccess) return RA_ERR_CUDA;
  }
  return RA_OK;
}

}  // namespace

int launch_bwd_tc(const AttnArgs& a, const void* out, const float* lse, const void* dout, void* dq, void* dk,
                  void* dv, void* workspace, int phase_mask, cudaStream_t stream) {
  if (a.D == 64) return launch_d<64>(a, out, lse, dout, dq, dk, dv, workspace, phase_mask, stream);
  if (a.D == 128) return launch_d<128>(a, out, lse, dout, dq, dk, dv, workspace, phase_mask, stream);
  return RA_ERR_UNSUPPORTED;
}

}  // namespace ra
