// Decoding against a sharded key/value cache: one new query token per
// (batch, head) attends to all N cached keys, which lie in S ring shards.
//
// The paper abstract names training *and inference*; for a decode step the
// query is tiny and the cache is long, so the ring's exact combine is used
// the other way around: every shard (and, to fill the GPU, every split of a
// shard) yields a normalised partial (o_s, lse_s) for the query, and the
// partials are folded together with the exact log-sum-exp merge (darcstar
// note, DarcStar commentary, first paragraph: online softmax is associative,
// partials of separate shards combine exactly).
//
// Two launches:
//   partial  one CTA per (batch, key/value head, split of C keys): the
//            key/value tiles (64 keys) stream through shared memory by TMA
//            (two stages, 128-byte swizzle; shared memory sized to the group
//            so three CTAs share an SM); all G query heads that share the
//            key/value head are served from the same tile (the cache is read
//            once per key/value head).  Writes (o_s, lse_s) in fp32.
//   merge    one warp per (batch, head): exact merge over the splits,
//            writes bf16 out and fp32 lse.
// HBM-bound: the cache is read once, 4 N D bytes per key/value head.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace ra {
namespace {

constexpr int kKeys = 64;         // keys per tile
constexpr int kThreads = 256;
constexpr int kStages = 2;
constexpr int kQuarters = kThreads / kKeys;  // partial dots per key in the score phase
constexpr float kLog2e = 1.4426950408889634f;

template <int D, int G>
struct DLayout {
  static constexpr int kTile = kKeys * D * 2;
  static constexpr int kK = 0;
  static constexpr int kV = kK + kStages * kTile;
  static constexpr int kQ = kV + kStages * kTile;            // fp32 [G][D]
  static constexpr int kS = kQ + G * D * 4;                  // fp32 [quarters][G][kKeys] partial scores
  static constexpr int kP = kS + kQuarters * G * kKeys * 4;  // fp32 [G][kKeys]
  static constexpr int kRed = kP + G * kKeys * 4;            // fp32 [2][2 warps][G]
  static constexpr int kBar = kRed + 4 * G * 4;
  static constexpr int kBytes = kBar + kStages * 8 + 8;
  static constexpr int kAlloc = kBytes + 1024;
};
static_assert(DLayout<128, 16>::kAlloc <= 232448, "decode tile set exceeds shared memory");

struct DParams {
  const __nv_bfloat16* q;  // [B*H, D]
  float* part_o;           // [B*H, splits, D]
  float* part_lse;         // [B*H, splits]
  int H, G, N, splits, chunk;
  int L, pieces;           // shard length, pieces per shard
  float scale_log2;
  DevStatus st;
};

// swizzled element (row, col) of a [kKeys][D] bf16 tile loaded as 64-column
// slabs with the 128-byte swizzle
__device__ __forceinline__ const __nv_bfloat16* tile_at(const uint8_t* tile, int row, int col) {
  const int slab = col >> 6, c = col & 63;
  const int chunk = (c >> 3) ^ (row & 7);
  return reinterpret_cast<const __nv_bfloat16*>(tile + slab * (kKeys * 128) + row * 128 + chunk * 16) + (c & 7);
}

// Threads: scores -- thread t takes key t % 64 over head dimensions
// [D/4 (t / 64), +D/4) for every query head of the group (four partial dots
// per key, summed through shared memory); softmax -- threads 0..63, one key
// each, block max and block sum per query head; P V -- thread t takes the
// column pair 2 (t % (D/2)) over its share of the tile's keys, with packed
// f32x2 multiply-adds; the key shares are summed once, at the end.
template <int D, int G>
__global__ void __launch_bounds__(kThreads) decode_partial_kernel(const __grid_constant__ CUtensorMap tmK,
                                                                  const __grid_constant__ CUtensorMap tmV,
                                                                  const DParams p) {
  using LY = DLayout<D, G>;
  constexpr int kDimQ = D / kQuarters;         // head dimensions per partial dot
  constexpr int kPairs = D / 2;                // column pairs
  constexpr int kShares = kThreads / kPairs;   // key shares in P V
  constexpr int kPerShare = kKeys / kShares;
  extern __shared__ uint8_t smem_d[];
  uint8_t* smem = smem_d + ((1024 - (smem_u32(smem_d) & 1023)) & 1023);
  uint8_t* sK = smem + LY::kK;
  uint8_t* sV = smem + LY::kV;
  float* sQ = reinterpret_cast<float*>(smem + LY::kQ);
  float* sS = reinterpret_cast<float*>(smem + LY::kS);
  float* sP = reinterpret_cast<float*>(smem + LY::kP);
  float* sRed = reinterpret_cast<float*>(smem + LY::kRed);
  uint64_t* bar_full = reinterpret_cast<uint64_t*>(smem + LY::kBar);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + LY::kBar + kStages * 8);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int split = (int)(blockIdx.x % p.splits);
  const int kvbh = (int)(blockIdx.x / p.splits);
  const int Hkv = p.H / G;
  const int qbh0 = (kvbh / Hkv) * p.H + (kvbh % Hkv) * G;  // first query head of the group
  // split -> (ring shard, piece of at most `chunk` keys inside it)
  const int shard = split / p.pieces, piece = split % p.pieces;
  const int s0 = shard * p.L, s1 = min(p.N, s0 + p.L);
  const int k0 = s0 + piece * p.chunk;
  const int k1 = min(s1, k0 + p.chunk);
  const int ntiles = k1 > k0 ? (k1 - k0 + kKeys - 1) / kKeys : 0;

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) mbar_init(&bar_full[s], 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  for (int i = tid; i < G * D; i += kThreads) sQ[i] = __bfloat162float(p.q[(size_t)(qbh0 + i / D) * D + i % D]);
  __syncthreads();

  auto load = [&](int t) {
    const int s = t % kStages;
    const int row = kvbh * p.N + k0 + t * kKeys;
    mbar_arrive_expect_tx(&bar_full[s], 2 * LY::kTile);
    tma_load_tile(sK + s * LY::kTile, &tmK, &bar_full[s], row);
    tma_load_tile(sV + s * LY::kTile, &tmV, &bar_full[s], row);
  };
  if (tid == 0) {
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    for (int t = 0; t < min(kStages - 1, ntiles); ++t) load(t);
  }

  const int skey = tid % kKeys, quarter = tid / kKeys;    // score role
  const int pair = tid % kPairs, share = tid / kPairs;    // P V role
  float m[G], l[G];                                       // running max (log2 units) and denominator
  float2 acc[G];                                          // O[g][2 pair, 2 pair + 1] over this key share
#pragma unroll
  for (int g = 0; g < G; ++g) {
    m[g] = -INFINITY;
    l[g] = 0.f;
    acc[g] = make_float2(0.f, 0.f);
  }
  bool ok = true;
  for (int t = 0; t < ntiles; ++t) {
    const int s = t % kStages;
    // the stage refilled here was last read in tile t - 1, which every
    // thread has left (barrier at the end of each tile)
    if (tid == 0 && t + kStages - 1 < ntiles) load(t + kStages - 1);
    ok = __syncthreads_and(mbar_wait(&bar_full[s], (t / kStages) & 1, p.st, abort_flag));
    if (!ok) break;
    const uint8_t* tK = sK + s * LY::kTile;
    const uint8_t* tV = sV + s * LY::kTile;
    {
      float2 sc[G];
#pragma unroll
      for (int g = 0; g < G; ++g) sc[g] = make_float2(0.f, 0.f);
#pragma unroll
      for (int c = quarter * kDimQ; c < quarter * kDimQ + kDimQ; c += 8) {
        const uint4 raw = *reinterpret_cast<const uint4*>(tile_at(tK, skey, c));
        const __nv_bfloat162* kv = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 kf = __bfloat1622float2(kv[e]);
#pragma unroll
          for (int g = 0; g < G; ++g)
            sc[g] = fma2(kf, *reinterpret_cast<const float2*>(&sQ[g * D + c + 2 * e]), sc[g]);
        }
      }
#pragma unroll
      for (int g = 0; g < G; ++g) sS[(quarter * G + g) * kKeys + skey] = sc[g].x + sc[g].y;
    }
    __syncthreads();
    // softmax pieces: one key per thread of the first two warps
    float sv[G];
    if (tid < kKeys) {
      const bool live = (k0 + t * kKeys + tid) < k1;
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float x = (sS[g * kKeys + tid] + sS[(G + g) * kKeys + tid]) +
                  (sS[(2 * G + g) * kKeys + tid] + sS[(3 * G + g) * kKeys + tid]);
        x = live ? x * p.scale_log2 : -INFINITY;
        sv[g] = x;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
        if (lane == 0) sRed[warp * G + g] = x;
      }
    }
    __syncthreads();
    float alpha[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float mn = fmaxf(m[g], fmaxf(sRed[g], sRed[G + g]));
      alpha[g] = (m[g] == -INFINITY) ? 0.f : ex2_approx(m[g] - mn);
      m[g] = mn;
    }
    if (tid < kKeys) {
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float pv = ex2_approx(sv[g] - m[g]);  // 0 for keys past the end
        sP[g * kKeys + tid] = pv;
        float x = pv;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
        if (lane == 0) sRed[(2 + warp) * G + g] = x;
      }
    }
    __syncthreads();
#pragma unroll
    for (int g = 0; g < G; ++g) {
      l[g] = l[g] * alpha[g] + (sRed[2 * G + g] + sRed[3 * G + g]);
      acc[g].x *= alpha[g];
      acc[g].y *= alpha[g];
    }
    // P V over this thread's key share for its column pair
#pragma unroll
    for (int kk = 0; kk < kPerShare; ++kk) {
      const int k = share * kPerShare + kk;
      const float2 vf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(tile_at(tV, k, 2 * pair)));
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float pk = sP[g * kKeys + k];
        acc[g] = fma2(vf, make_float2(pk, pk), acc[g]);
      }
    }
    __syncthreads();  // this tile's stage, partial scores and P are free
  }
  if (!ok) return;
  // sum the key shares (in the key/value stages, all consumed by now) and
  // write the partials
  float* sO = reinterpret_cast<float*>(sK);  // [kShares][G][D]
  static_assert(kShares * G * D * 4 <= 2 * kStages * LY::kTile, "key-share sums exceed the stages");
#pragma unroll
  for (int g = 0; g < G; ++g) *reinterpret_cast<float2*>(&sO[(share * G + g) * D + 2 * pair]) = acc[g];
  __syncthreads();
  for (int i = tid; i < G * D; i += kThreads) {
    const int g = i / D, c = i % D;
    float o = 0.f;
#pragma unroll
    for (int sh = 0; sh < kShares; ++sh) o += sO[(sh * G + g) * D + c];
    const size_t prow = (size_t)(qbh0 + g) * p.splits + split;
    const bool empty = (l[g] == 0.f);
    p.part_o[prow * D + c] = empty ? 0.f : o / l[g];
    if (c == 0) p.part_lse[prow] = empty ? -INFINITY : (m[g] + __log2f(l[g])) * 0.6931471805599453f;
  }
}

// Exact log-sum-exp merge of the splits of every (batch, head).
template <int D>
__global__ void __launch_bounds__(256) decode_merge_kernel(const float* __restrict__ part_o,
                                                           const float* __restrict__ part_lse,
                                                           __nv_bfloat16* __restrict__ out, float* __restrict__ lse,
                                                           int rows, int splits) {
  const int lane = threadIdx.x & 31;
  const int row = (int)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (row >= rows) return;
  const float* pl = part_lse + (size_t)row * splits;
  float mx = -INFINITY;
  for (int s = 0; s < splits; ++s) mx = fmaxf(mx, pl[s]);
  float den = 0.f;
  float o[D / 32];
#pragma unroll
  for (int x = 0; x < D / 32; ++x) o[x] = 0.f;
  for (int s = 0; s < splits; ++s) {
    if (pl[s] == -INFINITY) continue;
    const float w = expf(pl[s] - mx);
    den += w;
    const float* po = part_o + ((size_t)row * splits + s) * D;
#pragma unroll
    for (int x = 0; x < D / 32; ++x) o[x] = fmaf(w, po[lane + 32 * x], o[x]);
  }
#pragma unroll
  for (int x = 0; x < D / 32; ++x) out[(size_t)row * D + lane + 32 * x] = __float2bfloat16_rn(o[x] / den);
  if (lane == 0) lse[row] = mx + logf(den);
}

template <int D, int G>
int launch_partial(const CUtensorMap& tk, const CUtensorMap& tv, const DParams& p, int grid, cudaStream_t stream) {
  auto kern = decode_partial_kernel<D, G>;
  if (set_smem_attr((const void*)kern, DLayout<D, G>::kAlloc) != RA_OK) return RA_ERR_CUDA;
  kern<<<grid, kThreads, DLayout<D, G>::kAlloc, stream>>>(tk, tv, p);
  return cudaGetLastError() == cudaSuccess ? RA_OK : RA_ERR_CUDA;
}

template <int D>
int launch_d(const void* q, const void* k, const void* v, void* out, float* lse, int64_t B, int64_t H, int64_t Hkv,
             int64_t N, int S, int k_chunk, float scale, void* workspace, cudaStream_t stream) {
  const int splits = decode_splits(N, S, k_chunk);
  const int L = (int)((N + S - 1) / S);
  alignas(64) CUtensorMap tk, tv;
  const uint64_t kv_rows = (uint64_t)(B * Hkv * N);
  if (make_tmap_bf16_tile(&tk, k, D, kv_rows, kKeys) != RA_OK) return RA_ERR_CUDA;
  if (make_tmap_bf16_tile(&tv, v, D, kv_rows, kKeys) != RA_OK) return RA_ERR_CUDA;
  DParams p{};
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.part_lse = static_cast<float*>(workspace);
  const size_t lse_bytes = ((size_t)B * H * splits * 4 + 255) & ~(size_t)255;
  p.part_o = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + lse_bytes);
  p.H = (int)H;
  p.G = (int)(H / Hkv);
  p.N = (int)N;
  p.splits = splits;
  p.chunk = k_chunk;
  p.L = L;
  p.pieces = splits / S;
  p.scale_log2 = scale * kLog2e;
  int rc = current_status(&p.st);
  if (rc != RA_OK) return rc;
  const int grid = (int)(B * Hkv) * splits;
  switch (p.G) {
    case 1: rc = launch_partial<D, 1>(tk, tv, p, grid, stream); break;
    case 2: rc = launch_partial<D, 2>(tk, tv, p, grid, stream); break;
    case 4: rc = launch_partial<D, 4>(tk, tv, p, grid, stream); break;
    case 8: rc = launch_partial<D, 8>(tk, tv, p, grid, stream); break;
    case 16: rc = launch_partial<D, 16>(tk, tv, p, grid, stream); break;
    default: return RA_ERR_UNSUPPORTED;
  }
  if (rc != RA_OK) return rc;
  const int rows = (int)(B * H);
  decode_merge_kernel<D><<<(rows + 7) / 8, 256, 0, stream>>>(p.part_o, p.part_lse, static_cast<__nv_bfloat16*>(out),
                                                             lse, rows, splits);
  return cudaGetLastError() == cudaSuccess ? RA_OK : RA_ERR_CUDA;
}

}  // namespace

int decode_splits(int64_t N, int S, int k_chunk) {
  // every ring shard is cut into pieces of at most k_chunk keys
  const int64_t L = (N + S - 1) / S;
  const int64_t per_shard = (L + k_chunk - 1) / k_chunk;
  return (int)(S * per_shard);
}

int launch_decode(const void* q, const void* k, const void* v, void* out, float* lse, int64_t B, int64_t H,
                  int64_t Hkv, int64_t N, int64_t D, int S, int k_chunk, float scale, void* workspace,
                  cudaStream_t stream) {
  if (D == 64) return launch_d<64>(q, k, v, out, lse, B, H, Hkv, N, S, k_chunk, scale, workspace, stream);
  if (D == 128) return launch_d<128>(q, k, v, out, lse, B, H, Hkv, N, S, k_chunk, scale, workspace, stream);
  return RA_ERR_UNSUPPORTED;
}

}  // namespace ra
