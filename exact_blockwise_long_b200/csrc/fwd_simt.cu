// Exact fp32 ring forward on CUDA cores.
//
// Same schedule as the tensor-core kernel -- query shard i visits KV shards
// j = (i - t) mod S in ring order, causal pairs j > i skipped, the diagonal
// pair masked on global indices -- but all arithmetic in fp32 FFMA with the
// accurate expf/logf, so fp32 inputs meet a 1e-4 absolute bound.  Used for
// fp32 inputs and, with bf16 inputs, for the step-materialised mode.
//
// Per CTA: 64 query rows, 4 threads per row, each thread owning D/4 output
// columns; key/value tiles of 64 keys staged in shared memory as fp32.
// Inside a shard the tiles are folded in with the online-softmax update
// (shard-local max, denominator, unnormalised output); at the end of every
// visited shard that shard-local state is merged into the running state with
// the exact log-sum-exp combine (darcstar note, DarcStar commentary, first
// paragraph: online softmax is associative across shards).
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace ra {
namespace {

constexpr int kBQ = 64;   // query rows per CTA
constexpr int kBK = 64;   // keys per shared-memory tile
constexpr int kTPR = 4;   // threads per query row
constexpr int kThreads = kBQ * kTPR;

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ void from_f32(float* p, float x) { *p = x; }
__device__ __forceinline__ void from_f32(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }

// Exact combine of two unnormalised states (m, l, acc[DP]); m = -inf is the
// neutral element and never enters a subtraction.
template <int DP>
__device__ __forceinline__ void merge_state(float& m, float& l, float (&acc)[DP], float mb, float lb,
                                            const float (&accb)[DP]) {
  if (mb == -INFINITY) return;
  if (m == -INFINITY) {
    m = mb;
    l = lb;
#pragma unroll
    for (int x = 0; x < DP; ++x) acc[x] = accb[x];
    return;
  }
  const float mn = fmaxf(m, mb);
  const float fa = expf(m - mn), fb = expf(mb - mn);
  l = fa * l + fb * lb;
#pragma unroll
  for (int x = 0; x < DP; ++x) acc[x] = fa * acc[x] + fb * accb[x];
  m = mn;
}

template <int D, typename T, bool kStep>
__global__ void __launch_bounds__(kThreads) fwd_simt_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                            const T* __restrict__ v, T* __restrict__ out,
                                                            float* __restrict__ lse, float* __restrict__ o_acc,
                                                            float* __restrict__ lse_acc, int N, int S,
                                                            int causal, float scale, int step, int H, int G) {
  constexpr int DP = D / kTPR;
  extern __shared__ float smem_f[];
  float* sK = smem_f;             // [kBK][D]
  float* sV = smem_f + kBK * D;   // [kBK][D]

  const int tid = threadIdx.x;
  const int r = tid / kTPR;
  const int part = tid % kTPR;
  const int bh = blockIdx.y;
  const int q0 = blockIdx.x * kBQ;
  const int L = N / S;
  const int ishard = q0 / L;
  const int row = q0 + r;
  const size_t head = (size_t)bh * N * D;
  const size_t kv_head = (size_t)((bh / H) * (H / G) + (bh % H) / G) * N * D;

  float qr[DP];
#pragma unroll
  for (int x = 0; x < DP; ++x) qr[x] = to_f32(q[head + (size_t)row * D + part * DP + x]);

  float m_run = -INFINITY, l_run = 0.f;
  float acc_run[DP];
#pragma unroll
  for (int x = 0; x < DP; ++x) acc_run[x] = 0.f;

  for (int t = 0; t < S; ++t) {
    if (kStep && t != step) continue;
    int j = ishard - t;
    if (j < 0) j += S;
    if (causal && j > ishard) continue;  // whole pair in the future: skipped
    const int kbeg = j * L;
    int kend = kbeg + L;
    if (causal && j == ishard) kend = min(kend, q0 + kBQ);  // later keys are masked for every row here

    float m_s = -INFINITY, l_s = 0.f;
    float acc_s[DP];
#pragma unroll
    for (int x = 0; x < DP; ++x) acc_s[x] = 0.f;

    for (int kt = kbeg; kt < kend; kt += kBK) {
      __syncthreads();
      for (int e = tid; e < kBK * D; e += kThreads) {
        const size_t g = kv_head + (size_t)kt * D + e;
        sK[e] = to_f32(k[g]);
        sV[e] = to_f32(v[g]);
      }
      __syncthreads();

      float s[kBK];
      float tmax = -INFINITY;
#pragma unroll
      for (int c = 0; c < kBK; ++c) {
        float dot = 0.f;
#pragma unroll
        for (int x = 0; x < DP; ++x) dot = fmaf(qr[x], sK[c * D + part * DP + x], dot);
        dot += __shfl_xor_sync(0xffffffffu, dot, 1);
        dot += __shfl_xor_sync(0xffffffffu, dot, 2);
        float sc = dot * scale;
        if (causal && (kt + c) > row) sc = -INFINITY;
        s[c] = sc;
        tmax = fmaxf(tmax, sc);
      }
      if (tmax == -INFINITY) continue;  // every key of this tile masked for this row
      const float m_new = fmaxf(m_s, tmax);
      const float alpha = (m_s == -INFINITY) ? 0.f : expf(m_s - m_new);
      l_s *= alpha;
#pragma unroll
      for (int x = 0; x < DP; ++x) acc_s[x] *= alpha;
#pragma unroll
      for (int c = 0; c < kBK; ++c) {
        const float p = (s[c] == -INFINITY) ? 0.f : expf(s[c] - m_new);
        l_s += p;
#pragma unroll
        for (int x = 0; x < DP; ++x) acc_s[x] = fmaf(p, sV[c * D + part * DP + x], acc_s[x]);
      }
      m_s = m_new;
    }
    // cross-shard log-sum-exp merge of this shard's partial into the ring state
    merge_state<DP>(m_run, l_run, acc_run, m_s, l_s, acc_s);
  }

  const size_t orow = head + (size_t)row * D + part * DP;
  if (!kStep) {
    const float inv = 1.f / l_run;
#pragma unroll
    for (int x = 0; x < DP; ++x) from_f32(&out[orow + x], acc_run[x] * inv);
    if (part == 0) lse[(size_t)bh * N + row] = m_run + logf(l_run);
  } else {
    if (m_run == -INFINITY) return;  // pair skipped: accumulators unchanged
    const float lse_t = m_run + logf(l_run);
    const size_t li = (size_t)bh * N + row;
    const float lse_a = lse_acc[li];
    float wa, wb, lse_new;
    if (lse_a == -INFINITY) {
      wa = 0.f;
      wb = 1.f;
      lse_new = lse_t;
    } else {
      const float mx = fmaxf(lse_a, lse_t);
      const float ea = expf(lse_a - mx), eb = expf(lse_t - mx);
      const float tot = ea + eb;
      lse_new = mx + logf(tot);
      wa = ea / tot;
      wb = eb / tot;
    }
    const float inv = 1.f / l_run;
#pragma unroll
    for (int x = 0; x < DP; ++x) {
      const float ot = acc_run[x] * inv;
      o_acc[orow + x] = (wa == 0.f) ? wb * ot : wa * o_acc[orow + x] + wb * ot;
    }
    __syncwarp();
    if (part == 0) lse_acc[li] = lse_new;
  }
}

template <int D, typename T>
int launch_typed(const AttnArgs& a, void* out, float* lse, float* o_acc, float* lse_acc, int step,
                 cudaStream_t stream) {
  const int smem = 2 * kBK * D * (int)sizeof(float);
  dim3 grid((unsigned)(a.N / kBQ), (unsigned)(a.B * a.H));
  if (step < 0) {
    auto kern = fwd_simt_kernel<D, T, false>;
    if (set_smem_attr((const void*)kern, smem) != RA_OK) return RA_ERR_CUDA;
    kern<<<grid, kThreads, smem, stream>>>((const T*)a.q, (const T*)a.k, (const T*)a.v, (T*)out, lse, nullptr,
                                           nullptr, (int)a.N, a.S, a.causal, a.scale, 0, (int)a.H,
                                           (int)(a.H / a.Hkv));
  } else {
    auto kern = fwd_simt_kernel<D, T, true>;
    if (set_smem_attr((const void*)kern, smem) != RA_OK) return RA_ERR_CUDA;
    kern<<<grid, kThreads, smem, stream>>>((const T*)a.q, (const T*)a.k, (const T*)a.v, nullptr, nullptr,
                                           o_acc, lse_acc, (int)a.N, a.S, a.causal, a.scale, step, (int)a.H,
                                           (int)(a.H / a.Hkv));
  }
  return cudaGetLastError() == cudaSuccess ? RA_OK : RA_ERR_CUDA;
}

}  // namespace

int launch_fwd_simt(const AttnArgs& a, void* out, float* lse, float* o_acc, float* lse_acc, int step,
                    cudaStream_t stream) {
  if (a.N % kBQ || (a.N / a.S) % kBQ) return RA_ERR_SHAPE;
  if (a.dtype == RA_F32) {
    if (a.D == 64) return launch_typed<64, float>(a, out, lse, o_acc, lse_acc, step, stream);
    if (a.D == 128) return launch_typed<128, float>(a, out, lse, o_acc, lse_acc, step, stream);
  } else {
    if (a.D == 64) return launch_typed<64, __nv_bfloat16>(a, out, lse, o_acc, lse_acc, step, stream);
    if (a.D == 128) return launch_typed<128, __nv_bfloat16>(a, out, lse, o_acc, lse_acc, step, stream);
  }
  return RA_ERR_UNSUPPORTED;
}

}  // namespace ra
