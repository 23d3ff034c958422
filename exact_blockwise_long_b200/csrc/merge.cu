// Standalone exact log-sum-exp merge of two normalised partials in HBM:
//   (o_a, lse_a) <- (o_a, lse_a) (+) (o_b, lse_b)
//   lse = ln(e^lse_a + e^lse_b),  o = e^(lse_a - lse) o_a + e^(lse_b - lse) o_b
// darcstar note, DarcStar commentary, first paragraph: partial attention from
// separate shards combines exactly because online softmax is associative.
//
// HBM-bound: per row it reads 2*D + 2 floats and writes D + 1.  One warp per
// row; each lane moves 16-byte float4 vectors; grid-stride over rows with a
// grid sized to the SM count.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace ra {
namespace {

constexpr int kWarps = 8;

__global__ void __launch_bounds__(kWarps * 32) merge_kernel(float* __restrict__ o_a, float* __restrict__ lse_a,
                                                            const float* __restrict__ o_b,
                                                            const float* __restrict__ lse_b, int64_t rows,
                                                            int D4) {
  const int lane = threadIdx.x & 31;
  const int64_t warp0 = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5);
  const int64_t nwarps = (int64_t)gridDim.x * kWarps;
  for (int64_t row = warp0; row < rows; row += nwarps) {
    const float la = lse_a[row];
    const float lb = __ldg(&lse_b[row]);
    float4* pa = reinterpret_cast<float4*>(o_a + row * (int64_t)D4 * 4);
    const float4* pb = reinterpret_cast<const float4*>(o_b + row * (int64_t)D4 * 4);
    const bool a_empty = (la == -INFINITY), b_empty = (lb == -INFINITY);
    if (b_empty && !a_empty) continue;  // neutral element on the right
    float wa = 0.f, wb = 0.f, lse = -INFINITY;
    if (!a_empty && !b_empty) {
      const float m = fmaxf(la, lb);
      const float ea = expf(la - m), eb = expf(lb - m);
      const float tot = ea + eb;
      lse = m + logf(tot);
      wa = ea / tot;
      wb = eb / tot;
    } else if (!b_empty) {
      wb = 1.f;
      lse = lb;
    }
    for (int c = lane; c < D4; c += 32) {
      float4 r;
      if (a_empty && b_empty) {
        r = make_float4(0.f, 0.f, 0.f, 0.f);
      } else if (a_empty) {
        r = __ldg(&pb[c]);
      } else {
        const float4 x = pa[c];
        const float4 y = __ldg(&pb[c]);
        r = make_float4(wa * x.x + wb * y.x, wa * x.y + wb * y.y, wa * x.z + wb * y.z, wa * x.w + wb * y.w);
      }
      pa[c] = r;
    }
    if (lane == 0) lse_a[row] = lse;
  }
}

}  // namespace

int launch_merge(float* o_a, float* lse_a, const float* o_b, const float* lse_b, int64_t rows, int64_t D,
                 cudaStream_t stream) {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) != cudaSuccess) return RA_ERR_CUDA;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int64_t want = (rows + kWarps - 1) / kWarps;
  int64_t cap = (int64_t)sms * 8;
  unsigned grid = (unsigned)(want < cap ? want : cap);
  if (grid == 0) return RA_OK;
  merge_kernel<<<grid, kWarps * 32, 0, stream>>>(o_a, lse_a, o_b, lse_b, rows, (int)(D / 4));
  return cudaGetLastError() == cudaSuccess ? RA_OK : RA_ERR_CUDA;
}

}  // namespace ra
