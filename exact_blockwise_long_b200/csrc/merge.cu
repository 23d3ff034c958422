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

// Weights of the two partials of one row; (-inf, anything) is the neutral
// element and never enters a subtraction.
__device__ __forceinline__ void merge_weights(float la, float lb, float& wa, float& wb, float& lse) {
  const bool a_empty = (la == -INFINITY), b_empty = (lb == -INFINITY);
  if (!a_empty && !b_empty) {
    const float m = fmaxf(la, lb);
    const float ea = expf(la - m), eb = expf(lb - m);
    const float tot = ea + eb;
    lse = m + logf(tot);
    wa = ea / tot;
    wb = eb / tot;
  } else if (!b_empty) {
    wa = 0.f;
    wb = 1.f;
    lse = lb;
  } else {  // right side empty: the left one stands; both empty: zero row, lse -inf
    wa = a_empty ? 0.f : 1.f;
    wb = 0.f;
    lse = la;
  }
}

// One warp per row pair per iteration: every load of both rows (the two
// LSEs and the D-float rows of both partials) is issued before any of them
// is used, so a row costs one memory round trip, not two.
__global__ void __launch_bounds__(kWarps * 32) merge_kernel(float* __restrict__ o_a, float* __restrict__ lse_a,
                                                            const float* __restrict__ o_b,
                                                            const float* __restrict__ lse_b, int64_t rows,
                                                            int D4) {
  const int lane = threadIdx.x & 31;
  const int64_t warp0 = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5);
  const int64_t nwarps = (int64_t)gridDim.x * kWarps;
  for (int64_t r0 = warp0; r0 < rows; r0 += 2 * nwarps) {
    const int64_t r1 = r0 + nwarps;
    const bool has1 = r1 < rows;
    const float la0 = lse_a[r0], lb0 = __ldg(&lse_b[r0]);
    const float la1 = has1 ? lse_a[r1] : -INFINITY, lb1 = has1 ? __ldg(&lse_b[r1]) : -INFINITY;
    float4* pa0 = reinterpret_cast<float4*>(o_a + r0 * (int64_t)D4 * 4);
    const float4* pb0 = reinterpret_cast<const float4*>(o_b + r0 * (int64_t)D4 * 4);
    float4* pa1 = reinterpret_cast<float4*>(o_a + r1 * (int64_t)D4 * 4);
    const float4* pb1 = reinterpret_cast<const float4*>(o_b + r1 * (int64_t)D4 * 4);
    for (int c = lane; c < D4; c += 32) {
      const float4 x0 = pa0[c], y0 = __ldg(&pb0[c]);
      float4 x1 = make_float4(0.f, 0.f, 0.f, 0.f), y1 = x1;
      if (has1) {
        x1 = pa1[c];
        y1 = __ldg(&pb1[c]);
      }
      float wa, wb, l;
      merge_weights(la0, lb0, wa, wb, l);
      // an empty side contributes nothing even if its payload is not finite
      pa0[c] = make_float4((wa != 0.f ? wa * x0.x : 0.f) + (wb != 0.f ? wb * y0.x : 0.f),
                           (wa != 0.f ? wa * x0.y : 0.f) + (wb != 0.f ? wb * y0.y : 0.f),
                           (wa != 0.f ? wa * x0.z : 0.f) + (wb != 0.f ? wb * y0.z : 0.f),
                           (wa != 0.f ? wa * x0.w : 0.f) + (wb != 0.f ? wb * y0.w : 0.f));
      if (has1) {
        merge_weights(la1, lb1, wa, wb, l);
        pa1[c] = make_float4((wa != 0.f ? wa * x1.x : 0.f) + (wb != 0.f ? wb * y1.x : 0.f),
                             (wa != 0.f ? wa * x1.y : 0.f) + (wb != 0.f ? wb * y1.y : 0.f),
                             (wa != 0.f ? wa * x1.z : 0.f) + (wb != 0.f ? wb * y1.z : 0.f),
                             (wa != 0.f ? wa * x1.w : 0.f) + (wb != 0.f ? wb * y1.w : 0.f));
      }
    }
    // every lane has read lse_a of both rows (top of this iteration) before
    // lane 0 overwrites them
    __syncwarp();
    if (lane == 0) {
      float wa, wb, l;
      merge_weights(la0, lb0, wa, wb, l);
      lse_a[r0] = l;
      if (has1) {
        merge_weights(la1, lb1, wa, wb, l);
        lse_a[r1] = l;
      }
    }
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
