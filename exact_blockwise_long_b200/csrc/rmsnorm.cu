// RMS normalisation of the blockwise transformer layer (pre-norm before the
// attention and before the feed-forward), forward and backward.  Per token
// row of d_model values:
//   rstd = (mean(x^2) + eps)^-1/2,  out = x * rstd * g
// and, for dout = dL/dout, with xhat = x * rstd:
//   dx = rstd * (g*dout - xhat * mean(g*dout*xhat))     (+ a residual gradient)
//   dg = sum over rows of dout * xhat
// HBM-bound: one warp per row, 16-byte loads and stores, fp32 arithmetic,
// one rounding to bf16 per output.  The dg column sums are taken per block
// of rows into fp32 partials and then summed in a fixed order, so the result
// is deterministic.
#include "common.cuh"
#include "internal.h"

namespace ra {
namespace {

constexpr int kWarps = 8;
constexpr int kDgRows = 64;  // rows per dg partial

__device__ __forceinline__ void unpack8(const uint4& q, float (&f)[8]) {
  const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    f[2 * e] = __uint_as_float(w[e] << 16);
    f[2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u);
  }
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

template <int V>
__global__ void __launch_bounds__(kWarps * 32) rmsnorm_fwd_kernel(const uint4* __restrict__ x, const uint4* __restrict__ g,
                                                                uint4* __restrict__ out, float* __restrict__ rstd,
                                                                int T, float eps) {
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * kWarps + (threadIdx.x >> 5);
  if (row >= T) return;
  constexpr int kVec = V * 32;  // 16-byte vectors per row
  const uint4* xr = x + (size_t)row * kVec;
  float f[V][8];
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < V; ++i) {
    unpack8(xr[i * 32 + lane], f[i]);
#pragma unroll
    for (int e = 0; e < 8; ++e) ss = fmaf(f[i][e], f[i][e], ss);
  }
  ss = warp_sum(ss);
  const float r = rsqrtf(ss / (float)(kVec * 8) + eps);
  uint4* orow = out + (size_t)row * kVec;
#pragma unroll
  for (int i = 0; i < V; ++i) {
    float gv[8];
    unpack8(g[i * 32 + lane], gv);
    orow[i * 32 + lane] = make_uint4(pack_bf16x2(f[i][0] * r * gv[0], f[i][1] * r * gv[1]),
                                     pack_bf16x2(f[i][2] * r * gv[2], f[i][3] * r * gv[3]),
                                     pack_bf16x2(f[i][4] * r * gv[4], f[i][5] * r * gv[5]),
                                     pack_bf16x2(f[i][6] * r * gv[6], f[i][7] * r * gv[7]));
  }
  if (lane == 0) rstd[row] = r;
}

template <int V>
__global__ void __launch_bounds__(kWarps * 32)
    rmsnorm_bwd_kernel(const uint4* __restrict__ x, const uint4* __restrict__ g, const float* __restrict__ rstd,
                       const uint4* __restrict__ dxn, const uint4* __restrict__ dres, uint4* __restrict__ dx, int T) {
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * kWarps + (threadIdx.x >> 5);
  if (row >= T) return;
  constexpr int kVec = V * 32;
  const size_t base = (size_t)row * kVec;
  const float r = rstd[row];
  float gd[V][8], xh[V][8];
  float dot = 0.f;
#pragma unroll
  for (int i = 0; i < V; ++i) {
    float xv[8], dv[8], gv[8];
    unpack8(x[base + i * 32 + lane], xv);
    unpack8(dxn[base + i * 32 + lane], dv);
    unpack8(g[i * 32 + lane], gv);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      gd[i][e] = gv[e] * dv[e];
      xh[i][e] = xv[e] * r;
      dot = fmaf(gd[i][e], xh[i][e], dot);
    }
  }
  const float mean = warp_sum(dot) / (float)(kVec * 8);
#pragma unroll
  for (int i = 0; i < V; ++i) {
    float o[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) o[e] = r * (gd[i][e] - xh[i][e] * mean);
    if (dres) {
      float rv[8];
      unpack8(dres[base + i * 32 + lane], rv);
#pragma unroll
      for (int e = 0; e < 8; ++e) o[e] += rv[e];
    }
    dx[base + i * 32 + lane] = make_uint4(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]),
                                          pack_bf16x2(o[4], o[5]), pack_bf16x2(o[6], o[7]));
  }
}

// partial[blk][c] = sum over the rows of block blk of dxn[t][c] * x[t][c] * rstd[t].
// Each thread owns eight adjacent columns (16-byte loads) and walks the
// block's rows four at a time, so eight independent loads are in flight.
constexpr int kDgThreads = 128;  // x 8 columns = 1024 columns per CTA
__global__ void __launch_bounds__(kDgThreads) rmsnorm_dg_partial_kernel(const uint4* __restrict__ x,
                                                                        const uint4* __restrict__ dxn,
                                                                        const float* __restrict__ rstd,
                                                                        float* __restrict__ partial, int T, int dm) {
  const int v = blockIdx.x * kDgThreads + threadIdx.x;  // 8-column group
  const int nv = dm / 8;
  if (v >= nv) return;
  const int t0 = blockIdx.y * kDgRows;
  const int t1 = min(T, t0 + kDgRows);
  float a[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) a[e] = 0.f;
  int t = t0;
  for (; t + 4 <= t1; t += 4) {
    uint4 xv[4], dv[4];
    float r[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      xv[u] = x[(size_t)(t + u) * nv + v];
      dv[u] = dxn[(size_t)(t + u) * nv + v];
      r[u] = rstd[t + u];
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      float xf[8], df[8];
      unpack8(xv[u], xf);
      unpack8(dv[u], df);
#pragma unroll
      for (int e = 0; e < 8; ++e) a[e] = fmaf(df[e], xf[e] * r[u], a[e]);
    }
  }
  for (; t < t1; ++t) {
    float xf[8], df[8];
    unpack8(x[(size_t)t * nv + v], xf);
    unpack8(dxn[(size_t)t * nv + v], df);
    const float r = rstd[t];
#pragma unroll
    for (int e = 0; e < 8; ++e) a[e] = fmaf(df[e], xf[e] * r, a[e]);
  }
  float4* dst = reinterpret_cast<float4*>(partial + (size_t)blockIdx.y * dm + (size_t)v * 8);
  dst[0] = make_float4(a[0], a[1], a[2], a[3]);
  dst[1] = make_float4(a[4], a[5], a[6], a[7]);
}

// dg[c] = sum over the blocks of partial[blk][c], in a fixed order: warp w
// of a CTA sums blocks w, w + 8, ... for 32 adjacent columns, then the eight
// warp sums are added in warp order.
__global__ void __launch_bounds__(256) rmsnorm_dg_reduce_kernel(const float* __restrict__ partial, int nblk, int dm,
                                                                float* __restrict__ dg) {
  __shared__ float sh[8][32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int c = blockIdx.x * 32 + lane;
  float s = 0.f;
  if (c < dm)
    for (int b = warp; b < nblk; b += 8) s += partial[(size_t)b * dm + c];
  sh[warp][lane] = s;
  __syncthreads();
  if (warp == 0 && c < dm) {
    float t = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) t += sh[w][lane];
    dg[c] = t;
  }
}

template <int V>
int fwd_v(const void* x, const void* g, void* out, float* rstd, int64_t T, float eps, cudaStream_t stream) {
  const unsigned grid = (unsigned)((T + kWarps - 1) / kWarps);
  rmsnorm_fwd_kernel<V><<<grid, kWarps * 32, 0, stream>>>((const uint4*)x, (const uint4*)g, (uint4*)out, rstd,
                                                           (int)T, eps);
  return cudaGetLastError() == cudaSuccess ? RA_OK : RA_ERR_CUDA;
}

template <int V>
int bwd_v(const void* x, const void* g, const float* rstd, const void* dxn, const void* dres, void* dx, int64_t T,
          cudaStream_t stream) {
  const unsigned grid = (unsigned)((T + kWarps - 1) / kWarps);
  rmsnorm_bwd_kernel<V><<<grid, kWarps * 32, 0, stream>>>((const uint4*)x, (const uint4*)g, rstd, (const uint4*)dxn,
                                                           (const uint4*)dres, (uint4*)dx, (int)T);
  return cudaGetLastError() == cudaSuccess ? RA_OK : RA_ERR_CUDA;
}

}  // namespace

size_t rmsnorm_dg_partial_floats(int64_t T, int64_t d_model) {
  return (size_t)((T + kDgRows - 1) / kDgRows) * (size_t)d_model;
}

int launch_rmsnorm_fwd(const void* x, const void* g, void* out, float* rstd, int64_t T, int64_t d_model, float eps,
                       cudaStream_t stream) {
  if (T <= 0) return RA_OK;
  if (T > INT32_MAX) return RA_ERR_UNSUPPORTED;
  switch (d_model) {
    case 256: return fwd_v<1>(x, g, out, rstd, T, eps, stream);
    case 512: return fwd_v<2>(x, g, out, rstd, T, eps, stream);
    case 1024: return fwd_v<4>(x, g, out, rstd, T, eps, stream);
    case 2048: return fwd_v<8>(x, g, out, rstd, T, eps, stream);
    case 4096: return fwd_v<16>(x, g, out, rstd, T, eps, stream);
    default: return RA_ERR_UNSUPPORTED;
  }
}

int launch_rmsnorm_bwd(const void* x, const void* g, const float* rstd, const void* dxn, const void* dres, void* dx,
                       float* dg, float* partial, int64_t T, int64_t d_model, cudaStream_t stream) {
  if (T <= 0) return cudaMemsetAsync(dg, 0, (size_t)d_model * 4, stream) == cudaSuccess ? RA_OK : RA_ERR_CUDA;
  if (T > INT32_MAX) return RA_ERR_UNSUPPORTED;
  int rc;
  switch (d_model) {
    case 256: rc = bwd_v<1>(x, g, rstd, dxn, dres, dx, T, stream); break;
    case 512: rc = bwd_v<2>(x, g, rstd, dxn, dres, dx, T, stream); break;
    case 1024: rc = bwd_v<4>(x, g, rstd, dxn, dres, dx, T, stream); break;
    case 2048: rc = bwd_v<8>(x, g, rstd, dxn, dres, dx, T, stream); break;
    case 4096: rc = bwd_v<16>(x, g, rstd, dxn, dres, dx, T, stream); break;
    default: return RA_ERR_UNSUPPORTED;
  }
  if (rc != RA_OK) return rc;
  const int nblk = (int)((T + kDgRows - 1) / kDgRows);
  const dim3 pgrid((unsigned)((d_model / 8 + kDgThreads - 1) / kDgThreads), (unsigned)nblk);
  rmsnorm_dg_partial_kernel<<<pgrid, kDgThreads, 0, stream>>>((const uint4*)x, (const uint4*)dxn, rstd, partial,
                                                              (int)T, (int)d_model);
  rmsnorm_dg_reduce_kernel<<<(unsigned)((d_model + 31) / 32), 256, 0, stream>>>(partial, nblk, (int)d_model, dg);
  return cudaGetLastError() == cudaSuccess ? RA_OK : RA_ERR_CUDA;
}

}  // namespace ra
