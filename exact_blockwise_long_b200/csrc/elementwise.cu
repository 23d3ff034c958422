// Element-wise helpers for the multi-device ring (chapterpal "Ring
// Attention", definition: each device keeps its query block while key/value
// blocks circulate; the backward's key/value gradients travel with them):
// fp32 accumulation of per-pair gradients and the final rounding of fp32
// accumulators to the output dtype.  HBM-bound, 16-byte accesses.
#include "common.cuh"
#include "internal.h"

namespace ra {
namespace {

// acc[i] += x[i] for 8 elements per thread (x bf16 or fp32)
template <typename T>
__global__ void __launch_bounds__(256) accumulate_kernel(float* __restrict__ acc, const T* __restrict__ x, int64_t n) {
  const int64_t i = ((int64_t)blockIdx.x * 256 + threadIdx.x) * 8;
  if (i >= n) return;
  if (i + 8 <= n) {
    float4 a0 = *reinterpret_cast<float4*>(acc + i), a1 = *reinterpret_cast<float4*>(acc + i + 4);
    float v[8];
    if constexpr (sizeof(T) == 2) {
      const uint4 q = *reinterpret_cast<const uint4*>(x + i);
      const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        v[2 * e] = __uint_as_float(w[e] << 16);
        v[2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u);
      }
    } else {
      const float4 b0 = *reinterpret_cast<const float4*>(x + i), b1 = *reinterpret_cast<const float4*>(x + i + 4);
      v[0] = b0.x, v[1] = b0.y, v[2] = b0.z, v[3] = b0.w, v[4] = b1.x, v[5] = b1.y, v[6] = b1.z, v[7] = b1.w;
    }
    a0.x += v[0], a0.y += v[1], a0.z += v[2], a0.w += v[3];
    a1.x += v[4], a1.y += v[5], a1.z += v[6], a1.w += v[7];
    *reinterpret_cast<float4*>(acc + i) = a0;
    *reinterpret_cast<float4*>(acc + i + 4) = a1;
  } else {
    for (int64_t j = i; j < n; ++j) {
      if constexpr (sizeof(T) == 2)
        acc[j] += __bfloat162float(x[j]);
      else
        acc[j] += x[j];
    }
  }
}

__global__ void __launch_bounds__(256) cast_bf16_kernel(const float* __restrict__ x, __nv_bfloat16* __restrict__ out,
                                                        int64_t n) {
  const int64_t i = ((int64_t)blockIdx.x * 256 + threadIdx.x) * 8;
  if (i >= n) return;
  if (i + 8 <= n) {
    const float4 a = *reinterpret_cast<const float4*>(x + i), b = *reinterpret_cast<const float4*>(x + i + 4);
    *reinterpret_cast<uint4*>(out + i) =
        make_uint4(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w), pack_bf16x2(b.x, b.y), pack_bf16x2(b.z, b.w));
  } else {
    for (int64_t j = i; j < n; ++j) out[j] = __float2bfloat16_rn(x[j]);
  }
}

unsigned blocks_for(int64_t n) { return (unsigned)((n + 256 * 8 - 1) / (256 * 8)); }

}  // namespace

int launch_accumulate(float* acc, const void* x, int64_t n, int dtype, cudaStream_t stream) {
  if (n == 0) return RA_OK;
  if (dtype == RA_BF16)
    accumulate_kernel<__nv_bfloat16><<<blocks_for(n), 256, 0, stream>>>(acc, static_cast<const __nv_bfloat16*>(x), n);
  else
    accumulate_kernel<float><<<blocks_for(n), 256, 0, stream>>>(acc, static_cast<const float*>(x), n);
  return cudaGetLastError() == cudaSuccess ? RA_OK : RA_ERR_CUDA;
}

int launch_cast(const float* x, void* out, int64_t n, int dtype, cudaStream_t stream) {
  if (n == 0) return RA_OK;
  if (dtype == RA_BF16) {
    cast_bf16_kernel<<<blocks_for(n), 256, 0, stream>>>(x, static_cast<__nv_bfloat16*>(out), n);
    return cudaGetLastError() == cudaSuccess ? RA_OK : RA_ERR_CUDA;
  }
  return cudaMemcpyAsync(out, x, (size_t)n * 4, cudaMemcpyDeviceToDevice, stream) == cudaSuccess ? RA_OK
                                                                                               : RA_ERR_CUDA;
}

}  // namespace ra
