// The C ABI: argument validation, dispatch to the kernel launchers, the
// per-device status word and the tensor-map helper.
#include <cudaTypedefs.h>
#include <math.h>
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace ra {

// One status word per device (device variables are instantiated per device).
__device__ int g_status_word;

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_mu;
int* g_status_ptr[kMaxDevices] = {};

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

int current_status(DevStatus* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return RA_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_status_ptr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_status_word) != cudaSuccess || !ptr) return RA_ERR_CUDA;
    g_status_ptr[dev] = static_cast<int*>(ptr);
  }
  out->word = g_status_ptr[dev];
  out->timeout_ns = kDefaultTimeoutNs;
  return RA_OK;
}

namespace {
int make_tmap_2d(void* tmap, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t rows,
                 uint64_t row_pitch_bytes, uint32_t box_inner, uint32_t box_rows);
}

int make_tmap_bf16_2d(void* tmap, const void* base, uint64_t inner, uint64_t rows, uint64_t row_pitch_bytes,
                      uint32_t box_inner, uint32_t box_rows) {
  return make_tmap_2d(tmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, inner, rows, row_pitch_bytes, box_inner,
                      box_rows);
}

int make_tmap_bf16_tile(void* tmap, const void* base, uint64_t D, uint64_t rows, uint32_t box_rows) {
  if (D % 64 != 0 || D == 0) return RA_ERR_ARG;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_encode) {
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
          q != cudaDriverEntryPointSuccess || !fn)
        return RA_ERR_CUDA;
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
  }
  // dimensions: element within a 64-wide slab, row, slab (stride 128 B)
  cuuint64_t dims[3] = {64, rows, D / 64};
  cuuint64_t strides[2] = {D * 2, 128};
  cuuint32_t box[3] = {64, box_rows, (cuuint32_t)(D / 64)};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(reinterpret_cast<CUtensorMap*>(tmap), CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                        const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? RA_OK : RA_ERR_CUDA;
}

int make_tmap_f32_2d(void* tmap, const void* base, uint64_t inner, uint64_t rows, uint64_t row_pitch_bytes,
                     uint32_t box_inner, uint32_t box_rows) {
  return make_tmap_2d(tmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, base, inner, rows, row_pitch_bytes, box_inner,
                      box_rows);
}

namespace {
int make_tmap_2d(void* tmap, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t rows,
                 uint64_t row_pitch_bytes, uint32_t box_inner, uint32_t box_rows) {
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_encode) {
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
          q != cudaDriverEntryPointSuccess || !fn)
        return RA_ERR_CUDA;
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
  }
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {row_pitch_bytes};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(reinterpret_cast<CUtensorMap*>(tmap), dt, 2,
                        const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? RA_OK : RA_ERR_CUDA;
}
}  // namespace

int head_group(int per_head, int heads, double bytes_per_head, double budget_bytes) {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int g_waves = (2 * sms + per_head - 1) / per_head;
  const double g_fit = budget_bytes / (bytes_per_head > 1.0 ? bytes_per_head : 1.0);
  int g = g_fit > (double)g_waves ? (g_fit > 1e6 ? 1000000 : (int)g_fit) : g_waves;
  if (g < 1) g = 1;
  if (g > heads) g = heads;
  return g;
}

int set_smem_attr(const void* func, int bytes) {
  return cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) == cudaSuccess
             ? RA_OK
             : RA_ERR_CUDA;
}

// A kernel whose only job is to run a bounded wait out: one thread waits on
// an mbarrier that nothing arrives at, for timeout_ns, then latches
// RA_ERR_TIMEOUT and returns.
__global__ void selftest_timeout_kernel(DevStatus st) {
  __shared__ uint64_t bar;
  __shared__ volatile int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, st, &abort_flag);
  __syncthreads();
}

int launch_selftest_timeout(int timeout_us, cudaStream_t stream) {
  DevStatus st;
  int rc = current_status(&st);
  if (rc != RA_OK) return rc;
  st.timeout_ns = (unsigned long long)timeout_us * 1000ull;
  selftest_timeout_kernel<<<1, 32, 0, stream>>>(st);
  return cudaGetLastError() == cudaSuccess ? RA_OK : RA_ERR_CUDA;
}

}  // namespace ra

using namespace ra;

namespace {

// Internal marker: a valid request with an empty batch, head or sequence
// extent; the entry points return RA_OK without launching anything.
constexpr int kEmpty = 1;

int check_attn(const void* q, const void* k, const void* v, int64_t B, int64_t H, int64_t N, int64_t D,
               int dtype, int S, int q_chunk, int k_chunk, int causal) {
  if (B < 0 || H < 0 || N < 0 || S <= 0 || q_chunk <= 0 || k_chunk <= 0) return RA_ERR_ARG;
  if (causal != 0 && causal != 1) return RA_ERR_ARG;
  if (dtype != RA_BF16 && dtype != RA_F32) return RA_ERR_DTYPE;
  if (D != 64 && D != 128) return RA_ERR_UNSUPPORTED;
  if (B == 0 || H == 0 || N == 0) return kEmpty;  // nothing to compute
  if (!q || !k || !v) return RA_ERR_ARG;
  if (N % S) return RA_ERR_SHAPE;
  const int64_t L = N / S;
  if (L % q_chunk || L % k_chunk) return RA_ERR_SHAPE;
  const int tile = (dtype == RA_BF16) ? 128 : 64;
  if (q_chunk % tile || k_chunk % tile) return RA_ERR_SHAPE;
  if (B * H * N > (int64_t)INT32_MAX) return RA_ERR_UNSUPPORTED;  // row coordinate of the TMA tile maps (int32)
  if (!aligned16(q) || !aligned16(k) || !aligned16(v)) return RA_ERR_ALIGN;
  return RA_OK;
}

float resolve_scale(float scale, int64_t D) { return scale > 0.f ? scale : 1.0f / sqrtf((float)D); }

}  // namespace

extern "C" {

int ringattn_version(void) { return 100; }

const char* ringattn_status_string(int status) {
  switch (status) {
    case RA_OK: return "ok";
    case RA_ERR_ARG: return "invalid argument (null pointer or non-positive size)";
    case RA_ERR_SHAPE: return "shape rule violated (N % S, shard % chunk or chunk % tile)";
    case RA_ERR_DTYPE: return "unknown dtype";
    case RA_ERR_ALIGN: return "pointer not 16-byte aligned";
    case RA_ERR_UNSUPPORTED: return "unsupported configuration";
    case RA_ERR_CUDA: return "CUDA runtime error";
    case RA_ERR_TIMEOUT: return "device-side bounded wait timed out";
    case RA_ERR_WORKSPACE: return "workspace missing or too small";
    case RA_ERR_BOUNDS: return "bounds-checked build: an index fell outside its tensor";
    default: return "unknown status";
  }
}

const char* ringattn_kernel_plan(int op, int64_t N, int64_t D, int dtype, int S) {
  if (N <= 0 || S <= 0 || N % S) return nullptr;
  if (D != 64 && D != 128) return nullptr;
  if (dtype != RA_BF16 && dtype != RA_F32) return nullptr;
  if (op == 0) return dtype == RA_F32 ? "fwd_simt_kernel" : fwd_tc_kernel_name(N / S, D);
  if (op == 1) return dtype == RA_BF16 ? bwd_tc_kernel_names(D) : nullptr;
  return nullptr;
}

int ringattn_fwd(const void* q, const void* k, const void* v, void* out, float* lse, int64_t B, int64_t H,
                 int64_t N, int64_t D, int dtype, int S, int q_chunk, int k_chunk, int causal, float scale,
                 void* stream) {
  RA_NVTX_RANGE();
  return ringattn_fwd_gqa(q, k, v, out, lse, B, H, H, N, D, dtype, S, q_chunk, k_chunk, causal, scale, stream);
}

int ringattn_fwd_gqa(const void* q, const void* k, const void* v, void* out, float* lse, int64_t B, int64_t H,
                     int64_t Hkv, int64_t N, int64_t D, int dtype, int S, int q_chunk, int k_chunk, int causal,
                     float scale, void* stream) {
  RA_NVTX_RANGE();
  if (Hkv < 0 || (Hkv == 0 && H != 0) || (Hkv > 0 && H % Hkv != 0)) return RA_ERR_ARG;
  int rc = check_attn(q, k, v, B, H, N, D, dtype, S, q_chunk, k_chunk, causal);
  if (rc == kEmpty) return RA_OK;
  if (rc != RA_OK) return rc;
  if (!out || !lse) return RA_ERR_ARG;
  if (!aligned16(out) || !aligned16(lse)) return RA_ERR_ALIGN;
  AttnArgs a{q, k, v, B, H, N, D, dtype, S, q_chunk, k_chunk, causal, resolve_scale(scale, D), Hkv};
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dtype == RA_F32) return launch_fwd_simt(a, out, lse, nullptr, nullptr, -1, st);
  return launch_fwd_tc(a, out, lse, nullptr, nullptr, -1, st);
}

int ringattn_fwd_step(const void* q, const void* k, const void* v, float* o_acc, float* lse_acc, int64_t B,
                      int64_t H, int64_t N, int64_t D, int dtype, int S, int q_chunk, int k_chunk, int causal,
                      float scale, int t, void* stream) {
  RA_NVTX_RANGE();
  const int64_t Hkv = H;
  if (t < 0 || t >= S) return RA_ERR_ARG;
  int rc = check_attn(q, k, v, B, H, N, D, dtype, S, q_chunk, k_chunk, causal);
  if (rc == kEmpty) return RA_OK;
  if (rc != RA_OK) return rc;
  if (!o_acc || !lse_acc) return RA_ERR_ARG;
  if (!aligned16(o_acc) || !aligned16(lse_acc)) return RA_ERR_ALIGN;
  AttnArgs a{q, k, v, B, H, N, D, dtype, S, q_chunk, k_chunk, causal, resolve_scale(scale, D), Hkv};
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dtype == RA_F32) return launch_fwd_simt(a, nullptr, nullptr, o_acc, lse_acc, t, st);
  return launch_fwd_tc(a, nullptr, nullptr, o_acc, lse_acc, t, st);
}

int ringattn_merge(float* o_a, float* lse_a, const float* o_b, const float* lse_b, int64_t rows, int64_t D,
                   void* stream) {
  RA_NVTX_RANGE();
  if (!o_a || !lse_a || !o_b || !lse_b) return RA_ERR_ARG;
  if (rows < 0 || D <= 0) return RA_ERR_ARG;
  if (D % 4) return RA_ERR_SHAPE;
  if (!aligned16(o_a) || !aligned16(o_b) || !aligned16(lse_a) || !aligned16(lse_b)) return RA_ERR_ALIGN;
  if (rows == 0) return RA_OK;
  return launch_merge(o_a, lse_a, o_b, lse_b, rows, D, static_cast<cudaStream_t>(stream));
}

size_t ringattn_bwd_workspace_size(int64_t B, int64_t H, int64_t N, int64_t D) {
  return bwd_workspace_bytes(B, H, N, D, bwd_fused_supported(D));  // 0 for empty problems
}

}  // extern "C"

namespace ra {

int check_bwd_args(const void* q, const void* k, const void* v, const void* out, const float* lse, const void* dout,
                   const void* dq, const void* dk, const void* dv, int64_t B, int64_t H, int64_t Hkv, int64_t N,
                   int64_t D, int dtype, int S, int q_chunk, int k_chunk, int causal, int phase_mask) {
  if (phase_mask <= 0 || phase_mask > kPhaseAll) return RA_ERR_ARG;
  if (Hkv < 0 || (Hkv == 0 && H != 0) || (Hkv > 0 && H % Hkv != 0)) return RA_ERR_ARG;
  int rc = check_attn(q, k, v, B, H, N, D, dtype, S, q_chunk, k_chunk, causal);
  if (rc == kEmpty) return dtype == RA_BF16 ? kBwdEmpty : RA_ERR_UNSUPPORTED;
  if (rc != RA_OK) return rc;
  if (!out || !lse || !dout || !dq || !dk || !dv) return RA_ERR_ARG;
  if (!aligned16(out) || !aligned16(lse) || !aligned16(dout) || !aligned16(dq) || !aligned16(dk) ||
      !aligned16(dv))
    return RA_ERR_ALIGN;
  if (dtype != RA_BF16) return RA_ERR_UNSUPPORTED;
  if ((phase_mask & (kPhaseFused | kPhaseConvert)) && !bwd_fused_supported(D)) return RA_ERR_UNSUPPORTED;
  return RA_OK;
}

int run_bwd(const void* q, const void* k, const void* v, const void* out, const float* lse, const void* dout,
            void* dq, void* dk, void* dv, int64_t B, int64_t H, int64_t Hkv, int64_t N, int64_t D, int S,
            int q_chunk, int k_chunk, int causal, float scale, void* workspace, size_t workspace_bytes,
            int phase_mask, void* stream) {
  AttnArgs a{q, k, v, B, H, N, D, RA_BF16, S, q_chunk, k_chunk, causal, resolve_scale(scale, D), Hkv};
  return launch_bwd_tc(a, out, lse, dout, dq, dk, dv, workspace, workspace_bytes, phase_mask,
                       static_cast<cudaStream_t>(stream));
}

}  // namespace ra

namespace {
int bwd_impl(const void* q, const void* k, const void* v, const void* out, const float* lse, const void* dout,
             void* dq, void* dk, void* dv, int64_t B, int64_t H, int64_t Hkv, int64_t N, int64_t D, int dtype, int S,
             int q_chunk, int k_chunk, int causal, float scale, void* workspace, size_t workspace_bytes,
             int phase_mask, void* stream) {
  const int rc = check_bwd_args(q, k, v, out, lse, dout, dq, dk, dv, B, H, Hkv, N, D, dtype, S, q_chunk, k_chunk,
                                causal, phase_mask);
  if (rc == kBwdEmpty) return RA_OK;
  if (rc != RA_OK) return rc;
  const bool fused = (phase_mask & (kPhaseFused | kPhaseConvert)) != 0;
  if (!workspace || workspace_bytes < bwd_workspace_bytes(B, H, N, D, fused)) return RA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return RA_ERR_ALIGN;
  return run_bwd(q, k, v, out, lse, dout, dq, dk, dv, B, H, Hkv, N, D, S, q_chunk, k_chunk, causal, scale,
                 workspace, workspace_bytes, phase_mask, stream);
}
}  // namespace

extern "C" {

size_t ringattn_bwd_prepare_size(int64_t B, int64_t H, int64_t N) {
  return bwd_workspace_bytes(B, H, N, 1, false);  // two fp32 row vectors; 0 for empty problems
}

int ringattn_bwd_prepare(const void* out, const float* lse, const void* dout, void* prep, size_t prep_bytes,
                         int64_t B, int64_t H, int64_t N, int64_t D, int dtype, void* stream) {
  RA_NVTX_RANGE();
  if (B < 0 || H < 0 || N < 0) return RA_ERR_ARG;
  if (dtype != RA_BF16 && dtype != RA_F32) return RA_ERR_DTYPE;
  if (D != 64 && D != 128) return RA_ERR_UNSUPPORTED;
  if (dtype != RA_BF16) return RA_ERR_UNSUPPORTED;
  if (B == 0 || H == 0 || N == 0) return RA_OK;
  if (!out || !lse || !dout) return RA_ERR_ARG;
  if (!aligned16(out) || !aligned16(lse) || !aligned16(dout)) return RA_ERR_ALIGN;
  if (!prep || prep_bytes < ringattn_bwd_prepare_size(B, H, N)) return RA_ERR_WORKSPACE;
  if (!aligned16(prep)) return RA_ERR_ALIGN;
  AttnArgs a{nullptr, nullptr, nullptr, B, H, N, D, dtype, 1, 128, 128, 0, resolve_scale(0.f, D), H};
  return launch_bwd_tc(a, out, lse, dout, nullptr, nullptr, nullptr, prep, ringattn_bwd_prepare_size(B, H, N),
                       kPhasePre, static_cast<cudaStream_t>(stream));
}

int ringattn_bwd_pair(const void* q, const void* k, const void* v, const void* dout, const void* prep,
                      float* dq_acc, float* dk_acc, float* dv_acc, int64_t B, int64_t H, int64_t N, int64_t D,
                      int dtype, int q_chunk, int k_chunk, int diag, float scale, int kv_accumulate,
                      void* stream) {
  RA_NVTX_RANGE();
  if (kv_accumulate != 0 && kv_accumulate != 1) return RA_ERR_ARG;
  int rc = check_attn(q, k, v, B, H, N, D, dtype, 1, q_chunk, k_chunk, diag);
  if (rc == kEmpty) return dtype == RA_BF16 ? RA_OK : RA_ERR_UNSUPPORTED;
  if (rc != RA_OK) return rc;
  if (!dout || !dq_acc || !dk_acc || !dv_acc) return RA_ERR_ARG;
  if (!aligned16(dout) || !aligned16(dq_acc) || !aligned16(dk_acc) || !aligned16(dv_acc)) return RA_ERR_ALIGN;
  if (dtype != RA_BF16) return RA_ERR_UNSUPPORTED;
  if (!prep) return RA_ERR_WORKSPACE;
  if (!aligned16(prep)) return RA_ERR_ALIGN;
  AttnArgs a{q, k, v, B, H, N, D, dtype, 1, q_chunk, k_chunk, diag, resolve_scale(scale, D), H};
  return launch_bwd_pair(a, dout, prep, dq_acc, dk_acc, dv_acc, kv_accumulate, static_cast<cudaStream_t>(stream));
}

int ringattn_bwd_phase(const void* q, const void* k, const void* v, const void* out, const float* lse,
                       const void* dout, void* dq, void* dk, void* dv, int64_t B, int64_t H, int64_t N, int64_t D,
                       int dtype, int S, int q_chunk, int k_chunk, int causal, float scale, void* workspace,
                       size_t workspace_bytes, int phase_mask, void* stream) {
  RA_NVTX_RANGE();
  return bwd_impl(q, k, v, out, lse, dout, dq, dk, dv, B, H, H, N, D, dtype, S, q_chunk, k_chunk, causal, scale,
                  workspace, workspace_bytes, phase_mask, stream);
}

int ringattn_bwd_gqa(const void* q, const void* k, const void* v, const void* out, const float* lse,
                     const void* dout, void* dq, void* dk, void* dv, int64_t B, int64_t H, int64_t Hkv, int64_t N,
                     int64_t D, int dtype, int S, int q_chunk, int k_chunk, int causal, float scale,
                     void* workspace, size_t workspace_bytes, void* stream) {
  RA_NVTX_RANGE();
  return bwd_impl(q, k, v, out, lse, dout, dq, dk, dv, B, H, Hkv, N, D, dtype, S, q_chunk, k_chunk, causal, scale,
                  workspace, workspace_bytes, bwd_default_phases(D), stream);
}

int ringattn_bwd(const void* q, const void* k, const void* v, const void* out, const float* lse,
                 const void* dout, void* dq, void* dk, void* dv, int64_t B, int64_t H, int64_t N, int64_t D,
                 int dtype, int S, int q_chunk, int k_chunk, int causal, float scale, void* workspace,
                 size_t workspace_bytes, void* stream) {
  RA_NVTX_RANGE();
  return bwd_impl(q, k, v, out, lse, dout, dq, dk, dv, B, H, H, N, D, dtype, S, q_chunk, k_chunk, causal, scale,
                  workspace, workspace_bytes, bwd_default_phases(D), stream);
}

size_t ringattn_decode_workspace_size(int64_t B, int64_t H, int64_t N, int64_t D, int S, int k_chunk) {
  if (B <= 0 || H <= 0 || N <= 0 || D <= 0 || S <= 0 || k_chunk <= 0) return 0;
  const size_t splits = (size_t)decode_splits(N, S, k_chunk);
  const size_t lse_bytes = ((size_t)B * H * splits * 4 + 255) & ~(size_t)255;
  return lse_bytes + (size_t)B * H * splits * D * 4;
}

int ringattn_decode(const void* q, const void* k, const void* v, void* out, float* lse, int64_t B, int64_t H,
                    int64_t Hkv, int64_t N, int64_t D, int dtype, int S, int k_chunk, float scale, void* workspace,
                    size_t workspace_bytes, void* stream) {
  RA_NVTX_RANGE();
  if (B < 0 || H < 0 || N < 0 || Hkv <= 0 || S <= 0 || k_chunk <= 0) return RA_ERR_ARG;
  if (dtype != RA_BF16 && dtype != RA_F32) return RA_ERR_DTYPE;
  if (D != 64 && D != 128) return RA_ERR_UNSUPPORTED;
  if (H % Hkv) return RA_ERR_ARG;
  if (B == 0 || H == 0 || N == 0) return RA_OK;
  if (!q || !k || !v || !out || !lse) return RA_ERR_ARG;
  if (k_chunk % 128) return RA_ERR_SHAPE;
  if (dtype != RA_BF16) return RA_ERR_UNSUPPORTED;
  const int64_t G = H / Hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8 && G != 16) return RA_ERR_UNSUPPORTED;
  if (B * Hkv * N > (int64_t)INT32_MAX) return RA_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(lse)) return RA_ERR_ALIGN;
  if (!workspace || workspace_bytes < ringattn_decode_workspace_size(B, H, N, D, S, k_chunk)) return RA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return RA_ERR_ALIGN;
  return launch_decode(q, k, v, out, lse, B, H, Hkv, N, D, S, k_chunk, resolve_scale(scale, D), workspace,
                       static_cast<cudaStream_t>(stream));
}

size_t blockwise_ffn_workspace_size(int64_t chunk, int64_t d_ff, int dtype) {
  if (chunk <= 0 || d_ff <= 0) return 0;
  const size_t el = (dtype == RA_F32) ? 4 : 2;
  return (size_t)chunk * d_ff * el;
}

int blockwise_ffn(const void* x, const void* w1, const void* w2, const void* w3, void* y, int64_t T,
                  int64_t d_model, int64_t d_ff, int64_t chunk, int dtype, void* workspace,
                  size_t workspace_bytes, void* stream) {
  RA_NVTX_RANGE();
  if (T < 0 || d_model <= 0 || d_ff <= 0 || chunk <= 0) return RA_ERR_ARG;
  if (dtype != RA_BF16 && dtype != RA_F32) return RA_ERR_DTYPE;
  if (T == 0) return dtype == RA_BF16 ? RA_OK : RA_ERR_UNSUPPORTED;  // no tokens: nothing to compute
  if (!x || !w1 || !w2 || !w3 || !y) return RA_ERR_ARG;
  if (T % chunk || chunk % 128 || d_model % 128 || d_ff % 128) return RA_ERR_SHAPE;
  if (!aligned16(x) || !aligned16(w1) || !aligned16(w2) || !aligned16(w3) || !aligned16(y)) return RA_ERR_ALIGN;
  if (dtype != RA_BF16) return RA_ERR_UNSUPPORTED;
  if (!workspace || workspace_bytes < blockwise_ffn_workspace_size(chunk, d_ff, dtype)) return RA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return RA_ERR_ALIGN;
  return launch_ffn_tc(x, w1, w2, w3, y, T, d_model, d_ff, chunk, workspace, static_cast<cudaStream_t>(stream));
}

size_t blockwise_ffn_bwd_workspace_size(int64_t chunk, int64_t d_ff, int dtype) {
  if (chunk <= 0 || d_ff <= 0 || dtype != RA_BF16) return 0;
  return ffn_bwd_workspace_bytes(chunk, d_ff);
}

int blockwise_ffn_bwd(const void* x, const void* w1, const void* w2, const void* w3, const void* dy, void* dx,
                      float* dw1, float* dw2, float* dw3, int64_t T, int64_t d_model, int64_t d_ff, int64_t chunk,
                      int dtype, void* workspace, size_t workspace_bytes, void* stream) {
  RA_NVTX_RANGE();
  if (T < 0 || d_model <= 0 || d_ff <= 0 || chunk <= 0) return RA_ERR_ARG;
  if (dtype != RA_BF16 && dtype != RA_F32) return RA_ERR_DTYPE;
  if (dtype != RA_BF16) return RA_ERR_UNSUPPORTED;
  if (!w1 || !w2 || !w3 || !dw1 || !dw2 || !dw3) return RA_ERR_ARG;
  if (T > 0 && (!x || !dy || !dx)) return RA_ERR_ARG;  // token buffers may be null when there are no tokens
  if (T % chunk || chunk % 128 || d_model % 128 || d_ff % 128) return RA_ERR_SHAPE;
  if (!aligned16(x) || !aligned16(w1) || !aligned16(w2) || !aligned16(w3) || !aligned16(dy) || !aligned16(dx) ||
      !aligned16(dw1) || !aligned16(dw2) || !aligned16(dw3))
    return RA_ERR_ALIGN;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (T == 0) {  // no tokens: the weight gradients are zero
    const size_t wbytes = (size_t)d_ff * d_model * sizeof(float);
    if (cudaMemsetAsync(dw1, 0, wbytes, st) != cudaSuccess || cudaMemsetAsync(dw2, 0, wbytes, st) != cudaSuccess ||
        cudaMemsetAsync(dw3, 0, wbytes, st) != cudaSuccess)
      return RA_ERR_CUDA;
    return RA_OK;
  }
  if (!workspace || workspace_bytes < blockwise_ffn_bwd_workspace_size(chunk, d_ff, dtype)) return RA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return RA_ERR_ALIGN;
  return launch_ffn_bwd_tc(x, w1, w2, w3, dy, dx, dw1, dw2, dw3, T, d_model, d_ff, chunk, workspace, st);
}

int ringattn_accumulate(float* acc, const void* x, int64_t n, int dtype, void* stream) {
  RA_NVTX_RANGE();
  if (n < 0) return RA_ERR_ARG;
  if (dtype != RA_BF16 && dtype != RA_F32) return RA_ERR_DTYPE;
  if (n == 0) return RA_OK;
  if (!acc || !x) return RA_ERR_ARG;
  if (!aligned16(acc) || !aligned16(x)) return RA_ERR_ALIGN;
  return launch_accumulate(acc, x, n, dtype, static_cast<cudaStream_t>(stream));
}

int ringattn_cast(const float* x, void* out, int64_t n, int dtype, void* stream) {
  RA_NVTX_RANGE();
  if (n < 0) return RA_ERR_ARG;
  if (dtype != RA_BF16 && dtype != RA_F32) return RA_ERR_DTYPE;
  if (n == 0) return RA_OK;
  if (!x || !out) return RA_ERR_ARG;
  if (!aligned16(x) || !aligned16(out)) return RA_ERR_ALIGN;
  return launch_cast(x, out, n, dtype, static_cast<cudaStream_t>(stream));
}

int ringattn_get_error(void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return RA_ERR_CUDA;
  if (cudaGetLastError() != cudaSuccess) return RA_ERR_CUDA;
  int word = 0;
  if (cudaMemcpyFromSymbol(&word, ra::g_status_word, sizeof(int)) != cudaSuccess) return RA_ERR_CUDA;
  if (word != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(ra::g_status_word, &zero, sizeof(int)) != cudaSuccess) return RA_ERR_CUDA;
  }
  return word;
}

int ringattn_selftest_timeout(int timeout_us, void* stream) {
  RA_NVTX_RANGE();
  if (timeout_us <= 0 || timeout_us > 10000000) return RA_ERR_ARG;
  return launch_selftest_timeout(timeout_us, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
