// ringattn_step_host: one training step of ring attention on data that lives
// in host memory -- the inputs copied to the device, the forward and the
// backward run, the results copied back -- enqueued on the caller's streams.
// The forward's output and log-sum-exp go back while the backward runs; dO
// comes in while the forward runs.  With two device buffer sets used in
// turn and the caller's events ordering their reuse, one step's copies
// overlap the neighbouring steps' compute: a set's inputs may be refilled
// as soon as the backward that read them has run, its results overwritten
// once they have been copied out.
#include "common.cuh"
#include "internal.h"

namespace {

size_t up256(size_t x) { return (x + 255) & ~(size_t)255; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Device buffer set: q, k, v, dout, out, dq, dk, dv [B,H,N,D] bf16, lse
// [B,H,N] fp32, then the backward's workspace; every region 256-byte aligned.
struct StepBuffers {
  uint8_t* t[8];
  float* lse;
  void* ws;
  size_t ws_bytes;
};

size_t step_bytes(int64_t B, int64_t H, int64_t N, int64_t D, StepBuffers* out, void* base) {
  const size_t act = up256((size_t)B * H * N * D * 2);
  const size_t lse = up256((size_t)B * H * N * 4);
  const size_t ws = ringattn_bwd_workspace_size(B, H, N, D);
  if (out) {
    uint8_t* p = static_cast<uint8_t*>(base);
    for (int i = 0; i < 8; ++i) out->t[i] = p + i * act;
    out->lse = reinterpret_cast<float*>(p + 8 * act);
    out->ws = p + 8 * act + lse;
    out->ws_bytes = ws;
  }
  return 8 * act + lse + ws;
}

}  // namespace

extern "C" {

size_t ringattn_step_host_size(int64_t B, int64_t H, int64_t N, int64_t D) {
  if (B <= 0 || H <= 0 || N <= 0 || D <= 0) return 0;
  return step_bytes(B, H, N, D, nullptr, nullptr);
}

int ringattn_step_host(const void* h_q, const void* h_k, const void* h_v, const void* h_dout, void* h_out,
                       float* h_lse, void* h_dq, void* h_dk, void* h_dv, void* dev, size_t dev_bytes, int64_t B,
                       int64_t H, int64_t N, int64_t D, int dtype, int S, int q_chunk, int k_chunk, int causal,
                       float scale, void* compute_stream, void* in_stream, void* out_stream,
                       void* inputs_free_event, void* outputs_free_event, void* consumed_event, void* done_event) {
  RA_NVTX_RANGE();
  if (B < 0 || H < 0 || N < 0) return RA_ERR_ARG;
  if (dtype != RA_BF16 && dtype != RA_F32) return RA_ERR_DTYPE;
  if (dtype != RA_BF16) return RA_ERR_UNSUPPORTED;
  if (D != 64 && D != 128) return RA_ERR_UNSUPPORTED;
  if (B == 0 || H == 0 || N == 0) return RA_OK;
  const void* host[9] = {h_q, h_k, h_v, h_dout, h_out, h_lse, h_dq, h_dk, h_dv};
  for (const void* p : host)
    if (!p) return RA_ERR_ARG;
  for (const void* p : host)
    if (!aligned16(p)) return RA_ERR_ALIGN;
  if (!dev || dev_bytes < ringattn_step_host_size(B, H, N, D)) return RA_ERR_WORKSPACE;
  if (!aligned16(dev)) return RA_ERR_ALIGN;
  StepBuffers b;
  step_bytes(B, H, N, D, &b, dev);
  cudaStream_t cs = static_cast<cudaStream_t>(compute_stream);
  cudaStream_t is = static_cast<cudaStream_t>(in_stream);
  cudaStream_t os = static_cast<cudaStream_t>(out_stream);
  const size_t act = (size_t)B * H * N * D * 2, lse = (size_t)B * H * N * 4;

  // four events order the three streams inside the step; they are released
  // as soon as their work has completed
  cudaEvent_t ev[4] = {};
  for (auto& e : ev)
    if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return RA_ERR_CUDA;
  auto release = [&](int rc) {
    for (auto& e : ev)
      if (e) cudaEventDestroy(e);
    return rc;
  };
  auto ok = [](cudaError_t e) { return e == cudaSuccess; };
  if (inputs_free_event && !ok(cudaStreamWaitEvent(is, static_cast<cudaEvent_t>(inputs_free_event), 0)))
    return release(RA_ERR_CUDA);
  if (outputs_free_event && !ok(cudaStreamWaitEvent(cs, static_cast<cudaEvent_t>(outputs_free_event), 0)))
    return release(RA_ERR_CUDA);
  // q, k, v in; then dO, which the forward does not need
  for (int i = 0; i < 3; ++i)
    if (!ok(cudaMemcpyAsync(b.t[i], host[i], act, cudaMemcpyHostToDevice, is))) return release(RA_ERR_CUDA);
  if (!ok(cudaEventRecord(ev[0], is))) return release(RA_ERR_CUDA);
  if (!ok(cudaMemcpyAsync(b.t[3], h_dout, act, cudaMemcpyHostToDevice, is))) return release(RA_ERR_CUDA);
  if (!ok(cudaEventRecord(ev[1], is))) return release(RA_ERR_CUDA);
  // forward; its out and lse go back while the backward runs
  if (!ok(cudaStreamWaitEvent(cs, ev[0], 0))) return release(RA_ERR_CUDA);
  int rc = ringattn_fwd(b.t[0], b.t[1], b.t[2], b.t[4], b.lse, B, H, N, D, dtype, S, q_chunk, k_chunk, causal,
                        scale, cs);
  if (rc != RA_OK) return release(rc);
  if (!ok(cudaEventRecord(ev[2], cs)) || !ok(cudaStreamWaitEvent(os, ev[2], 0))) return release(RA_ERR_CUDA);
  if (!ok(cudaMemcpyAsync(h_out, b.t[4], act, cudaMemcpyDeviceToHost, os)) ||
      !ok(cudaMemcpyAsync(h_lse, b.lse, lse, cudaMemcpyDeviceToHost, os)))
    return release(RA_ERR_CUDA);
  // backward, then its gradients back
  if (!ok(cudaStreamWaitEvent(cs, ev[1], 0))) return release(RA_ERR_CUDA);
  rc = ringattn_bwd(b.t[0], b.t[1], b.t[2], b.t[4], b.lse, b.t[3], b.t[5], b.t[6], b.t[7], B, H, N, D, dtype, S,
                    q_chunk, k_chunk, causal, scale, b.ws, b.ws_bytes, cs);
  if (rc != RA_OK) return release(rc);
  if (!ok(cudaEventRecord(ev[3], cs)) || !ok(cudaStreamWaitEvent(os, ev[3], 0))) return release(RA_ERR_CUDA);
  if (consumed_event && !ok(cudaEventRecord(static_cast<cudaEvent_t>(consumed_event), cs))) return release(RA_ERR_CUDA);
  void* hg[3] = {h_dq, h_dk, h_dv};
  for (int i = 0; i < 3; ++i)
    if (!ok(cudaMemcpyAsync(hg[i], b.t[5 + i], act, cudaMemcpyDeviceToHost, os))) return release(RA_ERR_CUDA);
  if (done_event && !ok(cudaEventRecord(static_cast<cudaEvent_t>(done_event), os))) return release(RA_ERR_CUDA);
  return release(RA_OK);
}

}  // extern "C"
