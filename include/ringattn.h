/*
 * ringattn.h -- C ABI of the B200 (sm_100a) library for exact blockwise ring
 * attention and the blockwise feed-forward.
 *
 * What it computes (sources by page title and section):
 *
 *  - "Ring Attention with Blockwise Transformers for Near-Infinite Context",
 *    abstract: self-attention and the feed-forward computed blockwise, with
 *    no approximation, for training and inference.
 *  - chapterpal keyword page "Ring Attention", definition: the sequence is
 *    cut into blocks placed on a logical ring; each block keeps its queries
 *    while key/value blocks circulate around the ring.
 *  - sourcepulse project summary of the RingAttention package, "Highlighted
 *    Details": the query_chunk_size and key_chunk_size knobs.
 *  - darcstar.tech note on the paper, "DarcStar commentary", paragraphs one
 *    and two: online softmax is associative, so partial attention of separate
 *    shards combines exactly; the causal mask and the softmax denominator
 *    must be combined across chunks exactly; no all-gather of K/V.
 *
 * On one GPU the ring is virtual: the S shards are slices of the [B,H,N,D]
 * tensors in HBM and query shard i visits KV shard j = (i - t) mod S at ring
 * step t = 0..S-1.  Under the causal mask pairs j > i are skipped and the
 * diagonal pair j == i is masked inside its tiles.
 *
 * Conventions common to every call
 *  - All tensor pointers are DEVICE pointers owned by the caller; the library
 *    never frees or retains them.  The library allocates nothing per call.
 *    Its persistent device state, on every device that loads it, is one
 *    status word and the RINGATTN_NOALLOC_SCRATCH_BYTES array of
 *    ringattn_bwd_noalloc (held whether or not that call is used).
 *  - Attention tensors are contiguous [B, H, N, D] (D innermost).  LSE and
 *    the backward's D-vector are contiguous fp32 [B, H, N].  Pointers must be
 *    16-byte aligned.
 *  - `stream` is a cudaStream_t (NULL = legacy default stream).  Every call
 *    only enqueues work and returns; argument and launch errors come back
 *    synchronously as a negative ra_status, device-side failures (a bounded
 *    wait that ran out) are latched in the device status word and read back
 *    by ringattn_get_error().
 *  - Returns RA_OK (0) on success.  A request with an empty extent
 *    (B, H, N or T equal to 0) is valid and returns RA_OK without launching
 *    anything; negative sizes are RA_ERR_ARG.
 */
#ifndef RINGATTN_H_
#define RINGATTN_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define RA_API __attribute__((visibility("default")))
#else
#define RA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { RA_BF16 = 0, RA_F32 = 1 } ra_dtype;

typedef enum {
  RA_OK = 0,
  RA_ERR_ARG = -1,         /* null pointer or non-positive size             */
  RA_ERR_SHAPE = -2,       /* N % S, shard % chunk or chunk % tile != 0     */
  RA_ERR_DTYPE = -3,       /* dtype not RA_BF16 / RA_F32                    */
  RA_ERR_ALIGN = -4,       /* a pointer is not 16-byte aligned             */
  RA_ERR_UNSUPPORTED = -5, /* valid request this build does not implement   */
  RA_ERR_CUDA = -6,        /* a CUDA runtime call failed                    */
  RA_ERR_TIMEOUT = -7,     /* a kernel's bounded wait ran out (device word) */
  RA_ERR_WORKSPACE = -8,   /* workspace missing or smaller than required    */
  RA_ERR_BOUNDS = -9       /* a bounds-checked build (RA_CHECKED) caught an
                              index outside its tensor (device word)        */
} ra_status;

/* Library ABI version (major*100 + minor). */
RA_API int ringattn_version(void);

/* Human-readable text for an ra_status value (static storage). */
RA_API const char* ringattn_status_string(int status);

/*
 * ringattn_kernel_plan -- names of the kernels a call would launch on the
 * current device for a problem of N tokens in S shards with head dimension
 * D and `dtype` (static strings, several names joined by '+'):
 *   op 0: ringattn_fwd / ringattn_fwd_gqa, e.g. "fwd_tc2_kernel" (two
 *         128-row query tiles per CTA, used when the shard length is a
 *         multiple of 256 and this build's register split is usable on the
 *         device), "fwd_tc_kernel" or "fwd_simt_kernel" (RA_F32);
 *   op 1: ringattn_bwd / ringattn_bwd_gqa, e.g.
 *         "bwd_preprocess_kernel+bwd_fused_kernel+bwd_dq_convert_kernel".
 * NULL for an unknown op, a shape that breaks N % S, or an unsupported D or
 * dtype.  Lets a caller (or a benchmark) name what actually runs; the choice
 * is made once per device and does not change between calls.
 */
RA_API const char* ringattn_kernel_plan(int op, int64_t N, int64_t D, int dtype, int S);

/*
 * ringattn_fwd -- exact ring blockwise attention forward.
 *
 * For every (b, h) and query token i:
 *   s_ij = scale * q_i . k_j ;  visible(i, j) = !causal || j <= i
 *   lse_i = ln sum_{visible j} exp(s_ij)
 *   out_i = sum_{visible j} exp(s_ij - lse_i) v_j
 * computed shard by shard in ring order with an exact log-sum-exp merge of
 * the partial (max, denominator, unnormalised output) states.
 *
 *   q, k, v  [B,H,N,D] inputs of `dtype`                         (read)
 *   out      [B,H,N,D] output of `dtype` (bf16 rounded to nearest even)
 *   lse      [B,H,N] fp32 natural-log softmax denominator        (written)
 *   S        number of ring shards, N % S == 0, shard L = N / S
 *   q_chunk, k_chunk  query / key chunk sizes; both divide L.  RA_BF16 runs
 *            on the tensor cores in 128x128 tiles: chunks must be multiples
 *            of 128.  RA_F32 runs in exact fp32 on CUDA cores in 64-row
 *            tiles: chunks must be multiples of 64.
 *   causal   0 or 1 (mask j > i on global token indices)
 *   scale    softmax scale; <= 0 selects 1/sqrt(D)
 *   D        64 or 128
 * Errors: RA_ERR_ARG, RA_ERR_SHAPE, RA_ERR_DTYPE, RA_ERR_ALIGN, RA_ERR_CUDA.
 */
RA_API int ringattn_fwd(const void* q, const void* k, const void* v, void* out, float* lse,
                 int64_t B, int64_t H, int64_t N, int64_t D, int dtype,
                 int S, int q_chunk, int k_chunk, int causal, float scale,
                 void* stream);

/*
 * ringattn_fwd_gqa -- ringattn_fwd with grouped key/value heads (GQA; MQA
 * when Hkv == 1): query head h attends with key/value head h / (H / Hkv).
 * q, out [B,H,N,D]; k, v [B,Hkv,N,D]; lse [B,H,N].  H % Hkv == 0.  Fewer
 * key/value heads mean fewer bytes per ring step.  Other arguments and
 * errors as ringattn_fwd; ringattn_fwd is this call with Hkv = H.
 */
RA_API int ringattn_fwd_gqa(const void* q, const void* k, const void* v, void* out, float* lse,
                            int64_t B, int64_t H, int64_t Hkv, int64_t N, int64_t D, int dtype,
                            int S, int q_chunk, int k_chunk, int causal, float scale,
                            void* stream);

/*
 * ringattn_fwd_step -- one ring step t with a fused merge into running
 * fp32 accumulators (the per-step building block of a multi-device ring).
 *
 * Query shard i attends to KV shard j = (i - t) mod S only, and the partial
 * result is merged exactly into (o_acc, lse_acc):
 *   lse' = ln(e^lse_acc + e^lse_t),
 *   o'   = e^(lse_acc - lse') o_acc + e^(lse_t - lse') o_t
 * where (o_t, lse_t) is the normalised attention of the pair.  Pairs that
 * the causal mask skips (j > i) leave the accumulators unchanged.
 * Start from o_acc = 0 and lse_acc = -inf (the neutral element) and run
 * t = 0..S-1 in any order: the result equals ringattn_fwd's (in fp32).
 *
 *   o_acc    [B,H,N,D] fp32, read and written
 *   lse_acc  [B,H,N]   fp32, read and written
 * Other arguments as for ringattn_fwd; 0 <= t < S.
 */
RA_API int ringattn_fwd_step(const void* q, const void* k, const void* v,
                      float* o_acc, float* lse_acc,
                      int64_t B, int64_t H, int64_t N, int64_t D, int dtype,
                      int S, int q_chunk, int k_chunk, int causal, float scale,
                      int t, void* stream);

/*
 * ringattn_merge -- standalone exact log-sum-exp merge of two partials,
 * (o_a, lse_a) <- (o_a, lse_a) (+) (o_b, lse_b), all fp32:
 *   lse = ln(e^lse_a + e^lse_b);  o_a = e^(lse_a-lse) o_a + e^(lse_b-lse) o_b
 * (-inf, any) is the neutral element; two -inf rows give (0, -inf).
 *   o_a, o_b  [rows, D] fp32;  lse_a, lse_b  [rows] fp32;  D % 4 == 0.
 * Darcstar note, DarcStar commentary, paragraph one (associative combine).
 */
RA_API int ringattn_merge(float* o_a, float* lse_a, const float* o_b, const float* lse_b,
                   int64_t rows, int64_t D, void* stream);

/* Bytes of device workspace ringattn_bwd needs: two fp32 row vectors
 * [B,H,N] (D_i = dO_i . O_i and lse_i * log2(e)), each region 256-byte
 * aligned, followed by the fused pass's fp32 dQ accumulator [B,H,N,D].
 * Enough for every phase mask of ringattn_bwd_phase.  0 for empty
 * problems. */
RA_API size_t ringattn_bwd_workspace_size(int64_t B, int64_t H, int64_t N, int64_t D);

/*
 * ringattn_bwd -- gradient of sum(dout * out) for ringattn_fwd.
 *
 * With P_ij = exp(s_ij - lse_i) on visible pairs and D_i = dout_i . out_i:
 *   dv_j = sum_i P_ij dout_i
 *   dS_ij = P_ij (dout_i . v_j - D_i)
 *   dq_i = scale sum_j dS_ij k_j ;  dk_j = scale sum_i dS_ij q_i
 * Each key/value tile stays on chip while the query shards pass by in ring
 * order i = (j + t) mod S (causal: pairs in the future skipped, the
 * diagonal pair masked).  dK and dV accumulate on chip and are written once.
 * The same pass forms dQ's share of each tile pair and adds it into an
 * fp32 accumulator in the workspace; the sum over key tiles runs in the
 * order the CTAs reach memory, so dq is reproducible up to that fp32
 * summation order (dk, dv are bit-reproducible).  ringattn_bwd_phase with
 * mask 7 runs the deterministic split backward instead (a second,
 * query-stationary pass recomputes S and dP per tile pair and writes dq
 * once; every output bit-reproducible).
 *
 *   q,k,v,out,dout [B,H,N,D] of `dtype` (out and lse from ringattn_fwd)
 *   lse            [B,H,N] fp32
 *   dq,dk,dv       [B,H,N,D] of `dtype`, written
 *   workspace      device buffer of ringattn_bwd_workspace_size() bytes,
 *                  16-byte aligned; its contents on entry do not matter
 * Only RA_BF16 is implemented (RA_F32 returns RA_ERR_UNSUPPORTED).
 * Chunk rules as for ringattn_fwd with RA_BF16.  If a device cannot place
 * the fused pass's shared-memory tile set, the pass latches
 * RA_ERR_UNSUPPORTED in the status word (ringattn_get_error) and writes
 * nothing.
 */
RA_API int ringattn_bwd(const void* q, const void* k, const void* v, const void* out,
                 const float* lse, const void* dout,
                 void* dq, void* dk, void* dv,
                 int64_t B, int64_t H, int64_t N, int64_t D, int dtype,
                 int S, int q_chunk, int k_chunk, int causal, float scale,
                 void* workspace, size_t workspace_bytes, void* stream);

/*
 * ringattn_bwd_gqa -- ringattn_bwd with grouped key/value heads: k, v, dk,
 * dv are [B,Hkv,N,D]; dk and dv of a key/value head sum the contributions of
 * all H / Hkv query heads that share it (accumulated on chip, one write).
 * Other arguments as ringattn_bwd (same workspace size, computed with H).
 */
RA_API int ringattn_bwd_gqa(const void* q, const void* k, const void* v, const void* out,
                            const float* lse, const void* dout,
                            void* dq, void* dk, void* dv,
                            int64_t B, int64_t H, int64_t Hkv, int64_t N, int64_t D, int dtype,
                            int S, int q_chunk, int k_chunk, int causal, float scale,
                            void* workspace, size_t workspace_bytes, void* stream);

/*
 * ringattn_bwd_phase -- the backward's launches, selected by phase_mask
 * (1..31), for callers that schedule or time them separately:
 *   bit 0 (1)   preprocess: D_i and lse_i*log2(e) into the workspace; when
 *               the workspace is ringattn_bwd_workspace_size() bytes it
 *               also zeroes the fp32 dQ accumulator
 *   bit 1 (2)   key/value-stationary pass writing dk, dv     } the split,
 *   bit 2 (4)   query-stationary pass writing dq             } deterministic
 *                                                              backward
 *   bit 3 (8)   fused pass: dk, dv written, scale * dQ added into the
 *               accumulator
 *   bit 4 (16)  dq = bf16(accumulator)
 * Later bits read what bit 0 wrote into the same workspace; bit 4 reads what
 * bit 3 added.  Mask 7 is the deterministic backward, which needs only the
 * two row vectors (2 x round_up(B*H*N*4, 256) bytes); masks with bit 3 or 4
 * need the full ringattn_bwd_workspace_size().  ringattn_bwd runs mask 25
 * (1 + 8 + 16).  Arguments and errors as ringattn_bwd, plus RA_ERR_ARG for
 * a mask outside 1..31.
 */
RA_API int ringattn_bwd_phase(const void* q, const void* k, const void* v, const void* out,
                              const float* lse, const void* dout,
                              void* dq, void* dk, void* dv,
                              int64_t B, int64_t H, int64_t N, int64_t D, int dtype,
                              int S, int q_chunk, int k_chunk, int causal, float scale,
                              void* workspace, size_t workspace_bytes, int phase_mask,
                              void* stream);

/*
 * ringattn_bwd_prepare, ringattn_bwd_pair -- the backward one shard pair at
 * a time, for a ring spread over devices (chapterpal "Ring Attention",
 * definition: key/value blocks circulate while each device keeps its query
 * block; darcstar note, DarcStar commentary, paragraph one: per-block
 * results combine exactly).  A device holding query block i (N tokens of
 * [B,H,N,D] q, out, dout and [B,H,N] lse, all from the whole-sequence
 * forward) prepares once:
 *   prep <- D_n = dout_n . out_n and lse_n * log2(e), two fp32 row vectors
 *   [B,H,N], each region 256-byte aligned (ringattn_bwd_prepare_size bytes)
 * and then, for each key/value block j it holds in turn (same N):
 *   dq_acc += dq share of the pair   (fp32 [B,H,N,D], added into)
 *   dk_acc, dv_acc (fp32 [B,H,N,D])  = the pair's dk, dv share, or += with
 *                                      kv_accumulate = 1
 * with P, dS from the prepared lse and D (the global softmax statistics):
 * summed over all pairs these are ringattn_bwd's gradients.  diag = 1 is
 * the diagonal pair of a causal ring (mask j > i inside it); 0 is an
 * unmasked pair (the caller skips pairs that lie wholly in the future).
 * Chunk rules as ringattn_fwd with S = 1; only RA_BF16.  dq_acc additions
 * run in arrival order (fp32 summation order, as ringattn_bwd).
 * Errors: RA_ERR_ARG, RA_ERR_SHAPE, RA_ERR_ALIGN, RA_ERR_UNSUPPORTED,
 * RA_ERR_WORKSPACE (prep missing or too small), RA_ERR_CUDA.
 */
RA_API size_t ringattn_bwd_prepare_size(int64_t B, int64_t H, int64_t N);
RA_API int ringattn_bwd_prepare(const void* out, const float* lse, const void* dout, void* prep,
                                size_t prep_bytes, int64_t B, int64_t H, int64_t N, int64_t D, int dtype,
                                void* stream);
RA_API int ringattn_bwd_pair(const void* q, const void* k, const void* v, const void* dout, const void* prep,
                             float* dq_acc, float* dk_acc, float* dv_acc,
                             int64_t B, int64_t H, int64_t N, int64_t D, int dtype,
                             int q_chunk, int k_chunk, int diag, float scale, int kv_accumulate,
                             void* stream);

/*
 * ringattn_bwd_noalloc -- the backward without a workspace and without any
 * allocation.  The paper has no counterpart; it serves callers that cannot
 * allocate device memory when they run the backward (an allocator owned by
 * another framework, a device-memory budget fixed at start-up, or a hot
 * path where a cudaMalloc that may synchronise the device is not allowed).
 *
 * It runs the deterministic split backward (ringattn_bwd_phase, mask 7) and
 * gives its bits.  That backward's scratch -- two fp32 row vectors [B,H,N]
 * -- comes from one static device array of RINGATTN_NOALLOC_SCRATCH_BYTES
 * (64 MiB) that every GPU which loads this library keeps until the process
 * exits.  Arguments are checked first, exactly as by ringattn_bwd, with the
 * same errors; then a problem whose two row vectors exceed the array
 * returns RA_ERR_WORKSPACE (B*H*N up to about 8.3 million rows, e.g. H=32,
 * N=262144).
 * The first call on a device looks up the array's device address; make that
 * first call before any stream capture.  All calls share the one array and
 * it keeps the last call's contents (each call overwrites both vectors in
 * full before reading them), so calls that overlap on the GPU -- on
 * different streams, or from different host threads -- race and corrupt
 * each other's gradients: serialise them.
 */
#define RINGATTN_NOALLOC_SCRATCH_BYTES ((size_t)64 << 20)
RA_API int ringattn_bwd_noalloc(const void* q, const void* k, const void* v, const void* out,
                                const float* lse, const void* dout,
                                void* dq, void* dk, void* dv,
                                int64_t B, int64_t H, int64_t N, int64_t D, int dtype,
                                int S, int q_chunk, int k_chunk, int causal, float scale,
                                void* stream);

/*
 * ringattn_step_host -- one training step (ringattn_fwd, then ringattn_bwd)
 * on data in HOST memory, with every copy inside the call.  For callers whose
 * sequences and gradients live on the host (a data loader, an optimizer on
 * the CPU): the paper's training use (abstract) end to end.
 *
 *   h_q, h_k, h_v, h_dout    host [B,H,N,D] bf16 inputs (page-locked memory
 *                            lets the copies overlap compute)
 *   h_out, h_dq, h_dk, h_dv  host [B,H,N,D] bf16 results; h_lse host [B,H,N]
 *   dev                      device buffer of ringattn_step_host_size()
 *                            bytes (inputs, results and the backward's
 *                            workspace), 16-byte aligned
 *   compute_stream, in_stream, out_stream  cudaStream_t: kernels, host to
 *                            device copies, device to host copies
 *   inputs_free_event        cudaEvent_t or NULL: the copies of the inputs
 *                            into `dev` start after it (the consumed_event of
 *                            the step that last used `dev`)
 *   outputs_free_event       cudaEvent_t or NULL: the forward writes results
 *                            into `dev` after it (the done_event of the step
 *                            that last used `dev`)
 *   consumed_event           cudaEvent_t or NULL: recorded on compute_stream
 *                            once the backward has run (the inputs in `dev`
 *                            are no longer read)
 *   done_event               cudaEvent_t or NULL: recorded on out_stream once
 *                            the last result is on the host
 * q, k, v are copied first and the forward starts when they are in; dout
 * follows while the forward runs; out and lse go back while the backward
 * runs; dq, dk, dv go back last.  Asynchronous like every call: read the
 * host results after done_event.  Other arguments, rules and errors as
 * ringattn_fwd and ringattn_bwd; RA_ERR_WORKSPACE if `dev` is missing or
 * too small.  The call creates and releases a few CUDA events; it
 * allocates no memory.
 */
RA_API size_t ringattn_step_host_size(int64_t B, int64_t H, int64_t N, int64_t D);
RA_API int ringattn_step_host(const void* h_q, const void* h_k, const void* h_v, const void* h_dout,
                              void* h_out, float* h_lse, void* h_dq, void* h_dk, void* h_dv,
                              void* dev, size_t dev_bytes,
                              int64_t B, int64_t H, int64_t N, int64_t D, int dtype,
                              int S, int q_chunk, int k_chunk, int causal, float scale,
                              void* compute_stream, void* in_stream, void* out_stream,
                              void* inputs_free_event, void* outputs_free_event,
                              void* consumed_event, void* done_event);

/* Bytes of device workspace ringattn_decode needs: an fp32 partial output
 * and log-sum-exp per (batch, head, split). */
RA_API size_t ringattn_decode_workspace_size(int64_t B, int64_t H, int64_t N, int64_t D, int S, int k_chunk);

/*
 * ringattn_decode -- one new query token per (batch, head) against a key/
 * value cache of N tokens held as S ring shards (inference after a ring
 * prefill; paper abstract: training and inference).
 *
 *   out_bh = sum_j exp(s_j - lse_bh) v_j,  s_j = scale q_bh . k_j over all
 *   N cached keys (the new token sees the whole cache), with key/value head
 *   h / (H / Hkv) for query head h.
 * Each shard of ceil(N/S) keys is cut into pieces of k_chunk keys; every
 * piece yields an exact normalised partial and the partials are combined
 * with the exact log-sum-exp merge (darcstar note, DarcStar commentary,
 * paragraph one), so the result does not depend on S or k_chunk beyond
 * fp32 rounding.
 *
 *   q, out   [B,H,D] bf16        k, v  [B,Hkv,N,D] bf16 (contiguous)
 *   lse      [B,H] fp32 natural log
 *   k_chunk  multiple of 128;  H / Hkv in {1,2,4,8,16};  D 64 or 128
 *   workspace ringattn_decode_workspace_size() bytes, 16-byte aligned
 * Errors: RA_ERR_ARG, RA_ERR_SHAPE, RA_ERR_DTYPE, RA_ERR_ALIGN,
 * RA_ERR_UNSUPPORTED (fp32 or another group size), RA_ERR_WORKSPACE.
 */
RA_API int ringattn_decode(const void* q, const void* k, const void* v, void* out, float* lse,
                           int64_t B, int64_t H, int64_t Hkv, int64_t N, int64_t D, int dtype,
                           int S, int k_chunk, float scale,
                           void* workspace, size_t workspace_bytes, void* stream);

/* Bytes of device workspace blockwise_ffn needs for one chunk's hidden
 * activation h [chunk, d_ff] in `dtype`. */
RA_API size_t blockwise_ffn_workspace_size(int64_t chunk, int64_t d_ff, int dtype);

/*
 * blockwise_ffn -- SwiGLU feed-forward applied `chunk` tokens at a time.
 *
 *   y = (silu(x w1^T) * (x w3^T)) w2^T,   silu(z) = z / (1 + e^-z)
 * paper abstract: the feed-forward is computed blockwise, so only one
 * chunk's hidden activation [chunk, d_ff] exists at a time (in workspace).
 *
 *   x   [T, d_model]     w1, w3 [d_ff, d_model]     w2 [d_model, d_ff]
 *   y   [T, d_model] written.  Row-major, weights in [out, in] layout.
 *   T % chunk == 0; chunk, d_model multiples of 128; d_ff multiple of 128.
 *   workspace: blockwise_ffn_workspace_size(chunk, d_ff, dtype) bytes.
 * Only RA_BF16 is implemented (fp32 accumulation, h rounded to bf16).
 */
RA_API int blockwise_ffn(const void* x, const void* w1, const void* w2, const void* w3, void* y,
                  int64_t T, int64_t d_model, int64_t d_ff, int64_t chunk, int dtype,
                  void* workspace, size_t workspace_bytes, void* stream);

/* Bytes of device workspace blockwise_ffn_bwd needs: one chunk's dh
 * [chunk, d_ff] fp32 and dg, du, h [chunk, d_ff] bf16. */
RA_API size_t blockwise_ffn_bwd_workspace_size(int64_t chunk, int64_t d_ff, int dtype);

/*
 * blockwise_ffn_bwd -- gradient of sum(dy * y) for blockwise_ffn, chunk by
 * chunk (paper abstract: blockwise feed-forward, used for training).  With
 * g = x w1^T, u = x w3^T, s = 1/(1+e^-g), h = g s u:
 *   dh = dy w2;  du = dh * g s;  dg = dh * u * s (1 + g (1 - s))
 *   dx = dg w1 + du w3;  dw1 = sum dg^T x;  dw3 = sum du^T x;
 *   dw2 = sum dy^T h   (sums over all T tokens)
 * Each chunk recomputes its g and u; only one chunk's dg, du, h exist at a
 * time (in workspace).
 *
 *   x, dy [T, d_model] bf16;  w1, w3 [d_ff, d_model];  w2 [d_model, d_ff]
 *   dx  [T, d_model] bf16 written
 *   dw1, dw3 [d_ff, d_model] fp32 and dw2 [d_model, d_ff] fp32, written
 *   (summed over the chunks in fp32)
 *   T % chunk == 0; chunk, d_model, d_ff multiples of 128.  T == 0 zeroes
 *   the weight gradients (x, dy, dx may then be null).
 * Only RA_BF16 is implemented.  Errors: RA_ERR_ARG (null pointer, negative
 * size), RA_ERR_SHAPE, RA_ERR_ALIGN (any pointer not 16-byte aligned),
 * RA_ERR_WORKSPACE, RA_ERR_UNSUPPORTED (RA_F32), RA_ERR_CUDA.
 */
RA_API int blockwise_ffn_bwd(const void* x, const void* w1, const void* w2, const void* w3, const void* dy,
                             void* dx, float* dw1, float* dw2, float* dw3,
                             int64_t T, int64_t d_model, int64_t d_ff, int64_t chunk, int dtype,
                             void* workspace, size_t workspace_bytes, void* stream);

/*
 * ringattn_accumulate -- acc[i] += x[i] for i < n; acc fp32, x of `dtype`.
 * ringattn_cast       -- out[i] = x[i] rounded to `dtype` (RNE); x fp32.
 * The multi-device ring (chapterpal "Ring Attention", definition: key/value
 * blocks circulate between devices) uses them to sum per-pair gradients in
 * fp32 -- the key/value gradients travel with their blocks -- and to round
 * the fp32 accumulators at the end.  Pointers 16-byte aligned; n may be 0.
 */
RA_API int ringattn_accumulate(float* acc, const void* x, int64_t n, int dtype, void* stream);
RA_API int ringattn_cast(const float* x, void* out, int64_t n, int dtype, void* stream);

/* ---------------------------------------------------------------------------
 * One blockwise transformer layer (paper abstract: self-attention and the
 * feed-forward both computed blockwise, for training).  Pre-norm decoder
 * layer, no biases, no rotary embedding:
 *   xn  = x * rstd(x) * g_attn,          rstd(z) = (mean(z^2) + eps)^-1/2
 *   q, k, v = xn wq^T, xn wk^T, xn wv^T  (heads split: [B, H, N, D])
 *   o   = ring attention(q, k, v)        (scale 1/sqrt(D), S shards, chunks)
 *   x2  = x + o wo^T
 *   xn2 = x2 * rstd(x2) * g_ffn
 *   y   = x2 + (silu(xn2 w1^T) * (xn2 w3^T)) w2^T   (in ffn_chunk-token chunks)
 *
 *   x, y, dy, dx   [B*N, H*D] bf16 (token t = b*N + n)
 *   g_attn, g_ffn  [H*D] bf16;  wq, wk, wv, wo [H*D, H*D] bf16 ([out, in])
 *   w1, w3 [d_ff, H*D], w2 [H*D, d_ff] bf16
 *   saved: blockwise_layer_saved_size bytes, written by the forward (xn, q,
 *     k, v, o, x2, xn2, lse, both rstd) and read by the backward
 *   gradients: dx bf16; dg_attn, dg_ffn [H*D] fp32; dwq, dwk, dwv, dwo,
 *     dw1, dw2, dw3 fp32 in the weights' shapes (written, not accumulated)
 * B == 0 is valid: the forward does nothing and the backward zeroes the
 * nine parameter gradients (token pointers may then be null).
 * Rules: D in {64, 128}; H*D in {256, 512, 1024, 2048, 4096}; N % 128 == 0;
 * the attention's shard and chunk rules (N % S, shard % chunk, chunks
 * multiples of 128); (B*N) % ffn_chunk == 0, ffn_chunk and d_ff multiples
 * of 128; every pointer 16-byte aligned.  Errors: RA_ERR_ARG, RA_ERR_SHAPE,
 * RA_ERR_UNSUPPORTED, RA_ERR_ALIGN, RA_ERR_WORKSPACE, RA_ERR_CUDA.
 * marks: optional array of cudaEvent_t (null, or null entries, to skip);
 * entry i is recorded on `stream` after step i -- forward: 0 norm, 1 q/k/v
 * projections, 2 attention, 3 output projection, 4 norm, 5 feed-forward;
 * backward: 0 feed-forward, 1 norm, 2 dO, 3 dWo, 4 attention preprocess,
 * 5 dK/dV pass, 6 dQ pass, 7 dxn, 8 dWq/dWk/dWv, 9 norm.
 * ------------------------------------------------------------------------- */
RA_API size_t blockwise_layer_saved_size(int64_t B, int64_t N, int64_t H, int64_t D);
RA_API size_t blockwise_layer_fwd_workspace_size(int64_t ffn_chunk, int64_t d_ff);
RA_API size_t blockwise_layer_bwd_workspace_size(int64_t B, int64_t N, int64_t H, int64_t D, int64_t d_ff,
                                                 int64_t ffn_chunk);
RA_API int blockwise_layer_fwd(const void* x, const void* g_attn, const void* wq, const void* wk, const void* wv,
                               const void* wo, const void* g_ffn, const void* w1, const void* w2, const void* w3,
                               void* y, void* saved, size_t saved_bytes, int64_t B, int64_t N, int64_t H,
                               int64_t D, int64_t d_ff, int S, int q_chunk, int k_chunk, int causal, int ffn_chunk,
                               float eps, void* workspace, size_t workspace_bytes, void* const* marks,
                               void* stream);
RA_API int blockwise_layer_bwd(const void* x, const void* g_attn, const void* wq, const void* wk, const void* wv,
                               const void* wo, const void* g_ffn, const void* w1, const void* w2, const void* w3,
                               const void* saved, size_t saved_bytes, const void* dy, void* dx, float* dg_attn,
                               float* dwq, float* dwk, float* dwv, float* dwo, float* dg_ffn, float* dw1,
                               float* dw2, float* dw3, int64_t B, int64_t N, int64_t H, int64_t D, int64_t d_ff,
                               int S, int q_chunk, int k_chunk, int causal, int ffn_chunk, void* workspace,
                               size_t workspace_bytes, void* const* marks, void* stream);

/*
 * ringattn_get_error -- synchronise `stream`, return the device status word
 * of the current device (RA_OK, RA_ERR_TIMEOUT, RA_ERR_UNSUPPORTED from a
 * kernel that could not place its shared-memory tiles, or, in a library
 * built with RA_CHECKED, RA_ERR_BOUNDS from an index check that failed: the
 * access was skipped and the kernel wound down) and clear it.
 * Also reports a pending CUDA error as RA_ERR_CUDA.
 */
RA_API int ringattn_get_error(void* stream);

/*
 * ringattn_selftest_timeout -- launch one tiny kernel whose bounded wait on
 * an mbarrier that nothing arrives at runs out after `timeout_us`
 * microseconds; the kernel then latches RA_ERR_TIMEOUT in the device status
 * word and returns normally.  Lets a test exercise the timeout path without
 * hanging or faulting the GPU.  Read the result with ringattn_get_error().
 */
RA_API int ringattn_selftest_timeout(int timeout_us, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* RINGATTN_H_ */
