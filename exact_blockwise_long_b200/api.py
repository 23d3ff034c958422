"""torch-tensor front end of the C ABI: argument marshalling only.

Each function checks that its tensors are CUDA, contiguous and of the
expected dtype, passes their device pointers and sizes to the library entry
point of the same name on the current CUDA stream, and raises
``RingAttnError`` on a non-zero status.  Nothing is computed here.
"""

from __future__ import annotations

import ctypes

import torch

from ._lib import RA_BF16, RA_F32, call, lib

_DT = {torch.bfloat16: RA_BF16, torch.float32: RA_F32}


def _stream(stream=None) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return int(s.cuda_stream)


def _dev(t: torch.Tensor, name: str) -> int:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def _bhnd(q: torch.Tensor):
    if q.dim() != 4:
        raise ValueError("attention tensors are [B, H, N, D]")
    return tuple(int(x) for x in q.shape)


def _dtype(q: torch.Tensor) -> int:
    if q.dtype not in _DT:
        raise ValueError(f"unsupported dtype {q.dtype}")
    return _DT[q.dtype]


def ringattn_fwd(q, k, v, out, lse, S, q_chunk, k_chunk, causal, scale=0.0, stream=None):
    """out, lse <- exact ring blockwise attention of (q, k, v)."""
    B, H, N, D = _bhnd(q)
    for t in (k, v, out):
        if t.shape != q.shape or t.dtype != q.dtype:
            raise ValueError("q, k, v, out must share shape and dtype")
    if lse.dtype != torch.float32 or tuple(lse.shape) != (B, H, N):
        raise ValueError("lse must be float32 [B, H, N]")
    call("ringattn_fwd", _dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(out, "out"), _dev(lse, "lse"),
         B, H, N, D, _dtype(q), int(S), int(q_chunk), int(k_chunk), int(bool(causal)), float(scale),
         _stream(stream))
    return out, lse


def ringattn_fwd_gqa(q, k, v, out, lse, S, q_chunk, k_chunk, causal, scale=0.0, stream=None):
    """ringattn_fwd with grouped key/value heads: k, v are [B, Hkv, N, D]."""
    B, H, N, D = _bhnd(q)
    Hkv = int(k.shape[1])
    if tuple(k.shape) != (B, Hkv, N, D) or k.shape != v.shape or out.shape != q.shape:
        raise ValueError("q, out are [B, H, N, D]; k, v are [B, Hkv, N, D]")
    for t in (k, v, out):
        if t.dtype != q.dtype:
            raise ValueError("q, k, v, out must share dtype")
    if lse.dtype != torch.float32 or tuple(lse.shape) != (B, H, N):
        raise ValueError("lse must be float32 [B, H, N]")
    call("ringattn_fwd_gqa", _dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(out, "out"), _dev(lse, "lse"),
         B, H, Hkv, N, D, _dtype(q), int(S), int(q_chunk), int(k_chunk), int(bool(causal)), float(scale),
         _stream(stream))
    return out, lse


def ringattn_bwd_gqa(q, k, v, out, lse, dout, dq, dk, dv, S, q_chunk, k_chunk, causal, workspace,
                     scale=0.0, stream=None):
    """ringattn_bwd with grouped key/value heads: k, v, dk, dv are [B, Hkv, N, D]."""
    B, H, N, D = _bhnd(q)
    Hkv = int(k.shape[1])
    for t in (out, dout, dq):
        if t.shape != q.shape or t.dtype != q.dtype:
            raise ValueError("q, out, dout, dq must share shape and dtype")
    for t in (v, dk, dv):
        if t.shape != k.shape or t.dtype != q.dtype:
            raise ValueError("k, v, dk, dv must share shape [B, Hkv, N, D] and dtype")
    nbytes = workspace.numel() * workspace.element_size()
    call("ringattn_bwd_gqa", _dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(out, "out"), _dev(lse, "lse"),
         _dev(dout, "dout"), _dev(dq, "dq"), _dev(dk, "dk"), _dev(dv, "dv"), B, H, Hkv, N, D, _dtype(q),
         int(S), int(q_chunk), int(k_chunk), int(bool(causal)), float(scale), _dev(workspace, "workspace"),
         nbytes, _stream(stream))
    return dq, dk, dv


def ringattn_fwd_step(q, k, v, o_acc, lse_acc, S, q_chunk, k_chunk, causal, t, scale=0.0, stream=None):
    """Merge ring step t of (q, k, v) into the fp32 accumulators (o_acc, lse_acc)."""
    B, H, N, D = _bhnd(q)
    if o_acc.dtype != torch.float32 or tuple(o_acc.shape) != (B, H, N, D):
        raise ValueError("o_acc must be float32 [B, H, N, D]")
    if lse_acc.dtype != torch.float32 or tuple(lse_acc.shape) != (B, H, N):
        raise ValueError("lse_acc must be float32 [B, H, N]")
    call("ringattn_fwd_step", _dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(o_acc, "o_acc"),
         _dev(lse_acc, "lse_acc"), B, H, N, D, _dtype(q), int(S), int(q_chunk), int(k_chunk),
         int(bool(causal)), float(scale), int(t), _stream(stream))
    return o_acc, lse_acc


def ringattn_merge(o_a, lse_a, o_b, lse_b, stream=None):
    """(o_a, lse_a) <- exact log-sum-exp merge with (o_b, lse_b); fp32, [rows, D] / [rows]."""
    D = int(o_a.shape[-1])
    rows = o_a.numel() // D
    if o_b.shape != o_a.shape or lse_a.numel() != rows or lse_b.numel() != rows:
        raise ValueError("merge operands disagree in shape")
    for x in (o_a, o_b, lse_a, lse_b):
        if x.dtype != torch.float32:
            raise ValueError("merge operands are float32")
    call("ringattn_merge", _dev(o_a, "o_a"), _dev(lse_a, "lse_a"), _dev(o_b, "o_b"), _dev(lse_b, "lse_b"),
         rows, D, _stream(stream))
    return o_a, lse_a


def ringattn_kernel_plan(op, N, D, dtype, S):
    """Names of the kernels ringattn_fwd (op 0) or ringattn_bwd (op 1) launch
    for this shape on the current device, joined by '+'; None if invalid."""
    r = lib().ringattn_kernel_plan(int(op), int(N), int(D), _DT[dtype] if not isinstance(dtype, int) else dtype,
                                   int(S))
    return r.decode() if r is not None else None


def ringattn_bwd_workspace_size(B, H, N, D) -> int:
    return int(lib().ringattn_bwd_workspace_size(int(B), int(H), int(N), int(D)))


def ringattn_bwd(q, k, v, out, lse, dout, dq, dk, dv, S, q_chunk, k_chunk, causal, workspace,
                 scale=0.0, stream=None):
    """dq, dk, dv <- gradient of sum(dout * out) through ringattn_fwd."""
    B, H, N, D = _bhnd(q)
    for t in (k, v, out, dout, dq, dk, dv):
        if t.shape != q.shape or t.dtype != q.dtype:
            raise ValueError("attention tensors must share shape and dtype")
    if lse.dtype != torch.float32 or tuple(lse.shape) != (B, H, N):
        raise ValueError("lse must be float32 [B, H, N]")
    nbytes = workspace.numel() * workspace.element_size()
    call("ringattn_bwd", _dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(out, "out"), _dev(lse, "lse"),
         _dev(dout, "dout"), _dev(dq, "dq"), _dev(dk, "dk"), _dev(dv, "dv"), B, H, N, D, _dtype(q),
         int(S), int(q_chunk), int(k_chunk), int(bool(causal)), float(scale), _dev(workspace, "workspace"),
         nbytes, _stream(stream))
    return dq, dk, dv


def ringattn_bwd_phase(q, k, v, out, lse, dout, dq, dk, dv, S, q_chunk, k_chunk, causal, workspace, phase_mask,
                       scale=0.0, stream=None):
    """Run the selected backward launches: bit 0 preprocess, bits 1-2 the split
    (deterministic) dK/dV and dQ passes, bit 3 the fused pass, bit 4 the dQ
    conversion (include/ringattn.h, ringattn_bwd_phase)."""
    B, H, N, D = _bhnd(q)
    nbytes = workspace.numel() * workspace.element_size()
    call("ringattn_bwd_phase", _dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(out, "out"), _dev(lse, "lse"),
         _dev(dout, "dout"), _dev(dq, "dq"), _dev(dk, "dk"), _dev(dv, "dv"), B, H, N, D, _dtype(q),
         int(S), int(q_chunk), int(k_chunk), int(bool(causal)), float(scale), _dev(workspace, "workspace"),
         nbytes, int(phase_mask), _stream(stream))
    return dq, dk, dv


def ringattn_bwd_prepare_size(B, H, N) -> int:
    return int(lib().ringattn_bwd_prepare_size(int(B), int(H), int(N)))


def ringattn_bwd_prepare(out, lse, dout, prep, stream=None):
    """prep <- D_n = dout_n . out_n and lse_n * log2(e) of one query block."""
    B, H, N, D = _bhnd(out)
    if dout.shape != out.shape or dout.dtype != out.dtype:
        raise ValueError("out and dout must share shape and dtype")
    if lse.dtype != torch.float32 or tuple(lse.shape) != (B, H, N):
        raise ValueError("lse must be float32 [B, H, N]")
    call("ringattn_bwd_prepare", _dev(out, "out"), _dev(lse, "lse"), _dev(dout, "dout"), _dev(prep, "prep"),
         prep.numel() * prep.element_size(), B, H, N, D, _dtype(out), _stream(stream))
    return prep


def ringattn_bwd_pair(q, k, v, dout, prep, dq_acc, dk_acc, dv_acc, q_chunk, k_chunk, diag, kv_accumulate=False,
                      scale=0.0, stream=None):
    """One shard pair's gradient: dq_acc += its dq share; dk_acc, dv_acc <- (or +=) its dk, dv share (fp32)."""
    B, H, N, D = _bhnd(q)
    for t in (k, v, dout):
        if t.shape != q.shape or t.dtype != q.dtype:
            raise ValueError("q, k, v, dout must share shape and dtype")
    for t in (dq_acc, dk_acc, dv_acc):
        if t.dtype != torch.float32 or t.shape != q.shape:
            raise ValueError("the accumulators are float32 [B, H, N, D]")
    call("ringattn_bwd_pair", _dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(dout, "dout"), _dev(prep, "prep"),
         _dev(dq_acc, "dq_acc"), _dev(dk_acc, "dk_acc"), _dev(dv_acc, "dv_acc"), B, H, N, D, _dtype(q),
         int(q_chunk), int(k_chunk), int(bool(diag)), float(scale), int(bool(kv_accumulate)), _stream(stream))
    return dq_acc, dk_acc, dv_acc


def ringattn_bwd_noalloc(q, k, v, out, lse, dout, dq, dk, dv, S, q_chunk, k_chunk, causal, scale=0.0, stream=None):
    """The deterministic backward without a workspace: the library's fixed
    static scratch is used instead, for callers that cannot allocate device
    memory.  Calls must not overlap on the GPU (they share that scratch)."""
    B, H, N, D = _bhnd(q)
    for t in (k, v, out, dout, dq, dk, dv):
        if t.shape != q.shape or t.dtype != q.dtype:
            raise ValueError("attention tensors must share shape and dtype")
    call("ringattn_bwd_noalloc", _dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(out, "out"), _dev(lse, "lse"),
         _dev(dout, "dout"), _dev(dq, "dq"), _dev(dk, "dk"), _dev(dv, "dv"), B, H, N, D, _dtype(q),
         int(S), int(q_chunk), int(k_chunk), int(bool(causal)), float(scale), _stream(stream))
    return dq, dk, dv


def ringattn_step_host_size(B, H, N, D) -> int:
    return int(lib().ringattn_step_host_size(int(B), int(H), int(N), int(D)))


def ringattn_step_host(h_q, h_k, h_v, h_dout, h_out, h_lse, h_dq, h_dk, h_dv, dev, S, q_chunk, k_chunk, causal,
                       compute_stream, in_stream, out_stream, inputs_free_event=None, outputs_free_event=None,
                       consumed_event=None, done_event=None, scale=0.0):
    """One forward + backward step on host tensors (pinned), every copy inside
    the C call: inputs in on in_stream, kernels on compute_stream, results out
    on out_stream.  inputs_free_event and outputs_free_event guard the reuse
    of `dev` (pass the consumed_event and done_event of the step that last
    used it); consumed_event is recorded once the backward has run,
    done_event once the last result is on the host."""
    B, H, N, D = _bhnd(h_q)
    for t in (h_q, h_k, h_v, h_dout, h_out, h_dq, h_dk, h_dv):
        if t.is_cuda or t.shape != h_q.shape or t.dtype != h_q.dtype or not t.is_contiguous():
            raise ValueError("host tensors [B, H, N, D] of one dtype, contiguous")
    if h_lse.is_cuda or h_lse.dtype != torch.float32 or tuple(h_lse.shape) != (B, H, N):
        raise ValueError("h_lse must be a float32 host tensor [B, H, N]")

    def ev(e):
        if e is None:
            return None
        if e.cuda_event == 0:
            e.record()
        return e.cuda_event

    call("ringattn_step_host", *[t.data_ptr() for t in (h_q, h_k, h_v, h_dout, h_out, h_lse, h_dq, h_dk, h_dv)],
         _dev(dev, "dev"), _nbytes(dev), B, H, N, D, _dtype(h_q), int(S), int(q_chunk), int(k_chunk),
         int(bool(causal)), float(scale), int(compute_stream.cuda_stream), int(in_stream.cuda_stream),
         int(out_stream.cuda_stream), ev(inputs_free_event), ev(outputs_free_event), ev(consumed_event),
         ev(done_event))


def ringattn_decode_workspace_size(B, H, N, D, S, k_chunk) -> int:
    return int(lib().ringattn_decode_workspace_size(int(B), int(H), int(N), int(D), int(S), int(k_chunk)))


def ringattn_decode(q, k, v, out, lse, S, k_chunk, workspace, scale=0.0, stream=None):
    """out, lse <- one query token per (batch, head) against the [B, Hkv, N, D] cache."""
    if q.dim() != 3 or k.dim() != 4:
        raise ValueError("q, out are [B, H, D]; k, v are [B, Hkv, N, D]")
    B, H, D = (int(x) for x in q.shape)
    Hkv, N = int(k.shape[1]), int(k.shape[2])
    if tuple(k.shape) != (B, Hkv, N, D) or v.shape != k.shape or out.shape != q.shape:
        raise ValueError("shape mismatch")
    if lse.dtype != torch.float32 or tuple(lse.shape) != (B, H):
        raise ValueError("lse must be float32 [B, H]")
    nbytes = workspace.numel() * workspace.element_size()
    call("ringattn_decode", _dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(out, "out"), _dev(lse, "lse"),
         B, H, Hkv, N, D, _dtype(q), int(S), int(k_chunk), float(scale), _dev(workspace, "workspace"), nbytes,
         _stream(stream))
    return out, lse


def blockwise_ffn_workspace_size(chunk, d_ff, dtype=torch.bfloat16) -> int:
    return int(lib().blockwise_ffn_workspace_size(int(chunk), int(d_ff), _DT[dtype]))


def blockwise_ffn(x, w1, w2, w3, y, chunk, workspace, stream=None):
    """y <- (silu(x w1^T) * (x w3^T)) w2^T, chunk tokens at a time."""
    T, d_model = (int(s) for s in x.shape)
    d_ff = int(w1.shape[0])
    if tuple(w1.shape) != (d_ff, d_model) or tuple(w3.shape) != (d_ff, d_model):
        raise ValueError("w1, w3 are [d_ff, d_model]")
    if tuple(w2.shape) != (d_model, d_ff) or tuple(y.shape) != (T, d_model):
        raise ValueError("w2 is [d_model, d_ff], y is [T, d_model]")
    nbytes = workspace.numel() * workspace.element_size()
    call("blockwise_ffn", _dev(x, "x"), _dev(w1, "w1"), _dev(w2, "w2"), _dev(w3, "w3"), _dev(y, "y"),
         T, d_model, d_ff, int(chunk), _dtype(x), _dev(workspace, "workspace"), nbytes, _stream(stream))
    return y


def blockwise_ffn_bwd_workspace_size(chunk, d_ff, dtype=torch.bfloat16) -> int:
    return int(lib().blockwise_ffn_bwd_workspace_size(int(chunk), int(d_ff), _DT[dtype]))


def blockwise_ffn_bwd(x, w1, w2, w3, dy, dx, dw1, dw2, dw3, chunk, workspace, stream=None):
    """dx (bf16), dw1, dw2, dw3 (fp32) <- gradient of sum(dy * y) through blockwise_ffn."""
    T, d_model = (int(s) for s in x.shape)
    d_ff = int(w1.shape[0])
    if dy.shape != x.shape or dx.shape != x.shape:
        raise ValueError("x, dy, dx are [T, d_model]")
    for t, shp in ((dw1, (d_ff, d_model)), (dw3, (d_ff, d_model)), (dw2, (d_model, d_ff))):
        if t.dtype != torch.float32 or tuple(t.shape) != shp:
            raise ValueError("weight gradients are float32 in the weights' shapes")
    nbytes = workspace.numel() * workspace.element_size()
    call("blockwise_ffn_bwd", _dev(x, "x"), _dev(w1, "w1"), _dev(w2, "w2"), _dev(w3, "w3"), _dev(dy, "dy"),
         _dev(dx, "dx"), _dev(dw1, "dw1"), _dev(dw2, "dw2"), _dev(dw3, "dw3"), T, d_model, d_ff, int(chunk),
         _dtype(x), _dev(workspace, "workspace"), nbytes, _stream(stream))
    return dx, dw1, dw2, dw3


def blockwise_layer_saved_size(B, N, H, D) -> int:
    return int(lib().blockwise_layer_saved_size(int(B), int(N), int(H), int(D)))


def blockwise_layer_fwd_workspace_size(ffn_chunk, d_ff) -> int:
    return int(lib().blockwise_layer_fwd_workspace_size(int(ffn_chunk), int(d_ff)))


def blockwise_layer_bwd_workspace_size(B, N, H, D, d_ff, ffn_chunk) -> int:
    return int(lib().blockwise_layer_bwd_workspace_size(int(B), int(N), int(H), int(D), int(d_ff), int(ffn_chunk)))


def _nbytes(t):
    return t.numel() * t.element_size()


def _marks(events):
    """ctypes array of raw cudaEvent_t handles (recorded once so they exist), or None."""
    if not events:
        return None
    for e in events:
        if e.cuda_event == 0:
            e.record()
    arr = (ctypes.c_void_p * len(events))(*[e.cuda_event for e in events])
    return arr


def blockwise_layer_fwd(x, weights, y, saved, B, N, H, D, S, q_chunk, k_chunk, causal, ffn_chunk, workspace,
                        eps=1e-5, stream=None, marks=None):
    """y <- the blockwise transformer layer of x ([B*N, H*D] bf16); `saved`
    receives the activations the backward reads.  `weights` is the tuple
    (g_attn, wq, wk, wv, wo, g_ffn, w1, w2, w3)."""
    g_attn, wq, wk, wv, wo, g_ffn, w1, w2, w3 = weights
    d_ff = int(w1.shape[0])
    names = ("g_attn", "wq", "wk", "wv", "wo", "g_ffn", "w1", "w2", "w3")
    call("blockwise_layer_fwd", _dev(x, "x"), *[_dev(t, n) for t, n in zip(weights, names)], _dev(y, "y"),
         _dev(saved, "saved"), _nbytes(saved), int(B), int(N), int(H), int(D), d_ff, int(S), int(q_chunk),
         int(k_chunk), int(bool(causal)), int(ffn_chunk), float(eps), _dev(workspace, "workspace"),
         _nbytes(workspace), _marks(marks), _stream(stream))
    return y


def blockwise_layer_bwd(x, weights, saved, dy, dx, grads, B, N, H, D, S, q_chunk, k_chunk, causal, ffn_chunk,
                        workspace, stream=None, marks=None):
    """dx (bf16) and the fp32 parameter gradients `grads` = (dg_attn, dwq,
    dwk, dwv, dwo, dg_ffn, dw1, dw2, dw3) of sum(dy * layer(x))."""
    names = ("g_attn", "wq", "wk", "wv", "wo", "g_ffn", "w1", "w2", "w3")
    for t, w in zip(grads, weights):
        if t.dtype != torch.float32 or tuple(t.shape) != tuple(w.shape):
            raise ValueError("parameter gradients are float32 in the parameters' shapes")
    d_ff = int(weights[6].shape[0])
    call("blockwise_layer_bwd", _dev(x, "x"), *[_dev(t, n) for t, n in zip(weights, names)],
         _dev(saved, "saved"), _nbytes(saved), _dev(dy, "dy"), _dev(dx, "dx"),
         *[_dev(t, "d" + n) for t, n in zip(grads, names)], int(B), int(N), int(H), int(D), d_ff, int(S),
         int(q_chunk), int(k_chunk), int(bool(causal)), int(ffn_chunk), _dev(workspace, "workspace"),
         _nbytes(workspace), _marks(marks), _stream(stream))
    return dx, grads


def ringattn_accumulate(acc, x, stream=None):
    """acc (fp32) += x (bf16 or fp32), element-wise over the whole tensors."""
    if acc.dtype != torch.float32 or acc.numel() != x.numel():
        raise ValueError("acc must be float32 with as many elements as x")
    call("ringattn_accumulate", _dev(acc, "acc"), _dev(x, "x"), acc.numel(), _dtype(x), _stream(stream))
    return acc


def ringattn_cast(x, out, stream=None):
    """out (bf16 or fp32) <- x (fp32), rounded to nearest even."""
    if x.dtype != torch.float32 or x.numel() != out.numel():
        raise ValueError("x must be float32 with as many elements as out")
    call("ringattn_cast", _dev(x, "x"), _dev(out, "out"), x.numel(), _dtype(out), _stream(stream))
    return out


def ringattn_get_error(stream=None) -> int:
    """Synchronise the stream; return and clear the device status word."""
    return int(lib().ringattn_get_error(_stream(stream)))


def ringattn_selftest_timeout(timeout_us: int, stream=None) -> None:
    call("ringattn_selftest_timeout", int(timeout_us), _stream(stream))
