"""fp64 CPU oracle for one blockwise transformer layer, forward and backward.

TEST INFRASTRUCTURE ONLY -- see the package docstring.

"Ring Attention with Blockwise Transformers for Near-Infinite Context"
(paper abstract): the transformer layer -- self-attention and feed-forward --
is computed blockwise, and the method trains such layers.  Blocking changes
neither value (the attention is exact, the feed-forward is per token), so
the oracle is the plain layer.  The pages fix no layer details; the layer
here is the pre-norm decoder layer of the 7B shape the workloads name:

    xn  = rmsnorm(x) * g_attn,        rmsnorm(z) = z / sqrt(mean(z^2) + eps)
    q, k, v = xn wq^T, xn wk^T, xn wv^T   (each split into H heads of D)
    o   = softmax attention(q, k, v)      (scale 1/sqrt(D), causal or not)
    x2  = x + o wo^T
    xn2 = rmsnorm(x2) * g_ffn
    y   = x2 + swiglu_ffn(xn2)

Rows are tokens t = b*N + n of [B*N, H*D] matrices; weights are [out, in].
The backward is the chain rule through those steps, written out with the
pinned attention and feed-forward gradients as library steps.
"""

from __future__ import annotations

import numpy as np

from .attention import attention_backward, attention_forward
from .ffn import swiglu_ffn, swiglu_ffn_backward

PARAM_NAMES = ("g_attn", "wq", "wk", "wv", "wo", "g_ffn", "w1", "w2", "w3")


def rmsnorm(x, g, eps):
    """(x * r * g, r) with r = 1 / sqrt(mean(x^2) + eps) per row."""
    x = np.asarray(x, dtype=np.float64)
    r = 1.0 / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    return x * r * np.asarray(g, dtype=np.float64), r[..., 0]


def rmsnorm_backward(x, g, dout, eps):
    """(dx, dg) of sum(dout * rmsnorm(x, g)).

    With r = (mean(x^2) + eps)^-1/2 and d = row length:
    dr/dx_j = -r^3 x_j / d, so dx_j = r g_j dout_j - r^3 x_j sum_i(g_i dout_i x_i) / d,
    and dg = sum over rows of dout * x * r.
    """
    x = np.asarray(x, dtype=np.float64)
    g = np.asarray(g, dtype=np.float64)
    dout = np.asarray(dout, dtype=np.float64)
    d = x.shape[-1]
    r = 1.0 / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    s = np.sum(g * dout * x, axis=-1, keepdims=True)
    dx = r * g * dout - (r ** 3) * x * s / d
    dg = np.sum(dout * x * r, axis=0)
    return dx, dg


def _heads(m, B, N, H, D):
    """[B*N, H*D] -> [B, H, N, D]."""
    return m.reshape(B, N, H, D).transpose(0, 2, 1, 3)


def _tokens(a):
    """[B, H, N, D] -> [B*N, H*D]."""
    B, H, N, D = a.shape
    return a.transpose(0, 2, 1, 3).reshape(B * N, H * D)


def layer_forward(x, params, B, N, H, D, causal=True, eps=1e-5):
    """y [B*N, H*D] and the intermediates (a dict) of the layer."""
    g_attn, wq, wk, wv, wo, g_ffn, w1, w2, w3 = (np.asarray(p, dtype=np.float64) for p in params)
    x = np.asarray(x, dtype=np.float64)
    xn, r1 = rmsnorm(x, g_attn, eps)
    q, k, v = (_heads(xn @ w.T, B, N, H, D) for w in (wq, wk, wv))
    o, lse = attention_forward(q, k, v, causal)
    x2 = x + _tokens(o) @ wo.T
    xn2, r2 = rmsnorm(x2, g_ffn, eps)
    y = x2 + swiglu_ffn(xn2, w1, w2, w3)
    return y, dict(xn=xn, q=q, k=k, v=v, o=o, lse=lse, x2=x2, xn2=xn2, rstd1=r1, rstd2=r2)


def layer_backward(x, params, dy, B, N, H, D, causal=True, eps=1e-5):
    """(dx, grads) of sum(dy * layer_forward(x, params)); grads follow
    PARAM_NAMES."""
    g_attn, wq, wk, wv, wo, g_ffn, w1, w2, w3 = (np.asarray(p, dtype=np.float64) for p in params)
    x = np.asarray(x, dtype=np.float64)
    dy = np.asarray(dy, dtype=np.float64)
    _, a = layer_forward(x, params, B, N, H, D, causal, eps)
    # y = x2 + ffn(xn2)
    dxn2, dw1, dw2, dw3 = swiglu_ffn_backward(a["xn2"], w1, w2, w3, dy)
    # xn2 = rmsnorm(x2) * g_ffn
    dx2_norm, dg_ffn = rmsnorm_backward(a["x2"], g_ffn, dxn2, eps)
    dx2 = dy + dx2_norm
    # x2 = x + o_tok wo^T
    o_tok = _tokens(a["o"])
    do_tok = dx2 @ wo
    dwo = dx2.T @ o_tok
    # o = attention(q, k, v)
    dq, dk, dv = attention_backward(a["q"], a["k"], a["v"], _heads(do_tok, B, N, H, D), causal)
    dq, dk, dv = _tokens(dq), _tokens(dk), _tokens(dv)
    # q, k, v = xn w^T
    dxn = dq @ wq + dk @ wk + dv @ wv
    dwq, dwk, dwv = dq.T @ a["xn"], dk.T @ a["xn"], dv.T @ a["xn"]
    # xn = rmsnorm(x) * g_attn, plus the residual path x -> x2
    dx_norm, dg_attn = rmsnorm_backward(x, g_attn, dxn, eps)
    dx = dx2 + dx_norm
    return dx, (dg_attn, dwq, dwk, dwv, dwo, dg_ffn, dw1, dw2, dw3)
