"""fp64 CPU oracle for the blockwise feed-forward.

TEST INFRASTRUCTURE ONLY -- see the package docstring.

"Ring Attention with Blockwise Transformers for Near-Infinite Context"
(paper abstract): the method computes self-attention *and the feed-forward*
blockwise.  The feed-forward acts on each token on its own, so cutting the
sequence into chunks cannot change its value; the chunking only bounds the
size of the intermediate activation.

The layer shape is a 7B-style SwiGLU block (hidden 4096 -> 11008 -> 4096),
with weights in the [out, in] convention:
    w1 : [d_ff, d_model]  gate projection
    w3 : [d_ff, d_model]  up projection
    w2 : [d_model, d_ff]  down projection
    y  = (silu(x w1^T) * (x w3^T)) w2^T,   silu(z) = z / (1 + e^-z)
No biases.

Training (the abstract's setting) needs the gradient of a scalar loss through
this layer.  Given dy = dLoss/dy, the backward here is the chain rule written
out step by step in float64 (no fusion, no chunk-local shortcuts).  Like the
forward it is per token except for the weight gradients, which are sums over
tokens; the blockwise version sums per-chunk contributions.
"""

from __future__ import annotations

import numpy as np


def silu(z):
    """z * sigmoid(z) = z / (1 + exp(-z)), in float64."""
    z = np.asarray(z, dtype=np.float64)
    with np.errstate(over="ignore"):
        return z / (1.0 + np.exp(-z))


def swiglu_ffn(x, w1, w2, w3):
    """Unchunked SwiGLU feed-forward of every row of x [T, d_model]."""
    x = np.asarray(x, dtype=np.float64)
    w1 = np.asarray(w1, dtype=np.float64)
    w2 = np.asarray(w2, dtype=np.float64)
    w3 = np.asarray(w3, dtype=np.float64)
    h = silu(x @ w1.T) * (x @ w3.T)
    return h @ w2.T


def blockwise_ffn(x, w1, w2, w3, chunk: int):
    """The same feed-forward applied chunk by chunk (chunk rows at a time)."""
    x = np.asarray(x, dtype=np.float64)
    T = x.shape[0]
    if T % chunk:
        raise ValueError("chunk must divide the number of tokens")
    out = np.empty((T, np.asarray(w2).shape[0]))
    for c0 in range(0, T, chunk):
        out[c0:c0 + chunk] = swiglu_ffn(x[c0:c0 + chunk], w1, w2, w3)
    return out


def sigmoid(z):
    """1 / (1 + exp(-z)), in float64."""
    z = np.asarray(z, dtype=np.float64)
    with np.errstate(over="ignore"):
        return 1.0 / (1.0 + np.exp(-z))


def swiglu_ffn_backward(x, w1, w2, w3, dy):
    """Gradients (dx, dw1, dw2, dw3) of sum(dy * swiglu_ffn(x, ...)).

    Chain rule through g = x w1^T, u = x w3^T, a = silu(g), h = a * u,
    y = h w2^T, with d silu(g)/dg = s + g s (1 - s), s = sigmoid(g).
    """
    x = np.asarray(x, dtype=np.float64)
    w1 = np.asarray(w1, dtype=np.float64)
    w2 = np.asarray(w2, dtype=np.float64)
    w3 = np.asarray(w3, dtype=np.float64)
    dy = np.asarray(dy, dtype=np.float64)
    g = x @ w1.T
    u = x @ w3.T
    s = sigmoid(g)
    a = g * s
    h = a * u
    # y = h w2^T
    dh = dy @ w2
    dw2 = dy.T @ h
    # h = a * u
    da = dh * u
    du = dh * a
    # a = silu(g)
    dg = da * (s + g * s * (1.0 - s))
    # g = x w1^T, u = x w3^T
    dx = dg @ w1 + du @ w3
    dw1 = dg.T @ x
    dw3 = du.T @ x
    return dx, dw1, dw2, dw3


def blockwise_ffn_backward(x, w1, w2, w3, dy, chunk: int):
    """The backward chunk by chunk: dx rows per chunk, weight gradients
    summed over the chunks' contributions."""
    x = np.asarray(x, dtype=np.float64)
    T = x.shape[0]
    if T % chunk:
        raise ValueError("chunk must divide the number of tokens")
    dx = np.empty_like(x)
    dw1 = np.zeros(np.asarray(w1).shape)
    dw2 = np.zeros(np.asarray(w2).shape)
    dw3 = np.zeros(np.asarray(w3).shape)
    for c0 in range(0, T, chunk):
        sl = slice(c0, c0 + chunk)
        gx, g1, g2, g3 = swiglu_ffn_backward(x[sl], w1, w2, w3, np.asarray(dy)[sl])
        dx[sl] = gx
        dw1 += g1
        dw2 += g2
        dw3 += g3
    return dx, dw1, dw2, dw3


def swiglu_ffn_backward_terms(x, w1, w2, w3, dy):
    """Per-output sums of |term| of the gradient contractions, for error
    bounds: dx <- sum_f |dg w1| + |du w3|, dw1 <- sum_t |dg x|,
    dw3 <- sum_t |du x|, dw2 <- sum_t |dy h| (same shapes as the gradients)."""
    x = np.asarray(x, dtype=np.float64)
    w1 = np.asarray(w1, dtype=np.float64)
    w2 = np.asarray(w2, dtype=np.float64)
    w3 = np.asarray(w3, dtype=np.float64)
    dy = np.asarray(dy, dtype=np.float64)
    g = x @ w1.T
    u = x @ w3.T
    s = sigmoid(g)
    a = g * s
    dh = dy @ w2
    dg = np.abs(dh * u * (s + g * s * (1.0 - s)))
    du = np.abs(dh * a)
    ax = np.abs(x)
    return (dg @ np.abs(w1) + du @ np.abs(w3), dg.T @ ax, np.abs(dy).T @ np.abs(a * u), du.T @ ax)
