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
