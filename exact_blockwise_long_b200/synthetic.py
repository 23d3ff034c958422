"""Seeded synthetic inputs shared by the tests, the bench and the oracle side.

This module holds no part of the method's arithmetic: it only draws random
tensors and picks sample rows.  Both the CUDA path and the oracle receive
the very same bits (bf16 inputs are rounded once, here, and the oracle
upcasts those bf16 values exactly to float64).

Recipe (per workload): a torch.Generator on the target device seeded with
the workload seed draws float32 standard normals in the order q, k, v, dO
(then x, w1, w3, w2 and, for its backward, dy for the feed-forward), each scaled as the workload says
(k by 2 for the sharpened 32k workload, weights by 0.02), then rounded to the
compute dtype with round-to-nearest-even.
"""

from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch


@dataclass(frozen=True)
class AttnWorkload:
    name: str
    B: int
    H: int
    N: int
    D: int
    S: int
    q_chunk: int
    k_chunk: int
    causal: bool
    seed: int
    dtype: torch.dtype = torch.bfloat16
    k_scale: float = 1.0
    bwd: bool = True
    Hkv: int = 0  # key/value heads (grouped-query attention); 0 means H

    @property
    def kv_heads(self) -> int:
        return self.Hkv or self.H


@dataclass(frozen=True)
class FFNWorkload:
    name: str
    T: int
    d_model: int
    d_ff: int
    chunk: int
    seed: int
    w_std: float = 0.02
    dtype: torch.dtype = torch.bfloat16


WORKLOADS = {
    # tiny exact check, fp32, forward only
    "tiny_f32": AttnWorkload("tiny_f32", 1, 1, 512, 64, 4, 64, 64, True, 0, torch.float32, bwd=False),
    # B=2, H=16, N=8192, d=64, S=8, chunks 128, causal and non-causal
    "n8k_d64_causal": AttnWorkload("n8k_d64_causal", 2, 16, 8192, 64, 8, 128, 128, True, 1),
    "n8k_d64_full": AttnWorkload("n8k_d64_full", 2, 16, 8192, 64, 8, 128, 128, False, 1),
    # B=1, H=32, N=32768, d=128, S=16, q_chunk 512, k_chunk 1024, K scaled by 2
    "n32k_d128": AttnWorkload("n32k_d128", 1, 32, 32768, 128, 16, 512, 1024, True, 2, k_scale=2.0),
    # attention of the 7B-shaped layer: N=131072, 32 heads x 128, S=32, chunks 2048
    "layer7b_attn": AttnWorkload("layer7b_attn", 1, 32, 131072, 128, 32, 2048, 2048, True, 3),
    # million-token causal forward: S=64, q_chunk 1024, k_chunk 4096
    "n1m_d128": AttnWorkload("n1m_d128", 1, 32, 1048576, 128, 64, 1024, 4096, True, 4, bwd=False),
    # the 32k workload with grouped key/value heads: 8 KV heads for 32 query heads
    "n32k_d128_gqa8": AttnWorkload("n32k_d128_gqa8", 1, 32, 32768, 128, 16, 512, 1024, True, 5, k_scale=2.0,
                                   Hkv=8),
}

FFN_WORKLOADS = {
    # SwiGLU 4096 -> 11008 -> 4096 over N=131072 tokens in 2048-token chunks
    "layer7b_ffn": FFNWorkload("layer7b_ffn", 131072, 4096, 11008, 2048, 3),
}


@dataclass(frozen=True)
class DecodeWorkload:
    name: str
    B: int
    H: int
    Hkv: int
    N: int
    D: int
    S: int
    k_chunk: int
    seed: int


DECODE_WORKLOADS = {
    # one decode step after a ring prefill of 131072 tokens (S=32) for a batch of 8,
    # 32 query heads sharing 8 key/value heads of 128
    "decode_n128k": DecodeWorkload("decode_n128k", 8, 32, 8, 131072, 128, 32, 1024, 6),
}


@dataclass(frozen=True)
class LayerWorkload:
    name: str
    B: int
    N: int
    H: int
    D: int
    d_ff: int
    S: int
    q_chunk: int
    k_chunk: int
    ffn_chunk: int
    seed: int
    causal: bool = True
    w_std: float = 0.02
    eps: float = 1e-5

    @property
    def d_model(self) -> int:
        return self.H * self.D

    @property
    def T(self) -> int:
        return self.B * self.N


LAYER_WORKLOADS = {
    # the whole 7B-shaped layer (norms, projections, ring attention, SwiGLU FFN)
    # over N=131072 tokens, forward and backward
    "layer7b_full": LayerWorkload("layer7b_full", 1, 131072, 32, 128, 11008, 32, 2048, 2048, 2048, 3),
}


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _draw(shape, g, device, scale, dtype):
    x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if scale != 1.0:
        x.mul_(scale)
    return x.to(dtype)


def attention_inputs(w: AttnWorkload, device="cuda", with_dout: bool | None = None):
    """q, k, v (and dO when the workload has a backward) as [B,H,N,D] tensors."""
    shape = (w.B, w.H, w.N, w.D)
    kv_shape = (w.B, w.kv_heads, w.N, w.D)
    g = _gen(device, w.seed)
    q = _draw(shape, g, device, 1.0, w.dtype)
    k = _draw(kv_shape, g, device, w.k_scale, w.dtype)
    v = _draw(kv_shape, g, device, 1.0, w.dtype)
    want_do = w.bwd if with_dout is None else with_dout
    do = _draw(shape, g, device, 1.0, w.dtype) if want_do else None
    return q, k, v, do


def small_attention_inputs(B, H, N, D, seed, dtype=torch.bfloat16, device="cuda", k_scale=1.0, Hkv=0):
    """q, k, v, dO for ad-hoc test shapes (same recipe as the workloads)."""
    w = AttnWorkload("adhoc", B, H, N, D, 1, N, N, True, seed, dtype, k_scale, Hkv=Hkv)
    return attention_inputs(w, device, with_dout=True)


def decode_inputs(w: DecodeWorkload, device="cuda"):
    """q [B,H,D] (one new token per head), k, v [B,Hkv,N,D] (the cache)."""
    g = _gen(device, w.seed)
    q = _draw((w.B, w.H, w.D), g, device, 1.0, torch.bfloat16)
    k = _draw((w.B, w.Hkv, w.N, w.D), g, device, 1.0, torch.bfloat16)
    v = _draw((w.B, w.Hkv, w.N, w.D), g, device, 1.0, torch.bfloat16)
    return q, k, v


def ffn_inputs(w: FFNWorkload, device="cuda", T: int | None = None, with_dy: bool = False):
    """x [T, d_model], w1 [d_ff, d_model], w3 [d_ff, d_model], w2 [d_model, d_ff]
    (and, with with_dy, the output gradient dy [T, d_model], drawn last)."""
    T = w.T if T is None else T
    g = _gen(device, w.seed)
    x = _draw((T, w.d_model), g, device, 1.0, w.dtype)
    w1 = _draw((w.d_ff, w.d_model), g, device, w.w_std, w.dtype)
    w3 = _draw((w.d_ff, w.d_model), g, device, w.w_std, w.dtype)
    w2 = _draw((w.d_model, w.d_ff), g, device, w.w_std, w.dtype)
    if with_dy:
        return x, w1, w2, w3, _draw((T, w.d_model), g, device, 1.0, w.dtype)
    return x, w1, w2, w3


def sample_rows(B: int, H: int, N: int, n: int, seed: int, include_ends: bool = True) -> np.ndarray:
    """n seeded (b, h, i) triples (numpy default_rng(seed + 1000)).

    With include_ends the first two are the first and the last token of a
    head, so the first row of the causal diagonal and the longest row are
    always checked.
    """
    rng = np.random.default_rng(seed + 1000)
    rows = np.stack([rng.integers(0, B, n), rng.integers(0, H, n), rng.integers(0, N, n)], axis=1)
    if include_ends and n >= 2:
        rows[0] = (0, 0, 0)
        rows[1] = (B - 1, H - 1, N - 1)
    return rows.astype(np.int64)


def to_f64(t: torch.Tensor) -> np.ndarray:
    """Exact upcast of a (bf16 / fp32) tensor to a float64 numpy array."""
    return t.detach().to("cpu", torch.float32).numpy().astype(np.float64)


def layer_inputs(w: LayerWorkload, device="cuda"):
    """x [T, d_model]; params (g_attn, wq, wk, wv, wo, g_ffn, w1, w2, w3);
    dy [T, d_model].  Drawn in the order x, g_attn, wq, wk, wv, wo, g_ffn,
    w1, w3, w2, dy; norm gains are 1 + 0.1 z, weights w_std z."""
    g = _gen(device, w.seed)
    dm, dff = w.d_model, w.d_ff
    x = _draw((w.T, dm), g, device, 1.0, torch.bfloat16)
    g_attn = (1.0 + 0.1 * torch.randn(dm, generator=g, device=device)).to(torch.bfloat16)
    wq, wk, wv, wo = (_draw((dm, dm), g, device, w.w_std, torch.bfloat16) for _ in range(4))
    g_ffn = (1.0 + 0.1 * torch.randn(dm, generator=g, device=device)).to(torch.bfloat16)
    w1 = _draw((dff, dm), g, device, w.w_std, torch.bfloat16)
    w3 = _draw((dff, dm), g, device, w.w_std, torch.bfloat16)
    w2 = _draw((dm, dff), g, device, w.w_std, torch.bfloat16)
    dy = _draw((w.T, dm), g, device, 1.0, torch.bfloat16)
    return x, (g_attn, wq, wk, wv, wo, g_ffn, w1, w2, w3), dy

