"""Shared helpers for the GPU parity tests: tolerances, oracle comparison on
sampled rows, and small utilities.  Expected values always come from
``oracle`` on the exact input bits the GPU received."""

from __future__ import annotations

import numpy as np
import torch

import oracle
from exact_blockwise_long_b200.synthetic import to_f64

# Tolerances (max absolute error against the fp64 oracle).
TOL_F32 = 1e-4          # fp32 path, O and LSE
TOL_BF16_O = 2e-2       # bf16 inputs, fp32 accumulation: O
TOL_BF16_LSE = 1e-2     # bf16 path LSE: the pages state none; half the O bound
TOL_BF16_GRAD = 5e-2    # dQ, dK, dV


def max_abs(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.abs(a - b).max()) if a.size else 0.0


def check_rows(q, k, v, o, lse, rows, causal, scale=None):
    """Oracle forward on sampled (b, h, i) rows; returns (err_o, err_lse).

    K and V of each sampled head are upcast once; rows of one head are done
    together.
    """
    rows = np.asarray(rows)
    err_o = err_l = 0.0
    heads = sorted({(int(b), int(h)) for b, h, _ in rows})
    for b, h in heads:
        sel = rows[(rows[:, 0] == b) & (rows[:, 1] == h)]
        idx = torch.as_tensor(sel[:, 2], device=q.device)
        o_ref, l_ref = oracle.attention_head_rows(to_f64(q[b, h].index_select(0, idx)), to_f64(k[b, h]),
                                                  to_f64(v[b, h]), sel[:, 2], causal, scale)
        o_gpu = to_f64(o[b, h].index_select(0, idx))
        l_gpu = to_f64(lse[b, h].index_select(0, idx))
        err_o = max(err_o, max_abs(o_gpu, o_ref))
        err_l = max(err_l, max_abs(l_gpu, l_ref))
    return err_o, err_l


def run_fwd(q, k, v, S, qc, kc, causal):
    import exact_blockwise_long_b200 as ra
    B, H, N, D = q.shape
    out = torch.empty_like(q)
    lse = torch.empty((B, H, N), device=q.device, dtype=torch.float32)
    ra.ringattn_fwd(q, k, v, out, lse, S, qc, kc, causal)
    assert ra.ringattn_get_error() == 0
    return out, lse
