"""GPU parity of grouped key/value heads (GQA, MQA) in the ring forward and
backward against the fp64 oracle (attention_forward_gqa /
attention_backward_gqa) on the same seeded input bits."""

import numpy as np
import pytest
import torch

import oracle
from exact_blockwise_long_b200.synthetic import WORKLOADS, attention_inputs, sample_rows, small_attention_inputs, to_f64
from helpers import TOL_BF16_GRAD, TOL_BF16_LSE, TOL_BF16_O, TOL_F32, max_abs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from exact_blockwise_long_b200 import build
    build.build()
    import exact_blockwise_long_b200 as ra
    ra.lib()
    torch.cuda.set_device(0)


def fwd(q, k, v, S, qc, kc, causal):
    import exact_blockwise_long_b200 as ra
    B, H, N, D = q.shape
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), device="cuda", dtype=torch.float32)
    ra.ringattn_fwd_gqa(q, k, v, o, lse, S, qc, kc, causal)
    assert ra.ringattn_get_error() == 0
    return o, lse


def bwd(q, k, v, o, lse, do, S, qc, kc, causal):
    import exact_blockwise_long_b200 as ra
    B, H, N, D = q.shape
    ws = torch.empty(ra.ringattn_bwd_workspace_size(B, H, N, D), device="cuda", dtype=torch.uint8)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ra.ringattn_bwd_gqa(q, k, v, o, lse, do, dq, dk, dv, S, qc, kc, causal, ws)
    assert ra.ringattn_get_error() == 0
    return dq, dk, dv


CASES = [
    # (B, H, Hkv, N, D, S, qc, kc, causal)
    (1, 4, 2, 1024, 128, 4, 128, 256, True),    # GQA, two tiles per CTA forward
    (2, 4, 1, 768, 64, 3, 128, 128, False),     # MQA, shard of 256
    (1, 6, 3, 512, 128, 4, 128, 128, True),     # shard of 128 (one-tile forward)
    (1, 8, 2, 1024, 64, 2, 256, 512, True),
]


@pytest.mark.parametrize("B,H,Hkv,N,D,S,qc,kc,causal", CASES)
def test_gqa_fwd_bwd_full_oracle(B, H, Hkv, N, D, S, qc, kc, causal):
    q, k, v, do = small_attention_inputs(B, H, N, D, 300 + H + Hkv + N, k_scale=2.0, Hkv=Hkv)
    o, lse = fwd(q, k, v, S, qc, kc, causal)
    o_ref, l_ref = oracle.attention_forward_gqa(to_f64(q), to_f64(k), to_f64(v), causal)
    assert max_abs(to_f64(o), o_ref) <= TOL_BF16_O
    assert max_abs(to_f64(lse), l_ref) <= TOL_BF16_LSE
    dq, dk, dv = bwd(q, k, v, o, lse, do, S, qc, kc, causal)
    gq, gk, gv = oracle.attention_backward_gqa(to_f64(q), to_f64(k), to_f64(v), to_f64(do), causal)
    errs = [max_abs(to_f64(a), b) for a, b in ((dq, gq), (dk, gk), (dv, gv))]
    assert max(errs) <= TOL_BF16_GRAD, errs


def test_gqa_fp32_forward():
    q, k, v, _ = small_attention_inputs(1, 4, 512, 64, 31, dtype=torch.float32, Hkv=2)
    o, lse = fwd(q, k, v, 4, 64, 64, True)
    o_ref, l_ref = oracle.attention_forward_gqa(to_f64(q), to_f64(k), to_f64(v), True)
    assert max_abs(to_f64(o), o_ref) <= TOL_F32
    assert max_abs(to_f64(lse), l_ref) <= TOL_F32


def test_gqa_equals_expanded_kv():
    """Grouped heads give the same bits as the plain call on key/value heads
    repeated to H (the kernels are the same code on the same tiles)."""
    import exact_blockwise_long_b200 as ra
    q, k, v, do = small_attention_inputs(1, 8, 1024, 128, 41, Hkv=2)
    o1, l1 = fwd(q, k, v, 4, 256, 256, True)
    ke, ve = (t.repeat_interleave(4, dim=1).contiguous() for t in (k, v))
    o2 = torch.empty_like(q)
    l2 = torch.empty_like(l1)
    ra.ringattn_fwd(q, ke, ve, o2, l2, 4, 256, 256, True)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.slow
def test_gqa_workload_sampled():
    w = WORKLOADS["n32k_d128_gqa8"]
    q, k, v, do = attention_inputs(w)
    o, lse = fwd(q, k, v, w.S, w.q_chunk, w.k_chunk, w.causal)
    G = w.H // w.kv_heads
    rows = sample_rows(w.B, w.H, w.N, 256, w.seed)
    err_o = err_l = 0.0
    for b, h in sorted({(int(b), int(h)) for b, h, _ in rows}):
        sel = rows[(rows[:, 0] == b) & (rows[:, 1] == h)]
        idx = torch.as_tensor(sel[:, 2], device="cuda")
        o_r, l_r = oracle.attention_head_rows(to_f64(q[b, h][idx]), to_f64(k[b, h // G]), to_f64(v[b, h // G]),
                                              sel[:, 2], True)
        err_o = max(err_o, max_abs(to_f64(o[b, h][idx]), o_r))
        err_l = max(err_l, max_abs(to_f64(lse[b, h][idx]), l_r))
    assert err_o <= TOL_BF16_O and err_l <= TOL_BF16_LSE, (err_o, err_l)
    dq, dk, dv = bwd(q, k, v, o, lse, do, w.S, w.q_chunk, w.k_chunk, w.causal)
    # dk, dv of one key/value head on 64 key rows: sum over its 4 query heads
    rng = np.random.default_rng(w.seed + 2000)
    keys = np.sort(rng.choice(w.N, 64, replace=False))
    hk = 5
    gk = np.zeros((len(keys), w.D))
    gv = np.zeros((len(keys), w.D))
    kk, vv = to_f64(k[0:1, hk:hk + 1]), to_f64(v[0:1, hk:hk + 1])
    for h in range(hk * G, hk * G + G):
        a, b_ = oracle.attention_backward_key_rows(to_f64(q[0:1, h:h + 1]), kk, vv, to_f64(do[0:1, h:h + 1]),
                                                   0, 0, keys, True)
        gk += a
        gv += b_
    kidx = torch.as_tensor(keys, device="cuda")
    assert max_abs(to_f64(dk[0, hk][kidx]), gk) <= TOL_BF16_GRAD
    assert max_abs(to_f64(dv[0, hk][kidx]), gv) <= TOL_BF16_GRAD
