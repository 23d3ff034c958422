"""GPU parity of one blockwise transformer layer (RMS norms, projections,
ring attention, SwiGLU feed-forward; forward and backward) against the fp64
oracle layer on the same seeded bf16 input bits.

Error model: the GPU keeps every activation between kernels in bf16 (xn,
q, k, v, o, x2, xn2, h, and in the backward dxn2, dx2, dO, dq, dk, dv, dxn,
dg, du) and rounds P and dS to bf16 inside the attention; each rounding is
a relative error of at most 2^-9 (rms 2^-9/sqrt(3)), independent from
element to element, and about ten of them lie on the longest path: an
expected relative error of sqrt(10) 2^-9/sqrt(3), about 3.6e-3.  The bound
on the relative Frobenius error of every output is 2^-6 (a factor four for
amplification through the softmax and the norms), and no element may be off
by more than 2^-3 of the output's rms (about five standard deviations of the
same errors over a few million elements)."""

import numpy as np
import pytest
import torch

import oracle
from exact_blockwise_long_b200.synthetic import LayerWorkload, layer_inputs, to_f64

pytestmark = pytest.mark.gpu

FROB = 2.0 ** -6
ELEM = 2.0 ** -3


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from exact_blockwise_long_b200 import build
    build.build()
    import exact_blockwise_long_b200 as ra
    ra.lib()
    torch.cuda.set_device(0)


def run_layer(w, x, params, dy):
    import exact_blockwise_long_b200 as ra
    dm = w.d_model
    saved = torch.empty(ra.blockwise_layer_saved_size(w.B, w.N, w.H, w.D), device="cuda", dtype=torch.uint8)
    fws = torch.empty(ra.blockwise_layer_fwd_workspace_size(w.ffn_chunk, w.d_ff), device="cuda", dtype=torch.uint8)
    bws = torch.empty(ra.blockwise_layer_bwd_workspace_size(w.B, w.N, w.H, w.D, w.d_ff, w.ffn_chunk), device="cuda",
                      dtype=torch.uint8)
    y = torch.empty_like(x)
    ra.blockwise_layer_fwd(x, params, y, saved, w.B, w.N, w.H, w.D, w.S, w.q_chunk, w.k_chunk, w.causal,
                           w.ffn_chunk, fws, eps=w.eps)
    dx = torch.empty_like(x)
    grads = tuple(torch.empty(p.shape, device="cuda", dtype=torch.float32) for p in params)
    ra.blockwise_layer_bwd(x, params, saved, dy, dx, grads, w.B, w.N, w.H, w.D, w.S, w.q_chunk, w.k_chunk,
                           w.causal, w.ffn_chunk, bws)
    assert ra.ringattn_get_error() == 0
    assert dm == x.shape[1]
    return y, dx, grads


def check(name, got, ref):
    got, ref = np.asarray(got), np.asarray(ref)
    rms = float(np.sqrt(np.mean(ref * ref)))
    frob = float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30))
    worst = float(np.abs(got - ref).max() / max(rms, 1e-30))
    assert frob <= FROB and worst <= ELEM, (name, frob, worst)
    return frob, worst


CASES = [
    # B, N, H, D, d_ff, S, qc, kc, ffn_chunk, causal
    (1, 1024, 2, 128, 384, 4, 128, 128, 256, True),
    (2, 512, 4, 64, 512, 2, 128, 256, 512, True),
    (1, 768, 2, 128, 256, 3, 256, 128, 256, False),
    (1, 4096, 2, 128, 256, 2, 256, 512, 1024, True),  # four FFN chunks, long weight-gradient K
]


@pytest.mark.parametrize("B,N,H,D,dff,S,qc,kc,fc,causal", CASES)
def test_layer_full_oracle(B, N, H, D, dff, S, qc, kc, fc, causal):
    w = LayerWorkload("t", B, N, H, D, dff, S, qc, kc, fc, 50 + N + H, causal, w_std=(H * D) ** -0.5)
    x, params, dy = layer_inputs(w)
    y, dx, grads = run_layer(w, x, params, dy)
    xf, pf, dyf = to_f64(x), [to_f64(p) for p in params], to_f64(dy)
    ry, _ = oracle.layer_forward(xf, pf, B, N, H, D, causal, w.eps)
    rdx, rgrads = oracle.layer_backward(xf, pf, dyf, B, N, H, D, causal, w.eps)
    check("y", to_f64(y), ry)
    check("dx", to_f64(dx), rdx)
    for n, g, r in zip(oracle.PARAM_NAMES, grads, rgrads):
        check("d" + n, to_f64(g), r)


def test_layer_7b_width():
    """The 7B layer's widths (32 heads x 128, d_ff 11008) on 512 tokens in
    two shards, full oracle."""
    w = LayerWorkload("t", 1, 512, 32, 128, 11008, 2, 128, 256, 256, 61)
    x, params, dy = layer_inputs(w)
    y, dx, grads = run_layer(w, x, params, dy)
    xf, pf, dyf = to_f64(x), [to_f64(p) for p in params], to_f64(dy)
    ry, _ = oracle.layer_forward(xf, pf, w.B, w.N, w.H, w.D, True, w.eps)
    rdx, rgrads = oracle.layer_backward(xf, pf, dyf, w.B, w.N, w.H, w.D, True, w.eps)
    check("y", to_f64(y), ry)
    check("dx", to_f64(dx), rdx)
    for n, g, r in zip(oracle.PARAM_NAMES, grads, rgrads):
        check("d" + n, to_f64(g), r)


def test_layer_bad_shapes():
    import exact_blockwise_long_b200 as ra
    from exact_blockwise_long_b200 import RingAttnError
    w = LayerWorkload("t", 1, 1024, 2, 128, 384, 4, 128, 128, 256, 7)
    x, params, dy = layer_inputs(w)
    saved = torch.empty(ra.blockwise_layer_saved_size(1, 1024, 2, 128), device="cuda", dtype=torch.uint8)
    fws = torch.empty(ra.blockwise_layer_fwd_workspace_size(256, 384), device="cuda", dtype=torch.uint8)
    y = torch.empty_like(x)
    with pytest.raises(RingAttnError):   # 1024 tokens are not 3 equal shards
        ra.blockwise_layer_fwd(x, params, y, saved, 1, 1024, 2, 128, 3, 128, 128, True, 256, fws)
    with pytest.raises(RingAttnError):   # the saved buffer is too small
        ra.blockwise_layer_fwd(x, params, y, saved[:1024], 1, 1024, 2, 128, 4, 128, 128, True, 256, fws)


def test_layer_empty_batch():
    """No tokens: the forward does nothing, the backward zeroes the nine
    parameter gradients."""
    import exact_blockwise_long_b200 as ra
    w = LayerWorkload("t", 1, 256, 2, 128, 256, 2, 128, 128, 256, 8)
    x, params, dy = layer_inputs(w)
    grads = tuple(torch.full(p.shape, 3.0, device="cuda", dtype=torch.float32) for p in params)
    e = x[:0]
    empty = torch.empty(0, device="cuda", dtype=torch.uint8)
    assert ra.lib().blockwise_layer_fwd(*([None] * 12), 0, 0, 256, 2, 128, 256, 2, 128, 128, 1, 256, 1e-5, None,
                                        0, None, None) == 0
    ra.blockwise_layer_bwd(e, params, empty, dy[:0], torch.empty_like(e), grads, 0, 256, 2, 128, 2, 128, 128,
                           True, 256, empty)
    assert ra.ringattn_get_error() == 0
    assert all(torch.count_nonzero(g) == 0 for g in grads)


def test_layer_repeatable():
    """The forward reduces in a fixed order: repeated runs give identical
    bits.  The backward's attention sums dQ over key tiles with fp32
    additions in arrival order, so dx and the parameter gradients of repeats
    differ only by that order's rounding: far below the layer's tolerance
    (relative Frobenius 2^-6), bounded here by 2^-10."""
    w = LayerWorkload("t", 1, 1024, 2, 128, 384, 4, 128, 128, 256, 71, w_std=256 ** -0.5)
    x, params, dy = layer_inputs(w)
    a = run_layer(w, x, params, dy)

    def rel(p, q):
        p, q = p.float(), q.float()
        return float((p - q).norm() / q.norm().clamp_min(1e-30))

    for _ in range(3):
        b = run_layer(w, x, params, dy)
        assert torch.equal(a[0], b[0])
        assert rel(b[1], a[1]) <= 2.0 ** -10
        assert all(rel(p, q) <= 2.0 ** -10 for p, q in zip(b[2], a[2]))
