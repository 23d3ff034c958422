"""GPU parity of the blockwise SwiGLU feed-forward backward (tcgen05 GEMMs)
against the fp64 oracle gradient of sum(dy * y), on the same seeded bf16
input bits.

Bound (per element, derived from the arithmetic): the kernels round dg, du
and h to bf16 (relative error <= 2^-9 each) before the contractions that use
them, and round dx to bf16 once more at the end; everything else is fp32
accumulation of exact bf16 products.  So with `terms` the sum of |term| of
each contraction (oracle.swiglu_ffn_backward_terms),
    |dx_gpu  - dx_ref|  <= 2^-8 terms + 2^-8 |dx_ref|
    |dwX_gpu - dwX_ref| <= 2^-8 terms
(2^-8 doubles the rounding bound to absorb the fp32 sums and the sigmoid
approximation).  That bound is worst case; the rounding errors are
independent, so the relative Frobenius error must also stay below 2^-7."""

import numpy as np
import pytest
import torch

import oracle
from exact_blockwise_long_b200.synthetic import FFN_WORKLOADS, FFNWorkload, ffn_inputs, to_f64

pytestmark = pytest.mark.gpu

EPS = 2.0 ** -8
FROB = 2.0 ** -7


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from exact_blockwise_long_b200 import build
    build.build()
    import exact_blockwise_long_b200 as ra
    ra.lib()
    torch.cuda.set_device(0)


def run_ffn_bwd(x, w1, w2, w3, dy, chunk):
    import exact_blockwise_long_b200 as ra
    dx = torch.empty_like(x)
    dw1 = torch.empty(w1.shape, device="cuda", dtype=torch.float32)
    dw3 = torch.empty(w3.shape, device="cuda", dtype=torch.float32)
    dw2 = torch.empty(w2.shape, device="cuda", dtype=torch.float32)
    ws = torch.empty(ra.blockwise_ffn_bwd_workspace_size(chunk, w1.shape[0]), device="cuda", dtype=torch.uint8)
    ra.blockwise_ffn_bwd(x, w1, w2, w3, dy, dx, dw1, dw2, dw3, chunk, ws)
    assert ra.ringattn_get_error() == 0
    return dx, dw1, dw2, dw3


def check(got, ref, terms, final_round):
    err = np.abs(got - ref)
    bound = EPS * terms + (EPS * np.abs(ref) if final_round else 0.0)
    assert np.all(err <= bound), float((err / np.maximum(bound, 1e-30)).max())
    frob = np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30)
    assert frob <= FROB, frob


@pytest.mark.parametrize("T,dm,dff,chunk", [(512, 256, 384, 128), (256, 128, 256, 256), (384, 512, 128, 128),
                                            (1024, 384, 640, 256)])
def test_ffn_bwd_full_oracle(T, dm, dff, chunk):
    w = FFNWorkload("t", T, dm, dff, chunk, 21 + T + dm, w_std=0.06)
    x, w1, w2, w3, dy = ffn_inputs(w, with_dy=True)
    got = run_ffn_bwd(x, w1, w2, w3, dy, chunk)
    args = [to_f64(t) for t in (x, w1, w2, w3, dy)]
    ref = oracle.blockwise_ffn_backward(*args, chunk)
    terms = oracle.swiglu_ffn_backward_terms(*args)
    for i, (g, r, t) in enumerate(zip(got, ref, terms)):
        check(to_f64(g), r, t, final_round=(i == 0))


def test_ffn_bwd_chunking_keeps_dx_rows():
    """dx rows depend only on their own token: any chunk size gives the same
    bits; the weight gradients differ only by fp32 summation order."""
    w = FFNWorkload("t", 1024, 256, 512, 128, 31)
    x, w1, w2, w3, dy = ffn_inputs(w, with_dy=True)
    a = run_ffn_bwd(x, w1, w2, w3, dy, 128)
    b = run_ffn_bwd(x, w1, w2, w3, dy, 1024)
    assert torch.equal(a[0], b[0])
    for p, q in zip(a[1:], b[1:]):
        assert torch.allclose(p, q, rtol=1e-5, atol=1e-5)


def test_ffn_bwd_repeatable_and_zero_cases():
    w = FFNWorkload("t", 256, 256, 384, 128, 32)
    x, w1, w2, w3, dy = ffn_inputs(w, with_dy=True)
    a = run_ffn_bwd(x, w1, w2, w3, dy, 128)
    b = run_ffn_bwd(x, w1, w2, w3, dy, 128)
    assert all(torch.equal(p, q) for p, q in zip(a, b))  # no atomics: identical bits
    # no up projection: only dw3 survives
    dx, dw1, dw2, dw3 = run_ffn_bwd(x, w1, w2, torch.zeros_like(w3), dy, 128)
    assert torch.count_nonzero(dx) == 0 and torch.count_nonzero(dw1) == 0 and torch.count_nonzero(dw2) == 0
    assert torch.count_nonzero(dw3) > 0
    # zero output gradient: every gradient is zero
    for t in run_ffn_bwd(x, w1, w2, w3, torch.zeros_like(dy), 128):
        assert torch.count_nonzero(t) == 0


def test_ffn_bwd_empty_and_bad_shapes():
    import exact_blockwise_long_b200 as ra
    from exact_blockwise_long_b200 import RingAttnError
    w = FFNWorkload("t", 256, 128, 256, 128, 33)
    x, w1, w2, w3, dy = ffn_inputs(w, with_dy=True)
    dw = [torch.full(t.shape, 7.0, device="cuda") for t in (w1, w2, w3)]
    ws = torch.empty(ra.blockwise_ffn_bwd_workspace_size(128, 256), device="cuda", dtype=torch.uint8)
    e = x[:0]
    ra.blockwise_ffn_bwd(e, w1, w2, w3, dy[:0], torch.empty_like(e), dw[0], dw[1], dw[2], 128, ws)
    assert ra.ringattn_get_error() == 0
    assert all(torch.count_nonzero(t) == 0 for t in dw)  # no tokens: zero weight gradients
    with pytest.raises(RingAttnError):  # 192 tokens are not a whole number of 128-token chunks
        ra.blockwise_ffn_bwd(x[:192], w1, w2, w3, dy[:192], torch.empty_like(x[:192]), *dw, 128, ws)
    with pytest.raises(RingAttnError):  # workspace too small
        ra.blockwise_ffn_bwd(x, w1, w2, w3, dy, torch.empty_like(x), *dw, 128, ws[:1024])


def test_ffn_bwd_7b_shape_sampled():
    """The 7B layer's FFN shape (4096 -> 11008 -> 4096, 2048-token chunks) on
    two chunks: 32 seeded dx rows, and dw1/dw3 rows and dw2 columns of 32
    seeded hidden units (a subset of hidden units has exactly the weight
    gradients of those units, so the oracle runs on that subset alone)."""
    w = FFN_WORKLOADS["layer7b_ffn"]
    T = 4096
    x, w1, w2, w3, dy = ffn_inputs(w, T=T, with_dy=True)
    dx, dw1, dw2, dw3 = run_ffn_bwd(x, w1, w2, w3, dy, w.chunk)
    rng = np.random.default_rng(w.seed + 4000)
    rows = np.sort(rng.choice(T, 32, replace=False))
    rows[0], rows[-1] = 0, T - 1
    units = np.sort(rng.choice(w.d_ff, 32, replace=False))
    units[0], units[-1] = 0, w.d_ff - 1
    ri = torch.as_tensor(rows, device="cuda")
    ui = torch.as_tensor(units, device="cuda")
    xs, dys = to_f64(x[ri]), to_f64(dy[ri])
    W1, W2, W3 = to_f64(w1), to_f64(w2), to_f64(w3)
    rdx = oracle.swiglu_ffn_backward(xs, W1, W2, W3, dys)[0]
    tdx = oracle.swiglu_ffn_backward_terms(xs, W1, W2, W3, dys)[0]
    check(to_f64(dx[ri]), rdx, tdx, final_round=True)
    sub = (to_f64(x), W1[units], W2[:, units], W3[units], to_f64(dy))
    _, r1, r2, r3 = oracle.swiglu_ffn_backward(*sub)
    _, t1, t2, t3 = oracle.swiglu_ffn_backward_terms(*sub)
    check(to_f64(dw1[ui]), r1, t1, False)
    check(to_f64(dw2[:, ui]), r2, t2, False)
    check(to_f64(dw3[ui]), r3, t3, False)


@pytest.mark.slow
def test_ffn_bwd_7b_full_size_sampled():
    """The layer workload's FFN backward at full size (131072 tokens, 64
    chunks): 16 seeded dx rows, and the weight gradients of 8 seeded hidden
    units summed over all tokens (the oracle runs on 8192-token slices of
    those units and adds the slices up in fp64)."""
    w = FFN_WORKLOADS["layer7b_ffn"]
    x, w1, w2, w3, dy = ffn_inputs(w, with_dy=True)
    dx, dw1, dw2, dw3 = run_ffn_bwd(x, w1, w2, w3, dy, w.chunk)
    rng = np.random.default_rng(w.seed + 5000)
    rows = np.sort(rng.choice(w.T, 16, replace=False))
    rows[0], rows[-1] = 0, w.T - 1
    units = np.sort(rng.choice(w.d_ff, 8, replace=False))
    W1, W2, W3 = to_f64(w1), to_f64(w2), to_f64(w3)
    ri = torch.as_tensor(rows, device="cuda")
    xs, dys = to_f64(x[ri]), to_f64(dy[ri])
    check(to_f64(dx[ri]), oracle.swiglu_ffn_backward(xs, W1, W2, W3, dys)[0],
          oracle.swiglu_ffn_backward_terms(xs, W1, W2, W3, dys)[0], final_round=True)
    ref = [np.zeros((len(units), w.d_model)), np.zeros((w.d_model, len(units))), np.zeros((len(units), w.d_model))]
    trm = [np.zeros_like(r) for r in ref]
    for c0 in range(0, w.T, 8192):
        sub = (to_f64(x[c0:c0 + 8192]), W1[units], W2[:, units], W3[units], to_f64(dy[c0:c0 + 8192]))
        _, r1, r2, r3 = oracle.swiglu_ffn_backward(*sub)
        _, t1, t2, t3 = oracle.swiglu_ffn_backward_terms(*sub)
        for acc, part in zip(ref + trm, (r1, r2, r3, t1, t2, t3)):
            acc += part
    ui = torch.as_tensor(units, device="cuda")
    check(to_f64(dw1[ui]), ref[0], trm[0], False)
    check(to_f64(dw2[:, ui]), ref[1], trm[1], False)
    check(to_f64(dw3[ui]), ref[2], trm[2], False)
