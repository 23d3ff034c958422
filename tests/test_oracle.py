"""Pins for the fp64 oracle: each check is fixed by the pages or by mathematics,
not by re-running the oracle's own formula.

* hand-derived golden values (tests/golden/*.txt)
* closed forms: q = 0 gives mean(V) and lse = ln N; causal row 0 gives v_0
* library routines: scipy.special.softmax / logsumexp / expit
* brute force with explicit Python loops on tiny inputs
* the method itself: ring/blockwise result equals the full matrix for every
  S and chunk size, in any ring visiting order, and the step partials merge
  to it in any order
* gradients: central finite differences, shift and homogeneity invariants
"""

import itertools
import math

import numpy as np
import pytest
import scipy.special

import oracle
from golden_io import golden_path, load, stack


def _rand(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


# ---------------------------------------------------------------------------
# Golden worked examples
# ---------------------------------------------------------------------------

def _hand_attention():
    g = load(golden_path("attention_hand.txt"))
    q = stack(g, "q", 3)[None, None]
    k = stack(g, "k", 3)[None, None]
    v = stack(g, "v", 3)[None, None]
    do = stack(g, "do", 3)[None, None]
    return g, q, k, v, do


@pytest.mark.parametrize("causal", [False, True])
def test_golden_forward(causal):
    g, q, k, v, _ = _hand_attention()
    o, lse = oracle.attention_forward(q, k, v, causal)
    p = "c_" if causal else "nc_"
    np.testing.assert_allclose(o[0, 0], stack(g, p + "o", 3), rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse[0, 0], g[p + "lse"], rtol=0, atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_golden_backward(causal):
    g, q, k, v, do = _hand_attention()
    dq, dk, dv = oracle.attention_backward(q, k, v, do, causal)
    p = "c_" if causal else "nc_"
    np.testing.assert_allclose(dq[0, 0], stack(g, p + "dq", 3), rtol=0, atol=1e-13)
    np.testing.assert_allclose(dk[0, 0], stack(g, p + "dk", 3), rtol=0, atol=1e-13)
    np.testing.assert_allclose(dv[0, 0], stack(g, p + "dv", 3), rtol=0, atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_golden_ring_blockwise(causal):
    g, q, k, v, _ = _hand_attention()
    # N = 3: three shards of one token each, chunks of one token.
    o, lse = oracle.ring_blockwise_forward(q, k, v, S=3, q_chunk=1, k_chunk=1, causal=causal)
    p = "c_" if causal else "nc_"
    np.testing.assert_allclose(o[0, 0], stack(g, p + "o", 3), rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse[0, 0], g[p + "lse"], rtol=0, atol=1e-13)


def test_golden_wrong_scale_is_caught():
    """A dropped softmax scale (a plausible slip) moves the golden values."""
    g, q, k, v, _ = _hand_attention()
    o, _ = oracle.attention_forward(q, k, v, False, scale=1.0)
    assert np.abs(o[0, 0] - stack(g, "nc_o", 3)).max() > 0.1


def test_golden_ffn():
    g = load(golden_path("ffn_hand.txt"))
    x = stack(g, "x", 2)
    w1 = stack(g, "w1_", 2)
    w3 = stack(g, "w3_", 2)
    w2 = stack(g, "w2_", 2)
    y = oracle.swiglu_ffn(x, w1, w2, w3)
    np.testing.assert_allclose(y, stack(g, "y", 2), rtol=0, atol=1e-13)
    yb = oracle.blockwise_ffn(x, w1, w2, w3, chunk=1)
    np.testing.assert_allclose(yb, stack(g, "y", 2), rtol=0, atol=1e-13)
    # swapping the gate and up weights (a plausible slip) is caught
    assert np.abs(oracle.swiglu_ffn(x, w3, w2, w1) - stack(g, "y", 2)).max() > 0.1


# ---------------------------------------------------------------------------
# Closed forms and library routines
# ---------------------------------------------------------------------------

def test_zero_query_gives_mean_of_v():
    B, H, N, d = 2, 3, 37, 8
    q = np.zeros((B, H, N, d))
    k = _rand((B, H, N, d), 1)
    v = _rand((B, H, N, d), 2)
    o, lse = oracle.attention_forward(q, k, v, causal=False)
    np.testing.assert_allclose(o, np.broadcast_to(v.mean(axis=2, keepdims=True), o.shape), atol=1e-13)
    np.testing.assert_allclose(lse, np.log(N), atol=1e-13)


def test_zero_query_causal_gives_prefix_mean():
    N, d = 23, 4
    q = np.zeros((1, 1, N, d))
    k = _rand((1, 1, N, d), 3)
    v = _rand((1, 1, N, d), 4)
    o, lse = oracle.attention_forward(q, k, v, causal=True)
    prefix = np.cumsum(v[0, 0], axis=0) / np.arange(1, N + 1)[:, None]
    np.testing.assert_allclose(o[0, 0], prefix, atol=1e-13)
    np.testing.assert_allclose(lse[0, 0], np.log(np.arange(1, N + 1)), atol=1e-13)


def test_causal_row0_is_v0():
    B, H, N, d = 2, 2, 16, 8
    q, k, v = _rand((B, H, N, d), 5), _rand((B, H, N, d), 6), _rand((B, H, N, d), 7)
    o, lse = oracle.attention_forward(q, k, v, causal=True)
    np.testing.assert_allclose(o[:, :, 0], v[:, :, 0], atol=1e-14)
    s00 = (q[:, :, 0] * k[:, :, 0]).sum(-1) / np.sqrt(d)
    np.testing.assert_allclose(lse[:, :, 0], s00, atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_matches_scipy_softmax(causal):
    B, H, N, d = 1, 2, 40, 16
    q, k, v = _rand((B, H, N, d), 8), _rand((B, H, N, d), 9, 2.0), _rand((B, H, N, d), 10)
    o, lse = oracle.attention_forward(q, k, v, causal)
    for h in range(H):
        s = q[0, h] @ k[0, h].T / math.sqrt(d)
        if causal:
            s = np.where(np.tril(np.ones((N, N), bool)), s, -np.inf)
        p = scipy.special.softmax(s, axis=1)
        np.testing.assert_allclose(o[0, h], p @ v[0, h], atol=1e-12)
        np.testing.assert_allclose(lse[0, h], scipy.special.logsumexp(s, axis=1), atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_brute_force_loops(causal):
    """Explicit enumeration of visible pairs with math.exp, no arrays."""
    N, d = 7, 3
    q, k, v = _rand((1, 1, N, d), 11), _rand((1, 1, N, d), 12), _rand((1, 1, N, d), 13)
    o, lse = oracle.attention_forward(q, k, v, causal)
    sc = 1.0 / math.sqrt(d)
    for i in range(N):
        pairs = [j for j in range(N) if (j <= i or not causal)]
        w = [math.exp(sc * sum(q[0, 0, i, c] * k[0, 0, j, c] for c in range(d))) for j in pairs]
        tot = sum(w)
        for c in range(d):
            ref = sum(wj * v[0, 0, j, c] for wj, j in zip(w, pairs)) / tot
            assert abs(o[0, 0, i, c] - ref) < 1e-13
        assert abs(lse[0, 0, i] - math.log(tot)) < 1e-13


def test_sharp_scores_select_argmax():
    """A key aligned with the query and 100x longer dominates the softmax."""
    N, d = 16, 8
    rng = np.random.default_rng(14)
    q = rng.standard_normal((1, 1, N, d))
    k = rng.standard_normal((1, 1, N, d)) * 0.01
    v = rng.standard_normal((1, 1, N, d))
    k[0, 0, 5] = 100.0 * q[0, 0, 9] / np.linalg.norm(q[0, 0, 9])
    o, _ = oracle.attention_forward(q, k, v, causal=False)
    np.testing.assert_allclose(o[0, 0, 9], v[0, 0, 5], atol=1e-8)


def test_causal_locality():
    """Row i depends only on keys/values j <= i."""
    B, H, N, d = 1, 2, 24, 8
    q, k, v = _rand((B, H, N, d), 15), _rand((B, H, N, d), 16), _rand((B, H, N, d), 17)
    o1, l1 = oracle.attention_forward(q, k, v, causal=True)
    i = 10
    k2, v2 = k.copy(), v.copy()
    k2[:, :, i + 1:] += 5.0
    v2[:, :, i + 1:] -= 3.0
    o2, l2 = oracle.attention_forward(q, k2, v2, causal=True)
    np.testing.assert_array_equal(o1[:, :, : i + 1], o2[:, :, : i + 1])
    np.testing.assert_array_equal(l1[:, :, : i + 1], l2[:, :, : i + 1])
    assert np.abs(o1[:, :, i + 1:] - o2[:, :, i + 1:]).max() > 1e-3


# ---------------------------------------------------------------------------
# The method against the definition
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("S", [1, 2, 4, 8, 16])
def test_ring_blockwise_equals_full(S, causal):
    B, H, N, d = 1, 2, 64, 8
    q, k, v = _rand((B, H, N, d), 18), _rand((B, H, N, d), 19, 2.0), _rand((B, H, N, d), 20)
    o_ref, l_ref = oracle.attention_forward(q, k, v, causal)
    L = N // S
    chunks = [c for c in (1, 2, 4, 8, 16, 32, 64) if L % c == 0]
    for qc, kc in itertools.product(chunks, chunks):
        if qc < L // 4 and kc < L // 4 and L > 8:
            continue  # keep the sweep small; tiny chunks are covered at small L
        o, lse = oracle.ring_blockwise_forward(q, k, v, S, qc, kc, causal)
        np.testing.assert_allclose(o, o_ref, atol=1e-12, rtol=0)
        np.testing.assert_allclose(lse, l_ref, atol=1e-12, rtol=0)


@pytest.mark.parametrize("causal", [False, True])
def test_ring_order_invariance(causal):
    B, H, N, d, S = 1, 1, 48, 4, 6
    q, k, v = _rand((B, H, N, d), 21), _rand((B, H, N, d), 22), _rand((B, H, N, d), 23)
    o_ref, l_ref = oracle.attention_forward(q, k, v, causal)
    rng = np.random.default_rng(24)
    for _ in range(5):
        perms = {}
        for i in range(S):
            vis = oracle.ring_visit_order(i, S, causal)
            perms[i] = list(rng.permutation(vis))
        o, lse = oracle.ring_blockwise_forward(q, k, v, S, 4, 2, causal, order=lambda i: perms[i])
        np.testing.assert_allclose(o, o_ref, atol=1e-12)
        np.testing.assert_allclose(lse, l_ref, atol=1e-12)


def test_ring_visit_order_matches_statement():
    # step t: shard i holds KV shard (i - t) mod S
    assert oracle.ring_visit_order(2, 4, False) == [2, 1, 0, 3]
    assert oracle.ring_visit_order(2, 4, True) == [2, 1, 0]
    assert oracle.ring_visit_order(0, 4, True) == [0]
    assert oracle.ring_visit_order_bwd(1, 4, False) == [1, 2, 3, 0]
    assert oracle.ring_visit_order_bwd(1, 4, True) == [1, 2, 3]
    # forward and backward loop nests cover the same causal pairs
    S = 7
    fwd = {(i, j) for i in range(S) for j in oracle.ring_visit_order(i, S, True)}
    bwd = {(i, j) for j in range(S) for i in oracle.ring_visit_order_bwd(j, S, True)}
    assert fwd == bwd and len(fwd) == S * (S + 1) // 2


@pytest.mark.parametrize("causal", [False, True])
def test_step_partials_merge_to_full(causal):
    """Materialise each ring step, merge the partials in any order."""
    B, H, N, d, S = 1, 2, 32, 4, 4
    q, k, v = _rand((B, H, N, d), 25), _rand((B, H, N, d), 26), _rand((B, H, N, d), 27)
    o_ref, l_ref = oracle.attention_forward(q, k, v, causal)
    parts = [oracle.ring_blockwise_step(q, k, v, S, t, causal) for t in range(S)]
    for order in ([0, 1, 2, 3], [3, 1, 0, 2]):
        o = np.zeros_like(o_ref)
        lse = np.full(l_ref.shape, -np.inf)
        for t in order:
            o, lse = oracle.lse_merge(o, lse, *parts[t])
        np.testing.assert_allclose(o, o_ref, atol=1e-12)
        np.testing.assert_allclose(lse, l_ref, atol=1e-12)


def test_lse_merge_closed_form_and_algebra():
    rng = np.random.default_rng(28)
    n, d = 10, 5
    s = rng.standard_normal((n, 9)) * 3
    v = rng.standard_normal((9, d))
    # two disjoint key sets
    a, b = slice(0, 4), slice(4, 9)
    def part(sl):
        lse = scipy.special.logsumexp(s[:, sl], axis=1)
        return scipy.special.softmax(s[:, sl], axis=1) @ v[sl], lse
    oa, la = part(a)
    ob, lb = part(b)
    o, lse = oracle.lse_merge(oa, la, ob, lb)
    np.testing.assert_allclose(o, scipy.special.softmax(s, axis=1) @ v, atol=1e-13)
    np.testing.assert_allclose(lse, scipy.special.logsumexp(s, axis=1), atol=1e-13)
    # commutative
    o2, l2 = oracle.lse_merge(ob, lb, oa, la)
    np.testing.assert_allclose(o2, o, atol=1e-14)
    np.testing.assert_allclose(l2, lse, atol=1e-14)
    # associative over three parts
    c = [slice(0, 2), slice(2, 6), slice(6, 9)]
    p = [part(sl) for sl in c]
    left = oracle.lse_merge(*oracle.lse_merge(*p[0], *p[1]), *p[2])
    right = oracle.lse_merge(*p[0], *oracle.lse_merge(*p[1], *p[2]))
    np.testing.assert_allclose(left[0], right[0], atol=1e-13)
    np.testing.assert_allclose(left[1], right[1], atol=1e-13)
    # neutral element (o anything, lse = -inf), including both empty
    on, ln_ = oracle.lse_merge(oa, la, np.full_like(oa, 7.0), np.full(n, -np.inf))
    np.testing.assert_array_equal(on, oa)
    np.testing.assert_array_equal(ln_, la)
    oe, le = oracle.lse_merge(np.zeros((2, d)), np.full(2, -np.inf), np.zeros((2, d)), np.full(2, -np.inf))
    assert np.all(oe == 0) and np.all(np.isneginf(le))
    # the neutral element is neutral whatever output it carries (even NaN)
    junk = np.full_like(oa, np.nan)
    oj, lj = oracle.lse_merge(junk, np.full(n, -np.inf), ob, lb)
    np.testing.assert_array_equal(oj, ob)
    np.testing.assert_array_equal(lj, lb)
    oj2, lj2 = oracle.lse_merge(junk, np.full(n, -np.inf), junk, np.full(n, -np.inf))
    assert np.all(oj2 == 0) and np.all(np.isneginf(lj2))
    # large offsets do not overflow
    o3, l3 = oracle.lse_merge(oa, la + 800.0, ob, lb + 800.0)
    np.testing.assert_allclose(o3, o, atol=1e-12)
    np.testing.assert_allclose(l3, lse + 800.0, atol=1e-10)


# ---------------------------------------------------------------------------
# Gradients
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("causal", [False, True])
def test_backward_finite_differences(causal):
    B, H, N, d = 1, 1, 9, 5
    q, k, v = _rand((B, H, N, d), 29), _rand((B, H, N, d), 30), _rand((B, H, N, d), 31)
    do = _rand((B, H, N, d), 32)
    dq, dk, dv = oracle.attention_backward(q, k, v, do, causal)

    def loss(q_, k_, v_):
        return float((oracle.attention_forward(q_, k_, v_, causal)[0] * do).sum())

    eps = 1e-6
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            args_p = {"q": q, "k": k, "v": v}
            args_m = dict(args_p)
            args_p[name], args_m[name] = xp, xm
            num[idx] = (loss(**{f"{a}_": b for a, b in args_p.items()})
                        - loss(**{f"{a}_": b for a, b in args_m.items()})) / (2 * eps)
        err = np.abs(num - g).max() / max(1.0, np.abs(g).max())
        assert err < 1e-6, (name, err)


@pytest.mark.parametrize("causal", [False, True])
def test_backward_invariants(causal):
    B, H, N, d = 2, 2, 20, 6
    q, k, v = _rand((B, H, N, d), 33), _rand((B, H, N, d), 34), _rand((B, H, N, d), 35)
    do = _rand((B, H, N, d), 36)
    dq, dk, dv = oracle.attention_backward(q, k, v, do, causal)
    # adding one vector to every key shifts each score row by a constant:
    # the loss does not move, so the key gradients sum to zero
    np.testing.assert_allclose(dk.sum(axis=2), 0.0, atol=1e-12)
    # q -> a q, k -> k / a leaves every score unchanged
    np.testing.assert_allclose((q * dq).sum(axis=(2, 3)), (k * dk).sum(axis=(2, 3)), atol=1e-11)
    # upstream dO = 1 gives dv_j = column sums of the attention matrix
    ones = np.ones_like(do)
    _, _, dv1 = oracle.attention_backward(q, k, v, ones, causal)
    sc = 1 / math.sqrt(d)
    for b, h in itertools.product(range(B), range(H)):
        s = sc * q[b, h] @ k[b, h].T
        if causal:
            s = np.where(np.tril(np.ones((N, N), bool)), s, -np.inf)
        p = scipy.special.softmax(s, axis=1)
        np.testing.assert_allclose(dv1[b, h], np.repeat(p.sum(0)[:, None], d, 1), atol=1e-12)


# ---------------------------------------------------------------------------
# Sampled-row routines equal the full functions on the sample
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("causal", [False, True])
def test_sampled_rows(causal):
    B, H, N, d = 2, 3, 50, 8
    q, k, v = _rand((B, H, N, d), 37), _rand((B, H, N, d), 38), _rand((B, H, N, d), 39)
    do = _rand((B, H, N, d), 40)
    o, lse = oracle.attention_forward(q, k, v, causal)
    dq, dk, dv = oracle.attention_backward(q, k, v, do, causal)
    rng = np.random.default_rng(41)
    rows = np.stack([rng.integers(0, B, 20), rng.integers(0, H, 20), rng.integers(0, N, 20)], 1)
    rows[0] = (0, 0, 0)
    rows[1] = (1, 2, N - 1)
    o_r, l_r = oracle.attention_rows(q, k, v, rows, causal)
    o_h, l_h = oracle.attention_head_rows(q[1, 2, [3, 9]], k[1, 2], v[1, 2], [3, 9], causal)
    np.testing.assert_allclose(o_h, o[1, 2, [3, 9]], atol=1e-13)
    np.testing.assert_allclose(l_h, lse[1, 2, [3, 9]], atol=1e-13)
    np.testing.assert_allclose(o_r, o[rows[:, 0], rows[:, 1], rows[:, 2]], atol=1e-13)
    np.testing.assert_allclose(l_r, lse[rows[:, 0], rows[:, 1], rows[:, 2]], atol=1e-13)
    dq_r = oracle.attention_backward_query_rows(q, k, v, do, rows, causal)
    np.testing.assert_allclose(dq_r, dq[rows[:, 0], rows[:, 1], rows[:, 2]], atol=1e-12)
    keys = np.array([0, 3, 17, N - 1])
    dk_r, dv_r = oracle.attention_backward_key_rows(q, k, v, do, 1, 2, keys, causal, q_block=7)
    np.testing.assert_allclose(dk_r, dk[1, 2, keys], atol=1e-12)
    np.testing.assert_allclose(dv_r, dv[1, 2, keys], atol=1e-12)


# ---------------------------------------------------------------------------
# Feed-forward
# ---------------------------------------------------------------------------

def test_ffn_zero_cases_and_chunking():
    T, dm, dff = 24, 8, 12
    x = _rand((T, dm), 42)
    w1, w3 = _rand((dff, dm), 43), _rand((dff, dm), 44)
    w2 = _rand((dm, dff), 45)
    assert np.all(oracle.swiglu_ffn(np.zeros_like(x), w1, w2, w3) == 0)
    assert np.all(oracle.swiglu_ffn(x, w1, w2, np.zeros_like(w3)) == 0)
    y = oracle.swiglu_ffn(x, w1, w2, w3)
    for c in (1, 2, 3, 4, 6, 8, 12, 24):
        np.testing.assert_allclose(oracle.blockwise_ffn(x, w1, w2, w3, c), y, atol=1e-13)
    # explicit loops
    ref = np.zeros((T, dm))
    for t in range(T):
        h = []
        for f in range(dff):
            g = sum(x[t, a] * w1[f, a] for a in range(dm))
            u = sum(x[t, a] * w3[f, a] for a in range(dm))
            h.append(g / (1 + math.exp(-g)) * u)
        for a in range(dm):
            ref[t, a] = sum(h[f] * w2[a, f] for f in range(dff))
    np.testing.assert_allclose(y, ref, atol=1e-12)


def test_silu_matches_expit():
    z = np.linspace(-40, 40, 1001)
    np.testing.assert_allclose(oracle.silu(z), z * scipy.special.expit(z), rtol=1e-14, atol=1e-300)


def _ffn_case(T=5, dm=4, dff=6, seed=60, wscale=0.7):
    x = _rand((T, dm), seed)
    w1, w3 = _rand((dff, dm), seed + 1, wscale), _rand((dff, dm), seed + 2, wscale)
    w2 = _rand((dm, dff), seed + 3, wscale)
    dy = _rand((T, dm), seed + 4)
    return x, w1, w2, w3, dy


def test_ffn_backward_finite_differences():
    """Every entry of dx, dw1, dw2, dw3 against a central difference of
    sum(dy * y), y from the pinned forward."""
    x, w1, w2, w3, dy = _ffn_case()
    grads = oracle.swiglu_ffn_backward(x, w1, w2, w3, dy)
    args = [x, w1, w2, w3]
    eps = 1e-6
    for which, gi in zip((0, 1, 2, 3), grads):
        fd = np.empty_like(args[which])
        for idx in np.ndindex(*args[which].shape):
            plus = [a.copy() for a in args]
            minus = [a.copy() for a in args]
            plus[which][idx] += eps
            minus[which][idx] -= eps
            fd[idx] = (np.sum(dy * oracle.swiglu_ffn(*plus)) - np.sum(dy * oracle.swiglu_ffn(*minus))) / (2 * eps)
        np.testing.assert_allclose(gi, fd, rtol=1e-7, atol=1e-8)


def test_ffn_backward_zero_weight_closed_forms():
    x, w1, w2, w3, dy = _ffn_case(seed=70)
    # no up projection: h = 0, so only dw3 can be non-zero
    dx, dw1, dw2, dw3 = oracle.swiglu_ffn_backward(x, w1, w2, np.zeros_like(w3), dy)
    assert np.all(dx == 0) and np.all(dw1 == 0) and np.all(dw2 == 0) and np.abs(dw3).max() > 0.1
    # no down projection: dh = 0, so only dw2 can be non-zero
    dx, dw1, dw2, dw3 = oracle.swiglu_ffn_backward(x, w1, np.zeros_like(w2), w3, dy)
    assert np.all(dx == 0) and np.all(dw1 == 0) and np.all(dw3 == 0) and np.abs(dw2).max() > 0.1
    # zero input: g = u = h = 0 and every gradient vanishes (silu(0) = 0)
    for gr in oracle.swiglu_ffn_backward(np.zeros_like(x), w1, w2, w3, dy):
        assert np.all(gr == 0)
    # one token, one hidden unit, one feature: scalar calculus by hand
    # y = silu(a x) (b x) c; dy/dx = c b (silu(a x) + a x silu'(a x)) with
    # silu'(z) = expit(z) (1 + z (1 - expit(z)))
    a, b, c, xv = 0.8, -1.3, 0.6, 0.9
    z = a * xv
    sp = scipy.special.expit(z) * (1 + z * (1 - scipy.special.expit(z)))
    dx, dw1, dw2, dw3 = oracle.swiglu_ffn_backward(np.array([[xv]]), np.array([[a]]), np.array([[c]]),
                                                   np.array([[b]]), np.array([[1.0]]))
    silu_z = z * scipy.special.expit(z)
    assert math.isclose(dx[0, 0], c * b * (silu_z + a * xv * sp), rel_tol=1e-13)
    assert math.isclose(dw1[0, 0], c * b * xv * xv * sp, rel_tol=1e-13)
    assert math.isclose(dw2[0, 0], silu_z * b * xv, rel_tol=1e-13)
    assert math.isclose(dw3[0, 0], c * silu_z * xv, rel_tol=1e-13)


def test_ffn_backward_chunking_and_linearity():
    x, w1, w2, w3, dy = _ffn_case(T=24, dm=5, dff=7, seed=80)
    ref = oracle.swiglu_ffn_backward(x, w1, w2, w3, dy)
    for c in (1, 2, 3, 4, 6, 8, 12, 24):
        for a, b in zip(oracle.blockwise_ffn_backward(x, w1, w2, w3, dy, c), ref):
            np.testing.assert_allclose(a, b, atol=1e-12)
    dy2 = _rand(dy.shape, 81)
    g2 = oracle.swiglu_ffn_backward(x, w1, w2, w3, dy2)
    g12 = oracle.swiglu_ffn_backward(x, w1, w2, w3, 2.0 * dy - 3.0 * dy2)
    for a, b, c in zip(g12, ref, g2):
        np.testing.assert_allclose(a, 2.0 * b - 3.0 * c, atol=1e-12)
    # hidden units are independent: a subset of them has exactly the weight
    # gradients of those units in the full layer
    units = np.array([0, 3, 6])
    _, s1, s2, s3 = oracle.swiglu_ffn_backward(x, w1[units], w2[:, units], w3[units], dy)
    np.testing.assert_allclose(s1, ref[1][units], atol=1e-12)
    np.testing.assert_allclose(s2, ref[2][:, units], atol=1e-12)
    np.testing.assert_allclose(s3, ref[3][units], atol=1e-12)


def test_ffn_backward_terms_bound_gradients():
    x, w1, w2, w3, dy = _ffn_case(T=9, dm=5, dff=7, seed=90)
    for gr, tm in zip(oracle.swiglu_ffn_backward(x, w1, w2, w3, dy), oracle.swiglu_ffn_backward_terms(x, w1, w2, w3, dy)):
        assert np.all(np.abs(gr) <= tm + 1e-12) and np.all(tm > 0)
    # all inputs positive: every term is positive and the bound is attained
    pos = [np.abs(a) for a in (x, w1, w2, w3, dy)]
    for gr, tm in zip(oracle.swiglu_ffn_backward(*pos), oracle.swiglu_ffn_backward_terms(*pos)):
        np.testing.assert_allclose(gr, tm, rtol=1e-13)


# ---------------------------------------------------------------------------
# Grouped key/value heads
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("causal", [False, True])
def test_gqa_with_one_query_head_per_kv_head_is_plain(causal):
    B, H, N, d = 2, 3, 20, 8
    q, k, v, do = (_rand((B, H, N, d), 50 + i) for i in range(4))
    o1, l1 = oracle.attention_forward_gqa(q, k, v, causal)
    o2, l2 = oracle.attention_forward(q, k, v, causal)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)
    g1 = oracle.attention_backward_gqa(q, k, v, do, causal)
    g2 = oracle.attention_backward(q, k, v, do, causal)
    for a, b in zip(g1, g2):
        np.testing.assert_allclose(a, b, atol=1e-14)


def test_mqa_zero_queries_give_the_shared_mean():
    B, H, N, d = 1, 4, 15, 6
    q = np.zeros((B, H, N, d))
    k, v = _rand((B, 1, N, d), 60), _rand((B, 1, N, d), 61)
    o, lse = oracle.attention_forward_gqa(q, k, v, causal=False)
    np.testing.assert_allclose(o, np.broadcast_to(v.mean(axis=2, keepdims=True), o.shape), atol=1e-13)
    np.testing.assert_allclose(lse, np.log(N), atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_gqa_backward_finite_differences(causal):
    """dk, dv of a shared key/value head collect every query head's pull."""
    B, H, Hkv, N, d = 1, 4, 2, 6, 3
    q, do = _rand((B, H, N, d), 62), _rand((B, H, N, d), 63)
    k, v = _rand((B, Hkv, N, d), 64), _rand((B, Hkv, N, d), 65)
    dq, dk, dv = oracle.attention_backward_gqa(q, k, v, do, causal)

    def loss(k_, v_):
        return float((oracle.attention_forward_gqa(q, k_, v_, causal)[0] * do).sum())

    eps = 1e-6
    for x, g, is_k in ((k, dk, True), (v, dv, False)):
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            num[idx] = ((loss(xp, v) - loss(xm, v)) if is_k else (loss(k, xp) - loss(k, xm))) / (2 * eps)
        assert np.abs(num - g).max() / max(1.0, np.abs(g).max()) < 1e-6


def test_decode_is_the_last_causal_row():
    """A decode query at position N-1 equals row N-1 of causal attention over
    the same keys (reduction to the pinned full-matrix definition)."""
    B, H, Hkv, N, d = 2, 4, 2, 19, 8
    qfull = _rand((B, H, N, d), 70)
    k, v = _rand((B, Hkv, N, d), 71), _rand((B, Hkv, N, d), 72)
    o_full, l_full = oracle.attention_forward_gqa(qfull, k, v, causal=True)
    o, lse = oracle.attention_decode(qfull[:, :, N - 1], k, v)
    np.testing.assert_allclose(o, o_full[:, :, N - 1], atol=1e-13)
    np.testing.assert_allclose(lse, l_full[:, :, N - 1], atol=1e-13)


def test_decode_zero_query_gives_mean():
    B, H, N, d = 1, 2, 30, 4
    k, v = _rand((B, 1, N, d), 73), _rand((B, 1, N, d), 74)
    o, lse = oracle.attention_decode(np.zeros((B, H, d)), k, v)
    np.testing.assert_allclose(o, np.broadcast_to(v.mean(axis=2), o.shape), atol=1e-13)
    np.testing.assert_allclose(lse, np.log(N), atol=1e-13)


# ---------------------------------------------------------------------------
# RMS normalisation and the whole layer
# ---------------------------------------------------------------------------

def test_rmsnorm_closed_forms_and_gradient():
    x = _rand((6, 8), 300)
    y, r = oracle.rmsnorm(x, np.ones(8), 0.0)
    np.testing.assert_allclose(np.mean(y * y, axis=1), 1.0, rtol=1e-14)  # unit mean square
    y2, _ = oracle.rmsnorm(3.7 * x, np.ones(8), 0.0)
    np.testing.assert_allclose(y2, y, rtol=1e-13)                         # scale invariance
    c, eps = 0.3, 0.01
    yc, _ = oracle.rmsnorm(np.full((1, 8), c), np.arange(8.0), eps)       # constant row
    np.testing.assert_allclose(yc[0], c / math.sqrt(c * c + eps) * np.arange(8.0), rtol=1e-14)
    g = _rand(8, 301) + 1.0
    dout = _rand((6, 8), 302)
    dx, dg = oracle.rmsnorm_backward(x, g, dout, 1e-3)
    e = 1e-6
    for idx in np.ndindex(*x.shape):
        xp, xm = x.copy(), x.copy()
        xp[idx] += e
        xm[idx] -= e
        fd = (np.sum(dout * oracle.rmsnorm(xp, g, 1e-3)[0]) - np.sum(dout * oracle.rmsnorm(xm, g, 1e-3)[0])) / (2 * e)
        assert abs(fd - dx[idx]) <= 1e-7 * (1 + abs(fd))
    for j in range(8):
        gp, gm = g.copy(), g.copy()
        gp[j] += e
        gm[j] -= e
        fd = (np.sum(dout * oracle.rmsnorm(x, gp, 1e-3)[0]) - np.sum(dout * oracle.rmsnorm(x, gm, 1e-3)[0])) / (2 * e)
        assert abs(fd - dg[j]) <= 1e-7 * (1 + abs(fd))


def _layer_case(B=1, N=4, H=2, D=2, dff=3, seed=400, wscale=0.6):
    dm = H * D
    x = _rand((B * N, dm), seed)
    params = [1.0 + 0.2 * _rand(dm, seed + 1)] + [_rand((dm, dm), seed + 2 + i, wscale) for i in range(4)] + \
             [1.0 + 0.2 * _rand(dm, seed + 6), _rand((dff, dm), seed + 7, wscale), _rand((dm, dff), seed + 8, wscale),
              _rand((dff, dm), seed + 9, wscale)]
    dy = _rand((B * N, dm), seed + 10)
    return x, params, dy


@pytest.mark.parametrize("causal", [True, False])
def test_layer_backward_finite_differences(causal):
    """Every entry of dx and of all nine parameter gradients against a central
    difference of sum(dy * y) (two sequences, two heads)."""
    B, N, H, D = 2, 4, 2, 2
    x, params, dy = _layer_case(B, N, H, D)
    eps_n = 1e-3
    dx, grads = oracle.layer_backward(x, params, dy, B, N, H, D, causal, eps_n)

    def loss(xx, pp):
        return np.sum(dy * oracle.layer_forward(xx, pp, B, N, H, D, causal, eps_n)[0])

    e = 1e-6
    for idx in np.ndindex(*x.shape):
        xp, xm = x.copy(), x.copy()
        xp[idx] += e
        xm[idx] -= e
        fd = (loss(xp, params) - loss(xm, params)) / (2 * e)
        assert abs(fd - dx[idx]) <= 1e-6 * (1 + abs(fd)), ("x", idx)
    for pi, gr in enumerate(grads):
        for idx in np.ndindex(*params[pi].shape):
            pp = [p.copy() for p in params]
            pm = [p.copy() for p in params]
            pp[pi][idx] += e
            pm[pi][idx] -= e
            fd = (loss(x, pp) - loss(x, pm)) / (2 * e)
            assert abs(fd - gr[idx]) <= 1e-6 * (1 + abs(fd)), (oracle.PARAM_NAMES[pi], idx)


def test_layer_zero_output_projections_is_identity():
    """wo = 0 and w2 = 0 switch both branches off: y = x and dx = dy."""
    B, N, H, D = 1, 6, 2, 2
    x, params, dy = _layer_case(B, N, H, D, seed=420)
    params[4] = np.zeros_like(params[4])
    params[7] = np.zeros_like(params[7])
    y, _ = oracle.layer_forward(x, params, B, N, H, D)
    assert np.array_equal(y, x)
    dx, grads = oracle.layer_backward(x, params, dy, B, N, H, D)
    np.testing.assert_allclose(dx, dy, atol=1e-15)
    assert np.abs(grads[4]).max() > 0.01 and np.abs(grads[7]).max() > 0.01  # dwo, dw2 still flow
    for i in (0, 1, 2, 3, 5, 6, 8):
        assert np.all(grads[i] == 0), oracle.PARAM_NAMES[i]


def test_layer_causal_locality_and_batch_independence():
    B, N, H, D = 2, 6, 2, 2
    x, params, _ = _layer_case(B, N, H, D, seed=440)
    y, _ = oracle.layer_forward(x, params, B, N, H, D, causal=True)
    xp = x.copy()
    xp[4:6] += 5.0                   # later tokens of sequence 0
    yp, _ = oracle.layer_forward(xp, params, B, N, H, D, causal=True)
    np.testing.assert_allclose(yp[:4], y[:4], atol=1e-13)
    np.testing.assert_allclose(yp[6:], y[6:], atol=1e-13)   # the other sequence
    assert np.abs(yp[4:6] - y[4:6]).max() > 0.1

