"""GPU parity of the ring forward (fp32 CUDA-core path and bf16 tcgen05 path),
the fused ring-step + merge mode and the standalone merge kernel, against
the fp64 oracle on the same seeded input bits."""


import numpy as np
import pytest
import torch

import oracle
from exact_blockwise_long_b200.synthetic import (WORKLOADS, attention_inputs, sample_rows,
                                                 small_attention_inputs, to_f64)
from helpers import TOL_BF16_LSE, TOL_BF16_O, TOL_F32, check_rows, max_abs, run_fwd

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


def full_oracle(q, k, v, causal):
    return oracle.attention_forward(to_f64(q), to_f64(k), to_f64(v), causal)


# ---------------------------------------------------------------------------
# fp32 path (tiny exact workload and variants), tolerance 1e-4
# ---------------------------------------------------------------------------

def test_tiny_f32_workload():
    w = WORKLOADS["tiny_f32"]
    q, k, v, _ = attention_inputs(w)
    o, lse = run_fwd(q, k, v, w.S, w.q_chunk, w.k_chunk, w.causal)
    o_ref, l_ref = full_oracle(q, k, v, w.causal)
    assert max_abs(to_f64(o), o_ref) <= TOL_F32
    assert max_abs(to_f64(lse), l_ref) <= TOL_F32


@pytest.mark.parametrize("D,causal,S,qc,kc", [
    (64, False, 4, 64, 64), (128, True, 2, 128, 64), (128, False, 1, 256, 256),
    (64, True, 8, 64, 64), (128, True, 4, 64, 128),
])
def test_f32_variants(D, causal, S, qc, kc):
    q, k, v, _ = small_attention_inputs(2, 2, 256 * (2 if S == 8 else 1) * (1 if S < 4 else 2), D, 5,
                                        dtype=torch.float32)
    o, lse = run_fwd(q, k, v, S, qc, kc, causal)
    o_ref, l_ref = full_oracle(q, k, v, causal)
    assert max_abs(to_f64(o), o_ref) <= TOL_F32
    assert max_abs(to_f64(lse), l_ref) <= TOL_F32


# ---------------------------------------------------------------------------
# bf16 tcgen05 path: full oracle at small sizes spanning many tiles
# ---------------------------------------------------------------------------

BF16_CASES = [
    # (B, H, N, D, S, qc, kc, causal)
    (1, 2, 1024, 128, 4, 128, 128, True),
    (1, 2, 1024, 128, 4, 128, 256, False),
    (2, 1, 1024, 64, 2, 256, 128, True),
    (1, 3, 768, 64, 3, 128, 256, False),
    (1, 1, 128, 128, 1, 128, 128, True),    # a single tile
    (1, 1, 2048, 128, 16, 128, 128, True),  # one tile per shard
    (1, 2, 1536, 64, 1, 512, 1536, True),   # no ring (S = 1), one big chunk
    (1, 1, 2048, 128, 8, 256, 128, False),
]


@pytest.mark.parametrize("B,H,N,D,S,qc,kc,causal", BF16_CASES)
def test_bf16_full_oracle(B, H, N, D, S, qc, kc, causal):
    q, k, v, _ = small_attention_inputs(B, H, N, D, 11 + N + D + S, k_scale=2.0 if causal else 1.0)
    o, lse = run_fwd(q, k, v, S, qc, kc, causal)
    o_ref, l_ref = full_oracle(q, k, v, causal)
    e_o, e_l = max_abs(to_f64(o), o_ref), max_abs(to_f64(lse), l_ref)
    assert e_o <= TOL_BF16_O, e_o
    assert e_l <= TOL_BF16_LSE, e_l


def test_bf16_sharp_softmax_rescale_path():
    """Large, growing scores force many online-softmax rescales."""
    B, H, N, D = 1, 2, 1024, 128
    q, k, v, _ = small_attention_inputs(B, H, N, D, 99)
    ramp = torch.linspace(0.5, 6.0, N, device="cuda")[None, None, :, None]
    k = (k.float() * ramp).to(torch.bfloat16)
    o, lse = run_fwd(q, k, v, 4, 128, 128, True)
    o_ref, l_ref = full_oracle(q, k, v, True)
    assert max_abs(to_f64(o), o_ref) <= TOL_BF16_O
    assert max_abs(to_f64(lse), l_ref) <= TOL_BF16_LSE


def test_bf16_deterministic():
    """Race check by repetition: a missing wait would show up as run-to-run
    differences, so twenty runs must give identical bits."""
    q, k, v, _ = small_attention_inputs(1, 4, 2048, 128, 7)
    o1, l1 = run_fwd(q, k, v, 4, 256, 256, True)
    for _ in range(20):
        o2, l2 = run_fwd(q, k, v, 4, 256, 256, True)
        assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_bf16_chunk_and_shard_invariance():
    """Same inputs, different S and chunk sizes: the same exact result up to
    fp32 summation order."""
    q, k, v, _ = small_attention_inputs(1, 2, 2048, 64, 8)
    ref, lref = run_fwd(q, k, v, 1, 2048, 2048, True)
    for S, qc, kc in [(2, 512, 1024), (4, 128, 512), (16, 128, 128)]:
        o, lse = run_fwd(q, k, v, S, qc, kc, True)
        assert (o.float() - ref.float()).abs().max().item() <= 1e-2
        assert (lse - lref).abs().max().item() <= 1e-3


# ---------------------------------------------------------------------------
# ring-step mode with the fused merge, and the standalone merge kernel
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("dtype,tol", [(torch.bfloat16, TOL_BF16_O), (torch.float32, TOL_F32)])
@pytest.mark.parametrize("causal", [True, False])
def test_step_mode_any_order(dtype, tol, causal):
    import exact_blockwise_long_b200 as ra
    B, H, N, D, S = 1, 2, 1024, 128, 4
    q, k, v, _ = small_attention_inputs(B, H, N, D, 21, dtype=dtype)
    o_ref, l_ref = full_oracle(q, k, v, causal)
    for order in ([0, 1, 2, 3], [2, 0, 3, 1]):
        o_acc = torch.zeros((B, H, N, D), device="cuda", dtype=torch.float32)
        l_acc = torch.full((B, H, N), float("-inf"), device="cuda", dtype=torch.float32)
        for t in order:
            ra.ringattn_fwd_step(q, k, v, o_acc, l_acc, S, 128, 128, causal, t)
        assert ra.ringattn_get_error() == 0
        assert max_abs(to_f64(o_acc), o_ref) <= tol
        assert max_abs(to_f64(l_acc), l_ref) <= (tol if dtype == torch.float32 else TOL_BF16_LSE)


def test_step_partials_match_oracle_step():
    """One step into a neutral accumulator gives that step's partial."""
    import exact_blockwise_long_b200 as ra
    B, H, N, D, S = 1, 1, 512, 64, 4
    q, k, v, _ = small_attention_inputs(B, H, N, D, 23)
    for t in range(S):
        o_acc = torch.zeros((B, H, N, D), device="cuda")
        l_acc = torch.full((B, H, N), float("-inf"), device="cuda")
        ra.ringattn_fwd_step(q, k, v, o_acc, l_acc, S, 128, 128, True, t)
        o_t, l_t = oracle.ring_blockwise_step(to_f64(q), to_f64(k), to_f64(v), S, t, True)
        fin = np.isfinite(l_t)
        assert np.array_equal(np.isfinite(to_f64(l_acc)), fin)
        assert max_abs(to_f64(o_acc)[fin], o_t[fin]) <= TOL_BF16_O
        assert max_abs(to_f64(l_acc)[fin], l_t[fin]) <= TOL_BF16_LSE
        assert np.all(to_f64(o_acc)[~fin] == 0)


def test_merge_kernel():
    import exact_blockwise_long_b200 as ra
    g = torch.Generator(device="cuda").manual_seed(31)
    rows, D = 10007, 128
    o_a = torch.randn((rows, D), generator=g, device="cuda")
    o_b = torch.randn((rows, D), generator=g, device="cuda")
    l_a = torch.randn((rows,), generator=g, device="cuda") * 5
    l_b = torch.randn((rows,), generator=g, device="cuda") * 5
    l_a[::7] = float("-inf")
    l_b[::11] = float("-inf")
    o_a[::7] = float("nan")  # (-inf, anything) is neutral
    ref_o, ref_l = oracle.lse_merge(to_f64(o_a), to_f64(l_a), to_f64(o_b), to_f64(l_b))
    ra.ringattn_merge(o_a, l_a, o_b, l_b)
    assert ra.ringattn_get_error() == 0
    got_o, got_l = to_f64(o_a), to_f64(l_a)
    assert np.array_equal(np.isneginf(got_l), np.isneginf(ref_l))
    fin = np.isfinite(ref_l)
    assert max_abs(got_l[fin], ref_l[fin]) <= 1e-5
    assert not np.isnan(got_o).any()
    assert max_abs(got_o, ref_o) <= 1e-5


# ---------------------------------------------------------------------------
# Full-size workloads: sampled rows against fp64 brute force
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("name", ["n8k_d64_causal", "n8k_d64_full", "n32k_d128"])
def test_workload_sampled_rows(name):
    w = WORKLOADS[name]
    q, k, v, _ = attention_inputs(w, with_dout=False)
    o, lse = run_fwd(q, k, v, w.S, w.q_chunk, w.k_chunk, w.causal)
    rows = sample_rows(w.B, w.H, w.N, 256, w.seed)
    e_o, e_l = check_rows(q, k, v, o, lse, rows, w.causal)
    assert e_o <= TOL_BF16_O, e_o
    assert e_l <= TOL_BF16_LSE, e_l


def test_workload_n8k_full_oracle_two_heads():
    w = WORKLOADS["n8k_d64_causal"]
    q, k, v, _ = attention_inputs(w, with_dout=False)
    o, lse = run_fwd(q, k, v, w.S, w.q_chunk, w.k_chunk, w.causal)
    for b, h in [(0, 0), (1, 15)]:
        o_ref, l_ref = oracle.attention_forward(to_f64(q[b:b + 1, h:h + 1]), to_f64(k[b:b + 1, h:h + 1]),
                                                to_f64(v[b:b + 1, h:h + 1]), True)
        assert max_abs(to_f64(o[b:b + 1, h:h + 1]), o_ref) <= TOL_BF16_O
        assert max_abs(to_f64(lse[b:b + 1, h:h + 1]), l_ref) <= TOL_BF16_LSE


@pytest.mark.slow
def test_workload_million_tokens_sampled_rows():
    w = WORKLOADS["n1m_d128"]
    q, k, v, _ = attention_inputs(w, with_dout=False)
    o, lse = run_fwd(q, k, v, w.S, w.q_chunk, w.k_chunk, w.causal)
    rows = sample_rows(w.B, w.H, w.N, 256, w.seed)
    e_o, e_l = check_rows(q, k, v, o, lse, rows, w.causal)
    del q, k, v, o, lse
    torch.cuda.empty_cache()
    assert e_o <= TOL_BF16_O, e_o
    assert e_l <= TOL_BF16_LSE, e_l


# ---------------------------------------------------------------------------
# Bounded waits: a wait that nothing satisfies ends with a status, not a hang
# ---------------------------------------------------------------------------

def test_bounded_wait_reports_timeout():
    import exact_blockwise_long_b200 as ra
    assert ra.ringattn_get_error() == 0
    ra.ringattn_selftest_timeout(20000)          # 20 ms
    assert ra.ringattn_get_error() == -7         # RA_ERR_TIMEOUT, read and cleared
    assert ra.ringattn_get_error() == 0
    q, k, v, _ = small_attention_inputs(1, 1, 256, 64, 3)
    run_fwd(q, k, v, 2, 128, 128, True)          # the context is still usable
