"""The bounds-checked build (libringattn_checked.so, -DRA_CHECKED): every
tile and row index of the attention kernels is checked against its tensor
before the access, and a failed check latches RA_ERR_BOUNDS in the device
status word instead of making the access.  Run over small parity cases of
every attention entry point, the checked build must leave the status word
clear and give the unchecked build's bits (dq of the fused backward: up to
its fp32 summation order).  This is the race and bounds net that stands in
for compute-sanitizer, which is closed on this machine."""

import ctypes

import pytest
import torch

from exact_blockwise_long_b200.synthetic import small_attention_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def libs():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from exact_blockwise_long_b200 import _lib, build
    build.build()
    build.build(checked=True)
    torch.cuda.set_device(0)
    return _lib.lib(), _lib.load(_lib.CHECKED_LIB_PATH)


def _p(*ts):
    return [t.data_ptr() for t in ts]


def _fwd(L, q, k, v, S, qc, kc, causal, st):
    B, H, N, D = q.shape
    o = torch.full_like(q, float("nan"))
    lse = torch.full((B, H, N), float("nan"), device="cuda")
    dt = 0 if q.dtype == torch.bfloat16 else 1
    assert L.ringattn_fwd_gqa(*_p(q, k, v, o, lse), B, H, int(k.shape[1]), N, D, dt, S, qc, kc, causal, 0.0,
                              st) == 0
    return o, lse


def _bwd(L, q, k, v, o, lse, do, S, qc, kc, causal, mask, st):
    B, H, N, D = q.shape
    ws = torch.empty(L.ringattn_bwd_workspace_size(B, H, N, D), device="cuda", dtype=torch.uint8)
    g = [torch.full_like(t, float("nan")) for t in (q, k, v)]
    if mask is None:
        rc = L.ringattn_bwd_gqa(*_p(q, k, v, o, lse, do, *g), B, H, int(k.shape[1]), N, D, 0, S, qc, kc, causal,
                                0.0, ws.data_ptr(), ws.numel(), st)
    else:
        rc = L.ringattn_bwd_phase(*_p(q, k, v, o, lse, do, *g), B, H, N, D, 0, S, qc, kc, causal, 0.0,
                                  ws.data_ptr(), ws.numel(), mask, st)
    assert rc == 0
    return g


def _close(a, b):
    a, b = a.float(), b.float()
    return bool(((a - b).abs() <= 2.0 ** -7 * torch.maximum(a.abs(), b.abs()) + 1e-5).all())


CASES = [
    # (B, H, Hkv, N, D, S, qc, kc, causal)
    (1, 2, 2, 1024, 128, 4, 128, 256, 1),   # two-tile forward, fused backward
    (1, 2, 2, 640, 128, 5, 128, 128, 1),    # one-tile forward (shard of 128)
    (2, 2, 2, 768, 64, 3, 128, 256, 0),     # d = 64: fused backward, TMA-reduced dQ
    (1, 4, 1, 512, 128, 2, 256, 128, 1),    # MQA
]


@pytest.mark.parametrize("B,H,Hkv,N,D,S,qc,kc,causal", CASES)
def test_checked_build_is_clean_and_identical(libs, B, H, Hkv, N, D, S, qc, kc, causal):
    plain, checked = libs
    st = torch.cuda.current_stream().cuda_stream
    q, k, v, do = small_attention_inputs(B, H, N, D, 900 + N + D, k_scale=2.0, Hkv=Hkv)
    o1, l1 = _fwd(plain, q, k, v, S, qc, kc, causal, st)
    o2, l2 = _fwd(checked, q, k, v, S, qc, kc, causal, st)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    for mask in (None, 7) if Hkv == H else (None,):
        g1 = _bwd(plain, q, k, v, o1, l1, do, S, qc, kc, causal, mask, st)
        g2 = _bwd(checked, q, k, v, o1, l1, do, S, qc, kc, causal, mask, st)
        assert torch.equal(g1[1], g2[1]) and torch.equal(g1[2], g2[2])
        assert torch.equal(g1[0], g2[0]) if mask == 7 else _close(g1[0], g2[0])
    assert checked.ringattn_get_error(ctypes.c_void_p(st)) == 0
    assert plain.ringattn_get_error(ctypes.c_void_p(st)) == 0


def test_checked_build_pair_and_merge(libs):
    """The per-pair backward and the standalone merge through the checked build."""
    plain, checked = libs
    st = torch.cuda.current_stream().cuda_stream
    B, H, N, D = 1, 2, 512, 128
    q, k, v, do = small_attention_inputs(B, H, N, D, 931, k_scale=2.0)
    o, lse = _fwd(plain, q, k, v, 1, 128, 128, 1, st)
    outs = []
    for L in (plain, checked):
        prep = torch.empty(L.ringattn_bwd_prepare_size(B, H, N), device="cuda", dtype=torch.uint8)
        assert L.ringattn_bwd_prepare(*_p(o, lse, do, prep), prep.numel(), B, H, N, D, 0, st) == 0
        acc = [torch.zeros((B, H, N, D), device="cuda") for _ in range(3)]
        assert L.ringattn_bwd_pair(*_p(q, k, v, do, prep, *acc), B, H, N, D, 0, 128, 128, 1, 0.0, 0, st) == 0
        oa = torch.randn((1000, D), device="cuda", generator=torch.Generator("cuda").manual_seed(5))
        la = torch.randn(1000, device="cuda", generator=torch.Generator("cuda").manual_seed(6))
        ob, lb = oa.flip(0).contiguous(), la.flip(0).contiguous()
        assert L.ringattn_merge(*_p(oa, la, ob, lb), 1000, D, st) == 0
        outs.append(acc + [oa, la])
    a, b = outs
    assert _close(a[0], b[0]) and all(torch.equal(x, y) for x, y in zip(a[1:], b[1:]))
    assert checked.ringattn_get_error(ctypes.c_void_p(st)) == 0
