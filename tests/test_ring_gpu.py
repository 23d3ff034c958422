"""GPU checks of the multi-device ring's per-pair work (ring.DeviceOps) and
of the accumulate / cast kernels.  One GPU only: the ring's ranks are
emulated one after another in this process (no rank waits on another), or
run as a process group of one."""

import pytest
import torch

import oracle
from exact_blockwise_long_b200.synthetic import small_attention_inputs, to_f64
from helpers import TOL_BF16_GRAD, TOL_BF16_LSE, TOL_BF16_O, max_abs

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


def test_accumulate_and_cast_are_exact():
    import exact_blockwise_long_b200 as ra
    g = torch.Generator(device="cuda").manual_seed(3)
    for n in (0, 5, 4096, 100003):
        acc = torch.randn(n, generator=g, device="cuda")
        xb = torch.randn(n, generator=g, device="cuda").to(torch.bfloat16)
        xf = torch.randn(n, generator=g, device="cuda")
        ref = (acc + xb.float()) + xf
        ra.ringattn_accumulate(acc, xb)
        ra.ringattn_accumulate(acc, xf)
        assert torch.equal(acc, ref)
        out = torch.empty(n, device="cuda", dtype=torch.bfloat16)
        ra.ringattn_cast(acc, out)
        assert torch.equal(out, acc.to(torch.bfloat16))  # round to nearest even, like torch
    assert ra.ringattn_get_error() == 0


@pytest.mark.parametrize("S,causal,D", [(3, True, 128), (4, True, 128), (2, False, 128), (3, True, 64), (2, False, 64)])
def test_device_ops_over_an_emulated_ring(S, causal, D):
    """Each rank's schedule run in turn on one GPU: shard pairs in ring
    order with the causal skip and diagonal mask, exact merge, gradients
    summed per pair -- equal to full-sequence attention."""
    from exact_blockwise_long_b200.ring import DeviceOps
    B, H, L = 1, 2, 512
    N = S * L
    q, k, v, do = small_attention_inputs(B, H, N, D, 40 + S + D, k_scale=2.0 if causal else 1.0)
    ops = DeviceOps(128, 256)
    sh = lambda t, i: t[:, :, i * L:(i + 1) * L].contiguous()  # noqa: E731
    outs, lses = [], []
    for i in range(S):
        o_acc = torch.zeros((B, H, L, D), device="cuda", dtype=torch.float32)
        lse_acc = torch.full((B, H, L), float("-inf"), device="cuda", dtype=torch.float32)
        for t in range(S):
            j = (i - t) % S
            if not (causal and j > i):
                ops.fwd_pair(sh(q, i), sh(k, j), sh(v, j), o_acc, lse_acc, causal and j == i)
        o = torch.empty((B, H, L, D), device="cuda", dtype=torch.bfloat16)
        ops.cast(o_acc, o)
        outs.append(o)
        lses.append(lse_acc)
    out, lse = torch.cat(outs, 2), torch.cat(lses, 2)
    o_ref, l_ref = oracle.attention_forward(to_f64(q), to_f64(k), to_f64(v), causal)
    assert max_abs(to_f64(out), o_ref) <= TOL_BF16_O
    assert max_abs(to_f64(lse), l_ref) <= TOL_BF16_LSE

    f32 = dict(device="cuda", dtype=torch.float32)
    dq = [torch.zeros((B, H, L, D), **f32) for _ in range(S)]
    dk = [torch.zeros((B, H, L, D), **f32) for _ in range(S)]
    dv = [torch.zeros((B, H, L, D), **f32) for _ in range(S)]
    pk, pv = (torch.empty((B, H, L, D), **f32) for _ in range(2))
    for i in range(S):
        prep = ops.bwd_prepare(sh(out, i), sh(lse, i), sh(do, i))
        for t in range(S):
            j = (i - t) % S
            if causal and j > i:
                continue
            ops.bwd_pair(sh(q, i), sh(k, j), sh(v, j), sh(do, i), prep, dq[i], pk, pv, causal and j == i)
            ops.accumulate(dk[j], pk)
            ops.accumulate(dv[j], pv)
    gq, gk, gv = oracle.attention_backward(to_f64(q), to_f64(k), to_f64(v), to_f64(do), causal)
    for got, ref in ((dq, gq), (dk, gk), (dv, gv)):
        assert max_abs(to_f64(torch.cat(got, 2)), ref) <= TOL_BF16_GRAD
    import exact_blockwise_long_b200 as ra
    assert ra.ringattn_get_error() == 0


@pytest.mark.parametrize("D", [128, 64])
def test_pair_over_whole_sequence_equals_backward(D):
    """One diagonal pair over the whole sequence is the whole backward: its
    fp32 dk, dv round to ringattn_bwd's bf16 bits (same matmuls, same order),
    dq agrees up to fp32 summation order; kv_accumulate adds onto dk, dv."""
    import exact_blockwise_long_b200 as ra
    B, H, N = 1, 2, 1024
    q, k, v, do = small_attention_inputs(B, H, N, D, 61 + D, k_scale=2.0)
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), device="cuda", dtype=torch.float32)
    ra.ringattn_fwd(q, k, v, o, lse, 1, 128, 256, True)
    ws = torch.empty(ra.ringattn_bwd_workspace_size(B, H, N, D), device="cuda", dtype=torch.uint8)
    ref = [torch.empty_like(q) for _ in range(3)]
    ra.ringattn_bwd(q, k, v, o, lse, do, *ref, 1, 128, 256, True, ws)
    prep = torch.empty(ra.ringattn_bwd_prepare_size(B, H, N), device="cuda", dtype=torch.uint8)
    ra.ringattn_bwd_prepare(o, lse, do, prep)
    f32 = dict(device="cuda", dtype=torch.float32)
    dq_acc = torch.zeros((B, H, N, D), **f32)
    dk_acc, dv_acc = (torch.full((B, H, N, D), float("nan"), **f32) for _ in range(2))
    ra.ringattn_bwd_pair(q, k, v, do, prep, dq_acc, dk_acc, dv_acc, 128, 256, True)
    assert ra.ringattn_get_error() == 0
    assert torch.equal(dk_acc.to(torch.bfloat16), ref[1]) and torch.equal(dv_acc.to(torch.bfloat16), ref[2])
    a, b = dq_acc.to(torch.bfloat16).float(), ref[0].float()
    assert bool(((a - b).abs() <= 2.0 ** -7 * torch.maximum(a.abs(), b.abs()) + 1e-5).all())
    # the second call adds the same shares again: dq and (with kv_accumulate) dk, dv double
    dk1, dv1, dq1 = dk_acc.clone(), dv_acc.clone(), dq_acc.clone()
    ra.ringattn_bwd_pair(q, k, v, do, prep, dq_acc, dk_acc, dv_acc, 128, 256, True, kv_accumulate=True)
    assert torch.equal(dk_acc, 2 * dk1) and torch.equal(dv_acc, 2 * dv1)
    assert torch.allclose(dq_acc, 2 * dq1, rtol=1e-5, atol=1e-6)
    assert ra.ringattn_get_error() == 0


def test_ring_driver_with_one_rank():
    """The driver itself over NCCL with a group of one (no transfers)."""
    import os
    import socket
    import torch.distributed as dist
    from exact_blockwise_long_b200 import ring
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda", 0))
    try:
        q, k, v, do = small_attention_inputs(1, 2, 1024, 128, 51)
        out, lse = ring.ring_attention_forward(q, k, v, True, q_chunk=128, k_chunk=128)
        dq, dk, dv = ring.ring_attention_backward(q, k, v, out, lse, do, True, q_chunk=128, k_chunk=128)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    o_ref, l_ref = oracle.attention_forward(to_f64(q), to_f64(k), to_f64(v), True)
    gq, gk, gv = oracle.attention_backward(to_f64(q), to_f64(k), to_f64(v), to_f64(do), True)
    assert max_abs(to_f64(out), o_ref) <= TOL_BF16_O
    assert max_abs(to_f64(lse), l_ref) <= TOL_BF16_LSE
    for got, ref in ((dq, gq), (dk, gk), (dv, gv)):
        assert max_abs(to_f64(got), ref) <= TOL_BF16_GRAD
