"""ringattn_step_host: a forward + backward step on host buffers, every copy
inside the C call, must give the same results as the device-path calls
(forward, lse, dk, dv to the bit; dq up to the fp32 summation order of the
fused backward), also over several steps that use two device buffer sets in
turn with the consumed and done events guarding their reuse."""

import pytest
import torch

from exact_blockwise_long_b200.synthetic import small_attention_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from exact_blockwise_long_b200 import build
    build.build()
    torch.cuda.set_device(0)


def _close(a, b):
    a, b = a.float(), b.float()
    return bool(((a - b).abs() <= 2.0 ** -7 * torch.maximum(a.abs(), b.abs()) + 1e-5).all())


@pytest.mark.parametrize("D,S,qc,kc,causal", [(128, 4, 128, 256, True), (64, 2, 128, 128, False)])
def test_host_step_matches_device_path(D, S, qc, kc, causal):
    import exact_blockwise_long_b200 as ra
    B, H, N = 2, 2, 1024
    steps = []
    for seed in (11, 12, 13):  # three steps with different inputs
        q, k, v, do = small_attention_inputs(B, H, N, D, seed + D, k_scale=2.0)
        o = torch.empty_like(q)
        lse = torch.empty((B, H, N), device="cuda", dtype=torch.float32)
        ra.ringattn_fwd(q, k, v, o, lse, S, qc, kc, causal)
        ws = torch.empty(ra.ringattn_bwd_workspace_size(B, H, N, D), device="cuda", dtype=torch.uint8)
        g = [torch.empty_like(q) for _ in range(3)]
        ra.ringattn_bwd(q, k, v, o, lse, do, *g, S, qc, kc, causal, ws)
        steps.append(([t.cpu().pin_memory() for t in (q, k, v, do)], [o.cpu(), lse.cpu()] + [t.cpu() for t in g]))
    torch.cuda.synchronize()
    devs = [torch.empty(ra.ringattn_step_host_size(B, H, N, D), device="cuda", dtype=torch.uint8) for _ in range(2)]
    outs = [[torch.full(t.shape, float("nan"), dtype=t.dtype).pin_memory() for t in steps[0][1]] for _ in steps]
    cs, s_in, s_out = torch.cuda.current_stream(), torch.cuda.Stream(), torch.cuda.Stream()
    done = [torch.cuda.Event(), torch.cuda.Event()]
    consumed = [torch.cuda.Event(), torch.cuda.Event()]
    for j, (hin, _) in enumerate(steps):
        bi = j % 2
        ra.ringattn_step_host(*hin, *outs[j], devs[bi], S, qc, kc, causal, cs, s_in, s_out,
                              inputs_free_event=consumed[bi] if j >= 2 else None,
                              outputs_free_event=done[bi] if j >= 2 else None,
                              consumed_event=consumed[bi], done_event=done[bi])
    for e in done:
        e.synchronize()
    assert ra.ringattn_get_error() == 0
    for (_, ref), got in zip(steps, outs):
        o_r, l_r, dq_r, dk_r, dv_r = ref
        o_g, l_g, dq_g, dk_g, dv_g = got
        assert torch.equal(o_g, o_r) and torch.equal(l_g, l_r)
        assert torch.equal(dk_g, dk_r) and torch.equal(dv_g, dv_r)
        assert _close(dq_g, dq_r)


def test_host_step_rejects_bad_arguments():
    import exact_blockwise_long_b200 as ra
    L = ra.lib()
    B, H, N, D = 1, 1, 256, 128
    need = L.ringattn_step_host_size(B, H, N, D)
    assert need > 0 and L.ringattn_step_host_size(0, H, N, D) == 0
    h = [0x10000] * 9
    dev = torch.empty(need, device="cuda", dtype=torch.uint8)
    base = [B, H, N, D, 0, 2, 128, 128, 1, 0.0] + [None] * 7
    assert L.ringattn_step_host(*h, dev.data_ptr(), need - 1, *base) == -8         # device buffer too small
    assert L.ringattn_step_host(*h, None, need, *base) == -8                       # device buffer missing
    assert L.ringattn_step_host(*([None] + h[1:]), dev.data_ptr(), need, *base) == -1
    assert L.ringattn_step_host(*h, dev.data_ptr(), need, *(base[:4] + [1] + base[5:])) == -5  # fp32
