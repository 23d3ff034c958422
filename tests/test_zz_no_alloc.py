"""ringattn_bwd_noalloc: the backward for callers that cannot allocate device
memory (a framework-owned allocator, a fixed start-up memory budget, or a hot
path that must not call cudaMalloc).  It must give the same gradients as
ringattn_bwd with a caller workspace, on consecutive calls that reuse its one
static scratch array, and refuse problems larger than that array.

This file is collected last on purpose: it runs after every other test, and
it also passes on its own in a fresh process."""


import pytest
import torch

from exact_blockwise_long_b200.synthetic import small_attention_inputs
from helpers import TOL_BF16_GRAD

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def L():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from exact_blockwise_long_b200 import build
    build.build()
    from exact_blockwise_long_b200 import _lib
    torch.cuda.set_device(0)
    return _lib.lib()


def _ptrs(*ts):
    return [t.data_ptr() for t in ts]


def _bwd_with_workspace(L, q, k, v, o, lse, do, cfg, stream):
    B, H, N, D = q.shape
    ws = torch.empty(L.ringattn_bwd_workspace_size(B, H, N, D), device="cuda", dtype=torch.uint8)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    rc = L.ringattn_bwd(*_ptrs(q, k, v, o, lse, do, dq, dk, dv), B, H, N, D, 0, *cfg, 0.0,
                        ws.data_ptr(), ws.numel(), stream)
    assert rc == 0
    return dq, dk, dv


@pytest.mark.parametrize("B,H,N,D,S,qc,kc,causal", [
    (1, 2, 1024, 128, 4, 128, 256, True),
    (2, 2, 768, 64, 3, 128, 128, False),
])
def test_noalloc_matches_workspace_backward_twice(L, B, H, N, D, S, qc, kc, causal):
    q, k, v, do = small_attention_inputs(B, H, N, D, 77 + N)
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), device="cuda", dtype=torch.float32)
    stream = torch.cuda.current_stream().cuda_stream
    cfg = (S, qc, kc, int(causal))
    assert L.ringattn_fwd(*_ptrs(q, k, v, o, lse), B, H, N, D, 0, *cfg, 0.0, stream) == 0
    ref = _bwd_with_workspace(L, q, k, v, o, lse, do, cfg, stream)
    for _ in range(2):  # the second call finds the first call's scratch contents
        got = [torch.full_like(q, float("nan")) for _ in range(3)]
        rc = L.ringattn_bwd_noalloc(*_ptrs(q, k, v, o, lse, do, *got), B, H, N, D, 0, *cfg, 0.0, stream)
        assert rc == 0
        assert L.ringattn_get_error(stream) == 0
        for a, b in zip(got, ref):
            assert (a.float() - b.float()).abs().max().item() <= TOL_BF16_GRAD


def test_noalloc_rejects_problems_beyond_its_scratch(L):
    limit = 64 << 20
    B, H, N, D = 4, 32, 131072, 128        # needs about 134 MB of scratch
    assert L.ringattn_bwd_workspace_size(B, H, N, D) > limit
    fake = [0x10000] * 9                   # never touched: the size check comes first
    rc = L.ringattn_bwd_noalloc(*fake, B, H, N, D, 0, 16, 512, 1024, 1, 0.0, None)
    assert rc == -8                        # RA_ERR_WORKSPACE
