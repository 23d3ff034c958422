"""ringattn_bwd_noalloc: the backward for callers that cannot allocate device
memory (a framework-owned allocator, a fixed start-up memory budget, or a hot
path that must not call cudaMalloc).  It runs the deterministic split
backward with its scratch in one static array, so it must give the bits that
ringattn_bwd_phase (mask 7) gives with a caller workspace -- on consecutive
calls that reuse the array, also when a larger problem is followed by a
smaller one and the other way round -- and refuse problems larger than the
array only after the same argument checks as the workspace entry points.

This file is collected last on purpose: it runs after every other test, and
it also passes on its own in a fresh process."""


import pytest
import torch

from exact_blockwise_long_b200.synthetic import small_attention_inputs

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


DETERMINISTIC = 7  # phase mask: preprocess, key/value-stationary pass, query-stationary pass


def _problem(L, B, H, N, D, S, qc, kc, causal, seed, stream):
    """Seeded inputs, their forward, and the reference gradients from the
    split backward with a caller workspace."""
    q, k, v, do = small_attention_inputs(B, H, N, D, seed)
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), device="cuda", dtype=torch.float32)
    cfg = (S, qc, kc, int(causal))
    assert L.ringattn_fwd(*_ptrs(q, k, v, o, lse), B, H, N, D, 0, *cfg, 0.0, stream) == 0
    ws = torch.empty(L.ringattn_bwd_workspace_size(B, H, N, D), device="cuda", dtype=torch.uint8)
    ref = [torch.empty_like(q) for _ in range(3)]
    rc = L.ringattn_bwd_phase(*_ptrs(q, k, v, o, lse, do, *ref), B, H, N, D, 0, *cfg, 0.0,
                              ws.data_ptr(), ws.numel(), DETERMINISTIC, stream)
    assert rc == 0
    return (q, k, v, o, lse, do), cfg, ref


def _noalloc(L, tensors, cfg, stream):
    q = tensors[0]
    B, H, N, D = q.shape
    got = [torch.full_like(q, float("nan")) for _ in range(3)]
    rc = L.ringattn_bwd_noalloc(*_ptrs(*tensors, *got), B, H, N, D, 0, *cfg, 0.0, stream)
    assert rc == 0
    assert L.ringattn_get_error(stream) == 0
    return got


@pytest.mark.parametrize("B,H,N,D,S,qc,kc,causal", [
    (1, 2, 1024, 128, 4, 128, 256, True),
    (2, 2, 768, 64, 3, 128, 128, False),
])
def test_noalloc_matches_workspace_backward_twice(L, B, H, N, D, S, qc, kc, causal):
    stream = torch.cuda.current_stream().cuda_stream
    tensors, cfg, ref = _problem(L, B, H, N, D, S, qc, kc, causal, 77 + N, stream)
    for _ in range(2):  # the second call finds the first call's scratch contents
        got = _noalloc(L, tensors, cfg, stream)
        assert all(torch.equal(a, b) for a, b in zip(got, ref))


def test_noalloc_larger_then_smaller_and_back(L):
    """A larger problem leaves more of the shared array written than a smaller
    one that follows reads, and the reverse: every call still gives its own
    reference bits."""
    stream = torch.cuda.current_stream().cuda_stream
    big = _problem(L, 2, 4, 2048, 128, 8, 128, 256, True, 501, stream)
    small = _problem(L, 1, 1, 512, 64, 2, 128, 128, False, 502, stream)
    for tensors, cfg, ref in (big, small, big, small, small, big):
        got = _noalloc(L, tensors, cfg, stream)
        assert all(torch.equal(a, b) for a, b in zip(got, ref))


def test_noalloc_rejects_problems_beyond_its_scratch(L):
    limit = 64 << 20
    B, H, N, D = 4, 32, 131072, 128        # two fp32 row vectors: about 134 MB of scratch
    assert 2 * B * H * N * 4 > limit
    ptr = [0x10000] * 9                    # aligned, non-null: the argument checks pass, nothing launches
    rc = L.ringattn_bwd_noalloc(*ptr, B, H, N, D, 0, 16, 512, 1024, 1, 0.0, None)
    assert rc == -8                        # RA_ERR_WORKSPACE
    # argument errors come first, as from ringattn_bwd
    assert L.ringattn_bwd_noalloc(*ptr, B, H, N, D, 7, 16, 512, 1024, 1, 0.0, None) == -3       # dtype
    assert L.ringattn_bwd_noalloc(*ptr, B, H, N, D, 0, 3, 512, 1024, 1, 0.0, None) == -2        # N % S
    assert L.ringattn_bwd_noalloc(*([None] + ptr[1:]), B, H, N, D, 0, 16, 512, 1024, 1, 0.0, None) == -1
