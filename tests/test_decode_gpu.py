"""GPU parity of decoding against a sharded key/value cache (partials per
shard piece, exact merge) with the fp64 oracle's attention_decode."""

import numpy as np
import pytest
import torch

import oracle
from exact_blockwise_long_b200.synthetic import to_f64
from helpers import TOL_BF16_LSE, TOL_BF16_O, max_abs

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


def cache(B, H, Hkv, N, D, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    q = torch.randn((B, H, D), generator=g, device="cuda").to(torch.bfloat16)
    k = (2.0 * torch.randn((B, Hkv, N, D), generator=g, device="cuda")).to(torch.bfloat16)
    v = torch.randn((B, Hkv, N, D), generator=g, device="cuda").to(torch.bfloat16)
    return q, k, v


def decode(q, k, v, S, k_chunk):
    import exact_blockwise_long_b200 as ra
    B, H, D = q.shape
    N = k.shape[2]
    out = torch.empty_like(q)
    lse = torch.empty((B, H), device="cuda", dtype=torch.float32)
    ws = torch.empty(ra.ringattn_decode_workspace_size(B, H, N, D, S, k_chunk), device="cuda", dtype=torch.uint8)
    ra.ringattn_decode(q, k, v, out, lse, S, k_chunk, ws)
    assert ra.ringattn_get_error() == 0
    return out, lse


@pytest.mark.parametrize("B,H,Hkv,N,D,S,kc", [
    (2, 8, 2, 1000, 128, 4, 128),     # ragged cache length and shards
    (1, 4, 4, 4096, 64, 2, 256),      # one query head per KV head
    (3, 16, 1, 777, 128, 3, 128),     # MQA, 16 query heads share one KV head
    (1, 8, 1, 129, 64, 1, 128),       # one shard, one key past a tile
    (2, 4, 2, 5, 128, 8, 128),        # fewer keys than shards: empty shards
])
def test_decode_matches_oracle(B, H, Hkv, N, D, S, kc):
    q, k, v = cache(B, H, Hkv, N, D, 500 + N + H)
    out, lse = decode(q, k, v, S, kc)
    o_ref, l_ref = oracle.attention_decode(to_f64(q), to_f64(k), to_f64(v))
    assert max_abs(to_f64(out), o_ref) <= TOL_BF16_O
    assert max_abs(to_f64(lse), l_ref) <= TOL_BF16_LSE


def test_decode_shard_count_does_not_change_the_result():
    q, k, v = cache(2, 8, 2, 8192, 128, 7)
    o1, l1 = decode(q, k, v, 1, 8192)
    for S, kc in [(4, 512), (16, 128), (7, 256)]:
        o2, l2 = decode(q, k, v, S, kc)
        assert (o1.float() - o2.float()).abs().max().item() <= 1e-2
        assert (l1 - l2).abs().max().item() <= 1e-4


@pytest.mark.slow
def test_decode_full_size_sampled_heads():
    """B=8, H=32, Hkv=8, N=131072, d=128 (a 7B-style cache after a ring
    prefill of 131072 tokens, S=32): 16 (b, h) rows checked in fp64."""
    from exact_blockwise_long_b200.synthetic import DECODE_WORKLOADS, decode_inputs
    w = DECODE_WORKLOADS["decode_n128k"]
    q, k, v = decode_inputs(w)
    out, lse = decode(q, k, v, w.S, w.k_chunk)
    rng = np.random.default_rng(w.seed + 1000)
    G = w.H // w.Hkv
    for b, h in zip(rng.integers(0, w.B, 16), rng.integers(0, w.H, 16)):
        o_r, l_r = oracle.attention_decode(to_f64(q[b:b + 1, h:h + 1]), to_f64(k[b:b + 1, h // G:h // G + 1]),
                                           to_f64(v[b:b + 1, h // G:h // G + 1]))
        assert max_abs(to_f64(out[b, h]), o_r[0, 0]) <= TOL_BF16_O
        assert abs(float(lse[b, h]) - l_r[0, 0]) <= TOL_BF16_LSE
