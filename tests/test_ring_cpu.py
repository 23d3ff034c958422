"""The multi-device ring (exact_blockwise_long_b200.ring) on CPU ranks with
the gloo backend.  The per-pair work is done by fp64 reference arithmetic
(the oracle's attention plus the standard per-pair gradient with the global
softmax statistics), so this checks the driver itself: the ring order
(i - t) mod S, the causal skip and diagonal mask per shard pair, the
send/receive pairing, the exact merge of the forward partials, and the
key/value gradient accumulators following their blocks one step behind and
returning to their owners.  Gathered over the ranks, the results equal full-sequence
attention and its gradient from the oracle."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


class ReferenceOps:
    """Per-pair arithmetic in float64 numpy (test infrastructure)."""

    def __init__(self):
        import oracle
        self.oracle = oracle

    def fwd_pair(self, q, k, v, o_acc, lse_acc, causal):
        o_t, l_t = self.oracle.attention_forward(q.numpy(), k.numpy(), v.numpy(), causal)
        o_new, l_new = self.oracle.lse_merge(o_acc.double().numpy(), lse_acc.double().numpy(), o_t, l_t)
        o_acc.copy_(torch.from_numpy(o_new))
        lse_acc.copy_(torch.from_numpy(l_new))

    def bwd_prepare(self, o, lse, do):
        o, lse, do = (t.double().numpy() for t in (o, lse, do))
        return np.sum(do * o, axis=-1), lse                   # D_i with the global output; global lse

    def bwd_pair(self, q, k, v, do, prep, dq_acc, dk, dv, causal):
        dvec, lse = prep
        q, k, v, do = (t.double().numpy() for t in (q, k, v, do))
        scale = 1.0 / np.sqrt(q.shape[-1])
        s = np.einsum("bhid,bhjd->bhij", q, k) * scale
        if causal:
            L = q.shape[2]
            s = np.where(np.tril(np.ones((L, L), bool)), s, -np.inf)
        p = np.exp(s - lse[..., None])                       # global softmax statistics
        dp = np.einsum("bhid,bhjd->bhij", do, v)
        ds = p * (dp - dvec[..., None])
        dq_acc += torch.from_numpy(np.einsum("bhij,bhjd->bhid", ds, k) * scale).to(dq_acc.dtype)
        dk.copy_(torch.from_numpy(np.einsum("bhij,bhid->bhjd", ds, q) * scale))
        dv.copy_(torch.from_numpy(np.einsum("bhij,bhid->bhjd", p, do)))

    def accumulate(self, acc, x):
        acc += x

    def cast(self, x, out):
        out.copy_(x)


def _inputs(N, seed=77):
    rng = np.random.default_rng(seed)
    B, H, D = 1, 2, 4
    q, k, v, do = (rng.standard_normal((B, H, N, D)) for _ in range(4))
    return q, 1.5 * k, v, do


def _worker(rank, world, port, causal, N, out_dir):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    sys.path.insert(0, os.path.join(root, "tests"))
    from datetime import timedelta
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        from exact_blockwise_long_b200 import ring
        q, k, v, do = (torch.from_numpy(a) for a in _inputs(N))
        L = N // world
        sl = slice(rank * L, (rank + 1) * L)
        mine = [t[:, :, sl].contiguous() for t in (q, k, v, do)]
        ops = ReferenceOps()
        out, lse = ring.ring_attention_forward(mine[0], mine[1], mine[2], causal, ops=ops)
        dq, dk, dv = ring.ring_attention_backward(mine[0], mine[1], mine[2], out, lse, mine[3], causal, ops=ops)
        for name, t in (("o", out), ("l", lse), ("dq", dq), ("dk", dk), ("dv", dv)):
            np.save(os.path.join(out_dir, f"{name}{rank}.npy"), t.double().numpy())
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,causal", [(2, True), (3, True), (4, True), (4, False), (1, True)])
def test_ring_driver_matches_full_attention(tmp_path, world, causal):
    import oracle
    N = 8 * world
    mp.start_processes(_worker, args=(world, _free_port(), causal, N, str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    got = {n: np.concatenate([np.load(tmp_path / f"{n}{r}.npy") for r in range(world)], axis=2)
           for n in ("o", "l", "dq", "dk", "dv")}
    q, k, v, do = _inputs(N)
    o_ref, l_ref = oracle.attention_forward(q, k, v, causal)
    gq, gk, gv = oracle.attention_backward(q, k, v, do, causal)
    # fp32 accumulators in the forward: relative 1e-6 of unit-scale values
    np.testing.assert_allclose(got["o"], o_ref, atol=2e-6)
    np.testing.assert_allclose(got["l"], l_ref, atol=2e-6)
    for n, ref in (("dq", gq), ("dk", gk), ("dv", gv)):
        np.testing.assert_allclose(got[n], ref, atol=2e-5)
