"""Multi-process checks on CPU with the gloo backend (no GPU).

1. The multi-device ring the method describes (chapterpal "Ring Attention",
   definition: each device keeps its queries while key/value blocks
   circulate): S ranks each own one shard, pass their KV block to the next
   rank S-1 times with send/recv, and fold each step's partial into a running
   (O, LSE) with the exact merge (darcstar note, DarcStar commentary,
   paragraph one).  The gathered result equals full-matrix attention: the
   host-side schedule of a multi-GPU ring is correct by construction before
   any device runs it.  No all-gather of K/V takes place.
2. The bench's rank reduction: the step time is the maximum over ranks and
   the whole-job value counts every rank's work (weak scaling)."""

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


def _init(rank, world, port):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))


def _ring_worker(rank, world, port, causal, N, d, out_dir):
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import oracle
    _init(rank, world, port)
    try:
        L = N // world
        rng = np.random.default_rng(1234)
        q = rng.standard_normal((N, d))
        k = rng.standard_normal((N, d)) * 1.5
        v = rng.standard_normal((N, d))
        my_q = q[rank * L:(rank + 1) * L]
        kv = torch.from_numpy(np.concatenate([k[rank * L:(rank + 1) * L], v[rank * L:(rank + 1) * L]], 1).copy())
        o_run = np.zeros((L, d))
        lse_run = np.full(L, -np.inf)
        for t in range(world):
            j = (rank - t) % world          # the KV shard this rank holds at step t
            kj, vj = kv[:, :d].numpy(), kv[:, d:].numpy()
            if not (causal and j > rank):
                o_t, l_t = oracle.attention_head_rows(my_q, kj, vj, np.arange(L), causal and j == rank)
                o_run, lse_run = oracle.lse_merge(o_run, lse_run, o_t, l_t)
            if t < world - 1:
                nxt = torch.empty_like(kv)
                reqs = [dist.isend(kv, (rank + 1) % world), dist.irecv(nxt, (rank - 1) % world)]
                for r in reqs:
                    r.wait()
                kv = nxt
        np.save(os.path.join(out_dir, f"o{rank}.npy"), o_run)
        np.save(os.path.join(out_dir, f"l{rank}.npy"), lse_run)
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,causal", [(2, True), (4, True), (4, False), (3, True)])
def test_ring_exchange_matches_full_attention(tmp_path, world, causal):
    import oracle
    N, d = 48 * world, 8
    mp.start_processes(_ring_worker, args=(world, _free_port(), causal, N, d, str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    o = np.concatenate([np.load(tmp_path / f"o{r}.npy") for r in range(world)])
    lse = np.concatenate([np.load(tmp_path / f"l{r}.npy") for r in range(world)])
    rng = np.random.default_rng(1234)
    q = rng.standard_normal((N, d))
    k = rng.standard_normal((N, d)) * 1.5
    v = rng.standard_normal((N, d))
    o_ref, l_ref = oracle.attention_forward(q[None, None], k[None, None], v[None, None], causal)
    np.testing.assert_allclose(o, o_ref[0, 0], atol=1e-12)
    np.testing.assert_allclose(lse, l_ref[0, 0], atol=1e-12)


def _timing_worker(rank, world, port, out_dir):
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    _init(rank, world, port)
    try:
        ms = 10.0 + 5.0 * rank                      # rank 1 is the slowest
        worst = bench.max_over_ranks(ms, dist)
        val = bench.whole_job_tflops(1e12, world, worst)
        with open(os.path.join(out_dir, f"r{rank}.txt"), "w") as f:
            f.write(f"{worst} {val}")
    finally:
        dist.destroy_process_group()


def test_bench_takes_max_over_ranks_and_counts_all_work(tmp_path):
    world = 2
    mp.start_processes(_timing_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    for r in range(world):
        worst, val = (float(x) for x in open(tmp_path / f"r{r}.txt").read().split())
        assert worst == 15.0
        assert abs(val - 2 * 1e12 / 15e-3 / 1e12) < 1e-9
