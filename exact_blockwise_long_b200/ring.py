"""Ring attention across devices: one process per GPU, one sequence shard
per rank, key/value blocks passed around the ring.

chapterpal keyword page "Ring Attention" (definition paragraph): the
sequence is cut into blocks, one per device; each device keeps its query
block while the key/value blocks circulate around a ring, so no device ever
holds the whole sequence.  darcstar.tech note, "DarcStar commentary"
(paragraphs one and two): the partial attentions of separate blocks combine
exactly through the log-sum-exp merge, and the causal mask is applied per
block pair -- there is no all-gather of K/V.

Rank i of a group of S ranks owns shard i (tokens [i L, (i+1) L), L = N/S)
of q, k, v as [B, H, L, D] tensors.  At ring step t it holds key/value
shard j = (i - t) mod S and computes the pair (q_i, kv_j) on this library's
kernels: the whole pair when j < i, the masked diagonal when j = i, nothing
when j > i (causal).  Meanwhile the key/value block moves on to rank i+1
and the next arrives from rank i-1 (peer-to-peer send/receive through
torch.distributed, NCCL on GPUs, issued before the step's compute so the
transfer overlaps it).  The forward merges each pair into fp32 (O, LSE)
accumulators; the backward sums each pair's dq locally and lets the dk, dv
accumulators travel with their key/value block, which returns to its owner
after the last step.

The per-pair computations go through an `ops` object; `DeviceOps` (the
default) calls the C ABI.  Tests substitute reference arithmetic to check
the schedule on CPU ranks.
"""

from __future__ import annotations

import torch
import torch.distributed as dist


class DeviceOps:
    """Per-pair work on this library's CUDA kernels."""

    def __init__(self, q_chunk: int, k_chunk: int):
        from . import api
        self.api = api
        self.q_chunk, self.k_chunk = int(q_chunk), int(k_chunk)
        self._ws = None

    def fwd_pair(self, q, k, v, o_acc, lse_acc, causal):
        """Merge the attention of q against (k, v) -- one shard pair, the
        causal mask only on the diagonal pair -- into (o_acc, lse_acc)."""
        self.api.ringattn_fwd_step(q, k, v, o_acc, lse_acc, 1, self.q_chunk, self.k_chunk, causal, 0)

    def bwd_pair(self, q, k, v, o, lse, do, dq, dk, dv, causal):
        """This pair's share of the gradients, with the global o and lse."""
        B, H, L, D = q.shape
        n = self.api.ringattn_bwd_workspace_size(B, H, L, D)
        if self._ws is None or self._ws.numel() < n:
            self._ws = torch.empty(n, device=q.device, dtype=torch.uint8)
        self.api.ringattn_bwd(q, k, v, o, lse, do, dq, dk, dv, 1, self.q_chunk, self.k_chunk, causal, self._ws)

    def accumulate(self, acc, x):
        self.api.ringattn_accumulate(acc, x)

    def cast(self, x, out):
        self.api.ringattn_cast(x, out)


def _exchange(tensors_out, tensors_in, rank, world, group):
    """Send `tensors_out` to rank+1 and receive `tensors_in` from rank-1;
    returns the requests (issued on the communication side; waiting on them
    orders later work of the current stream after the transfer)."""
    nxt, prv = (rank + 1) % world, (rank - 1) % world
    ops = [dist.P2POp(dist.isend, t, nxt, group) for t in tensors_out]
    ops += [dist.P2POp(dist.irecv, t, prv, group) for t in tensors_in]
    return dist.batch_isend_irecv(ops)


def ring_attention_forward(q, k, v, causal=True, ops=None, group=None, q_chunk=128, k_chunk=128):
    """O and LSE of this rank's query shard against the whole sequence.

    q, k, v: this rank's shards [B, H, L, D].  Returns (out, lse): out in
    q's dtype, lse [B, H, L] fp32 (natural log).
    """
    ops = ops or DeviceOps(q_chunk, k_chunk)
    rank, world = dist.get_rank(group), dist.get_world_size(group)
    B, H, L, D = q.shape
    o_acc = torch.zeros((B, H, L, D), device=q.device, dtype=torch.float32)
    lse_acc = torch.full((B, H, L), float("-inf"), device=q.device, dtype=torch.float32)
    # the caller's k, v are only read; blocks arrive alternately in two
    # buffers of our own (the one received at step t is read and sent on at
    # step t + 1 while the other receives)
    cur = [k.contiguous(), v.contiguous()]
    bufs = [[torch.empty_like(cur[0]), torch.empty_like(cur[1])] for _ in range(2 if world > 2 else 1)]
    for t in range(world):
        j = (rank - t) % world
        nxt = bufs[t % len(bufs)]
        reqs = _exchange(cur, nxt, rank, world, group) if t < world - 1 else []
        if not (causal and j > rank):
            ops.fwd_pair(q, cur[0], cur[1], o_acc, lse_acc, causal and j == rank)
        for r in reqs:
            r.wait()
        cur = nxt
    out = torch.empty_like(q)
    ops.cast(o_acc, out)
    return out, lse_acc


def ring_attention_backward(q, k, v, out, lse, dout, causal=True, ops=None, group=None, q_chunk=128, k_chunk=128):
    """dq, dk, dv of sum(dout * out) for this rank's shards.

    out and lse are this rank's rows of the global forward result.  Each
    key/value block carries fp32 dk, dv accumulators around the ring; after
    the last step they take one more hop, back to the block's owner.
    """
    ops = ops or DeviceOps(q_chunk, k_chunk)
    rank, world = dist.get_rank(group), dist.get_world_size(group)
    shape = q.shape
    f32 = dict(device=q.device, dtype=torch.float32)
    dq_acc = torch.zeros(shape, **f32)
    # k, v of the caller are only read (see ring_attention_forward); blocks
    # and their gradient accumulators arrive alternately in two buffer sets
    cur = [k.contiguous(), v.contiguous(), torch.zeros(shape, **f32), torch.zeros(shape, **f32)]
    bufs = [[torch.empty_like(x) for x in cur] for _ in range(2)]
    dq_p, dk_p, dv_p = (torch.empty_like(q) for _ in range(3))
    for t in range(world):
        j = (rank - t) % world
        if not (causal and j > rank):
            ops.bwd_pair(q, cur[0], cur[1], out, lse, dout, dq_p, dk_p, dv_p, causal and j == rank)
            ops.accumulate(dq_acc, dq_p)
            ops.accumulate(cur[2], dk_p)
            ops.accumulate(cur[3], dv_p)
        if world == 1:
            break
        # the block (with its gradients) moves on; after the last step only
        # the gradients travel, home to the block's owner
        nxt = bufs[t % 2]
        if t < world - 1:
            reqs = _exchange(cur, nxt, rank, world, group)
        else:
            reqs = _exchange(cur[2:], nxt[2:], rank, world, group)
        for r in reqs:
            r.wait()
        cur = nxt
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ops.cast(dq_acc, dq)
    ops.cast(cur[2], dk)
    ops.cast(cur[3], dv)
    return dq, dk, dv
