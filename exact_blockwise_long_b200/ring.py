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
accumulators.  The backward adds each pair's dq share into a local fp32
accumulator; each key/value block's dk, dv accumulators follow the block
one step behind it: at step t a rank computes its share of the block it
holds into a buffer of its own while the block's accumulator -- finished by
the previous rank at step t - 1 -- is on its way, and adds the two once both
are there.  So the key/value blocks and the accumulators both move while
pairs are computed; after the last step the accumulators take one more hop,
home to their blocks' owners.

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

    def fwd_pair(self, q, k, v, o_acc, lse_acc, causal):
        """Merge the attention of q against (k, v) -- one shard pair, the
        causal mask only on the diagonal pair -- into (o_acc, lse_acc)."""
        self.api.ringattn_fwd_step(q, k, v, o_acc, lse_acc, 1, self.q_chunk, self.k_chunk, causal, 0)

    def bwd_prepare(self, o, lse, do):
        """The query block's row statistics (D_n = dO_n . O_n, lse), once per backward."""
        B, H, L, D = o.shape
        prep = torch.empty(self.api.ringattn_bwd_prepare_size(B, H, L), device=o.device, dtype=torch.uint8)
        return self.api.ringattn_bwd_prepare(o, lse, do, prep)

    def bwd_pair(self, q, k, v, do, prep, dq_acc, dk, dv, causal):
        """dq_acc += this pair's dq share; dk, dv <- its dk, dv share (fp32)."""
        self.api.ringattn_bwd_pair(q, k, v, do, prep, dq_acc, dk, dv, self.q_chunk, self.k_chunk, causal)

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
    key/value block's fp32 dk, dv accumulators follow it around the ring one
    step behind; after the last step they take one more hop, back to the
    block's owner.
    """
    ops = ops or DeviceOps(q_chunk, k_chunk)
    rank, world = dist.get_rank(group), dist.get_world_size(group)
    shape = q.shape
    f32 = dict(device=q.device, dtype=torch.float32)
    prep = ops.bwd_prepare(out, lse, dout)
    dq_acc = torch.zeros(shape, **f32)
    # k, v of the caller are only read (see ring_attention_forward)
    kv = [k.contiguous(), v.contiguous()]
    kv_bufs = [[torch.empty_like(kv[0]), torch.empty_like(kv[1])] for _ in range(2 if world > 2 else 1)]
    # dk, dv accumulator pairs in three roles: `part` takes this step's share,
    # `recv` receives the accumulator of the block held now, `done` is the
    # finished accumulator of the previous step's block (being sent on)
    part = [torch.empty(shape, **f32), torch.empty(shape, **f32)]
    recv = [torch.empty(shape, **f32), torch.empty(shape, **f32)]
    spare = [torch.empty(shape, **f32), torch.empty(shape, **f32)]
    done = None
    for t in range(world):
        j = (rank - t) % world
        reqs = []
        if t < world - 1:  # the block moves on while this step computes with it
            nxt = kv_bufs[t % len(kv_bufs)]
            reqs += _exchange(kv, nxt, rank, world, group)
        if t > 0:  # the previous step's finished accumulator on; this block's in
            reqs += _exchange(done, recv, rank, world, group)
        visible = not (causal and j > rank)  # always true at t == 0 (the diagonal pair)
        if visible:
            ops.bwd_pair(q, kv[0], kv[1], dout, prep, dq_acc, part[0], part[1], causal and j == rank)
        for r in reqs:
            r.wait()
        if t == 0:
            done, part, spare = part, spare, None  # the block's first share is its accumulator
        else:
            if visible:
                ops.accumulate(recv[0], part[0])
                ops.accumulate(recv[1], part[1])
            done, recv = recv, done  # the sent buffer is free again: it receives next
        if t < world - 1:
            kv = nxt
    if world > 1:
        # the finished accumulators go home: this rank's block comes from rank - 1
        for r in _exchange(done, recv, rank, world, group):
            r.wait()
        done = recv
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ops.cast(dq_acc, dq)
    ops.cast(done[0], dk)
    ops.cast(done[1], dv)
    return dq, dk, dv
