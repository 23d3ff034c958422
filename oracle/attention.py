"""fp64 CPU oracle for exact (ring) blockwise softmax attention.

TEST INFRASTRUCTURE ONLY -- see the package docstring.  Plain NumPy in
float64; no blocking, fusion or reordering beyond what each docstring states.

Notation (the pages' problem statement, made concrete):
    q, k, v, do : [B, H, N, d] arrays; scale defaults to 1/sqrt(d).
    s_ij  = scale * q_i . k_j
    causal: key j is visible to query i iff j <= i (global token indices).
    lse_i = ln sum_{j visible} exp(s_ij)          (natural log)
    o_i   = sum_j exp(s_ij - lse_i) v_j

Sources:
    "Ring Attention with Blockwise Transformers for Near-Infinite Context",
    abstract: exact blockwise self-attention ("without resorting to
    approximations").
    chapterpal keyword page "Ring Attention", definition: sequence
    partitioned into blocks on a logical ring; each device keeps its query
    block while key/value blocks circulate.
    darcstar.tech note on the same paper, DarcStar commentary, paragraph one:
    online softmax is associative, partial attention from separate shards
    combines exactly; paragraph two: causal mask and softmax denominator are
    combined across chunks exactly.
"""

from __future__ import annotations

import numpy as np

NEG_INF = -np.inf


def _f64(x):
    return np.asarray(x, dtype=np.float64)


def _scale(d: int, scale) -> float:
    """Softmax scale: 1/sqrt(d) unless a positive value is given."""
    if scale is None or scale <= 0:
        return 1.0 / np.sqrt(d)
    return float(scale)


# ---------------------------------------------------------------------------
# The plain definition (full matrix).
# ---------------------------------------------------------------------------

def attention_forward(q, k, v, causal: bool, scale=None):
    """Full-matrix softmax attention, the exact result the method reaches.

    Returns (o [B,H,N,d], lse [B,H,N]) in float64.  lse is the natural-log
    softmax denominator of each query row (max plus log of the shifted sum,
    which is the same number computed without overflow).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, N, d = q.shape
    Nk = k.shape[2]
    sc = _scale(d, scale)
    o = np.empty((B, H, N, v.shape[3]))
    lse = np.empty((B, H, N))
    visible = np.tril(np.ones((N, Nk), dtype=bool)) if causal else None
    for b in range(B):
        for h in range(H):
            s = sc * (q[b, h] @ k[b, h].T)
            if causal:
                s = np.where(visible, s, NEG_INF)
            m = s.max(axis=1, keepdims=True)
            e = np.exp(s - m)
            den = e.sum(axis=1, keepdims=True)
            o[b, h] = (e / den) @ v[b, h]
            lse[b, h] = (m + np.log(den))[:, 0]
    return o, lse


def attention_backward(q, k, v, do, causal: bool, scale=None):
    """Gradient of sum(do * o) with respect to q, k and v (plain definition).

    With P_ij = exp(s_ij - lse_i) (zero where masked), D_i = do_i . o_i:
        dv_j = sum_i P_ij do_i
        dP_ij = do_i . v_j
        dS_ij = P_ij (dP_ij - D_i)
        dq_i = scale sum_j dS_ij k_j
        dk_j = scale sum_i dS_ij q_i
    This is the chain rule through the softmax; the pages use the method for
    training ("training and inference", paper abstract) but print no
    backward algorithm.
    Returns (dq, dk, dv) in float64.
    """
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    B, H, N, d = q.shape
    Nk = k.shape[2]
    sc = _scale(d, scale)
    dq = np.empty_like(q)
    dk = np.empty_like(k)
    dv = np.empty_like(v)
    visible = np.tril(np.ones((N, Nk), dtype=bool)) if causal else None
    for b in range(B):
        for h in range(H):
            s = sc * (q[b, h] @ k[b, h].T)
            if causal:
                s = np.where(visible, s, NEG_INF)
            m = s.max(axis=1, keepdims=True)
            e = np.exp(s - m)
            p = e / e.sum(axis=1, keepdims=True)
            o = p @ v[b, h]
            D = (do[b, h] * o).sum(axis=1)
            dp = do[b, h] @ v[b, h].T
            ds = p * (dp - D[:, None])
            dq[b, h] = sc * (ds @ k[b, h])
            dk[b, h] = sc * (ds.T @ q[b, h])
            dv[b, h] = p.T @ do[b, h]
    return dq, dk, dv


# ---------------------------------------------------------------------------
# Grouped key/value heads (GQA; MQA when there is one key/value head).
# ---------------------------------------------------------------------------

def attention_forward_gqa(q, k, v, causal: bool, scale=None):
    """Attention where query head h reads key/value head h // (H // Hkv).

    q: [B,H,N,d]; k, v: [B,Hkv,N,d] with H % Hkv == 0.  Each query head is
    plain softmax attention against its group's keys and values.
    Returns (o [B,H,N,d], lse [B,H,N]).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H = q.shape[:2]
    G = H // k.shape[1]
    o = np.empty(q.shape[:3] + (v.shape[3],))
    lse = np.empty(q.shape[:3])
    for b in range(B):
        for h in range(H):
            hk = h // G
            ob, lb = attention_forward(q[b:b + 1, h:h + 1], k[b:b + 1, hk:hk + 1], v[b:b + 1, hk:hk + 1],
                                       causal, scale)
            o[b, h], lse[b, h] = ob[0, 0], lb[0, 0]
    return o, lse


def attention_backward_gqa(q, k, v, do, causal: bool, scale=None):
    """Gradient of sum(do * o) for attention_forward_gqa.

    dq of each query head as in the plain case; dk and dv of a key/value
    head are the sums over the query heads that read it (chain rule through
    the shared operand).  Returns (dq [B,H,N,d], dk, dv [B,Hkv,N,d]).
    """
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    B, H = q.shape[:2]
    G = H // k.shape[1]
    dq = np.empty_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for b in range(B):
        for h in range(H):
            hk = h // G
            gq, gk, gv = attention_backward(q[b:b + 1, h:h + 1], k[b:b + 1, hk:hk + 1], v[b:b + 1, hk:hk + 1],
                                            do[b:b + 1, h:h + 1], causal, scale)
            dq[b, h] = gq[0, 0]
            dk[b, hk] += gk[0, 0]
            dv[b, hk] += gv[0, 0]
    return dq, dk, dv


def attention_decode(q, k, v, scale=None):
    """One new query token per (batch, head) against a cache of N keys.

    q: [B,H,d]; k, v: [B,Hkv,N,d]; query head h reads key/value head
    h // (H // Hkv).  The new token sees every cached key.
    Returns (o [B,H,d], lse [B,H]).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, d = q.shape
    G = H // k.shape[1]
    sc = _scale(d, scale)
    o = np.empty((B, H, v.shape[3]))
    lse = np.empty((B, H))
    for b in range(B):
        for h in range(H):
            s = sc * (k[b, h // G] @ q[b, h])
            m = s.max()
            e = np.exp(s - m)
            den = e.sum()
            o[b, h] = (e / den) @ v[b, h // G]
            lse[b, h] = m + np.log(den)
    return o, lse


# ---------------------------------------------------------------------------
# Sampled rows: the same definition restricted to chosen rows.
# ---------------------------------------------------------------------------

def attention_head_rows(q_sel, K, V, idx, causal: bool, scale=None):
    """Forward definition for chosen query rows of one head.

    q_sel: [n, d] query vectors of tokens idx [n]; K, V: [N, d] of the head.
    Each row is computed on its own from the full key/value sequence, so the
    result is exact for that row, not an estimate.  Returns (o [n, d], lse [n]).
    """
    q_sel = _f64(q_sel)
    K = _f64(K)
    V = _f64(V)
    sc = _scale(q_sel.shape[1], scale)
    o = np.empty((len(idx), V.shape[1]))
    lse = np.empty(len(idx))
    for r, i in enumerate(np.asarray(idx, dtype=np.int64)):
        kk, vv = (K[: i + 1], V[: i + 1]) if causal else (K, V)
        s = sc * (kk @ q_sel[r])
        m = s.max()
        e = np.exp(s - m)
        den = e.sum()
        o[r] = (e / den) @ vv
        lse[r] = m + np.log(den)
    return o, lse


def attention_rows(q, k, v, rows, causal: bool, scale=None):
    """Forward definition for selected query rows only.

    rows: integer array [n, 3] of (b, h, i).  Returns (o [n, d], lse [n]).
    """
    rows = np.asarray(rows, dtype=np.int64)
    o = np.empty((len(rows), v.shape[3]))
    lse = np.empty(len(rows))
    for r, (b, h, i) in enumerate(rows):
        o[r:r + 1], lse[r:r + 1] = attention_head_rows(_f64(q[b, h, i])[None], k[b, h], v[b, h], [i],
                                                       causal, scale)
    return o, lse


def attention_backward_query_rows(q, k, v, do, rows, causal: bool, scale=None):
    """dq for selected query rows: dq_i = scale sum_j P_ij (do_i.v_j - D_i) k_j.

    Row i needs only its own scores, so each row is exact on its own.
    rows: [n, 3] of (b, h, i).  Returns dq [n, d].
    """
    rows = np.asarray(rows, dtype=np.int64)
    d = q.shape[3]
    sc = _scale(d, scale)
    out = np.empty((len(rows), d))
    for r, (b, h, i) in enumerate(rows):
        kk = _f64(k[b, h])
        vv = _f64(v[b, h])
        if causal:
            kk = kk[: i + 1]
            vv = vv[: i + 1]
        qi = _f64(q[b, h, i])
        doi = _f64(do[b, h, i])
        s = sc * (kk @ qi)
        e = np.exp(s - s.max())
        p = e / e.sum()
        oi = p @ vv
        Di = doi @ oi
        ds = p * (vv @ doi - Di)
        out[r] = sc * (ds @ kk)
    return out


def attention_backward_key_rows(q, k, v, do, b, h, keys, causal: bool,
                                scale=None, q_block: int = 2048):
    """dk and dv for selected key rows j of one head (b, h).

    dv_j = sum_i P_ij do_i ;  dk_j = scale sum_i P_ij (do_i.v_j - D_i) q_i.
    These need lse_i and D_i = do_i . o_i of every query i that sees key j,
    so the full forward of the head is recomputed here, in blocks of q_block
    query rows (the blocking only bounds memory; each row is computed whole).
    Under the causal mask only queries i >= min(keys) contribute.
    Returns (dk [n, d], dv [n, d]).
    """
    keys = np.asarray(keys, dtype=np.int64)
    N, d = q.shape[2], q.shape[3]
    sc = _scale(d, scale)
    K = _f64(k[b, h])
    V = _f64(v[b, h])
    Ksel = K[keys]
    Vsel = V[keys]
    dk = np.zeros((len(keys), d))
    dv = np.zeros((len(keys), V.shape[1]))
    lo = int(keys.min()) if causal else 0
    for i0 in range(lo, N, q_block):
        i1 = min(N, i0 + q_block)
        Q = _f64(q[b, h, i0:i1])
        dO = _f64(do[b, h, i0:i1])
        idx = np.arange(i0, i1)
        s = sc * (Q @ K.T)
        if causal:
            s = np.where(np.arange(K.shape[0])[None, :] <= idx[:, None], s, NEG_INF)
        m = s.max(axis=1, keepdims=True)
        e = np.exp(s - m)
        den = e.sum(axis=1, keepdims=True)
        lse = m + np.log(den)
        o = (e / den) @ V
        D = (dO * o).sum(axis=1)
        ssel = sc * (Q @ Ksel.T)
        psel = np.exp(ssel - lse)
        if causal:
            psel = np.where(keys[None, :] <= idx[:, None], psel, 0.0)
        dpsel = dO @ Vsel.T
        dssel = psel * (dpsel - D[:, None])
        dv += psel.T @ dO
        dk += sc * (dssel.T @ Q)
    return dk, dv


# ---------------------------------------------------------------------------
# The method's steps: shards, ring order, chunk tiles, log-sum-exp merge.
# Used to pin the definition against the method, not for GPU parity.
# ---------------------------------------------------------------------------

def ring_visit_order(i: int, S: int, causal: bool):
    """KV shards that query shard i visits, in ring order.

    At ring step t = 0..S-1 query shard i holds KV shard j = (i - t) mod S
    (the KV blocks move one device along the ring per step while each device
    keeps its queries).  Under the causal mask a shard j > i lies entirely
    in the future of every query of shard i and is skipped.
    """
    out = []
    for t in range(S):
        j = (i - t) % S
        if causal and j > i:
            continue
        out.append(j)
    return out


def ring_visit_order_bwd(j: int, S: int, causal: bool):
    """Query shards that KV shard j meets, in ring order, for the backward.

    With the key/value block stationary, step t brings query shard
    i = (j + t) mod S; under the causal mask shards i < j are skipped.
    The set of pairs is the same as in the forward; only the loop nest is
    turned around.
    """
    out = []
    for t in range(S):
        i = (j + t) % S
        if causal and i < j:
            continue
        out.append(i)
    return out


def _merge_state(a, b):
    """Exact combine of two unnormalised partial states (m, l, acc).

    m: running max [n]; l: denominator [n] relative to m; acc: unnormalised
    output [n, d] relative to m.  The neutral element is (-inf, 0, 0); the
    factor exp(m_x - m) is taken as 0 when m_x = -inf so that -inf - -inf is
    never formed.
    """
    ma, la, aa = a
    mb, lb, ab = b
    m = np.maximum(ma, mb)
    fin = np.isfinite(m)
    with np.errstate(invalid="ignore"):
        fa = np.where(np.isfinite(ma) & fin, np.exp(np.where(fin, ma - m, 0.0)), 0.0)
        fb = np.where(np.isfinite(mb) & fin, np.exp(np.where(fin, mb - m, 0.0)), 0.0)
    return m, fa * la + fb * lb, fa[:, None] * aa + fb[:, None] * ab


def _block_state(s, vblk):
    """Partial state of one score block s [n, c] (masked entries -inf)."""
    m = s.max(axis=1)
    fin = np.isfinite(m)
    with np.errstate(invalid="ignore"):
        p = np.where(fin[:, None], np.exp(s - np.where(fin, m, 0.0)[:, None]), 0.0)
    return m, p.sum(axis=1), p @ vblk


def ring_blockwise_forward(q, k, v, S: int, q_chunk: int, k_chunk: int,
                           causal: bool, scale=None, order=None):
    """The method written out: S shards, ring order, chunk tiles, exact merge.

    For every query shard i (one virtual device) and every query chunk of
    q_chunk rows inside it, the KV shards are visited in ring order
    (``ring_visit_order``, or ``order(i)`` when given, to test that the
    visiting order does not matter).  Inside a visited shard the keys are
    taken k_chunk at a time; each chunk's partial state (max, denominator,
    unnormalised output) is merged into the shard-local state, and at the
    end of the shard the shard-local state is merged into the running state
    (the cross-shard log-sum-exp merge).  The causal mask is applied on
    global token indices inside the tiles of the diagonal pair.
    Returns (o, lse) in float64.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, N, d = q.shape
    if N % S:
        raise ValueError("N must be divisible by S")
    L = N // S
    if L % q_chunk or L % k_chunk:
        raise ValueError("chunk sizes must divide the shard length")
    sc = _scale(d, scale)
    dv = v.shape[3]
    o = np.empty((B, H, N, dv))
    lse = np.empty((B, H, N))
    for b in range(B):
        for h in range(H):
            for i in range(S):
                visits = ring_visit_order(i, S, causal) if order is None else order(i)
                for c0 in range(0, L, q_chunk):
                    rows = i * L + c0 + np.arange(q_chunk)
                    Q = q[b, h, rows]
                    n = len(rows)
                    run = (np.full(n, NEG_INF), np.zeros(n), np.zeros((n, dv)))
                    for j in visits:
                        shard = (np.full(n, NEG_INF), np.zeros(n), np.zeros((n, dv)))
                        for k0 in range(0, L, k_chunk):
                            cols = j * L + k0 + np.arange(k_chunk)
                            s = sc * (Q @ k[b, h, cols].T)
                            if causal:
                                s = np.where(cols[None, :] <= rows[:, None], s, NEG_INF)
                            shard = _merge_state(shard, _block_state(s, v[b, h, cols]))
                        run = _merge_state(run, shard)
                    m, l, acc = run
                    o[b, h, rows] = acc / l[:, None]
                    lse[b, h, rows] = m + np.log(l)
    return o, lse


def ring_blockwise_step(q, k, v, S: int, t: int, causal: bool, scale=None):
    """Normalised partial result of ring step t alone.

    Query shard i attends only to KV shard j = (i - t) mod S.  Returns
    (o_t, lse_t): o_t is that shard pair's softmax-normalised output and
    lse_t its log denominator.  Rows with no visible key in the pair (the
    causal pairs j > i, skipped by the method) get o_t = 0, lse_t = -inf,
    the neutral element of ``lse_merge``.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, N, d = q.shape
    L = N // S
    sc = _scale(d, scale)
    o = np.zeros((B, H, N, v.shape[3]))
    lse = np.full((B, H, N), NEG_INF)
    for b in range(B):
        for h in range(H):
            for i in range(S):
                j = (i - t) % S
                if causal and j > i:
                    continue
                rows = i * L + np.arange(L)
                cols = j * L + np.arange(L)
                s = sc * (q[b, h, rows] @ k[b, h, cols].T)
                if causal:
                    s = np.where(cols[None, :] <= rows[:, None], s, NEG_INF)
                m = s.max(axis=1, keepdims=True)
                e = np.exp(s - m)
                den = e.sum(axis=1, keepdims=True)
                o[b, h, rows] = (e / den) @ v[b, h, cols]
                lse[b, h, rows] = (m + np.log(den))[:, 0]
    return o, lse


def lse_merge(o_a, lse_a, o_b, lse_b):
    """Exact merge of two normalised partials (o_a, lse_a) and (o_b, lse_b).

    lse = ln(e^lse_a + e^lse_b);  o = e^(lse_a - lse) o_a + e^(lse_b - lse) o_b.
    This is softmax over the union of the two key sets, written in terms of
    each part's own normalised output and log denominator.  (-inf, any o) is
    the neutral element; when both are -inf the result is (0, -inf).
    """
    o_a, lse_a, o_b, lse_b = _f64(o_a), _f64(lse_a), _f64(o_b), _f64(lse_b)
    m = np.maximum(lse_a, lse_b)
    fin = np.isfinite(m)
    msafe = np.where(fin, m, 0.0)
    with np.errstate(invalid="ignore", divide="ignore"):
        ea = np.where(np.isfinite(lse_a), np.exp(lse_a - msafe), 0.0)
        eb = np.where(np.isfinite(lse_b), np.exp(lse_b - msafe), 0.0)
        tot = ea + eb
        lse = np.where(fin, msafe + np.log(np.where(fin, tot, 1.0)), NEG_INF)
        wa = np.where(fin, ea / np.where(fin, tot, 1.0), 0.0)
        wb = np.where(fin, eb / np.where(fin, tot, 1.0), 0.0)
    # an empty partial (lse = -inf) contributes nothing, whatever o it holds
    a_in = np.isfinite(lse_a)[..., None]
    b_in = np.isfinite(lse_b)[..., None]
    with np.errstate(invalid="ignore"):
        o = np.where(a_in, wa[..., None] * np.where(a_in, o_a, 0.0), 0.0) + \
            np.where(b_in, wb[..., None] * np.where(b_in, o_b, 0.0), 0.0)
    return o, lse
