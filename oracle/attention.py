"""Plain exact softmax attention in float64 -- oracle (test infrastructure).

Definition followed (Ring Attention with Blockwise Transformers for
Near-Infinite Context, Summary: attention stays exact while computed block by
block; sourcepulse project card of the 1M-context recipe, How It Works: full
attention, no approximations).  The pages print no formula; the one written
out here is the textbook definition:

    s_ij   = (q_i . k_j) * scale,          scale = 1/sqrt(d) by default
    mask   : causal keeps j <= i (query and key positions share one axis)
    lse_i  = ln sum_j exp(s_ij)           (over visible j, whole row at once)
    P_ij   = exp(s_ij - lse_i)
    O_i    = sum_j P_ij v_j

Grouped-query heads: query head h reads key/value head h // (Hq / Hkv).

Backward of L = sum(dO * O) (the pages are silent; analytic gradient):

    dV_j  = sum_i P_ij dO_i
    dP_ij = dO_i . v_j
    D_i   = sum_j P_ij dP_ij
    dS_ij = P_ij (dP_ij - D_i)
    dQ_i  = scale * sum_j dS_ij k_j
    dK_j  = scale * sum_i dS_ij q_i

Layouts: q, out, dout, dq are [B, S, Hq, d]; k, v, dk, dv are [B, S, Hkv, d];
lse is [B, Hq, S].  Rows are processed in blocks only to bound memory; each
block is the whole-row definition above (no online rescaling).
"""

from __future__ import annotations

import math

import numpy as np

from .merge import lse_merge


def _f64(x):
    """Host float64 copy of a numpy array or torch tensor."""
    if hasattr(x, "detach"):
        x = x.detach().to("cpu")
        import torch  # local: torch is only needed to convert tensors
        x = x.to(torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def _scale(d, scale):
    return 1.0 / math.sqrt(d) if not scale else float(scale)


def _row_block(s_q, keys, causal, rows):
    """Logits of the given query rows against all keys, masked."""
    s = s_q
    if causal:
        j = np.arange(keys)[None, :]
        s = np.where(j <= rows[:, None], s, -np.inf)
    return s


def _row_dot_terms(p, dP):
    """D_i = sum_j P_ij dP_ij, the row term of dS = P o (dP - D)."""
    return np.sum(p * dP, axis=1)


def _softmax_rows(s):
    """Return (P, lse) of each row of s (row max subtracted for range)."""
    mx = np.max(s, axis=1)
    mx_safe = np.where(np.isfinite(mx), mx, 0.0)
    e = np.exp(s - mx_safe[:, None])
    tot = np.sum(e, axis=1)
    with np.errstate(divide="ignore"):
        lse = mx_safe + np.log(tot)
    lse = np.where(tot > 0, lse, -np.inf)
    p = np.where(tot[:, None] > 0, e / np.where(tot > 0, tot, 1.0)[:, None], 0.0)
    return p, lse


def attention_forward(q, k, v, causal: bool, scale=None, row_block: int = 2048,
                      heads=None):
    """Exact attention.  Returns (out [B,S,H,d], lse [B,H,S]) in float64.

    ``heads`` restricts the computation to those query heads (the returned
    arrays then hold only them, in the given order)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, S, Hq, d = q.shape
    Hkv = k.shape[2]
    assert Hq % Hkv == 0
    rep = Hq // Hkv
    sc = _scale(d, scale)
    hs = list(range(Hq)) if heads is None else list(heads)
    out = np.zeros((B, S, len(hs), d))
    lse = np.zeros((B, len(hs), S))
    for b in range(B):
        for hi, h in enumerate(hs):
            g = h // rep
            Q, K, V = q[b, :, h], k[b, :, g], v[b, :, g]
            for r0 in range(0, S, row_block):
                r1 = min(S, r0 + row_block)
                rows = np.arange(r0, r1)
                kend = r1 if causal else S
                s = (Q[r0:r1] @ K[:kend].T) * sc
                s = _row_block(s, kend, causal, rows)
                p, l = _softmax_rows(s)
                out[b, r0:r1, hi] = p @ V[:kend]
                lse[b, hi, r0:r1] = l
    return out, lse


def attention_rows(q, k, v, causal: bool, b: int, h: int, rows, scale=None):
    """Exact (out, lse) of the given query rows of one (batch, head).

    Each sampled row is the full-row definition over every visible key, so it
    can be checked at sequence lengths where the whole output is too costly.
    Returns (out [R, d], lse [R])."""
    rows = np.asarray(rows, dtype=np.int64)
    if hasattr(q, "detach"):
        import torch
        Q = _f64(q[b, torch.as_tensor(rows, device=q.device), h])
    else:
        Q = _f64(np.asarray(q)[b, rows, h])
    Hq, Hkv = q.shape[2], k.shape[2]
    g = h // (Hq // Hkv)
    K = _f64(k[b, :, g])
    V = _f64(v[b, :, g])
    d = Q.shape[-1]
    sc = _scale(d, scale)
    S = K.shape[0]
    s = (Q @ K.T) * sc
    s = _row_block(s, S, causal, rows)
    p, lse = _softmax_rows(s)
    return p @ V, lse


def attention_backward(q, k, v, dout, causal: bool, scale=None,
                       row_block: int = 2048, kv_heads=None):
    """Analytic gradients of L = sum(dout * out).  Returns (dq, dk, dv).

    P is recomputed from the definition.  ``kv_heads`` restricts the work to
    those key/value heads and the query heads that read them; the returned
    dq then holds only those query heads (ascending), dk/dv only those kv
    heads (in the given order)."""
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    B, S, Hq, d = q.shape
    Hkv = k.shape[2]
    rep = Hq // Hkv
    sc = _scale(d, scale)
    gs = list(range(Hkv)) if kv_heads is None else list(kv_heads)
    qheads = [h for g in gs for h in range(g * rep, (g + 1) * rep)]
    dq = np.zeros((B, S, len(qheads), d))
    dk = np.zeros((B, S, len(gs), d))
    dv = np.zeros((B, S, len(gs), d))
    for b in range(B):
        for gi, g in enumerate(gs):
            K, V = k[b, :, g], v[b, :, g]
            for r in range(rep):
                h = g * rep + r
                hi = gi * rep + r
                Q, dO = q[b, :, h], dout[b, :, h]
                for r0 in range(0, S, row_block):
                    r1 = min(S, r0 + row_block)
                    rows = np.arange(r0, r1)
                    kend = r1 if causal else S
                    s = (Q[r0:r1] @ K[:kend].T) * sc
                    s = _row_block(s, kend, causal, rows)
                    p, _ = _softmax_rows(s)
                    dP = dO[r0:r1] @ V[:kend].T
                    D = _row_dot_terms(p, dP)
                    dS = p * (dP - D[:, None])
                    dv[b, :kend, gi] += p.T @ dO[r0:r1]
                    dq[b, r0:r1, hi] = sc * (dS @ K[:kend])
                    dk[b, :kend, gi] += sc * (dS.T @ Q[r0:r1])
    return dq, dk, dv


def chunked_attention_forward(q, k, v, causal: bool, chunk: int, order,
                              scale=None):
    """Blockwise attention as the Ring Attention summary describes it: each
    query row attends to the key/value chunks one at a time, and the partial
    (O, lse) results are combined with ``lse_merge`` in the given chunk
    ``order``.  A chunk in which a row sees no key contributes (0, -inf).

    Used by the pins to show order independence; the oracle's forward does
    not use it."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, S, Hq, d = q.shape
    rep = Hq // k.shape[2]
    sc = _scale(d, scale)
    out = np.zeros((B, S, Hq, d))
    lse = np.full((B, Hq, S), -np.inf)
    rows = np.arange(S)
    for b in range(B):
        for h in range(Hq):
            g = h // rep
            Q, K, V = q[b, :, h], k[b, :, g], v[b, :, g]
            o_run = np.zeros((S, d))
            l_run = np.full(S, -np.inf)
            for c in order:
                j0, j1 = c * chunk, min(S, (c + 1) * chunk)
                s = (Q @ K[j0:j1].T) * sc
                if causal:
                    j = np.arange(j0, j1)[None, :]
                    s = np.where(j <= rows[:, None], s, -np.inf)
                p, l_c = _softmax_rows(s)
                o_c = p @ V[j0:j1]
                o_run, l_run = lse_merge(o_run, l_run, o_c, l_c)
            out[b, :, h] = o_run
            lse[b, h] = l_run
    return out, lse


def attention_backward_rows(q, k, v, dout, causal: bool, b: int, g: int, rows,
                            scale=None):
    """Backward restricted to query ``rows`` of every query head that reads
    key/value head ``g`` (batch ``b``).  Each row is the full-row definition.

    Returns (dq [R, rep, d] for those rows, dk_part [S, d], dv_part [S, d])
    where the *_part arrays hold only the rows' contributions
    (dK_j += scale * sum_{i in rows} dS_ij q_i, dV_j += sum_{i in rows} P_ij dO_i).
    Under a causal mask, a key j receives contributions only from rows
    i >= j, so when ``rows`` is the tail [r0, S) the parts equal the full dK_j
    and dV_j for every j >= r0."""
    import torch  # noqa: F401  (tensor inputs are converted by _f64)
    rows = np.asarray(rows, dtype=np.int64)
    Hq, Hkv = q.shape[2], k.shape[2]
    rep = Hq // Hkv
    K = _f64(k[b, :, g])
    V = _f64(v[b, :, g])
    S, d = K.shape
    sc = _scale(d, scale)
    dq = np.zeros((len(rows), rep, d))
    dk = np.zeros((S, d))
    dv = np.zeros((S, d))
    for r in range(rep):
        h = g * rep + r
        Q = _f64(q[b, :, h])[rows]
        dO = _f64(dout[b, :, h])[rows]
        s = _row_block((Q @ K.T) * sc, S, causal, rows)
        p, _ = _softmax_rows(s)
        dP = dO @ V.T
        D = _row_dot_terms(p, dP)
        dS = p * (dP - D[:, None])
        dq[:, r] = sc * (dS @ K)
        dk += sc * (dS.T @ Q)
        dv += p.T @ dO
    return dq, dk, dv


def _position_mask(qpos, kpos):
    """Causal visibility over absolute positions: [len(qpos), len(kpos)]."""
    return kpos[None, :] <= qpos[:, None]


def block_attention(q, k, v, q_pos0: int, k_pos0: int, causal: bool, scale=None):
    """Partial attention of a query block over one key/value block, as a host
    of the ring computes it (Ring Attention with Blockwise Transformers for
    Near-Infinite Context, Summary: each host attends its own query block to
    the key/value block it holds, and the per-block results are merged).

    q [B, Sq, Hq, d] holds the queries at positions q_pos0 .. q_pos0+Sq-1,
    k, v [B, Sk, Hkv, d] the keys at positions k_pos0 .. k_pos0+Sk-1 of the
    same position axis; with ``causal`` key j is visible to query i iff
    k_pos0 + j <= q_pos0 + i.  Returns the block's partial (out [B, Sq, Hq,
    d], lse [B, Hq, Sq]) over the visible keys of this block only; a row
    that sees none of them gets the empty partial (0, -inf)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Sq, Hq, d = q.shape
    Sk, Hkv = k.shape[1], k.shape[2]
    rep = Hq // Hkv
    sc = _scale(d, scale)
    visible = _position_mask(q_pos0 + np.arange(Sq), k_pos0 + np.arange(Sk))
    out = np.zeros((B, Sq, Hq, d))
    lse = np.zeros((B, Hq, Sq))
    for b in range(B):
        for h in range(Hq):
            g = h // rep
            s = (q[b, :, h] @ k[b, :, g].T) * sc
            if causal:
                s = np.where(visible, s, -np.inf)
            p, l = _softmax_rows(s)
            out[b, :, h] = p @ v[b, :, g]
            lse[b, h] = l
    return out, lse
