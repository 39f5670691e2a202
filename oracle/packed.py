"""Exact attention over a packed batch of variable-length sequences, float64
-- oracle (test infrastructure).

The pages train on fixed-length sequences and say nothing about packing;
the plainest reading, taken here, is that each packed sequence is an
independent attention problem: sequence b holds tokens
[cu_seqlens[b], cu_seqlens[b+1]) of one token axis and attends only to
itself, causal by position inside the sequence.  So this module slices the
packed axis and applies the plain definition in ``attention`` to each
slice; nothing else.

Layouts: q, out, dout, dq are [T, Hq, d]; k, v, dk, dv are [T, Hkv, d]; lse
is [Hq, T].  Token rows outside every sequence are NaN in out, lse, dk and
dv (undefined) and zero in dq.
"""

from __future__ import annotations

import numpy as np

from .attention import _f64, attention_backward, attention_forward


def _bounds(cu_seqlens):
    cu = [int(x) for x in np.asarray(cu_seqlens).reshape(-1)]
    if any(b < a for a, b in zip(cu, cu[1:])) or cu[0] < 0:
        raise ValueError("cu_seqlens must be nondecreasing and start at >= 0")
    return list(zip(cu, cu[1:]))


def packed_attention_forward(q, k, v, cu_seqlens, causal: bool, scale=None):
    """Returns (out [T,Hq,d], lse [Hq,T]) in float64."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    T, Hq, d = q.shape
    out = np.full((T, Hq, d), np.nan)
    lse = np.full((Hq, T), np.nan)
    for c0, c1 in _bounds(cu_seqlens):
        if c1 == c0:
            continue
        o, l = attention_forward(q[None, c0:c1], k[None, c0:c1], v[None, c0:c1], causal,
                                 scale=scale)
        out[c0:c1] = o[0]
        lse[:, c0:c1] = l[0]
    return out, lse


def packed_attention_backward(q, k, v, dout, cu_seqlens, causal: bool, scale=None):
    """Gradients of sum(dout * out) over the packed batch.  Returns
    (dq, dk, dv) in float64."""
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    T = q.shape[0]
    dq = np.zeros(q.shape)
    dk = np.full(k.shape, np.nan)
    dv = np.full(v.shape, np.nan)
    for c0, c1 in _bounds(cu_seqlens):
        if c1 == c0:
            continue
        gq, gk, gv = attention_backward(q[None, c0:c1], k[None, c0:c1], v[None, c0:c1],
                                        dout[None, c0:c1], causal, scale=scale)
        dq[c0:c1] = gq[0]
        dk[c0:c1] = gk[0]
        dv[c0:c1] = gv[0]
    assert dq.shape[0] == T
    return dq, dk, dv
