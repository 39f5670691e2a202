"""(O, lse) merge of partial attention results -- oracle (test infrastructure).

Ring Attention with Blockwise Transformers for Near-Infinite Context
(Summary): each host attends its query block to one key/value block at a
time and the per-block results are combined; blockwise attention gives the
same answer whatever order the blocks are processed in.  The pages do not
print the combination rule; written out, for partials (o_a, lse_a) and
(o_b, lse_b) over disjoint key sets:

    lse = M + ln(exp(lse_a - M) + exp(lse_b - M)),   M = max(lse_a, lse_b)
    o   = exp(lse_a - lse) * o_a + exp(lse_b - lse) * o_b

A partial over an empty key set is (0, -inf) and is the identity.
"""

from __future__ import annotations

import numpy as np


def lse_merge(o_a, lse_a, o_b, lse_b):
    """Merge two partial results.  o_*: [..., d], lse_*: [...].  float64."""
    o_a = np.asarray(o_a, dtype=np.float64)
    o_b = np.asarray(o_b, dtype=np.float64)
    lse_a = np.asarray(lse_a, dtype=np.float64)
    lse_b = np.asarray(lse_b, dtype=np.float64)
    M = np.maximum(lse_a, lse_b)
    empty = ~np.isfinite(M)
    Ms = np.where(empty, 0.0, M)
    ea = np.exp(lse_a - Ms)
    eb = np.exp(lse_b - Ms)
    with np.errstate(divide="ignore"):
        lse = np.where(empty, -np.inf, Ms + np.log(ea + eb))
    ls = np.where(empty, 0.0, lse)
    wa = np.where(empty, 0.0, np.exp(lse_a - ls))
    wb = np.where(empty, 0.0, np.exp(lse_b - ls))
    o = wa[..., None] * o_a + wb[..., None] * o_b
    return o, lse
