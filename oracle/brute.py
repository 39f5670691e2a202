"""Pure-Python brute force for tiny inputs -- oracle pins (test infrastructure).

An independent restatement of exact attention used only to pin the
vectorised oracle: nested Python loops, ``math.exp`` and ``math.fsum``, no
numpy in the arithmetic.  The visibility of key j to query i is given as a
predicate, so S2-Attn can be stated here as a mask over ORIGINAL token
positions (no rolling at all), which checks the oracle's roll/unroll steps
from a second direction (LongLoRA, Summary: attention inside groups of the
shifted sequence).
"""

from __future__ import annotations

import math


def attend(q, k, v, visible, scale):
    """q: [S][d], k: [T][d], v: [T][dv] as nested lists.  Returns (out, lse)
    with out[i] = sum_j softmax_j(scale * q_i.k_j over visible j) v_j."""
    out, lses = [], []
    for i, qi in enumerate(q):
        logits = []
        for j, kj in enumerate(k):
            if visible(i, j):
                logits.append((j, scale * math.fsum(a * b for a, b in zip(qi, kj))))
        if not logits:
            out.append([0.0] * len(v[0]))
            lses.append(-math.inf)
            continue
        mx = max(s for _, s in logits)
        tot = math.fsum(math.exp(s - mx) for _, s in logits)
        lse = mx + math.log(tot)
        row = []
        for c in range(len(v[0])):
            row.append(math.fsum(math.exp(s - lse) * v[j][c] for j, s in logits))
        out.append(row)
        lses.append(lse)
    return out, lses


def s2_visible(S: int, group: int, shifted: bool, causal: bool):
    """Mask of S2-Attn over original token indices: token t sits at shifted
    position (t - G/2) mod S when its head is shifted, else at t; two tokens
    see each other iff their positions fall in the same group of G, and (if
    causal) the key's position is not after the query's."""
    def pos(t):
        return (t - group // 2) % S if shifted else t

    def vis(i, j):
        pi, pj = pos(i), pos(j)
        if pi // group != pj // group:
            return False
        return (pj <= pi) if causal else True
    return vis


def full_visible(causal: bool):
    return (lambda i, j: j <= i) if causal else (lambda i, j: True)
