"""LongLoRA shifted sparse attention (S2-Attn), taken literally -- oracle.

LongLoRA: Efficient Fine-tuning of Long-Context Large Language Models
(Summary; Key points): tokens are split into groups, attention runs inside
each group, and in half of the heads the tokens are shifted by half a group
so information passes between neighbouring groups; a group of 2048 stands
in for training at 8192.  Steps, in that order:

  1. for the shifted heads, roll the sequence so that shifted position p
     holds original token (p + G/2) mod S (the last group wraps around);
  2. split the (shifted) sequence into S/G groups of G positions;
  3. run exact attention (``attention_forward``) independently in each
     group, causal by position inside the group when asked;
  4. roll the outputs (and lse) of the shifted heads back.

Readings where the page is silent: the shift is half a group, the shifted
heads are the trailing ``shift_heads`` query heads, and with grouped-query
heads a key/value head is shifted together with the query heads that read it
(so the boundary must fall on a group of query heads).  ``direction=-1``
rolls the other way; it yields the same ordered groups, which a pin checks.
"""

from __future__ import annotations

import numpy as np

from .attention import _f64, attention_forward, attention_backward


def s2_token_of_position(p, S: int, group: int, shifted: bool):
    """Original token held by shifted position p."""
    return (p + group // 2) % S if shifted else p


def _check(S, Hq, Hkv, group, shift_heads):
    if group <= 0 or S % group or group % 2:
        raise ValueError("group must be even and divide S")
    if not (0 <= shift_heads <= Hq):
        raise ValueError("shift_heads out of range")
    rep = Hq // Hkv
    if (Hq - shift_heads) % rep:
        raise ValueError("shifted heads must cover whole grouped-query groups")
    return rep


def _roll_heads(x, heads, amount):
    """Roll axis 1 (sequence) of the given heads (axis 2) by ``amount``."""
    y = x.copy()
    if len(heads):
        y[:, :, heads] = np.roll(x[:, :, heads], amount, axis=1)
    return y


def _group_split(x, group):
    B, S, H, d = x.shape
    return x.reshape(B * (S // group), group, H, d)


def _group_join(x, B):
    n, G, H, d = x.shape
    return x.reshape(B, n // B * G, H, d)


def _lse_join(lse, B):
    n, H, G = lse.shape
    nG = n // B
    return lse.reshape(B, nG, H, G).transpose(0, 2, 1, 3).reshape(B, H, nG * G)


def s2attn_forward(q, k, v, group: int, shift_heads: int, causal: bool = True,
                   scale=None, direction: int = 1):
    """Returns (out [B,S,Hq,d], lse [B,Hq,S]) in original token order."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, S, Hq, d = q.shape
    Hkv = k.shape[2]
    rep = _check(S, Hq, Hkv, group, shift_heads)
    qh = list(range(Hq - shift_heads, Hq))
    kh = list(range((Hq - shift_heads) // rep, Hkv)) if shift_heads else []
    amt = -direction * (group // 2)
    q2, k2, v2 = _roll_heads(q, qh, amt), _roll_heads(k, kh, amt), _roll_heads(v, kh, amt)
    o, lse = attention_forward(_group_split(q2, group), _group_split(k2, group),
                               _group_split(v2, group), causal, scale)
    o = _group_join(o, B)
    lse = _lse_join(lse, B)
    o = _roll_heads(o, qh, -amt)
    if qh:
        lse = lse.copy()
        lse[:, qh] = np.roll(lse[:, qh], -amt, axis=2)
    return o, lse


def s2attn_backward(q, k, v, dout, group: int, shift_heads: int,
                    causal: bool = True, scale=None, direction: int = 1):
    """Gradients of sum(dout * out) for S2-Attn.  Returns (dq, dk, dv)."""
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    B, S, Hq, d = q.shape
    Hkv = k.shape[2]
    rep = _check(S, Hq, Hkv, group, shift_heads)
    qh = list(range(Hq - shift_heads, Hq))
    kh = list(range((Hq - shift_heads) // rep, Hkv)) if shift_heads else []
    amt = -direction * (group // 2)
    args = [_group_split(_roll_heads(x, hs, amt), group)
            for x, hs in ((q, qh), (k, kh), (v, kh), (dout, qh))]
    dq, dk, dv = attention_backward(*args, causal, scale)
    dq = _roll_heads(_group_join(dq, B), qh, -amt)
    dk = _roll_heads(_group_join(dk, B), kh, -amt)
    dv = _roll_heads(_group_join(dv, B), kh, -amt)
    return dq, dk, dv
