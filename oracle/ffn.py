"""Blockwise feedforward in float64 -- oracle (test infrastructure).

What the pages fix: a host "computes attention and feedforward for its
query block block by block", and the blockwise feedforward of BPT lowers
the feedforward's activation memory (Ring Attention with Blockwise
Transformers for Near-Infinite Context, Summary and Key points).  They
print no feedforward; the workloads are Llama models, whose feedforward is
the gated SiLU unit (reading adopted):

    FFN(x) = W_down (silu(W_gate x) * (W_up x)),   silu(g) = g / (1 + e^-g)

with PyTorch's Linear weight layout (W_gate, W_up: [f, h]; W_down: [h, f]).
Blockwise: the token rows are processed ``block`` at a time, so the [., f]
intermediate only ever exists for one block.  Each row's result depends on
that row alone, so the blocking changes nothing in the result -- the pins
check exactly that.

Backward of L = sum(dout * out) (the analytic gradient; the pages are
silent), with s = silu(g), sigma = 1 / (1 + e^-g), h = s * u:

    dH = dout W_down               dW_down = dout^T H
    dU = dH * s                    dW_up   = dU^T x
    dG = dH * u * sigma (1 + g (1 - sigma))
                                   dW_gate = dG^T x
    dx = dG W_gate + dU W_up

also block by block (the weight gradients summed over the blocks).

Layouts: x, out [T, h]; returns float64.
"""

from __future__ import annotations

import numpy as np

from .attention import _f64


def silu(g):
    """g * sigmoid(g), written to stay finite for large |g|."""
    g = np.asarray(g, dtype=np.float64)
    out = np.empty_like(g)
    pos = g >= 0
    out[pos] = g[pos] / (1.0 + np.exp(-g[pos]))
    e = np.exp(g[~pos])
    out[~pos] = g[~pos] * e / (1.0 + e)
    return out


def ffn_forward(x, w_gate, w_up, w_down, block: int = 0):
    """Blockwise gated-SiLU feedforward.  block = 0: all rows at once."""
    x, wg, wu, wd = _f64(x), _f64(w_gate), _f64(w_up), _f64(w_down)
    T = x.shape[0]
    block = block or T
    out = np.empty((T, wd.shape[0]))
    for r0 in range(0, T, block):
        xb = x[r0:r0 + block]
        h = silu(xb @ wg.T) * (xb @ wu.T)
        out[r0:r0 + block] = h @ wd.T
    return out


def ffn_rows(x, w_gate, w_up, w_down, rows):
    """The feedforward of the given rows only (each row is independent)."""
    x = _f64(x)
    return ffn_forward(x[np.asarray(rows)], w_gate, w_up, w_down)


def _sigmoid(g):
    g = np.asarray(g, dtype=np.float64)
    out = np.empty_like(g)
    pos = g >= 0
    out[pos] = 1.0 / (1.0 + np.exp(-g[pos]))
    e = np.exp(g[~pos])
    out[~pos] = e / (1.0 + e)
    return out


def ffn_backward(x, w_gate, w_up, w_down, dout, block: int = 0):
    """Gradients of sum(dout * ffn_forward(...)).  Returns (dx, dw_gate,
    dw_up, dw_down) in float64."""
    x, wg, wu, wd, do = _f64(x), _f64(w_gate), _f64(w_up), _f64(w_down), _f64(dout)
    T = x.shape[0]
    block = block or T
    dx = np.empty_like(x)
    dwg, dwu, dwd = np.zeros_like(wg), np.zeros_like(wu), np.zeros_like(wd)
    for r0 in range(0, T, block):
        xb, dob = x[r0:r0 + block], do[r0:r0 + block]
        g, u = xb @ wg.T, xb @ wu.T
        sig = _sigmoid(g)
        s = g * sig
        dh = dob @ wd
        du = dh * s
        dg = dh * u * sig * (1.0 + g * (1.0 - sig))
        dx[r0:r0 + block] = dg @ wg + du @ wu
        dwg += dg.T @ xb
        dwu += du.T @ xb
        dwd += dob.T @ (s * u)
    return dx, dwg, dwu, dwd


def ffn_backward_columns(x, w_gate, w_up, w_down, dout, cols):
    """The weight gradients that involve feedforward columns ``cols`` only:
    rows cols of dw_gate and dw_up, columns cols of dw_down.  Column j needs
    g[:, j], u[:, j] and dH[:, j] over all tokens, O(T h) each, so large
    shapes can be checked column by column.  Returns (dwg_rows, dwu_rows,
    dwd_cols) in float64."""
    x, wg, wu, wd, do = _f64(x), _f64(w_gate), _f64(w_up), _f64(w_down), _f64(dout)
    cols = np.asarray(cols)
    g, u = x @ wg[cols].T, x @ wu[cols].T          # [T, len(cols)]
    sig = _sigmoid(g)
    s = g * sig
    dh = do @ wd[:, cols]
    du = dh * s
    dg = dh * u * sig * (1.0 + g * (1.0 - sig))
    return dg.T @ x, du.T @ x, do.T @ (s * u)
