"""Pins for the blockwise feedforward oracle (oracle/ffn.py), CPU only:
pure-Python brute force on tiny inputs, invariance to the block size (the
blockwise claim of the Ring Attention summary: blocking changes memory, not
the result), closed forms of the gated SiLU, central finite differences of
the backward, and planted mistakes that the pins must catch."""

import math

import numpy as np
import pytest

from oracle import ffn as F


def brute(x, wg, wu, wd):
    """Nested loops, math.exp and math.fsum: out_k = sum_j a_j wd[k, j] with
    a_j = silu(sum_i x_i wg[j, i]) * sum_i x_i wu[j, i]."""
    out = []
    for row in x:
        a = []
        for j in range(len(wg)):
            g = math.fsum(float(xi) * float(w) for xi, w in zip(row, wg[j]))
            u = math.fsum(float(xi) * float(w) for xi, w in zip(row, wu[j]))
            a.append(g / (1.0 + math.exp(-g)) * u)
        out.append([math.fsum(aj * float(w) for aj, w in zip(a, wd[k])) for k in range(len(wd))])
    return np.array(out)


def weights(rng, h, f, std=0.5):
    return (rng.standard_normal((f, h)) * std, rng.standard_normal((f, h)) * std,
            rng.standard_normal((h, f)) * std)


@pytest.mark.parametrize("T,h,f", [(1, 3, 2), (4, 5, 7), (6, 8, 3)])
def test_matches_brute(T, h, f):
    rng = np.random.default_rng(T * 100 + h * 10 + f)
    x = rng.standard_normal((T, h))
    wg, wu, wd = weights(rng, h, f)
    np.testing.assert_allclose(F.ffn_forward(x, wg, wu, wd), brute(x, wg, wu, wd),
                               rtol=0, atol=1e-12)


@pytest.mark.parametrize("block", [1, 2, 5, 7, 64])
def test_block_size_does_not_change_the_result(block):
    rng = np.random.default_rng(7)
    x = rng.standard_normal((23, 6))
    wg, wu, wd = weights(rng, 6, 9)
    ref = F.ffn_forward(x, wg, wu, wd, block=0)
    np.testing.assert_allclose(F.ffn_forward(x, wg, wu, wd, block=block), ref,
                               rtol=0, atol=1e-13)


def test_rows_match_full():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((17, 5))
    wg, wu, wd = weights(rng, 5, 4)
    rows = [0, 9, 16]
    np.testing.assert_allclose(F.ffn_rows(x, wg, wu, wd, rows),
                               F.ffn_forward(x, wg, wu, wd)[rows], atol=1e-14)


def test_silu_closed_forms():
    assert F.silu(np.array([0.0]))[0] == 0.0
    np.testing.assert_allclose(F.silu(np.array([1.0]))[0], 1.0 / (1.0 + math.exp(-1.0)),
                               rtol=1e-15)
    # large positive: the identity; large negative: g e^g
    np.testing.assert_allclose(F.silu(np.array([40.0]))[0], 40.0, rtol=1e-15)
    np.testing.assert_allclose(F.silu(np.array([-40.0]))[0], -40.0 * math.exp(-40.0),
                               rtol=1e-12)
    # finite for any input
    assert np.isfinite(F.silu(np.array([-1e4, 1e4]))).all()


def test_ffn_closed_forms():
    rng = np.random.default_rng(5)
    h, f = 4, 3
    wg, wu, wd = weights(rng, h, f)
    x = rng.standard_normal((5, h))
    # no up projection: nothing passes the gate
    assert np.all(F.ffn_forward(x, wg, np.zeros_like(wu), wd) == 0.0)
    # one-hot input, one-hot weights: out = wd[:, 0] * silu(a) * b
    a, b = 1.7, -0.6
    x1 = np.zeros((1, h)); x1[0, 2] = 1.0
    g = np.zeros((f, h)); g[0, 2] = a
    u = np.zeros((f, h)); u[0, 2] = b
    want = wd[:, 0] * (a / (1 + math.exp(-a))) * b
    np.testing.assert_allclose(F.ffn_forward(x1, g, u, wd)[0], want, atol=1e-15)


@pytest.mark.parametrize("mutant", ["sigmoid_not_silu", "gate_up_swapped", "no_gate"])
def test_pins_catch_planted_mistakes(monkeypatch, mutant):
    if mutant == "sigmoid_not_silu":
        monkeypatch.setattr(F, "silu", lambda g: 1.0 / (1.0 + np.exp(-np.asarray(g))))
    elif mutant == "no_gate":
        monkeypatch.setattr(F, "silu", lambda g: np.asarray(g))
    else:
        orig = F.ffn_forward

        def swapped(x, wg, wu, wd, block=0):
            return orig(x, wu, wg, wd, block)
        monkeypatch.setattr(F, "ffn_forward", swapped)
    with pytest.raises(AssertionError):
        test_matches_brute(4, 5, 7)


def _fd(fwd, tensors, do, eps=1e-6):
    num = []
    for t in tensors:
        g = np.zeros_like(t)
        for idx in np.ndindex(*t.shape):
            old = t[idx]
            t[idx] = old + eps
            lp = np.sum(fwd() * do)
            t[idx] = old - eps
            lm = np.sum(fwd() * do)
            t[idx] = old
            g[idx] = (lp - lm) / (2 * eps)
        num.append(g)
    return num


@pytest.mark.parametrize("block", [0, 2])
def test_backward_finite_differences(block):
    rng = np.random.default_rng(41 + block)
    T, h, f = 5, 3, 4
    x = rng.standard_normal((T, h))
    wg, wu, wd = weights(rng, h, f, std=0.8)
    do = rng.standard_normal((T, h))
    got = F.ffn_backward(x, wg, wu, wd, do, block=block)
    num = _fd(lambda: F.ffn_forward(x, wg, wu, wd), [x, wg, wu, wd], do)
    for name, a, b in zip(("dx", "dw_gate", "dw_up", "dw_down"), got, num):
        err = np.linalg.norm(a - b) / np.linalg.norm(b)
        assert err <= 1e-6, (name, err)


def test_backward_block_size_does_not_change_the_result():
    rng = np.random.default_rng(43)
    x = rng.standard_normal((19, 6))
    wg, wu, wd = weights(rng, 6, 5)
    do = rng.standard_normal((19, 6))
    ref = F.ffn_backward(x, wg, wu, wd, do)
    for block in (1, 4, 7):
        for a, b in zip(F.ffn_backward(x, wg, wu, wd, do, block=block), ref):
            np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)


def test_backward_catches_a_wrong_silu_derivative(monkeypatch):
    # the derivative of silu dropped to sigma alone must fail the pin
    orig = F._sigmoid

    def bad_backward(x, w_gate, w_up, w_down, dout, block=0):
        x, wg, wu, wd, do = (np.asarray(t, np.float64) for t in (x, w_gate, w_up, w_down, dout))
        g, u = x @ wg.T, x @ wu.T
        sig = orig(g)
        dh = do @ wd
        dg = dh * u * sig
        du = dh * g * sig
        return dg @ wg + du @ wu, dg.T @ x, du.T @ x, do.T @ (g * sig * u)
    monkeypatch.setattr(F, "ffn_backward", bad_backward)
    with pytest.raises(AssertionError):
        test_backward_finite_differences(0)


def test_backward_columns_match_full():
    rng = np.random.default_rng(47)
    x = rng.standard_normal((11, 5))
    wg, wu, wd = weights(rng, 5, 7)
    do = rng.standard_normal((11, 5))
    _, dwg, dwu, dwd = F.ffn_backward(x, wg, wu, wd, do)
    cols = [0, 3, 6]
    a, b, c = F.ffn_backward_columns(x, wg, wu, wd, do, cols)
    np.testing.assert_allclose(a, dwg[cols], atol=1e-13)
    np.testing.assert_allclose(b, dwu[cols], atol=1e-13)
    np.testing.assert_allclose(c, dwd[:, cols], atol=1e-13)
