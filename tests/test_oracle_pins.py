"""Pins for the fp64 oracle: checks against facts the mathematics fixes, not
against the oracle itself.  CPU only.

* brute force: pure-Python loops (``oracle.brute``) on tiny inputs;
* closed forms: causal row 0, all-zero keys, a two-key case that exposes the
  softmax scale;
* invariants: rows of P sum to one, lse bounds, convex-hull outputs, the
  global gradient identities;
* merge: commutative, associative, identity element, chunk-order independence
  (Ring Attention with Blockwise Transformers, Summary);
* S2-Attn special cases (LongLoRA, Summary): group = sequence with no shift
  is full attention, both shift directions agree, no shift is per-group
  attention, and a mask-based restatement over original tokens agrees;
* gradients: central finite differences.

The last block plants mistakes in a copy of the oracle and checks that these
pins catch them.
"""

import itertools
import math

import numpy as np
import pytest

import oracle
from oracle import attention as A
from oracle import brute
from oracle.merge import lse_merge

RNG = np.random.default_rng(1234)


def rand(*shape, rng=RNG, std=1.0):
    return rng.standard_normal(shape) * std


def as_lists(x):
    return [list(map(float, r)) for r in x]


# ---------------------------------------------------------------- brute force

@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("S,d,Hq,Hkv", [(1, 3, 1, 1), (7, 5, 2, 2), (12, 4, 4, 2),
                                        (16, 8, 4, 1)])
def test_vectorised_matches_brute(causal, S, d, Hq, Hkv):
    rng = np.random.default_rng(S * 100 + d * 10 + Hq + causal)
    q, k, v = rand(2, S, Hq, d, rng=rng), rand(2, S, Hkv, d, rng=rng), rand(2, S, Hkv, d, rng=rng)
    out, lse = oracle.attention_forward(q, k, v, causal, row_block=5)
    sc = 1 / math.sqrt(d)
    for b in range(2):
        for h in range(Hq):
            g = h // (Hq // Hkv)
            o_b, l_b = brute.attend(as_lists(q[b, :, h]), as_lists(k[b, :, g]),
                                    as_lists(v[b, :, g]), brute.full_visible(causal), sc)
            np.testing.assert_allclose(out[b, :, h], np.array(o_b), rtol=0, atol=1e-12)
            np.testing.assert_allclose(lse[b, h], np.array(l_b), rtol=0, atol=1e-12)


def test_rows_match_full():
    rng = np.random.default_rng(7)
    q, k, v = rand(1, 40, 4, 8, rng=rng), rand(1, 40, 2, 8, rng=rng), rand(1, 40, 2, 8, rng=rng)
    out, lse = oracle.attention_forward(q, k, v, True)
    rows = [0, 5, 39, 17]
    o_r, l_r = oracle.attention_rows(q, k, v, True, 0, 3, rows)
    np.testing.assert_allclose(o_r, out[0, rows, 3], atol=1e-13)
    np.testing.assert_allclose(l_r, lse[0, 3, rows], atol=1e-13)


# ---------------------------------------------------------------- closed forms

def test_causal_row0_is_v0():
    q, k, v = rand(1, 9, 2, 4), rand(1, 9, 2, 4), rand(1, 9, 2, 4)
    out, lse = oracle.attention_forward(q, k, v, True)
    np.testing.assert_allclose(out[0, 0], v[0, 0], atol=1e-15)
    s00 = np.sum(q[0, 0] * k[0, 0], axis=-1) / 2.0
    np.testing.assert_allclose(lse[0, :, 0], s00, atol=1e-14)


@pytest.mark.parametrize("causal", [False, True])
def test_zero_keys_give_running_mean(causal):
    S = 11
    q, v = rand(1, S, 2, 4), rand(1, S, 2, 4)
    k = np.zeros_like(q)
    out, lse = oracle.attention_forward(q, k, v, causal)
    for i in range(S):
        n = i + 1 if causal else S
        np.testing.assert_allclose(out[0, i], v[0, :n].mean(axis=0), atol=1e-14)
        np.testing.assert_allclose(lse[0, :, i], math.log(n), atol=1e-14)


def test_two_key_closed_form_exposes_scale():
    d = 16
    a = 1.7
    q = np.zeros((1, 2, 1, d)); k = np.zeros((1, 2, 1, d)); v = rand(1, 2, 1, d)
    q[0, 1, 0, 3] = a
    k[0, 0, 0, 3] = a          # row 1 sees key 0 with logit a^2/sqrt(d), key 1 with 0
    out, lse = oracle.attention_forward(q, k, v, True)
    s = a * a / math.sqrt(d)
    p0 = math.exp(s) / (math.exp(s) + 1.0)
    np.testing.assert_allclose(lse[0, 0, 1], math.log(math.exp(s) + 1.0), atol=1e-14)
    np.testing.assert_allclose(out[0, 1, 0], p0 * v[0, 0, 0] + (1 - p0) * v[0, 1, 0], atol=1e-14)


def test_one_hot_row():
    d = 8
    S = 6
    k = rand(1, S, 1, d)
    q = np.zeros((1, S, 1, d))
    q[0, 4, 0] = 60.0 * k[0, 2, 0]     # row 4 picks key 2 by a wide margin
    v = rand(1, S, 1, d)
    out, _ = oracle.attention_forward(q, k, v, True)
    np.testing.assert_allclose(out[0, 4, 0], v[0, 2, 0], atol=1e-8)


# ---------------------------------------------------------------- invariants

@pytest.mark.parametrize("causal", [False, True])
def test_rows_of_p_sum_to_one_and_bounds(causal):
    S, d = 30, 6
    q, k, v = rand(1, S, 2, d, std=2.0), rand(1, S, 2, d), rand(1, S, 2, d)
    ones = np.ones_like(v)
    out1, lse = oracle.attention_forward(q, k, ones, causal)
    np.testing.assert_allclose(out1, 1.0, atol=1e-12)        # sum_j P_ij = 1
    out, _ = oracle.attention_forward(q, k, v, causal)
    for h in range(2):
        s = q[0, :, h] @ k[0, :, h].T / math.sqrt(d)
        for i in range(S):
            n = i + 1 if causal else S
            mx = s[i, :n].max()
            assert mx - 1e-12 <= lse[0, h, i] <= mx + math.log(n) + 1e-12
            lo, hi = v[0, :n, h].min(axis=0), v[0, :n, h].max(axis=0)
            assert np.all(out[0, i, h] >= lo - 1e-12) and np.all(out[0, i, h] <= hi + 1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_gradient_global_identities(causal):
    S, d, Hq, Hkv = 24, 8, 4, 2
    q, k, v, do = rand(2, S, Hq, d), rand(2, S, Hkv, d), rand(2, S, Hkv, d), rand(2, S, Hq, d)
    dq, dk, dv = oracle.attention_backward(q, k, v, do, causal, row_block=7)
    rep = Hq // Hkv
    # sum_j dK_j = scale * sum_i (sum_j dS_ij) q_i = 0 because sum_j dS_ij = D_i - D_i
    np.testing.assert_allclose(dk.sum(axis=1), 0.0, atol=1e-12 * np.abs(dk).sum())
    # sum_j dV_j = sum_i dO_i (rows of P sum to one), summed over the query heads
    want = do.sum(axis=1).reshape(2, Hkv, rep, d).sum(axis=2)
    np.testing.assert_allclose(dv.sum(axis=1), want, atol=1e-12)


def _d_identity_holds(monkeypatch, causal):
    """Record the rows D_i = sum_j P_ij dP_ij that the oracle's backward uses
    and compare them with dO_i . O_i, O_i from the oracle's forward (the two
    are equal because O_i = sum_j P_ij v_j and dP_ij = dO_i . v_j).  Returns
    False if any row differs."""
    B, S, d, Hq, Hkv = 2, 13, 8, 4, 2
    rng = np.random.default_rng(77)
    q, k, v, do = (rand(B, S, Hq, d, rng=rng), rand(B, S, Hkv, d, rng=rng),
                   rand(B, S, Hkv, d, rng=rng), rand(B, S, Hq, d, rng=rng))
    seen = []
    inner = A._row_dot_terms

    def record(p, dP):
        D = inner(p, dP)
        seen.append(np.array(D))
        return D

    monkeypatch.setattr(A, "_row_dot_terms", record)
    oracle.attention_backward(q, k, v, do, causal, row_block=S)  # one row block per head
    monkeypatch.setattr(A, "_row_dot_terms", inner)
    out, _ = oracle.attention_forward(q, k, v, causal)
    rep = Hq // Hkv
    # the backward visits batch entries, then key/value heads, then their query heads
    order = [(b, g * rep + r) for b in range(B) for g in range(Hkv) for r in range(rep)]
    assert len(seen) == len(order)
    return all(np.allclose(D, np.sum(do[b, :, h] * out[b, :, h], axis=1), rtol=0, atol=1e-12)
               for D, (b, h) in zip(seen, order))


@pytest.mark.parametrize("causal", [False, True])
def test_d_rows_equal_dout_dot_out(monkeypatch, causal):
    """D_i = sum_j P_ij dP_ij (as the backward computes it) equals dO_i . O_i."""
    assert _d_identity_holds(monkeypatch, causal)


def test_d_identity_catches_rows_taken_from_the_wrong_row(monkeypatch):
    """A planted mistake in the oracle -- D of row i taken from row i - 1 --
    breaks the identity, and the backward's gradients too."""
    S, d = 9, 4
    q, k, v, do = rand(1, S, 1, d), rand(1, S, 1, d), rand(1, S, 1, d), rand(1, S, 1, d)
    good = oracle.attention_backward(q, k, v, do, True)
    orig = A._row_dot_terms
    monkeypatch.setattr(A, "_row_dot_terms", lambda p, dP: np.roll(orig(p, dP), 1))
    assert not _d_identity_holds(monkeypatch, True)
    monkeypatch.setattr(A, "_row_dot_terms", lambda p, dP: np.roll(orig(p, dP), 1))
    bad = oracle.attention_backward(q, k, v, do, True)
    assert np.abs(bad[0] - good[0]).max() > 1e-3  # dQ moves; dV does not depend on D
    np.testing.assert_allclose(bad[2], good[2], atol=1e-14)


def test_backward_kv_head_subset_matches_full():
    S, d, Hq, Hkv = 20, 4, 4, 2
    q, k, v, do = rand(1, S, Hq, d), rand(1, S, Hkv, d), rand(1, S, Hkv, d), rand(1, S, Hq, d)
    dq, dk, dv = oracle.attention_backward(q, k, v, do, True)
    dq1, dk1, dv1 = oracle.attention_backward(q, k, v, do, True, kv_heads=[1])
    np.testing.assert_allclose(dq1, dq[:, :, 2:4], atol=1e-14)
    np.testing.assert_allclose(dk1[:, :, 0], dk[:, :, 1], atol=1e-14)
    np.testing.assert_allclose(dv1[:, :, 0], dv[:, :, 1], atol=1e-14)


# ---------------------------------------------------------------- merge

def _rand_partial(n, d, rng):
    return rng.standard_normal((n, d)), rng.standard_normal(n) * 3


def test_merge_commutative_associative_identity():
    rng = np.random.default_rng(3)
    a, b, c = (_rand_partial(10, 4, rng) for _ in range(3))
    ab = lse_merge(*a, *b)
    ba = lse_merge(*b, *a)
    np.testing.assert_allclose(ab[0], ba[0], atol=1e-14)
    np.testing.assert_allclose(ab[1], ba[1], atol=1e-14)
    left = lse_merge(*ab, *c)
    right = lse_merge(*a, *lse_merge(*b, *c))
    np.testing.assert_allclose(left[0], right[0], atol=1e-13)
    np.testing.assert_allclose(left[1], right[1], atol=1e-13)
    ident = lse_merge(*a, np.zeros((10, 4)), np.full(10, -np.inf))
    np.testing.assert_allclose(ident[0], a[0], atol=1e-15)
    np.testing.assert_allclose(ident[1], a[1], atol=1e-15)
    empty = lse_merge(np.zeros((2, 4)), np.full(2, -np.inf), np.zeros((2, 4)), np.full(2, -np.inf))
    assert np.all(empty[1] == -np.inf) and np.all(empty[0] == 0)


def test_merge_two_halves_is_softmax_of_union():
    rng = np.random.default_rng(5)
    s = rng.standard_normal(9) * 2
    vv = rng.standard_normal((9, 3))
    def part(ix):
        m = s[ix].max(); e = np.exp(s[ix] - m); l = m + math.log(e.sum())
        return (np.exp(s[ix] - l) @ vv[ix])[None], np.array([l])
    o, l = lse_merge(*part(slice(0, 4)), *part(slice(4, 9)))
    m = s.max(); e = np.exp(s - m)
    np.testing.assert_allclose(l[0], m + math.log(e.sum()), atol=1e-14)
    np.testing.assert_allclose(o[0], (e / e.sum()) @ vv, atol=1e-14)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("S,chunk", [(24, 6), (23, 5), (10, 7)])
def test_chunk_order_independence(causal, S, chunk):
    rng = np.random.default_rng(11 + S + chunk)
    d = 4
    q, k, v = rand(1, S, 2, d, rng=rng), rand(1, S, 1, d, rng=rng), rand(1, S, 1, d, rng=rng)
    ref_o, ref_l = oracle.attention_forward(q, k, v, causal)
    n = -(-S // chunk)
    orders = [list(range(n)), list(reversed(range(n)))] + \
             [list(rng.permutation(n)) for _ in range(4)]
    for order in orders:
        o, l = oracle.chunked_attention_forward(q, k, v, causal, chunk, order)
        np.testing.assert_allclose(o, ref_o, atol=1e-12)
        np.testing.assert_allclose(l, ref_l, atol=1e-12)


# ---------------------------------------------------------------- S2-Attn

def test_s2_group_is_sequence_no_shift_equals_full():
    q, k, v = rand(1, 16, 4, 4), rand(1, 16, 4, 4), rand(1, 16, 4, 4)
    for causal in (False, True):
        o, l = oracle.s2attn_forward(q, k, v, 16, 0, causal)
        o2, l2 = oracle.attention_forward(q, k, v, causal)
        assert np.array_equal(o, o2) and np.array_equal(l, l2)


def test_s2_shift_direction_irrelevant():
    q, k, v, do = rand(2, 16, 4, 4), rand(2, 16, 4, 4), rand(2, 16, 4, 4), rand(2, 16, 4, 4)
    for causal in (False, True):
        o, l = oracle.s2attn_forward(q, k, v, 8, 2, causal, direction=1)
        o2, l2 = oracle.s2attn_forward(q, k, v, 8, 2, causal, direction=-1)
        np.testing.assert_allclose(o, o2, atol=1e-15)
        np.testing.assert_allclose(l, l2, atol=1e-15)
        g1 = oracle.s2attn_backward(q, k, v, do, 8, 2, causal, direction=1)
        g2 = oracle.s2attn_backward(q, k, v, do, 8, 2, causal, direction=-1)
        for a, b in zip(g1, g2):
            np.testing.assert_allclose(a, b, atol=1e-14)


def test_s2_no_shift_is_per_group_attention():
    q, k, v = rand(1, 24, 2, 4), rand(1, 24, 2, 4), rand(1, 24, 2, 4)
    o, l = oracle.s2attn_forward(q, k, v, 8, 0, True)
    for g in range(3):
        sl = slice(8 * g, 8 * g + 8)
        og, lg = oracle.attention_forward(q[:, sl], k[:, sl], v[:, sl], True)
        np.testing.assert_allclose(o[:, sl], og, atol=1e-15)
        np.testing.assert_allclose(l[:, :, sl], lg, atol=1e-15)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("S,G,H,shift,Hkv", [(16, 8, 4, 2, 4), (12, 4, 2, 1, 2),
                                             (16, 16, 2, 2, 2), (16, 8, 4, 2, 2)])
def test_s2_matches_mask_restatement(causal, S, G, H, shift, Hkv):
    rng = np.random.default_rng(S + G + H + shift)
    d = 4
    q, k, v = rand(1, S, H, d, rng=rng), rand(1, S, Hkv, d, rng=rng), rand(1, S, Hkv, d, rng=rng)
    o, l = oracle.s2attn_forward(q, k, v, G, shift, causal)
    sc = 1 / math.sqrt(d)
    rep = H // Hkv
    for h in range(H):
        vis = brute.s2_visible(S, G, h >= H - shift, causal)
        ob, lb = brute.attend(as_lists(q[0, :, h]), as_lists(k[0, :, h // rep]),
                              as_lists(v[0, :, h // rep]), vis, sc)
        np.testing.assert_allclose(o[0, :, h], np.array(ob), atol=1e-12)
        np.testing.assert_allclose(l[0, h], np.array(lb), atol=1e-12)


def test_s2_wrap_group_contents():
    # shifted position p holds token (p + G/2) mod S; the last group wraps
    S, G = 16, 8
    toks = [oracle.s2_token_of_position(p, S, G, True) for p in range(S)]
    assert toks[:8] == [4, 5, 6, 7, 8, 9, 10, 11]
    assert toks[8:] == [12, 13, 14, 15, 0, 1, 2, 3]


# ---------------------------------------------------------------- gradients

def _fd_check(fwd, bwd, tensors, do, eps=1e-6, tol=1e-6):
    grads = bwd(*tensors, do)
    for ti, t in enumerate(tensors):
        num = np.zeros_like(t)
        for idx in itertools.product(*[range(s) for s in t.shape]):
            old = t[idx]
            t[idx] = old + eps
            lp = np.sum(fwd(*tensors)[0] * do)
            t[idx] = old - eps
            lm = np.sum(fwd(*tensors)[0] * do)
            t[idx] = old
            num[idx] = (lp - lm) / (2 * eps)
        err = np.linalg.norm(num - grads[ti]) / max(np.linalg.norm(num), 1e-30)
        assert err <= tol, (ti, err)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Hq,Hkv", [(1, 1), (4, 2)])
def test_finite_differences_attention(causal, Hq, Hkv):
    rng = np.random.default_rng(21 + Hq + causal)
    S, d = 6, 3
    q, k, v = rand(1, S, Hq, d, rng=rng), rand(1, S, Hkv, d, rng=rng), rand(1, S, Hkv, d, rng=rng)
    do = rand(1, S, Hq, d, rng=rng)
    _fd_check(lambda a, b, c: oracle.attention_forward(a, b, c, causal),
              lambda a, b, c, g: oracle.attention_backward(a, b, c, g, causal),
              [q, k, v], do)


@pytest.mark.parametrize("causal", [False, True])
def test_finite_differences_s2(causal):
    rng = np.random.default_rng(99)
    S, d, H, G = 8, 2, 2, 4
    q, k, v, do = (rand(1, S, H, d, rng=rng) for _ in range(4))
    _fd_check(lambda a, b, c: oracle.s2attn_forward(a, b, c, G, 1, causal),
              lambda a, b, c, g: oracle.s2attn_backward(a, b, c, g, G, 1, causal),
              [q, k, v], do)


# ---------------------------------------------------------------- packed batches

def _segment_visible(cu, causal):
    """Block-diagonal mask over the whole packed axis: tokens see each other
    iff they lie in the same sequence (and, causal, the key is not later)."""
    seg = {}
    for b, (c0, c1) in enumerate(zip(cu, cu[1:])):
        for t in range(c0, c1):
            seg[t] = b

    def vis(i, j):
        if i not in seg or seg.get(j) != seg[i]:
            return False
        return (j <= i) if causal else True
    return vis


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("cu", [[0, 4, 4, 9, 13], [0, 13], [0, 1, 2, 13], [2, 5, 11]])
def test_packed_matches_block_diagonal_brute(causal, cu):
    """Slicing per sequence (oracle.packed) against one masked attention over
    the packed axis (brute force): a wrong offset, a leak across sequences or
    a mask counted from the packed axis instead of the sequence fails."""
    rng = np.random.default_rng(sum(cu) + causal)
    T, Hq, Hkv, d = 13, 2, 1, 3
    q, k, v = rand(T, Hq, d, rng=rng), rand(T, Hkv, d, rng=rng), rand(T, Hkv, d, rng=rng)
    out, lse = oracle.packed_attention_forward(q, k, v, cu, causal)
    vis = _segment_visible(cu, causal)
    covered = [t for t in range(T) if cu[0] <= t < cu[-1]]
    for h in range(Hq):
        o_b, l_b = brute.attend(as_lists(q[:, h]), as_lists(k[:, h // (Hq // Hkv)]),
                                as_lists(v[:, h // (Hq // Hkv)]), vis, 1 / math.sqrt(d))
        np.testing.assert_allclose(out[covered, h], np.array(o_b)[covered], atol=1e-12)
        np.testing.assert_allclose(lse[h, covered], np.array(l_b)[covered], atol=1e-12)
    outside = [t for t in range(T) if t not in covered]
    assert np.isnan(out[outside]).all() and np.isnan(lse[:, outside]).all()


@pytest.mark.parametrize("causal", [False, True])
def test_finite_differences_packed(causal):
    rng = np.random.default_rng(77 + causal)
    cu = [0, 3, 3, 7]
    T, Hq, Hkv, d = 7, 2, 1, 2
    q, k, v = rand(T, Hq, d, rng=rng), rand(T, Hkv, d, rng=rng), rand(T, Hkv, d, rng=rng)
    do = rand(T, Hq, d, rng=rng)
    _fd_check(lambda a, b, c: oracle.packed_attention_forward(a, b, c, cu, causal),
              lambda a, b, c, g: oracle.packed_attention_backward(a, b, c, g, cu, causal),
              [q, k, v], do)


def test_packed_backward_outside_rows():
    rng = np.random.default_rng(5)
    cu = [1, 4, 6]
    T, H, d = 8, 1, 2
    q, k, v, do = (rand(T, H, d, rng=rng) for _ in range(4))
    dq, dk, dv = oracle.packed_attention_backward(q, k, v, do, cu, True)
    assert (dq[[0, 6, 7]] == 0).all()
    assert np.isnan(dk[[0, 6, 7]]).all() and np.isnan(dv[[0, 6, 7]]).all()
    assert np.isfinite(dk[1:6]).all()


# ---------------------------------------------------------------- planted mistakes

def _pins_pass():
    """Run a handful of forward pins; return False if any fails."""
    checks = [test_causal_row0_is_v0, test_two_key_closed_form_exposes_scale,
              lambda: test_zero_keys_give_running_mean(True),
              lambda: test_vectorised_matches_brute(True, 7, 5, 2, 2),
              lambda: test_s2_matches_mask_restatement(True, 16, 8, 4, 2, 4)]
    for c in checks:
        try:
            c()
        except AssertionError:
            return False
    return True


def test_pins_pass_unmutated():
    assert _pins_pass()


@pytest.mark.parametrize("mutant", ["no_scale", "strict_mask", "transposed_v",
                                    "unshift_wrong_way"])
def test_pins_catch_planted_mistakes(monkeypatch, mutant):
    from oracle import s2attn as S2
    if mutant == "no_scale":
        monkeypatch.setattr(A, "_scale", lambda d, s: 1.0)
    elif mutant == "strict_mask":
        def bad(s, keys, causal, rows):
            if causal:
                j = np.arange(keys)[None, :]
                s = np.where(j < rows[:, None], s, -np.inf)
            return s
        monkeypatch.setattr(A, "_row_block", bad)
    elif mutant == "transposed_v":
        orig = A._softmax_rows
        def bad(s):
            p, l = orig(s)
            return (p[::-1] if p.shape[0] > 1 else p), l
        monkeypatch.setattr(A, "_softmax_rows", bad)
    elif mutant == "unshift_wrong_way":
        orig = S2._roll_heads
        calls = {"n": 0}
        def bad(x, heads, amount):
            calls["n"] += 1
            # the fourth roll of a forward call is the un-shift of the output
            return orig(x, heads, amount if calls["n"] % 4 else -amount)
        monkeypatch.setattr(S2, "_roll_heads", bad)
    assert not _pins_pass()


@pytest.mark.parametrize("causal", [False, True])
def test_backward_rows_matches_full(causal):
    rng = np.random.default_rng(31)
    S, d, Hq, Hkv = 20, 4, 4, 2
    q, k, v, do = rand(1, S, Hq, d, rng=rng), rand(1, S, Hkv, d, rng=rng), \
        rand(1, S, Hkv, d, rng=rng), rand(1, S, Hq, d, rng=rng)
    dq, dk, dv = oracle.attention_backward(q, k, v, do, causal)
    rows = [3, 11, 19]
    dqr, _, _ = oracle.attention_backward_rows(q, k, v, do, causal, 0, 1, rows)
    np.testing.assert_allclose(dqr, dq[0, rows, 2:4], atol=1e-13)
    # all rows: the parts are the full gradients
    dqa, dka, dva = oracle.attention_backward_rows(q, k, v, do, causal, 0, 1, range(S))
    np.testing.assert_allclose(dka, dk[0, :, 1], atol=1e-13)
    np.testing.assert_allclose(dva, dv[0, :, 1], atol=1e-13)
    if causal:  # tail rows give exact dK/dV for keys in the tail
        _, dkt, dvt = oracle.attention_backward_rows(q, k, v, do, True, 0, 0, range(12, S))
        np.testing.assert_allclose(dkt[12:], dk[0, 12:, 0], atol=1e-13)
        np.testing.assert_allclose(dvt[12:], dv[0, 12:, 0], atol=1e-13)


# ---------------------------------------------------------------- power of the parity gates

def test_lse_tolerance_catches_a_dropped_chunk():
    """Dropping one key chunk from the merge moves lse by ln(1 - n_c/n_vis),
    far beyond the 1e-3 lse bound (Ring Attention, Summary: every block must
    be merged), on the bf16 workloads' 0.5-scaled inputs."""
    rng = np.random.default_rng(71)
    S, d, chunk = 512, 16, 64
    q, k, v = (rand(1, S, 1, d, rng=rng, std=0.5) for _ in range(3))
    _, ref = oracle.attention_forward(q, k, v, True)
    n = S // chunk
    _, dropped = oracle.chunked_attention_forward(q, k, v, True, chunk, list(range(1, n)))
    later = slice(chunk, S)  # rows that should have seen chunk 0
    assert np.min(np.abs(dropped[0, 0, later] - ref[0, 0, later])) > 1e-3


def test_relative_output_gate_catches_a_zero_output():
    """With 0.5-scaled inputs attention is near uniform and |O| shrinks like
    1/sqrt(row), so at the 32K workload's length an all-zero output passes
    the 2e-2 absolute bound; the per-head relative Frobenius bound of 1e-2
    does not.  Sampled tail rows, each exact over every visible key."""
    rng = np.random.default_rng(73)
    S, d = 32768, 128
    q, k, v = (rand(1, S, 1, d, rng=rng, std=0.5) for _ in range(3))
    rows = np.sort(rng.choice(np.arange(S // 2, S), 64, replace=False))
    ref, _ = oracle.attention_rows(q, k, v, True, 0, 0, rows)
    zero = np.zeros_like(ref)
    assert np.max(np.abs(zero - ref)) <= 2e-2                        # the loose gate passes
    assert np.linalg.norm(zero - ref) / np.linalg.norm(ref) > 1e-2   # the strict gate fails it


# ---------------------------------------------------------------- blocks

@pytest.mark.parametrize("q_pos0,k_pos0,Sq,Sk", [(0, 0, 6, 6), (5, 2, 4, 7), (2, 9, 5, 3),
                                                 (3, 3, 4, 2), (0, 6, 3, 4)])
@pytest.mark.parametrize("causal", [False, True])
def test_block_matches_brute_with_positions(q_pos0, k_pos0, Sq, Sk, causal):
    """A query block at q_pos0 against a key block at k_pos0, against the
    pure-Python loops with the mask stated over absolute positions (rows
    that see no key of the block give (0, -inf))."""
    rng = np.random.default_rng(q_pos0 * 31 + k_pos0)
    d = 4
    q, k, v = rand(1, Sq, 2, d, rng=rng), rand(1, Sk, 1, d, rng=rng), rand(1, Sk, 1, d, rng=rng)
    out, lse = oracle.block_attention(q, k, v, q_pos0, k_pos0, causal)
    vis = (lambda i, j: k_pos0 + j <= q_pos0 + i) if causal else (lambda i, j: True)
    for h in range(2):
        bo, bl = brute.attend(as_lists(q[0, :, h]), as_lists(k[0, :, 0]), as_lists(v[0, :, 0]),
                              vis, 1 / math.sqrt(d))
        np.testing.assert_allclose(out[0, :, h], bo, atol=1e-12)
        np.testing.assert_array_equal(np.isinf(lse[0, h]), np.isinf(bl))
        fin = np.isfinite(bl)
        np.testing.assert_allclose(lse[0, h][fin], np.asarray(bl)[fin], atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_block_at_equal_positions_is_full_attention(causal):
    q, k, v = rand(2, 11, 4, 3), rand(2, 11, 2, 3), rand(2, 11, 2, 3)
    bo, bl = oracle.block_attention(q, k, v, 7, 7, causal)
    fo, fl = oracle.attention_forward(q, k, v, causal)
    np.testing.assert_allclose(bo, fo, atol=1e-13)
    np.testing.assert_allclose(bl, fl, atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("cuts", [(0, 5, 12, 20), (0, 1, 2, 20), (0, 13, 20)])
def test_merged_blocks_are_the_whole_row(causal, cuts):
    """Splitting the keys of a sequence into blocks, attending a query block
    to each at its own position and merging the partials in any order gives
    the rows of full attention (Ring Attention, Summary)."""
    S, d = 20, 5
    rng = np.random.default_rng(len(cuts))
    q, k, v = rand(1, S, 2, d, rng=rng), rand(1, S, 2, d, rng=rng), rand(1, S, 2, d, rng=rng)
    fo, fl = oracle.attention_forward(q, k, v, causal)
    r0, r1 = 4, 17  # the query block
    parts = [oracle.block_attention(q[:, r0:r1], k[:, a:b], v[:, a:b], r0, a, causal)
             for a, b in zip(cuts[:-1], cuts[1:])]
    for order in (range(len(parts)), reversed(range(len(parts)))):
        o = np.zeros((1, r1 - r0, 2, d))
        l = np.full((1, 2, r1 - r0), -np.inf)
        for i in order:
            po, pl = parts[i]
            o_t, l_t = lse_merge(o.transpose(0, 2, 1, 3), l, po.transpose(0, 2, 1, 3), pl)
            o, l = o_t.transpose(0, 2, 1, 3), l_t
        np.testing.assert_allclose(o, fo[:, r0:r1], atol=1e-12)
        np.testing.assert_allclose(l, fl[:, :, r0:r1], atol=1e-12)


def test_block_pins_catch_a_mask_off_by_one(monkeypatch):
    """Planted in the oracle: the block mask uses < instead of <= (the
    diagonal key dropped); the brute-force pin catches it."""
    q, k, v = rand(1, 6, 1, 3), rand(1, 6, 1, 3), rand(1, 6, 1, 3)
    bo, _ = brute.attend(as_lists(q[0, :, 0]), as_lists(k[0, :, 0]), as_lists(v[0, :, 0]),
                         brute.full_visible(True), 1 / math.sqrt(3))
    good = oracle.block_attention(q, k, v, 0, 0, True)
    monkeypatch.setattr(A, "_position_mask", lambda qp, kp: kp[None, :] < qp[:, None])
    bad = oracle.block_attention(q, k, v, 0, 0, True)
    assert np.abs(good[0][0, :, 0] - np.asarray(bo)).max() < 1e-12
    assert np.abs(bad[0][0, :, 0] - np.asarray(bo)).max() > 1e-3
