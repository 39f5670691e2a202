"""Host-side checks of index logic compiled for the CPU: the feedforward
kernel's tile raster visits every output tile exactly once, in bands of a
given number of row tiles walked column by column; and the packed-sequence view accepts
exactly the in-order, in-range offsets no longer than the longest sequence
(the kernels skip anything else and report it); and the S2 roll's position
-> token map is the oracle's, a permutation of each head's tokens."""

import os
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "host", "layout_probe.cu")
BIN = os.path.join(HERE, "host", "layout_probe.bin")
CSRC = os.path.join(HERE, "..", "long_context_exact_attention_b200", "csrc")


@pytest.fixture(scope="module")
def probe():
    deps = [SRC] + [os.path.join(CSRC, f) for f in ("ffn_sm100.cuh", "sched.cuh", "ptx.cuh",
                                                     "aux_kernels.cuh")]
    if not os.path.exists(BIN) or os.path.getmtime(BIN) < max(map(os.path.getmtime, deps)):
        subprocess.run(["nvcc", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a",
                        "-x", "cu", SRC, "-o", BIN], check=True)

    def run(*args):
        out = subprocess.run([BIN] + [str(a) for a in args], capture_output=True, text=True,
                             check=True).stdout
        return [tuple(int(x) for x in line.split()) for line in out.splitlines()]
    return run


@pytest.mark.parametrize("band", [1, 16, 32, 64])
@pytest.mark.parametrize("n_tm,n_tn", [(1, 1), (64, 86), (64, 16), (86, 16), (17, 3), (33, 43),
                                       (16, 1), (5, 7), (172, 16)])
def test_tile_raster_is_a_bijection_in_bands(probe, n_tm, n_tn, band):
    rows = probe("tiles", n_tm, n_tn, band)
    coords = [(tm, tn) for _, tm, tn in rows]
    assert sorted(coords) == [(m, n) for m in range(n_tm) for n in range(n_tn)]
    for t, tm, tn in rows:
        b = t // (band * n_tn)
        assert b * band <= tm < min((b + 1) * band, n_tm)   # its own band of row tiles
    # inside a band, consecutive tiles walk down a column before moving right
    for (t0, m0, n0), (t1, m1, n1) in zip(rows, rows[1:]):
        if t0 // (band * n_tn) == t1 // (band * n_tn):
            assert (n1 == n0 and m1 == m0 + 1) or (n1 == n0 + 1)


@pytest.mark.parametrize("cu,S_max,T,want", [
    ([0, 300, 300, 700], 400, 800, [(1, 0, 300, 3), (1, 300, 0, 0), (1, 300, 400, 4)]),
    ([64, 300, 700], 400, 700, [(1, 64, 236, 2), (1, 300, 400, 4)]),
    ([0, 300, 200, 500], 300, 600, [(1, 0, 300, 3), (0, None, None, None), (1, 200, 300, 3)]),
    ([0, 300, 600], 299, 600, [(0, None, None, None), (0, None, None, None)]),
    ([0, 300, 900], 600, 600, [(1, 0, 300, 3), (0, None, None, None)]),
    ([-5, 10], 100, 100, [(0, None, None, None)]),
])
def test_packed_sequence_view(probe, cu, S_max, T, want):
    rows = probe("seq", S_max, 128, T, *cu)
    assert len(rows) == len(want)
    for (b, ok, tokb, ln, nt), w in zip(rows, want):
        assert ok == w[0], (b, rows)
        if ok:
            assert (tokb, ln, nt) == w[1:], (b, rows)


@pytest.mark.parametrize("S,G,H,shift", [(6000, 1500, 4, 2), (1200, 200, 2, 2), (400, 100, 2, 1),
                                         (16, 4, 3, 0)])
def test_s2_roll_map_matches_the_oracle(probe, S, G, H, shift):
    import oracle
    rows = probe("s2", S, G // 2, H, H - shift)
    first = H - shift
    for h in range(H):
        toks = [t for hh, p, t in rows if hh == h]
        assert sorted(toks) == list(range(S))             # a permutation of the tokens
        want = [oracle.s2_token_of_position(p, S, G, h >= first) for p in range(S)]
        assert toks == want


def test_random_tile_rasters(probe):
    import random
    rng = random.Random(7)
    for _ in range(20):
        n_tm, n_tn, band = rng.randint(1, 60), rng.randint(1, 50), rng.randint(1, 70)
        rows = probe("tiles", n_tm, n_tn, band)
        assert sorted((tm, tn) for _, tm, tn in rows) == \
            [(m, n) for m in range(n_tm) for n in range(n_tn)]
