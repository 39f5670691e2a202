"""Host-side check of the kernels' tile walks (csrc/sched.cuh), compiled for
the CPU: every query tile visits each visible key tile exactly once, chunks
come in the requested order (in-order, ring, custom), S2-Attn walks stay in
the query's group, and the backward's query ranges are the transpose of the
forward's visibility."""

import os
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "host", "sched_probe.cu")
BIN = os.path.join(HERE, "host", "sched_probe.bin")


@pytest.fixture(scope="module")
def probe():
    if not os.path.exists(BIN) or os.path.getmtime(BIN) < max(
            os.path.getmtime(SRC),
            os.path.getmtime(os.path.join(HERE, "..", "long_context_exact_attention_b200",
                                          "csrc", "sched.cuh"))):
        subprocess.run(["nvcc", "-std=c++17", "-x", "cu", SRC, "-o", BIN], check=True)

    def run(n_tiles, causal, s2=0, tpc=None, n_chunks=1, order=0, qb=None, gt=0, st=0, fsh=0,
            perm=()):
        tpc = tpc or -(-n_tiles // n_chunks)
        qb = qb or tpc
        args = [BIN] + [str(a) for a in (n_tiles, causal, s2, tpc, n_chunks, order, qb, gt, st,
                                         fsh)] + [str(p) for p in perm]
        out = subprocess.run(args, capture_output=True, text=True, check=True).stdout
        walks, qr, tok = {}, {}, {}
        for line in out.splitlines():
            tag, rest = line.split(" ", 1)
            key, vals = rest.split(":")
            vals = [int(v) for v in vals.split()]
            if tag == "Q":
                walks[int(key)] = vals
            elif tag == "K":
                qr[int(key)] = tuple(vals)
            else:
                tok[int(key)] = tuple(vals)
        return walks, qr, tok
    return run


@pytest.mark.parametrize("causal", [0, 1])
@pytest.mark.parametrize("n_chunks,order,qb,perm", [
    (1, 0, None, ()), (4, 0, None, ()), (4, 1, None, ()), (4, 1, 4, ()),
    (4, 2, None, (2, 0, 3, 1)), (8, 1, 1, ())])
def test_chunk_walks(probe, causal, n_chunks, order, qb, perm):
    n = 16
    walks, qr, _ = probe(n, causal, n_chunks=n_chunks, order=order, qb=qb, perm=perm)
    tpc = n // n_chunks
    qb = qb or tpc
    for qt, seq in walks.items():
        visible = [t for t in range(n) if (t <= qt or not causal)]
        assert sorted(seq) == visible, (qt, seq)
        # chunk order
        chunks = []
        for t in seq:
            c = t // tpc
            if not chunks or chunks[-1] != c:
                chunks.append(c)
        if order == 0:
            want = list(range(n_chunks))
        elif order == 1:
            i = qt // qb
            want = [(i - j) % n_chunks for j in range(n_chunks)]
        else:
            want = list(perm)
        want = [c for c in want if any(t // tpc == c for t in visible)]
        assert chunks == want, (qt, chunks, want)
        # tiles inside a chunk ascend
        for c in chunks:
            ts = [t for t in seq if t // tpc == c]
            assert ts == sorted(ts)
    for kt, (a, b) in qr.items():
        assert list(range(a, b)) == [qt for qt in range(n) if kt in walks[qt]]


@pytest.mark.parametrize("causal", [0, 1])
@pytest.mark.parametrize("n,tpc,order,perm", [(10, 4, 0, ()), (10, 4, 1, ()), (7, 3, 2, (2, 0, 1)),
                                             (5, 8, 0, ())])
def test_partial_last_chunk(probe, causal, n, tpc, order, perm):
    n_chunks = -(-n // tpc)
    walks, qr, _ = probe(n, causal, tpc=tpc, n_chunks=n_chunks, order=order, perm=perm)
    for qt, seq in walks.items():
        visible = [t for t in range(n) if (t <= qt or not causal)]
        assert sorted(seq) == visible, (qt, seq)
        assert max(seq) < n
    for kt, (a, b) in qr.items():
        assert list(range(a, b)) == [qt for qt in range(n) if kt in walks[qt]]


@pytest.mark.parametrize("causal", [0, 1])
@pytest.mark.parametrize("n,gt,st", [(16, 4, 2), (16, 16, 8), (8, 2, 1)])
def test_s2_walks(probe, causal, n, gt, st):
    walks, qr, tok = probe(n, causal, s2=1, gt=gt, st=st, fsh=2)
    for qt, seq in walks.items():
        g0 = qt // gt * gt
        want = list(range(g0, qt + 1)) if causal else list(range(g0, g0 + gt))
        assert seq == want
    for kt, (a, b) in qr.items():
        assert list(range(a, b)) == [qt for qt in range(n) if kt in walks[qt]]
    for t, (plain, shifted) in tok.items():
        assert plain == t and shifted == (t + st) % n
