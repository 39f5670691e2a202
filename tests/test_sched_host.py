"""Host-side check of the kernels' tile walks (csrc/sched.cuh), compiled for
the CPU: every query tile visits each visible key exactly once, chunks come
in the requested order (in-order, ring, custom), tiles that straddle a chunk
boundary are split at it, S2-Attn walks stay in the query's group, and the
backward's query ranges are the transpose of the forward's visibility."""

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

    def run(S, tile, causal, s2=0, kv_chunk=0, order=0, q_block=0, gt=0, st=0, fsh=0,
            perm=()):
        kv_chunk = kv_chunk or S
        q_block = q_block or kv_chunk
        args = [BIN] + [str(a) for a in (S, tile, causal, s2, kv_chunk, order, q_block, gt, st,
                                         fsh)] + [str(p) for p in perm]
        out = subprocess.run(args, capture_output=True, text=True, check=True).stdout
        walks, qr, tok, tiles = {}, {}, {}, {}
        for line in out.splitlines():
            tag, rest = line.split(" ", 1)
            key, vals = rest.split(":")
            if tag == "Q":
                walks[int(key)] = [tuple(int(x) for x in v.split(",")) for v in vals.split()]
            elif tag == "W":
                tiles[int(key)] = [int(v) for v in vals.split()]
            elif tag == "K":
                qr[int(key)] = tuple(int(v) for v in vals.split())
            else:
                tok[int(key)] = tuple(int(v) for v in vals.split())
        if tiles:
            # the tile-only walk visits the same tiles in the same order
            assert tiles == {qt: [t for (t, _, _) in v] for qt, v in walks.items()}
        run.tile_walks_checked += bool(tiles)
        return walks, qr, tok
    run.tile_walks_checked = 0
    yield run
    assert run.tile_walks_checked > 0


def keys_of(visits, tile):
    """The keys a walk covers, in visit order."""
    return [t * tile + i for (t, lo, hi) in visits for i in range(lo, hi)]


def check_chunk_walks(probe, S, tile, causal, kv_chunk, order, q_block=0, perm=()):
    walks, qr, _ = probe(S, tile, causal, kv_chunk=kv_chunk, order=order, q_block=q_block,
                         perm=perm)
    n_tiles = -(-S // tile)
    n_chunks = -(-S // kv_chunk)
    q_block = q_block or kv_chunk
    for qt, visits in walks.items():
        end = min(S, (qt + 1) * tile) if causal else S
        keys = keys_of(visits, tile)
        # every visible key exactly once, nothing else
        assert sorted(keys) == list(range(end)), (qt, visits)
        for (t, lo, hi) in visits:
            assert 0 <= lo < hi <= tile
            # a visit never crosses a chunk boundary
            assert (t * tile + lo) // kv_chunk == (t * tile + hi - 1) // kv_chunk
        # chunk order
        chunks = []
        for k in keys:
            c = k // kv_chunk
            if not chunks or chunks[-1] != c:
                chunks.append(c)
        if order == 0:
            want = list(range(n_chunks))
        elif order == 1:
            i = qt * tile // q_block
            want = [(i - j) % n_chunks for j in range(n_chunks)]
        else:
            want = list(perm)
        want = [c for c in want if c * kv_chunk < end]
        assert chunks == want, (qt, chunks, want)
        # keys inside a chunk ascend
        for c in chunks:
            ks = [k for k in keys if k // kv_chunk == c]
            assert ks == sorted(ks)
    for kt, (a, b) in qr.items():
        assert list(range(a, b)) == [qt for qt in range(n_tiles)
                                     if any(t == kt for (t, _, _) in walks[qt])]


@pytest.mark.parametrize("causal", [0, 1])
@pytest.mark.parametrize("n_chunks,order,qb,perm", [
    (1, 0, None, ()), (4, 0, None, ()), (4, 1, None, ()), (4, 1, 4, ()),
    (4, 2, None, (2, 0, 3, 1)), (8, 1, 1, ())])
def test_chunk_walks(probe, causal, n_chunks, order, qb, perm):
    tile, n = 4, 16
    S = n * tile
    kv_chunk = S // n_chunks
    check_chunk_walks(probe, S, tile, causal, kv_chunk, order,
                      q_block=(qb * tile if qb else 0), perm=perm)


@pytest.mark.parametrize("causal", [0, 1])
@pytest.mark.parametrize("S,kv_chunk,order,perm", [
    (40, 16, 0, ()), (40, 16, 1, ()), (28, 12, 2, (2, 0, 1)), (20, 32, 0, ()),
    (37, 16, 1, ())])
def test_partial_last_chunk(probe, causal, S, kv_chunk, order, perm):
    check_chunk_walks(probe, S, 4, causal, kv_chunk, order, perm=perm)


@pytest.mark.parametrize("causal", [0, 1])
@pytest.mark.parametrize("S,kv_chunk,order,q_block,perm", [
    (64, 6, 0, 0, ()), (64, 6, 1, 0, ()), (61, 10, 1, 8, ()), (30, 7, 2, 0, (3, 1, 4, 0, 2)),
    (45, 1, 1, 0, ()), (64, 17, 0, 0, ())])
def test_unaligned_chunks(probe, causal, S, kv_chunk, order, q_block, perm):
    """kv_chunk not a multiple of the tile: a straddling tile is visited once
    per chunk, each visit masked to that chunk's keys."""
    check_chunk_walks(probe, S, 4, causal, kv_chunk, order, q_block=q_block, perm=perm)


@pytest.mark.parametrize("causal", [0, 1])
@pytest.mark.parametrize("n,gt,st", [(16, 4, 2), (16, 16, 8), (8, 2, 1)])
def test_s2_walks(probe, causal, n, gt, st):
    tile = 4
    walks, qr, tok = probe(n * tile, tile, causal, s2=1, gt=gt, st=st, fsh=2)
    for qt, visits in walks.items():
        g0 = qt // gt * gt
        want = list(range(g0, qt + 1)) if causal else list(range(g0, g0 + gt))
        assert [t for (t, _, _) in visits] == want
        assert all(lo == 0 and hi == tile for (_, lo, hi) in visits)
    for kt, (a, b) in qr.items():
        assert list(range(a, b)) == [qt for qt in range(n)
                                     if any(t == kt for (t, _, _) in walks[qt])]
    for t, (plain, shifted) in tok.items():
        assert plain == t and shifted == (t + st) % n


def test_random_walks(probe):
    """Seeded random schedules: lengths, tile sizes, chunk lengths (aligned
    or not), orders and query blocks; every property above must hold."""
    import random
    rng = random.Random(2024)
    for _ in range(40):
        tile = rng.choice([2, 4, 8])
        S = rng.randint(1, 70)
        causal = rng.randint(0, 1)
        kv_chunk = rng.choice([rng.randint(1, S), tile * rng.randint(1, 4), S])
        order = rng.randint(0, 2)
        n_chunks = -(-S // kv_chunk)
        perm = tuple(rng.sample(range(n_chunks), n_chunks)) if order == 2 else ()
        q_block = rng.choice([0, rng.randint(1, S)])
        check_chunk_walks(probe, S, tile, causal, kv_chunk, order, q_block=q_block, perm=perm)
