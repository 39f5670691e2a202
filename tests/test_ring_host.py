"""The ring driver's host logic on CPU (no GPU, no oracle): the zig-zag
partition, the per-step launch plan, and the rotation of key/value blocks
and of their gradient accumulators over gloo ranks.

The kernels are replaced by recording stand-ins that check which block they
were handed and add distinct powers of two, so every result is an exact
integer in float64: a block that is visited twice, skipped, sent to the
wrong rank, or whose accumulators do not return home changes a result or the
record of visits.  Bit-exact comparisons throughout."""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from long_context_exact_attention_b200 import ring


# ---------------------------------------------------------------- plan

@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
@pytest.mark.parametrize("causal", [True, False])
def test_every_visible_chunk_pair_is_launched_once(world, causal):
    seen = []
    for r in range(world):
        for s in range(world):
            for qi, kj, gq, gk in ring.step_pairs(r, world, s, causal):
                assert ring.zigzag_chunks(r, world)[qi] == gq
                assert ring.zigzag_chunks((r - s) % world, world)[kj] == gk
                seen.append((gq, gk))
    n = 2 * world
    want = [(a, b) for a in range(n) for b in range(n) if not causal or b <= a]
    assert sorted(seen) == sorted(want)


@pytest.mark.parametrize("world", [1, 2, 4, 8, 16])
def test_causal_work_is_balanced_at_every_step(world):
    for s in range(world):
        work = [sum(ring.pair_work(gq, gk, True) for _, _, gq, gk in ring.step_pairs(r, world, s, True))
                for r in range(world)]
        assert work == [2.0] * world, (s, work)


@pytest.mark.parametrize("world", [1, 2, 4])
def test_shard_unshard_roundtrip(world):
    x = torch.arange(2 * 8 * world * 3 * 2).reshape(2, 8 * world, 3, 2)
    blocks = [ring.shard(x, r, world) for r in range(world)]
    c = x.shape[1] // (2 * world)
    for r, b in enumerate(blocks):
        a, z = ring.zigzag_chunks(r, world)
        assert torch.equal(b[:, :c], x[:, a * c:(a + 1) * c])
        assert torch.equal(b[:, c:], x[:, z * c:(z + 1) * c])
    assert torch.equal(ring.unshard(blocks), x)


def test_shard_rejects_indivisible_lengths():
    with pytest.raises(ValueError):
        ring.shard(torch.zeros(1, 10, 1, 1), 0, 4)


# ---------------------------------------------------------------- stand-ins

class RecordingOps:
    """Stand-ins for the block kernels on float64 CPU tensors.  Query chunk
    g holds the value g + 1, key chunk g the value 1000 (g + 1), value chunk
    g the value -(g + 1): each call checks that it was handed the chunks its
    positions name.  Forward: o += 2^gk, lse += 1.  Backward: dq += 2^gk,
    dk += 2^gq, dv += 3 * 2^gq."""

    def __init__(self):
        self.calls = []

    @staticmethod
    def _check(q, k, v, gq, gk):
        assert bool((q == gq + 1).all()), ("query chunk", gq)
        assert bool((k == 1000 * (gk + 1)).all()), ("key chunk", gk)
        assert bool((v == -(gk + 1)).all()), ("value chunk", gk)

    def fwd_block(self, q, k, v, q_pos0, k_pos0, causal, accumulate, o_acc, lse_acc, scale):
        c = q.shape[1]
        gq, gk = q_pos0 // c, k_pos0 // c
        self._check(q, k, v, gq, gk)
        self.calls.append(("fwd", gq, gk))
        if accumulate:
            o_acc += 2.0 ** gk
            lse_acc += 1.0
        else:
            o_acc.fill_(2.0 ** gk)
            lse_acc.fill_(1.0)
        return o_acc, lse_acc, None

    def bwd_block_prep(self, q, out, lse, dout, scale):
        return torch.zeros(q.shape, dtype=torch.float64)

    def bwd_block(self, q, k, v, dout, q_pos0, k_pos0, ws, causal, dk_acc, dv_acc,
                  accumulate_kv, scale):
        c = q.shape[1]
        gq, gk = q_pos0 // c, k_pos0 // c
        self._check(q, k, v, gq, gk)
        self.calls.append(("bwd", gq, gk))
        ws += 2.0 ** gk
        if accumulate_kv:
            dk_acc += 2.0 ** gq
            dv_acc += 3 * 2.0 ** gq
        else:
            dk_acc.fill_(2.0 ** gq)
            dv_acc.fill_(3 * 2.0 ** gq)
        return dk_acc, dv_acc

    def bwd_block_dq(self, q, ws, scale):
        return ws.clone()

    def cast_bf16(self, src):
        return src.clone()

    def accumulate(self, src, dst):
        dst += src
        return dst

    @staticmethod
    def empty_like(t, dtype=None):
        return torch.full(t.shape, float("nan"), dtype=torch.float64)


def _marked_inputs(world, c, B=2, Hq=2, Hkv=1, d=4):
    """Full-sequence q, k, v whose chunk g carries the markers above."""
    n = 2 * world
    g = torch.arange(n, dtype=torch.float64).repeat_interleave(c)  # chunk of every token
    shape = lambda H: (B, n * c, H, d)
    q = (g + 1).view(1, -1, 1, 1).expand(shape(Hq)).contiguous()
    k = (1000 * (g + 1)).view(1, -1, 1, 1).expand(shape(Hkv)).contiguous()
    v = (-(g + 1)).view(1, -1, 1, 1).expand(shape(Hkv)).contiguous()
    return q, k, v, g


def _expected(world, causal, g):
    """Per token: (out, lse, dq) of its query chunk and (dk, dv) of its key
    chunk, from the definition of the stand-ins."""
    n = 2 * world
    vis = lambda a, b: (not causal) or b <= a
    out = torch.tensor([sum(2.0 ** b for b in range(n) if vis(a, b)) for a in range(n)])
    cnt = torch.tensor([float(sum(1 for b in range(n) if vis(a, b))) for a in range(n)])
    dk = torch.tensor([sum(2.0 ** a for a in range(n) if vis(a, b)) for b in range(n)])
    idx = g.long()
    return out[idx], cnt[idx], dk[idx]


def _check_rank(world, rank, causal, c, ops_calls):
    q, k, v, g = _marked_inputs(world, c)
    blk = lambda x: ring.shard(x, rank, world)
    ops = RecordingOps()
    out, lse = ring.ring_attn_fwd(blk(q), blk(k), blk(v), causal=causal, ops=ops)
    dout = torch.zeros_like(blk(q))
    dq, dk, dv = ring.ring_attn_bwd(blk(q), blk(k), blk(v), out, lse, dout, causal=causal,
                                    ops=ops)
    want_out, want_cnt, want_dk = (blk(t.view(1, -1, 1, 1)) for t in _expected(world, causal, g))
    B, S2, Hq, d = out.shape
    assert torch.equal(out, want_out.expand(B, S2, Hq, d))
    assert torch.equal(lse, want_cnt.view(1, S2, 1, 1).expand(B, S2, Hq, 1)[..., 0]
                       .transpose(1, 2))
    assert torch.equal(dq, want_out.expand(B, S2, Hq, d))
    assert torch.equal(dk, want_dk.expand(B, S2, dk.shape[2], d))
    assert torch.equal(dv, 3 * want_dk.expand(B, S2, dv.shape[2], d))
    ops_calls[rank] = ops.calls


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, causal, c, calls):
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        _check_rank(world, rank, causal, c, calls)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
@pytest.mark.parametrize("causal", [True, False])
def test_ring_over_gloo_ranks_is_exact(world, causal):
    """Every rank runs the real ring driver over gloo; the key/value blocks
    and their accumulators really travel between processes."""
    c = 3
    mgr = mp.Manager()
    calls = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), causal, c, calls), nprocs=world,
                       start_method="spawn")
    n = 2 * world
    vis = [(a, b) for a in range(n) for b in range(n) if not causal or b <= a]
    for kind in ("fwd", "bwd"):
        got = sorted((gq, gk) for r in range(world) for (kd, gq, gk) in calls[r] if kd == kind)
        assert got == sorted(vis), kind


@pytest.mark.parametrize("world", [1, 2, 3, 5])
def test_single_process_emulation_matches_the_definition(world):
    """The same per-rank code driven in one process (the one-device stand-in
    for W devices)."""
    causal, c = True, 2
    q, k, v, g = _marked_inputs(world, c)
    blk = lambda x: [ring.shard(x, r, world) for r in range(world)]
    ops = RecordingOps()
    fw = ring.emulate_fwd(blk(q), blk(k), blk(v), causal=causal, ops=ops)
    outs = [o for o, _ in fw]
    lses = [l for _, l in fw]
    bw = ring.emulate_bwd(blk(q), blk(k), blk(v), outs, lses, [torch.zeros_like(x) for x in blk(q)],
                          causal=causal, ops=ops)
    want_out, want_cnt, want_dk = _expected(world, causal, g)
    B, S, Hq, d = q.shape
    assert torch.equal(ring.unshard(outs), want_out.view(1, -1, 1, 1).expand(B, S, Hq, d))
    assert torch.equal(ring.unshard([x[0] for x in bw]),
                       want_out.view(1, -1, 1, 1).expand(B, S, Hq, d))
    dk = ring.unshard([x[1] for x in bw])
    assert torch.equal(dk, want_dk.view(1, -1, 1, 1).expand(B, S, k.shape[2], d))
    assert torch.equal(ring.unshard(lses, dim=2),
                       want_cnt.view(1, 1, -1).expand(B, Hq, S))


@pytest.mark.parametrize("causal", [True, False])
def test_one_rank_ring_without_a_process_group(causal):
    """No process group: the driver runs a ring of one rank, which holds its
    own key/value block throughout and sends nothing (its backward must not
    try to hand the block's accumulators on)."""
    assert not (dist.is_available() and dist.is_initialized())
    calls = {}
    _check_rank(1, 0, causal, 3, calls)
    want = [(0, 0), (1, 0), (1, 1)] if causal else [(a, b) for a in range(2) for b in range(2)]
    for kind in ("fwd", "bwd"):
        assert sorted((gq, gk) for kd, gq, gk in calls[0] if kd == kind) == want, kind
