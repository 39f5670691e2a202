"""Ring attention across ranks: exact causal attention with the sequence
split over devices.

Ring Attention with Blockwise Transformers for Near-Infinite Context
(Summary and Key points): every host keeps its own block of queries; the
key/value blocks move from host to host around a ring, each host attends its
queries to every block as it arrives and overlaps sending the block on with
that computation; the partial results combine into the exact answer because
the log-sum-exp merge does not depend on the order of the blocks.  In the
backward pass the key/value gradients are accumulated in buffers that travel
with their block and end where the block started.

Partitioning (load-balanced for the causal mask): the S tokens are cut into
2W chunks of c = S / (2W) tokens and rank r holds chunks r and 2W-1-r, in
that order, as one local block of 2c rows ("zig-zag").  A key chunk is
visible in full to a later query chunk, on the diagonal to its own, and not
at all to an earlier one, so at every step every rank attends exactly two
chunk-pairs' worth of keys:

  step 0 (its own keys):   (r, r) diagonal, (2W-1-r, r) full, (2W-1-r, 2W-1-r) diagonal
  keys of rank src < r:    both query chunks against key chunk src, full
  keys of rank src > r:    query chunk 2W-1-r against both key chunks, full

The per-step work goes through the library's block entry points
(lca_attn_fwd_block, lca_attn_bwd_block, ...): every launch is one query
chunk against one key chunk, so every operand is a contiguous tensor for any
batch size.  Transfers are point-to-point sends to rank r+1 and receives
from rank r-1 (NCCL over NVLink on GPUs), posted before the step's kernels
so they overlap them.

The per-rank algorithm is written once, as a generator that yields its
transfers; three drivers run it:
  * ``ring_attn_fwd`` / ``ring_attn_bwd``: one rank per process over
    torch.distributed (NCCL for device tensors; gloo with host staging for
    testing several ranks on one device);
  * ``emulate_fwd`` / ``emulate_bwd``: all W ranks in one process on one
    device, the transfers done as device copies (no two kernels ever wait on
    each other), for checking and measuring the per-rank work on one GPU.
"""

from __future__ import annotations

import dataclasses
from typing import Callable, List, Optional

import torch

from . import lca


# ---------------------------------------------------------------- partition

def zigzag_chunks(rank: int, world: int):
    """Global chunk indices held by `rank` (of 2*world chunks), in local order."""
    return rank, 2 * world - 1 - rank


def shard(x: torch.Tensor, rank: int, world: int, dim: int = 1) -> torch.Tensor:
    """This rank's zig-zag block of a full-sequence tensor (token axis `dim`)."""
    S = x.shape[dim]
    if S % (2 * world):
        raise ValueError(f"sequence length {S} is not a multiple of 2 * world = {2 * world}")
    c = S // (2 * world)
    a, b = zigzag_chunks(rank, world)
    return torch.cat([x.narrow(dim, a * c, c), x.narrow(dim, b * c, c)], dim=dim).contiguous()


def unshard(blocks: List[torch.Tensor], dim: int = 1) -> torch.Tensor:
    """Reassemble the full sequence from every rank's zig-zag block."""
    world = len(blocks)
    c = blocks[0].shape[dim] // 2
    chunks = [None] * (2 * world)
    for r, blk in enumerate(blocks):
        a, b = zigzag_chunks(r, world)
        chunks[a] = blk.narrow(dim, 0, c)
        chunks[b] = blk.narrow(dim, c, c)
    return torch.cat(chunks, dim=dim)


def step_pairs(rank: int, world: int, step: int, causal: bool):
    """Launches of one step: (local query chunk, local key chunk, global
    query chunk, global key chunk) for every pair with a visible key."""
    src = (rank - step) % world
    gq = zigzag_chunks(rank, world)
    gk = zigzag_chunks(src, world)
    return [(qi, kj, gq[qi], gk[kj]) for qi in (0, 1) for kj in (0, 1)
            if not causal or gk[kj] <= gq[qi]]


def pair_work(gq: int, gk: int, causal: bool) -> float:
    """Work of one chunk pair in units of c*c visible (query, key) pairs
    (a diagonal pair counts half)."""
    if not causal or gk < gq:
        return 1.0
    return 0.5 if gk == gq else 0.0


# ---------------------------------------------------------------- protocol

@dataclasses.dataclass
class Exchange:
    """Send `send` to rank r+1 and receive `recv` from rank r-1."""
    send: torch.Tensor
    recv: torch.Tensor


@dataclasses.dataclass
class Wait:
    """Block the stream (or the host) until an earlier exchange is done."""
    handle: object


class KernelOps:
    """The library's block entry points (what a step computes).  Tests of the
    schedule substitute recording stand-ins with the same signatures."""

    fwd_block = staticmethod(lca.attn_fwd_block)
    bwd_block_prep = staticmethod(lca.attn_bwd_block_prep)
    bwd_block = staticmethod(lca.attn_bwd_block)
    bwd_block_dq = staticmethod(lca.attn_bwd_block_dq)
    cast_bf16 = staticmethod(lca.cast_bf16)
    accumulate = staticmethod(lca.accumulate)

    @staticmethod
    def empty_like(t, dtype=None):
        return torch.empty(t.shape, device=t.device, dtype=dtype or t.dtype)


def _chunks(x: torch.Tensor, c: int):
    return x[:, :c].contiguous(), x[:, c:].contiguous()


def _fwd_rank(rank: int, world: int, q, k, v, causal: bool, scale, ops):
    """One rank's forward.  q [B, 2c, Hq, d], k/v [B, 2c, Hkv, d] (its zig-zag
    block).  Returns (out [B, 2c, Hq, d] bf16, lse [B, Hq, 2c] float32)."""
    c = q.shape[1] // 2
    qc = _chunks(q, c)
    kv = torch.stack([*_chunks(k, c), *_chunks(v, c)])  # k0 k1 v0 v1, one buffer to send
    nxt = torch.empty_like(kv)
    B, _, Hq, d = q.shape
    o_acc = torch.empty((2, B, c, Hq, d), device=q.device, dtype=torch.float32)
    lse = torch.empty((2, B, Hq, c), device=q.device, dtype=torch.float32)
    started = [False, False]
    for step in range(world):
        h = (yield Exchange(kv, nxt)) if step + 1 < world else None
        for qi, kj, gq, gk in step_pairs(rank, world, step, causal):
            ops.fwd_block(qc[qi], kv[kj], kv[2 + kj], gq * c, gk * c, causal=causal,
                          accumulate=started[qi], o_acc=o_acc[qi], lse_acc=lse[qi], scale=scale)
            started[qi] = True
        if step + 1 < world:
            yield Wait(h)
            kv, nxt = nxt, kv
    out = ops.cast_bf16(o_acc)
    return torch.cat([out[0], out[1]], dim=1), torch.cat([lse[0], lse[1]], dim=2)


def _bwd_rank(rank: int, world: int, q, k, v, out, lse, dout, causal: bool, scale, ops):
    """One rank's backward from the forward's out and lse (the zig-zag
    layouts of ``_fwd_rank``).  Returns (dq, dk, dv), bf16."""
    c = q.shape[1] // 2
    qc, oc, dc = _chunks(q, c), _chunks(out, c), _chunks(dout, c)
    lc = lse[:, :, :c].contiguous(), lse[:, :, c:].contiguous()
    ws = [ops.bwd_block_prep(qc[i], oc[i], lc[i], dc[i], scale=scale) for i in (0, 1)]
    kv = torch.stack([*_chunks(k, c), *_chunks(v, c)])  # k0 k1 v0 v1
    kv_nxt = torch.empty_like(kv)
    # accumulators of the key/value block held: dk0 dk1 dv0 dv1 (float32)
    acc = ops.empty_like(kv, torch.float32)
    acc_nxt = ops.empty_like(kv, torch.float32)
    part = ops.empty_like(kv, torch.float32)
    h_acc = None
    for step in range(world):
        h_kv = (yield Exchange(kv, kv_nxt)) if step + 1 < world else None
        # step 0 writes straight into the own block's accumulators (both key
        # chunks are touched); later steps write a partial that is added
        # once the block's accumulators have arrived
        tgt = acc if step == 0 else part
        touched = [False, False]
        for qi, kj, gq, gk in step_pairs(rank, world, step, causal):
            ops.bwd_block(qc[qi], kv[kj], kv[2 + kj], dc[qi], gq * c, gk * c, ws[qi],
                          causal=causal, dk_acc=tgt[kj], dv_acc=tgt[2 + kj],
                          accumulate_kv=touched[kj], scale=scale)
            touched[kj] = True
        if step == 0:
            assert all(touched), "the own block's first step touches both key chunks"
        else:
            yield Wait(h_acc)
            for kj in (0, 1):
                if touched[kj]:
                    ops.accumulate(part[kj], acc[kj])
                    ops.accumulate(part[2 + kj], acc[2 + kj])
        # hand the block's accumulators on; after the last step this sends
        # every block home (rank r then holds its own block's gradients).
        # A ring of one rank holds its own block throughout.
        if world > 1:
            h_acc = yield Exchange(acc, acc_nxt)
            acc, acc_nxt = acc_nxt, acc
        if step + 1 < world:
            yield Wait(h_kv)
            kv, kv_nxt = kv_nxt, kv
    yield Wait(h_acc)
    dq = [ops.bwd_block_dq(qc[i], ws[i], scale=scale) for i in (0, 1)]
    g = ops.cast_bf16(acc)
    cat = lambda a, b: torch.cat([a, b], dim=1)
    return cat(dq[0], dq[1]), cat(g[0], g[1]), cat(g[2], g[3])


# ---------------------------------------------------------------- drivers

class DistTransport:
    """Point-to-point ring transfers over torch.distributed: NCCL moves
    device tensors directly (its own stream; ``wait`` orders the current
    stream after it); any other backend (gloo) is staged through host
    memory, synchronously."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)
        self.nccl = dist.get_backend(group) == "nccl"

    def _peer(self, r):
        g = self.group
        return r if g is None else self.dist.get_global_rank(g, r)

    def exchange(self, send, recv):
        dist = self.dist
        nxt, prv = self._peer((self.rank + 1) % self.world), self._peer((self.rank - 1) % self.world)
        if self.nccl:
            ops = [dist.P2POp(dist.isend, send, nxt, self.group),
                   dist.P2POp(dist.irecv, recv, prv, self.group)]
            return dist.batch_isend_irecv(ops)
        staged = send.is_cuda
        if staged:
            torch.cuda.current_stream(send.device).synchronize()
        s_host = send.cpu() if staged else send
        r_host = torch.empty(recv.shape, dtype=recv.dtype) if staged else recv
        ops = [dist.P2POp(dist.isend, s_host, nxt, self.group),
               dist.P2POp(dist.irecv, r_host, prv, self.group)]
        for w in dist.batch_isend_irecv(ops):
            w.wait()
        if staged:
            recv.copy_(r_host)
        return None

    def wait(self, handle):
        if handle is not None:
            for w in handle:
                w.wait()


def _drive(gen, transport):
    """Run one rank's generator against a transport; returns its result."""
    reply = None
    while True:
        try:
            msg = gen.send(reply)
        except StopIteration as stop:
            return stop.value
        if isinstance(msg, Exchange):
            reply = transport.exchange(msg.send, msg.recv)
        else:
            transport.wait(msg.handle)
            reply = None


class _NoTransport:
    """A ring of one rank exchanges nothing."""
    rank, world = 0, 1

    def exchange(self, send, recv):
        raise RuntimeError("a ring of one rank has nothing to exchange")

    def wait(self, handle):
        pass


def _transport(group):
    import torch.distributed as dist
    if group is None and not (dist.is_available() and dist.is_initialized()):
        return _NoTransport()
    return DistTransport(group)


def ring_attn_fwd(q, k, v, causal: bool = True, group=None, scale=None, ops=None):
    """Ring attention forward on this rank.  q [B, 2c, Hq, d], k/v
    [B, 2c, Hkv, d]: this rank's zig-zag block (``shard``) of the sequence;
    c must be a multiple of 128 when causal.  Every rank of `group` calls
    it together (without a process group: a ring of one rank).  Returns
    (out, lse) of this rank's block."""
    t = _transport(group)
    return _drive(_fwd_rank(t.rank, t.world, q, k, v, causal, scale, ops or KernelOps), t)


def ring_attn_bwd(q, k, v, out, lse, dout, causal: bool = True, group=None, scale=None,
                  ops=None):
    """Ring attention backward on this rank (zig-zag blocks, as
    ``ring_attn_fwd``; out and lse are its results).  Returns (dq, dk, dv)
    of this rank's block."""
    t = _transport(group)
    return _drive(_bwd_rank(t.rank, t.world, q, k, v, out, lse, dout, causal, scale,
                            ops or KernelOps), t)


def launches_per_step(world: int, causal: bool = True) -> int:
    """This library's kernel launches of one ring forward + backward on one
    rank (block forwards and a cast; per query chunk a row-dot and a dq
    finalize; block backwards, the accumulator additions of the later steps
    and a cast)."""
    pairs = [step_pairs(0, world, s, causal) for s in range(world)]
    n_blocks = sum(len(p) for p in pairs)
    adds = sum(2 * len({kj for _, kj, _, _ in p}) for p in pairs[1:])
    return (n_blocks + 1) + (2 + n_blocks + adds + 2 + 1)


def _emulate(gens):
    """Run W ranks' generators in lock step in one process: each exchange
    point is reached by every rank, then rank r's send is copied into rank
    r+1's receive buffer (stream-ordered device copies)."""
    W = len(gens)
    replies = [None] * W
    results = [None] * W
    live = list(range(W))
    while live:
        msgs = {}
        for r in live:
            try:
                msgs[r] = gens[r].send(replies[r])
            except StopIteration as stop:
                results[r] = stop.value
        done = [r for r in live if r not in msgs]
        if done and len(done) != len(live):
            raise RuntimeError("ranks of the emulated ring fell out of step")
        live = [r for r in live if r in msgs]
        if not live:
            break
        kinds = {type(msgs[r]) for r in live}
        if len(kinds) != 1:
            raise RuntimeError("ranks of the emulated ring fell out of step")
        if kinds == {Exchange}:
            for r in live:
                msgs[(r + 1) % W].recv.copy_(msgs[r].send)
        replies = [None] * W
    return results


def emulate_fwd(q_blocks, k_blocks, v_blocks, causal: bool = True, scale=None, ops=None):
    """Every rank's forward, run in one process (one device stands in for W).
    Lists of per-rank zig-zag blocks in, list of per-rank (out, lse) out."""
    W = len(q_blocks)
    ops = ops or KernelOps
    return _emulate([_fwd_rank(r, W, q_blocks[r], k_blocks[r], v_blocks[r], causal, scale, ops)
                     for r in range(W)])


def emulate_bwd(q_blocks, k_blocks, v_blocks, out_blocks, lse_blocks, dout_blocks,
                causal: bool = True, scale=None, ops=None):
    """Every rank's backward in one process; list of per-rank (dq, dk, dv)."""
    W = len(q_blocks)
    ops = ops or KernelOps
    return _emulate([_bwd_rank(r, W, q_blocks[r], k_blocks[r], v_blocks[r], out_blocks[r],
                               lse_blocks[r], dout_blocks[r], causal, scale, ops)
                     for r in range(W)])
