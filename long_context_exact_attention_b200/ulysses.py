"""Ulysses sequence parallelism: exact attention with the sequence split over
ranks, by trading the sequence split for a head split around the kernels.

The 1M-context training recipe (sourcepulse project card, How It Works)
names Ulysses beside ring attention as the sequence-parallel methods it
trains with: each rank holds a contiguous shard of S/W tokens of every
head; an all-to-all turns that into all S tokens of H/W heads, each rank
runs ordinary exact attention over the whole sequence for its heads (the
library's lca_attn_fwd / lca_attn_bwd, unchanged), and a second all-to-all
returns the output to the sequence split.  The backward does the same with
q, k, v, out and dout in and dq, dk, dv out.

Grouped-query heads: query heads are split into W groups of Hq/W and
key/value heads into W groups of Hkv/W, so the query heads a rank holds read
exactly the key/value heads it holds (query head h reads key/value head
h // (Hq/Hkv)); W must divide Hkv.

The all-to-all is torch.distributed's (NCCL for device tensors; for gloo the
tensors are staged through host memory).  The packing around it is a
permutation of whole [S/W, H/W, d] slabs (``heads_to_front`` /
``from_front``), checked bit-exactly on CPU ranks.
"""

from __future__ import annotations

from typing import List

import torch

from . import lca


# ---------------------------------------------------------------- layout

def heads_to_front(x: torch.Tensor, world: int) -> torch.Tensor:
    """[B, S/W, H, d] sequence shard -> [W, B, S/W, H/W, d]: slab j holds the
    heads destined to rank j (contiguous, ready for an all-to-all)."""
    B, s, H, d = x.shape
    if H % world:
        raise ValueError(f"{H} heads do not split over {world} ranks")
    return x.view(B, s, world, H // world, d).permute(2, 0, 1, 3, 4).contiguous()


def seq_from_front(y: torch.Tensor) -> torch.Tensor:
    """[W (source rank), B, S/W, H/W, d] after the all-to-all -> [B, S, H/W, d]:
    rank i's shard holds sequence positions [i S/W, (i+1) S/W)."""
    W, B, s, h, d = y.shape
    return y.permute(1, 0, 2, 3, 4).reshape(B, W * s, h, d)


def seq_to_front(x: torch.Tensor, world: int) -> torch.Tensor:
    """[B, S, H/W, d] head shard -> [W, B, S/W, H/W, d]: slab j holds the
    sequence positions of rank j."""
    B, S, h, d = x.shape
    if S % world:
        raise ValueError(f"sequence length {S} does not split over {world} ranks")
    return x.view(B, world, S // world, h, d).permute(1, 0, 2, 3, 4).contiguous()


def heads_from_front(y: torch.Tensor) -> torch.Tensor:
    """[W (source rank = head group), B, S/W, H/W, d] -> [B, S/W, H, d]."""
    W, B, s, h, d = y.shape
    return y.permute(1, 2, 0, 3, 4).reshape(B, s, W * h, d)


def lse_seq_shard(lse: torch.Tensor, rank: int, world: int) -> torch.Tensor:
    """This rank's sequence shard of a [B, H, S] tensor."""
    S = lse.shape[-1]
    return lse[..., rank * (S // world):(rank + 1) * (S // world)]


# ---------------------------------------------------------------- transport

class DistAllToAll:
    """All-to-all of a [W, ...] slab tensor over torch.distributed: slab j
    goes to rank j, slab i of the result came from rank i."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        if group is None and not (dist.is_available() and dist.is_initialized()):
            # no process group: one rank holding the whole sequence
            self.rank, self.world, self.nccl = 0, 1, False
            return
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)
        self.nccl = dist.get_backend(group) == "nccl"

    def __call__(self, x: torch.Tensor) -> torch.Tensor:
        if self.world == 1:
            return x
        if self.nccl or not x.is_cuda:
            out = torch.empty_like(x)
            self.dist.all_to_all_single(out, x, group=self.group)
            return out
        torch.cuda.current_stream(x.device).synchronize()
        h = x.cpu()
        out = torch.empty_like(h)
        self.dist.all_to_all_single(out, h, group=self.group)
        return out.to(x.device)


def _gqa_check(Hq, Hkv, world):
    if Hq % world or Hkv % world:
        raise ValueError(f"Ulysses over {world} ranks needs it to divide both Hq={Hq} and "
                         f"Hkv={Hkv}")


def ulysses_attn_fwd(q, k, v, causal: bool = True, group=None, scale=None, a2a=None):
    """Forward on this rank.  q [B, S/W, Hq, d], k/v [B, S/W, Hkv, d]: this
    rank's contiguous shard (rank r holds positions [r S/W, (r+1) S/W)).
    Returns (out [B, S/W, Hq, d], lse [B, Hq/W, S]): the output in the
    sequence split, the lse of this rank's heads over the whole sequence
    (what ``ulysses_attn_bwd`` takes back)."""
    a2a = a2a or DistAllToAll(group)
    W = a2a.world
    _gqa_check(q.shape[2], k.shape[2], W)
    qh, kh, vh = (seq_from_front(a2a(heads_to_front(t, W))) for t in (q, k, v))
    out_h, lse_h = lca.attn_fwd(qh, kh, vh, causal=causal, scale=scale)
    out = heads_from_front(a2a(seq_to_front(out_h, W)))
    return out, lse_h


def ulysses_attn_bwd(q, k, v, out, lse_h, dout, causal: bool = True, group=None, scale=None,
                     a2a=None):
    """Backward on this rank: q, k, v, out, dout in the sequence split, lse_h
    as ``ulysses_attn_fwd`` returned it.  Returns (dq, dk, dv) in the
    sequence split."""
    a2a = a2a or DistAllToAll(group)
    W = a2a.world
    _gqa_check(q.shape[2], k.shape[2], W)
    qh, kh, vh, oh, doh = (seq_from_front(a2a(heads_to_front(t, W)))
                           for t in (q, k, v, out, dout))
    dqh, dkh, dvh = lca.attn_bwd(qh, kh, vh, oh, lse_h, doh, causal=causal, scale=scale)
    return tuple(heads_from_front(a2a(seq_to_front(t, W))) for t in (dqh, dkh, dvh))


def launches_per_step(world: int) -> int:
    """This library's kernel launches of one Ulysses forward + backward on
    one rank: the forward over the rank's heads, then the backward's row-dot,
    main kernel and dq finalize (the re-layouts around the all-to-alls are
    tensor copies, the all-to-alls the process group's)."""
    return 1 + 3


# ---------------------------------------------------------------- one-device stand-in

def emulate_all_to_all(slabs: List[torch.Tensor]) -> List[torch.Tensor]:
    """The all-to-all of W ranks done in one process: slab j of rank i
    becomes slab i of rank j."""
    W = len(slabs)
    return [torch.stack([slabs[i][j] for i in range(W)]) for j in range(W)]


def emulate_fwd(q_shards, k_shards, v_shards, causal: bool = True, scale=None):
    """Every rank's forward in one process (one device standing in for W).
    Returns per-rank (out, lse_h)."""
    W = len(q_shards)
    _gqa_check(q_shards[0].shape[2], k_shards[0].shape[2], W)
    heads = [[seq_from_front(y) for y in emulate_all_to_all([heads_to_front(t, W) for t in s])]
             for s in (q_shards, k_shards, v_shards)]
    res = [lca.attn_fwd(heads[0][r], heads[1][r], heads[2][r], causal=causal, scale=scale)
           for r in range(W)]
    outs = emulate_all_to_all([seq_to_front(o, W) for o, _ in res])
    return [(heads_from_front(outs[r]), res[r][1]) for r in range(W)]


def emulate_bwd(q_shards, k_shards, v_shards, out_shards, lse_hs, dout_shards,
                causal: bool = True, scale=None):
    """Every rank's backward in one process.  Returns per-rank (dq, dk, dv)."""
    W = len(q_shards)
    _gqa_check(q_shards[0].shape[2], k_shards[0].shape[2], W)
    heads = [[seq_from_front(y) for y in emulate_all_to_all([heads_to_front(t, W) for t in s])]
             for s in (q_shards, k_shards, v_shards, out_shards, dout_shards)]
    grads = [lca.attn_bwd(heads[0][r], heads[1][r], heads[2][r], heads[3][r], lse_hs[r],
                          heads[4][r], causal=causal, scale=scale) for r in range(W)]
    back = [emulate_all_to_all([seq_to_front(g[i], W) for g in grads]) for i in range(3)]
    return [tuple(heads_from_front(back[i][r]) for i in range(3)) for r in range(W)]
