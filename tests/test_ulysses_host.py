"""Ulysses' re-layout on CPU (no GPU, no oracle): the all-to-all that turns a
sequence split into a head split and back is a permutation of whole slabs,
checked bit for bit against slices of a global tensor, in one process and
over gloo ranks."""

import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from long_context_exact_attention_b200 import ulysses as U


def _global(B, S, H, d):
    return torch.arange(B * S * H * d, dtype=torch.float64).reshape(B, S, H, d)


def _shard(x, r, W):
    s = x.shape[1] // W
    return x[:, r * s:(r + 1) * s].contiguous()


@pytest.mark.parametrize("W,B,S,H", [(1, 1, 8, 4), (2, 2, 8, 4), (4, 1, 16, 8), (4, 3, 12, 4)])
def test_emulated_layout_roundtrip_is_exact(W, B, S, H):
    d = 3
    x = _global(B, S, H, d)
    shards = [_shard(x, r, W) for r in range(W)]
    heads = [U.seq_from_front(y) for y in
             U.emulate_all_to_all([U.heads_to_front(t, W) for t in shards])]
    h = H // W
    for j in range(W):
        assert torch.equal(heads[j], x[:, :, j * h:(j + 1) * h])   # all tokens, own heads
    back = [U.heads_from_front(y) for y in
            U.emulate_all_to_all([U.seq_to_front(t, W) for t in heads])]
    for r in range(W):
        assert torch.equal(back[r], shards[r])


def test_lse_seq_shard():
    lse = torch.arange(2 * 3 * 8.).reshape(2, 3, 8)
    assert torch.equal(U.lse_seq_shard(lse, 1, 4), lse[..., 2:4])


def test_head_counts_must_split():
    with pytest.raises(ValueError):
        U.heads_to_front(torch.zeros(1, 4, 6, 2), 4)
    with pytest.raises(ValueError):
        U._gqa_check(32, 2, 4)
    U._gqa_check(32, 8, 8)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port):
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        B, S, H, d = 2, 4 * world, 2 * world, 3
        x = _global(B, S, H, d)
        a2a = U.DistAllToAll()
        heads = U.seq_from_front(a2a(U.heads_to_front(_shard(x, rank, world), world)))
        h = H // world
        assert torch.equal(heads, x[:, :, rank * h:(rank + 1) * h])
        back = U.heads_from_front(a2a(U.seq_to_front(heads, world)))
        assert torch.equal(back, _shard(x, rank, world))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_gloo_all_to_all_layout_is_exact(world):
    mp.start_processes(_worker, args=(world, _free_port()), nprocs=world, start_method="spawn")
