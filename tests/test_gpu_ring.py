"""GPU parity of the block entry points (one ring step) and of the ring
driver, against the fp64 oracle.

* lca_attn_fwd_block vs ``oracle.block_attention`` element by element: the
  diagonal, full, empty and partial relations, ragged blocks, non-causal
  blocks at arbitrary positions;
* a query block folded over several key blocks (both orders) vs the rows of
  full attention;
* the block backward (prep, one call per key block, dq) vs the oracle's
  gradients of those rows, per key block;
* the ring over W emulated ranks in one process, and over two processes
  sharing the one GPU with host-staged gloo transfers (no kernel waits on
  another process), vs full-sequence attention and its gradients.
"""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from long_context_exact_attention_b200 import lca, ring
from long_context_exact_attention_b200.inputs import WORKLOADS, make_inputs, shrink

from gpu_util import (BF16_LSE_ABS, BF16_OUT_ABS, BF16_OUT_REL, GRAD_REL, assert_fwd_close,
                      assert_grads_close, host, max_abs, rel_fro)

pytestmark = pytest.mark.gpu

BASE = WORKLOADS["llama3_8b_gqa_s128k"]


def _inputs(B, S, Hq, Hkv, seed):
    w = shrink(BASE, B=B, S=S, Hq=Hq, Hkv=Hkv, seed=seed)
    return make_inputs(w, "cuda", with_dout=True)


def _rand(B, S, H, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    return (torch.randn((B, S, H, 128), generator=g, device="cuda") * 0.5).to(torch.bfloat16)


def _assert_block_close(o_acc, lse, out, ro, rl):
    """Block partial vs the oracle; rows that see no key are (0, -inf)."""
    o, l = host(o_acc), host(lse)
    empty = np.isinf(rl)
    assert np.array_equal(np.isinf(l), empty)
    assert (l[np.isinf(l)] < 0).all()
    assert max_abs(l[~empty], rl[~empty]) <= BF16_LSE_ABS if (~empty).any() else True
    assert max_abs(o, ro) <= BF16_OUT_ABS, max_abs(o, ro)
    e_rows = empty.transpose(0, 2, 1)  # [B, Sq, Hq]
    assert (o[e_rows] == 0).all()
    if out is not None:
        assert max_abs(host(out), ro) <= BF16_OUT_ABS
    for b in range(o.shape[0]):
        for h in range(o.shape[2]):
            if np.linalg.norm(ro[b, :, h]) > 0:
                assert rel_fro(o[b, :, h], ro[b, :, h]) <= BF16_OUT_REL, (b, h)


@pytest.mark.parametrize("Sq,Sk,q_pos0,k_pos0,causal", [
    (256, 256, 0, 0, True),         # diagonal
    (384, 256, 512, 0, True),       # keys wholly before the queries: full
    (256, 384, 128, 0, True),       # the diagonal one tile into the key block
    (256, 300, 0, 128, True),       # the first query tile sees nothing; ragged keys
    (300, 200, 100, 100, True),     # ragged queries and keys on the diagonal
    (256, 256, 0, 512, True),       # keys wholly after the queries: empty
    (200, 333, 7, 1000, False),     # non-causal, arbitrary positions
])
def test_fwd_block_matches_oracle(Sq, Sk, q_pos0, k_pos0, causal):
    B, Hq, Hkv = 2, 4, 2
    q, k, v = _rand(B, Sq, Hq, 1), _rand(B, Sk, Hkv, 2), _rand(B, Sk, Hkv, 3)
    out = torch.full_like(q, float("nan"))
    o_acc, lse, _ = lca.attn_fwd_block(q, k, v, q_pos0, k_pos0, causal=causal, out=out)
    torch.cuda.synchronize()
    lca.check()
    ro, rl = oracle.block_attention(q, k, v, q_pos0, k_pos0, causal)
    _assert_block_close(o_acc, lse, out, ro, rl)


@pytest.mark.parametrize("reverse", [False, True])
def test_fwd_blocks_fold_to_full_attention(reverse):
    B, S, Hq, Hkv = 1, 1024, 4, 2
    x = _inputs(B, S, Hq, Hkv, 21)
    r0, r1 = 256, 768
    q = x["q"][:, r0:r1].contiguous()
    cuts = [0, 100, 256, 640, 1024]  # full (ragged), full, diagonal, diagonal
    blocks = list(zip(cuts[:-1], cuts[1:]))
    if reverse:
        blocks = blocks[::-1]
    o_acc = lse = None
    out = torch.empty_like(q)
    for i, (a, b) in enumerate(blocks):
        o_acc, lse, _ = lca.attn_fwd_block(q, x["k"][:, a:b].contiguous(),
                                           x["v"][:, a:b].contiguous(), r0, a, causal=True,
                                           accumulate=i > 0, o_acc=o_acc, lse_acc=lse,
                                           out=out if i == len(blocks) - 1 else None)
    torch.cuda.synchronize()
    lca.check()
    ro, rl = oracle.attention_forward(x["q"], x["k"], x["v"], True)
    assert_fwd_close(host(out), host(lse), ro[:, r0:r1], rl[:, :, r0:r1])
    assert max_abs(host(o_acc), ro[:, r0:r1]) <= BF16_OUT_ABS


@pytest.mark.parametrize("mode", ["accumulate", "overwrite", "bf16"])
def test_bwd_blocks_match_oracle_per_key_block(mode):
    B, S, Hq, Hkv = 2, 768, 4, 2
    x = _inputs(B, S, Hq, Hkv, 22)
    out, lse = lca.attn_fwd(x["q"], x["k"], x["v"], causal=True)
    r0, r1 = 128, 640
    sl = lambda t: t[:, r0:r1].contiguous()
    q, do = sl(x["q"]), sl(x["dout"])
    ws = lca.attn_bwd_block_prep(q, sl(out), lse[:, :, r0:r1].contiguous(), do)
    got = {}
    for a, b in [(0, 256), (256, 512), (512, 768)]:
        k, v = x["k"][:, a:b].contiguous(), x["v"][:, a:b].contiguous()
        if mode == "bf16":
            dk, dv = lca.attn_bwd_block(q, k, v, do, r0, a, ws, causal=True)
        else:
            dk = torch.full(k.shape, 0.0 if mode == "accumulate" else float("nan"),
                            device="cuda", dtype=torch.float32)
            dv = torch.full_like(dk, 0.0 if mode == "accumulate" else float("nan"))
            lca.attn_bwd_block(q, k, v, do, r0, a, ws, causal=True, dk_acc=dk, dv_acc=dv,
                               accumulate_kv=mode == "accumulate")
        got[a, b] = (dk, dv)
    dq = lca.attn_bwd_block_dq(q, ws)
    torch.cuda.synchronize()
    lca.check()
    rows = np.arange(r0, r1)
    rep = Hq // Hkv
    for bb in range(B):
        for g in range(Hkv):
            dq_r, dk_r, dv_r = oracle.attention_backward_rows(x["q"], x["k"], x["v"], x["dout"],
                                                              True, bb, g, rows)
            assert rel_fro(host(dq[bb, :, g * rep:(g + 1) * rep]), dq_r) <= GRAD_REL
            for (a, b), (dk, dv) in got.items():
                assert rel_fro(host(dk[bb, :, g]), dk_r[a:b]) <= GRAD_REL, (bb, g, a)
                assert rel_fro(host(dv[bb, :, g]), dv_r[a:b]) <= GRAD_REL, (bb, g, a)


@pytest.mark.parametrize("world,B", [(1, 1), (2, 2), (4, 1)])
def test_ring_emulated_matches_oracle(world, B):
    c = 256
    S, Hq, Hkv = 2 * world * c, 4, 2
    x = _inputs(B, S, Hq, Hkv, 30 + world)
    blk = lambda t: [ring.shard(t, r, world) for r in range(world)]
    fw = ring.emulate_fwd(blk(x["q"]), blk(x["k"]), blk(x["v"]), causal=True)
    bw = ring.emulate_bwd(blk(x["q"]), blk(x["k"]), blk(x["v"]), [o for o, _ in fw],
                          [l for _, l in fw], blk(x["dout"]), causal=True)
    torch.cuda.synchronize()
    lca.check()
    out = ring.unshard([o for o, _ in fw])
    lse = ring.unshard([l for _, l in fw], dim=2)
    ro, rl = oracle.attention_forward(x["q"], x["k"], x["v"], True)
    assert_fwd_close(host(out), host(lse), ro, rl)
    grads = [host(ring.unshard([g[i] for g in bw])) for i in range(3)]
    assert_grads_close(grads, oracle.attention_backward(x["q"], x["k"], x["v"], x["dout"], True))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _ring_worker(rank, world, port, path, B, S, Hq, Hkv, seed):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    sys.path.insert(0, os.path.join(root, "tests"))
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        torch.cuda.set_device(0)
        x = _inputs(B, S, Hq, Hkv, seed)  # the same seeded draw on every rank
        blk = {n: ring.shard(t, rank, world) for n, t in x.items()}
        out, lse = ring.ring_attn_fwd(blk["q"], blk["k"], blk["v"], causal=True)
        dq, dk, dv = ring.ring_attn_bwd(blk["q"], blk["k"], blk["v"], out, lse, blk["dout"],
                                        causal=True)
        torch.cuda.synchronize()
        lca.check()
        torch.save({n: t.cpu() for n, t in dict(out=out, lse=lse, dq=dq, dk=dk, dv=dv).items()},
                   os.path.join(path, f"rank{rank}.pt"))
    finally:
        dist.destroy_process_group()


def test_ring_two_processes_on_one_gpu(tmp_path):
    """Two ranks as two processes on the one GPU; the blocks travel through
    host memory over gloo, so no kernel ever waits for the other process."""
    world, B, S, Hq, Hkv, seed = 2, 1, 1024, 4, 2, 40
    mp.start_processes(_ring_worker, args=(world, _free_port(), str(tmp_path), B, S, Hq, Hkv,
                                           seed),
                       nprocs=world, start_method="spawn")
    res = [torch.load(os.path.join(tmp_path, f"rank{r}.pt")) for r in range(world)]
    x = _inputs(B, S, Hq, Hkv, seed)
    ro, rl = oracle.attention_forward(x["q"], x["k"], x["v"], True)
    out = ring.unshard([r["out"] for r in res])
    lse = ring.unshard([r["lse"] for r in res], dim=2)
    assert_fwd_close(host(out), host(lse), ro, rl)
    grads = [host(ring.unshard([r[n] for r in res])) for n in ("dq", "dk", "dv")]
    assert_grads_close(grads, oracle.attention_backward(x["q"], x["k"], x["v"], x["dout"], True))
