"""Ulysses sequence parallelism on the GPU against the fp64 oracle: W ranks
emulated in one process (the all-to-all as tensor moves on one device), and
two ranks as two processes sharing the one GPU with a host-staged gloo
all-to-all (no kernel waits on the other process).  Outputs and gradients
in the sequence split are reassembled and compared with full-sequence
attention."""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from long_context_exact_attention_b200 import lca, ulysses as U
from long_context_exact_attention_b200.inputs import WORKLOADS, make_inputs, shrink

from gpu_util import assert_fwd_close, assert_grads_close, host

pytestmark = pytest.mark.gpu


def _inputs(B, S, Hq, Hkv, seed):
    w = shrink(WORKLOADS["llama3_8b_gqa_s128k"], B=B, S=S, Hq=Hq, Hkv=Hkv, seed=seed)
    return make_inputs(w, "cuda", with_dout=True)


def _shard(x, r, W):
    s = x.shape[1] // W
    return x[:, r * s:(r + 1) * s].contiguous()


@pytest.mark.parametrize("W,B,S,Hq,Hkv", [(2, 1, 768, 4, 2), (4, 2, 512, 8, 4)])
def test_ulysses_emulated_matches_oracle(W, B, S, Hq, Hkv):
    x = _inputs(B, S, Hq, Hkv, 50 + W)
    sh = {n: [_shard(t, r, W) for r in range(W)] for n, t in x.items()}
    fw = U.emulate_fwd(sh["q"], sh["k"], sh["v"], causal=True)
    bw = U.emulate_bwd(sh["q"], sh["k"], sh["v"], [o for o, _ in fw], [l for _, l in fw],
                       sh["dout"], causal=True)
    torch.cuda.synchronize()
    lca.check()
    out = torch.cat([o for o, _ in fw], dim=1)
    lse = torch.cat([l for _, l in fw], dim=1)  # rank j holds heads [j Hq/W, (j+1) Hq/W)
    ro, rl = oracle.attention_forward(x["q"], x["k"], x["v"], True)
    assert_fwd_close(host(out), host(lse), ro, rl)
    grads = [host(torch.cat([g[i] for g in bw], dim=1)) for i in range(3)]
    assert_grads_close(grads, oracle.attention_backward(x["q"], x["k"], x["v"], x["dout"], True))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, path, B, S, Hq, Hkv, seed):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    sys.path.insert(0, os.path.join(root, "tests"))
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        torch.cuda.set_device(0)
        x = _inputs(B, S, Hq, Hkv, seed)
        sh = {n: _shard(t, rank, world) for n, t in x.items()}
        out, lse_h = U.ulysses_attn_fwd(sh["q"], sh["k"], sh["v"], causal=True)
        dq, dk, dv = U.ulysses_attn_bwd(sh["q"], sh["k"], sh["v"], out, lse_h, sh["dout"],
                                        causal=True)
        torch.cuda.synchronize()
        lca.check()
        torch.save({n: t.cpu() for n, t in dict(out=out, lse=lse_h, dq=dq, dk=dk, dv=dv).items()},
                   os.path.join(path, f"rank{rank}.pt"))
    finally:
        dist.destroy_process_group()


def test_ulysses_two_processes_on_one_gpu(tmp_path):
    world, B, S, Hq, Hkv, seed = 2, 1, 1024, 4, 2, 60
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path), B, S, Hq, Hkv, seed),
                       nprocs=world, start_method="spawn")
    res = [torch.load(os.path.join(tmp_path, f"rank{r}.pt")) for r in range(world)]
    x = _inputs(B, S, Hq, Hkv, seed)
    ro, rl = oracle.attention_forward(x["q"], x["k"], x["v"], True)
    out = torch.cat([r["out"] for r in res], dim=1)
    lse = torch.cat([r["lse"] for r in res], dim=1)
    assert_fwd_close(host(out), host(lse), ro, rl)
    grads = [host(torch.cat([r[n] for r in res], dim=1)) for n in ("dq", "dk", "dv")]
    assert_grads_close(grads, oracle.attention_backward(x["q"], x["k"], x["v"], x["dout"], True))
