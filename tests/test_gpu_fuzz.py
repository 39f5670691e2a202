"""Seeded random sweep over the entry points' parameter space, each case
against the fp64 oracle: dense attention (batch, grouped-query heads, any
length, causal or not, any key/value chunk length, in-order / ring /
permuted chunk order, forward and backward), packed batches of random
lengths, S2-Attn with random groups and shifted heads, and block calls at
random positions.  The cases are drawn once from a fixed seed, so a failure
names a reproducible configuration; the sizes stay small enough for the
oracle (at most a few hundred rows per head) while spanning several tiles
and ragged tails."""

import itertools
import random

import numpy as np
import pytest
import torch

import oracle
from long_context_exact_attention_b200 import lca
from long_context_exact_attention_b200.inputs import WORKLOADS, chunk_permutation, shrink

from gpu_util import (BF16_LSE_ABS, BF16_OUT_ABS, BF16_OUT_REL, GRAD_REL, assert_fwd_close,
                      assert_grads_close, device_inputs, host, max_abs, rel_fro)

pytestmark = pytest.mark.gpu

HEADS = [(1, 1), (2, 1), (2, 2), (4, 2), (4, 1), (6, 2), (8, 2)]


def _dense_cases(n, seed):
    rnd = random.Random(seed)
    out = []
    for _ in range(n):
        S = rnd.randint(1, 700)
        Hq, Hkv = rnd.choice(HEADS)
        B = rnd.choice([1, 1, 2])
        causal = rnd.random() < 0.7
        kv_chunk = rnd.choice([0, 0, rnd.randint(1, 300), 128 * rnd.randint(1, 4)])
        order = rnd.choice(["inorder", "ring", "custom"])
        out.append((S, B, Hq, Hkv, causal, kv_chunk, order, rnd.randint(0, 10 ** 6)))
    return out


@pytest.mark.parametrize("S,B,Hq,Hkv,causal,kv_chunk,order,seed", _dense_cases(48, 2024))
def test_dense_random(S, B, Hq, Hkv, causal, kv_chunk, order, seed):
    w = shrink(WORKLOADS["llama2_7b_s32k"], S=S, B=B, Hq=Hq, Hkv=Hkv, causal=causal,
               rope=False, seed=seed % 1000)
    x = device_inputs(w)
    chunk = kv_chunk or S
    n = -(-S // chunk)
    perm = chunk_permutation(n, seed % 97) if order == "custom" else None
    out, lse = lca.attn_fwd(x["q"], x["k"], x["v"], causal=causal, kv_chunk=kv_chunk,
                            order=order, chunk_perm=perm)
    dq, dk, dv = lca.attn_bwd(x["q"], x["k"], x["v"], out, lse, x["dout"], causal=causal)
    torch.cuda.synchronize()
    lca.check()
    ro, rl = oracle.attention_forward(x["q"], x["k"], x["v"], causal)
    assert_fwd_close(host(out), host(lse), ro, rl)
    rg = oracle.attention_backward(x["q"], x["k"], x["v"], x["dout"], causal)
    assert_grads_close([host(dq), host(dk), host(dv)], rg)


def _packed_cases(n, seed):
    rnd = random.Random(seed)
    out = []
    for i in range(n):
        lengths = [rnd.randint(1, 400) for _ in range(rnd.randint(1, 5))]
        Hq, Hkv = rnd.choice(HEADS)
        out.append((tuple(lengths), Hq, Hkv, i % 3 != 2, rnd.randint(0, 10 ** 6)))
    return out


@pytest.mark.parametrize("lengths,Hq,Hkv,causal,seed", _packed_cases(16, 7))
def test_packed_random(lengths, Hq, Hkv, causal, seed):
    T = sum(lengths)
    g = torch.Generator(device="cuda").manual_seed(seed)
    mk = lambda H: (torch.randn((T, H, 128), generator=g, device="cuda") * 0.5).to(torch.bfloat16)
    q, k, v, do = mk(Hq), mk(Hkv), mk(Hkv), mk(Hq)
    cu = torch.tensor([0] + list(itertools.accumulate(lengths)), dtype=torch.int32,
                      device="cuda")
    ml = max(lengths)
    out, lse = lca.attn_fwd_varlen(q, k, v, cu, ml, causal=causal)
    dq, dk, dv = lca.attn_bwd_varlen(q, k, v, out, lse, do, cu, ml, causal=causal)
    torch.cuda.synchronize()
    lca.check()
    cu_h = cu.cpu().numpy()
    ro, rl = oracle.packed_attention_forward(q, k, v, cu_h, causal)
    assert_fwd_close(host(out)[None], host(lse)[None], ro[None], rl[None])
    rg = oracle.packed_attention_backward(q, k, v, do, cu_h, causal)
    assert_grads_close([host(dq)[None], host(dk)[None], host(dv)[None]], [r[None] for r in rg])


def _s2_cases(n, seed):
    rnd = random.Random(seed)
    out = []
    for i in range(n):
        Hq, Hkv = rnd.choice([(2, 1), (2, 2), (4, 2), (4, 4)])
        # whole-tile halves take the tile-coordinate path, others the roll
        half = rnd.choice([128, 256]) if i % 2 == 0 else rnd.randint(1, 300)
        G = 2 * half
        S = G * rnd.randint(1, 3)
        rep = Hq // Hkv
        shift = rnd.choice([s for s in range(0, Hq + 1) if (Hq - s) % rep == 0])
        out.append((S, G, Hq, Hkv, shift, rnd.random() < 0.8, rnd.randint(0, 10 ** 6)))
    return out


@pytest.mark.parametrize("S,G,Hq,Hkv,shift,causal,seed", _s2_cases(16, 11))
def test_s2_random(S, G, Hq, Hkv, shift, causal, seed):
    w = shrink(WORKLOADS["llama2_7b_s32k"], S=S, B=1, Hq=Hq, Hkv=Hkv, causal=causal,
               rope=False, seed=seed % 1000)
    x = device_inputs(w)
    out, lse = lca.s2attn_fwd(x["q"], x["k"], x["v"], G, shift, causal=causal)
    dq, dk, dv = lca.s2attn_bwd(x["q"], x["k"], x["v"], out, lse, x["dout"], G, shift,
                                causal=causal)
    torch.cuda.synchronize()
    lca.check()
    ro, rl = oracle.s2attn_forward(x["q"], x["k"], x["v"], G, shift, causal)
    assert_fwd_close(host(out), host(lse), ro, rl)
    rg = oracle.s2attn_backward(x["q"], x["k"], x["v"], x["dout"], G, shift, causal)
    assert_grads_close([host(dq), host(dk), host(dv)], rg)


def _block_cases(n, seed):
    rnd = random.Random(seed)
    out = []
    for _ in range(n):
        Sq, Sk = rnd.randint(1, 400), rnd.randint(1, 400)
        causal = rnd.random() < 0.7
        q_pos0 = 128 * rnd.randint(0, 4)
        if causal:
            k_pos0 = max(0, q_pos0 + 128 * rnd.randint(-3, 3))  # diagonal a tile multiple apart
        else:
            k_pos0 = rnd.randint(0, 600)
        out.append((Sq, Sk, q_pos0, k_pos0, causal, rnd.randint(0, 10 ** 6)))
    return out


@pytest.mark.parametrize("Sq,Sk,q_pos0,k_pos0,causal,seed", _block_cases(20, 13))
def test_block_random(Sq, Sk, q_pos0, k_pos0, causal, seed):
    B, Hq, Hkv = 1, 4, 2
    g = torch.Generator(device="cuda").manual_seed(seed)
    mk = lambda S, H: (torch.randn((B, S, H, 128), generator=g, device="cuda") * 0.5).to(
        torch.bfloat16)
    q, k, v = mk(Sq, Hq), mk(Sk, Hkv), mk(Sk, Hkv)
    out = torch.full_like(q, float("nan"))
    o_acc, lse, _ = lca.attn_fwd_block(q, k, v, q_pos0, k_pos0, causal=causal, out=out)
    torch.cuda.synchronize()
    lca.check()
    ro, rl = oracle.block_attention(q, k, v, q_pos0, k_pos0, causal)
    o, l = host(o_acc), host(lse)
    empty = np.isinf(rl)
    assert np.array_equal(np.isinf(l), empty)
    if (~empty).any():
        assert max_abs(l[~empty], rl[~empty]) <= BF16_LSE_ABS
    assert max_abs(o, ro) <= BF16_OUT_ABS
    assert max_abs(host(out), ro) <= BF16_OUT_ABS
    for h in range(Hq):
        if np.linalg.norm(ro[0, :, h]) > 0:
            assert rel_fro(o[0, :, h], ro[0, :, h]) <= BF16_OUT_REL, h
