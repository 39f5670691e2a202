"""GPU parity: the CUDA library (through its C ABI) against the fp64 oracle on
the same seeded inputs.  Small cases span several tiles, several chunks and
every chunk order and are compared element by element in full."""

import math

import numpy as np
import pytest
import torch

import oracle
from long_context_exact_attention_b200 import lca
from long_context_exact_attention_b200.inputs import WORKLOADS, chunk_permutation, shrink

from gpu_util import (assert_fwd_close, assert_grads_close, device_inputs, host, max_abs,
                      rel_fro)

pytestmark = pytest.mark.gpu

BASE = WORKLOADS["llama2_7b_s32k"]


def small(S=512, Hq=4, Hkv=4, B=2, causal=True, seed=11, rope=False, **kw):
    return shrink(BASE, S=S, Hq=Hq, Hkv=Hkv, B=B, causal=causal, seed=seed, rope=rope, **kw)


# --------------------------------------------------------------- float32 path

@pytest.mark.parametrize("order", ["inorder", "ring", "custom"])
def test_fp32_tiny_workload_fwd_bwd(order):
    w = WORKLOADS["tiny_fp32_s256"]
    x = device_inputs(w)
    perm = chunk_permutation(w.S // w.kv_chunk, 5) if order == "custom" else None
    out, lse = lca.attn_fwd(x["q"], x["k"], x["v"], causal=True, kv_chunk=w.kv_chunk,
                            order=order, chunk_perm=perm)
    dq, dk, dv = lca.attn_bwd(x["q"], x["k"], x["v"], out, lse, x["dout"], causal=True)
    torch.cuda.synchronize()
    lca.check()
    ro, rl = oracle.attention_forward(x["q"], x["k"], x["v"], True)
    assert_fwd_close(host(out), host(lse), ro, rl, fp32=True)
    rg = oracle.attention_backward(x["q"], x["k"], x["v"], x["dout"], True)
    assert_grads_close([host(dq), host(dk), host(dv)], rg, fp32=True)


@pytest.mark.parametrize("d,Hkv,causal", [(128, 2, False), (64, 1, True)])
def test_fp32_other_shapes(d, Hkv, causal):
    w = shrink(WORKLOADS["tiny_fp32_s256"], B=2, Hq=2, Hkv=Hkv, S=192, d=d, seed=3,
               causal=causal)
    x = device_inputs(w)
    out, lse = lca.attn_fwd(x["q"], x["k"], x["v"], causal=causal, kv_chunk=64, order="ring")
    dq, dk, dv = lca.attn_bwd(x["q"], x["k"], x["v"], out, lse, x["dout"], causal=causal)
    torch.cuda.synchronize()
    ro, rl = oracle.attention_forward(x["q"], x["k"], x["v"], causal)
    assert_fwd_close(host(out), host(lse), ro, rl, fp32=True)
    rg = oracle.attention_backward(x["q"], x["k"], x["v"], x["dout"], causal)
    assert_grads_close([host(dq), host(dk), host(dv)], rg, fp32=True)


# --------------------------------------------------------------- bf16 forward

@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("Hkv", [4, 2, 1])
def test_bf16_fwd_small(causal, Hkv):
    w = small(Hkv=Hkv, causal=causal)
    x = device_inputs(w, with_dout=False)
    out, lse = lca.attn_fwd(x["q"], x["k"], x["v"], causal=causal, kv_chunk=128)
    torch.cuda.synchronize()
    lca.check()
    ro, rl = oracle.attention_forward(x["q"], x["k"], x["v"], causal)
    assert_fwd_close(host(out), host(lse), ro, rl)


@pytest.mark.parametrize("order", ["inorder", "ring", "custom"])
@pytest.mark.parametrize("kv_chunk,q_block", [(128, 0), (256, 0), (128, 256), (0, 0)])
def test_bf16_chunk_orders(order, kv_chunk, q_block):
    w = small(S=1024, B=1, Hq=2, Hkv=2, seed=12)
    x = device_inputs(w, with_dout=False)
    n = w.S // (kv_chunk or w.S)
    perm = chunk_permutation(n, 9) if order == "custom" else None
    out, lse = lca.attn_fwd(x["q"], x["k"], x["v"], causal=True, kv_chunk=kv_chunk, order=order,
                            chunk_perm=perm, q_block=q_block)
    torch.cuda.synchronize()
    ro, rl = oracle.attention_forward(x["q"], x["k"], x["v"], True)
    assert_fwd_close(host(out), host(lse), ro, rl)


def test_bf16_zero_keys_closed_form():
    # all logits 0: O_i = mean of v_0..v_i, lse_i = ln(i + 1)
    w = small(S=384, B=1, Hq=2, Hkv=2)
    x = device_inputs(w, with_dout=False)
    k = torch.zeros_like(x["k"])
    out, lse = lca.attn_fwd(x["q"], k, x["v"], causal=True, kv_chunk=128)
    torch.cuda.synchronize()
    v = host(x["v"])
    want = np.cumsum(v, axis=1) / np.arange(1, w.S + 1)[None, :, None, None]
    assert max_abs(host(out), want) <= 2e-2
    assert max_abs(host(lse), np.log(np.arange(1, w.S + 1))[None, None, :]) <= 1e-3


def test_bf16_peaky_attention():
    # q_i = alpha * k_t(i) with t(i) <= i: attention is close to one-hot, so a
    # wrong row/key pairing or a dropped tile shows up as an O(1) error.
    w = small(S=512, B=1, Hq=2, Hkv=2, seed=13)
    x = device_inputs(w, with_dout=False)
    g = torch.Generator(device="cpu").manual_seed(77)
    t = torch.stack([torch.randint(0, i + 1, (1,), generator=g) for i in range(w.S)]).view(-1)
    q = (8.0 * x["k"].float()[:, t]).to(torch.bfloat16).contiguous()
    out, lse = lca.attn_fwd(q, x["k"], x["v"], causal=True, kv_chunk=128, order="ring")
    torch.cuda.synchronize()
    ro, rl = oracle.attention_forward(q, x["k"], x["v"], True)
    assert_fwd_close(host(out), host(lse), ro, rl)
    assert max_abs(host(out), ro) <= 2e-2


def test_bf16_outputs_fully_written():
    w = small(S=256, B=1, Hq=2, Hkv=2)
    x = device_inputs(w, with_dout=False)
    out = torch.full_like(x["q"], float("nan"))
    lse = torch.full((1, 2, w.S), float("nan"), device="cuda")
    lca.attn_fwd(x["q"], x["k"], x["v"], causal=True, out=out, lse=lse)
    torch.cuda.synchronize()
    assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()


# --------------------------------------------------------------- bf16 backward

@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("Hkv", [4, 2])
def test_bf16_bwd_small(causal, Hkv):
    w = small(Hkv=Hkv, causal=causal, seed=21)
    x = device_inputs(w)
    out, lse = lca.attn_fwd(x["q"], x["k"], x["v"], causal=causal, kv_chunk=256)
    dq, dk, dv = lca.attn_bwd(x["q"], x["k"], x["v"], out, lse, x["dout"], causal=causal)
    torch.cuda.synchronize()
    lca.check()
    rg = oracle.attention_backward(x["q"], x["k"], x["v"], x["dout"], causal)
    assert_grads_close([host(dq), host(dk), host(dv)], rg)


def test_bf16_bwd_repeatable():
    w = small(S=384, B=1, Hq=2, Hkv=1, seed=22)
    x = device_inputs(w)
    out, lse = lca.attn_fwd(x["q"], x["k"], x["v"], causal=True)
    g1 = lca.attn_bwd(x["q"], x["k"], x["v"], out, lse, x["dout"], causal=True)
    g1 = [t.clone() for t in g1]
    g2 = lca.attn_bwd(x["q"], x["k"], x["v"], out, lse, x["dout"], causal=True)
    torch.cuda.synchronize()
    for a, b in zip(g1, g2):
        # dq sums float32 atomics in arbitrary order; dk/dv are deterministic
        assert rel_fro(host(a), host(b)) <= 1e-3


# --------------------------------------------------------------- S2-Attn

@pytest.mark.parametrize("S,G,H,shift,Hkv,causal", [
    (1024, 512, 4, 2, 4, True), (1024, 256, 4, 2, 4, True), (1024, 512, 4, 4, 4, False),
    (768, 256, 4, 0, 4, True), (1024, 512, 4, 2, 2, True)])
def test_s2_small(S, G, H, shift, Hkv, causal):
    w = small(S=S, B=2, Hq=H, Hkv=Hkv, seed=31)
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


def test_s2_full_group_no_shift_equals_full_attention():
    w = small(S=512, B=1, Hq=2, Hkv=2, seed=32)
    x = device_inputs(w, with_dout=False)
    o1, l1 = lca.s2attn_fwd(x["q"], x["k"], x["v"], 512, 0, causal=True)
    o2, l2 = lca.attn_fwd(x["q"], x["k"], x["v"], causal=True)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


# --------------------------------------------------------------- (O, lse) merge

def test_lse_merge_kernel():
    g = torch.Generator(device="cpu").manual_seed(5)
    rows, d = 1000, 128
    oa = torch.randn(rows, d, generator=g)
    ob = torch.randn(rows, d, generator=g)
    la = torch.randn(rows, generator=g) * 4
    lb = torch.randn(rows, generator=g) * 4
    la[::7] = -math.inf
    lb[::11] = -math.inf
    o, l = lca.lse_merge(oa.cuda(), la.cuda(), ob.cuda(), lb.cuda())
    torch.cuda.synchronize()
    ro, rl = oracle.lse_merge(oa.double().numpy(), la.double().numpy(), ob.double().numpy(),
                              lb.double().numpy())
    np.testing.assert_allclose(host(o), ro, atol=1e-5)
    np.testing.assert_array_equal(np.isinf(host(l)), np.isinf(rl))
    fin = np.isfinite(rl)
    np.testing.assert_allclose(host(l)[fin], rl[fin], atol=1e-5)


def test_merge_of_two_chunk_calls_equals_full():
    # Ring step by hand: attention of every query to key half A and to key
    # half B as two separate calls, merged on the GPU, equals full attention
    # (Ring Attention: per-block results combine in any order).  A call sees
    # only half A by duplicating it: [K_A; K_A] gives the same weights, and
    # lse grows by ln 2.
    w = shrink(WORKLOADS["tiny_fp32_s256"], B=1, Hq=2, Hkv=2, S=512, d=128, seed=33,
               causal=False)
    x = device_inputs(w, with_dout=False)
    q, k, v = x["q"], x["k"], x["v"]
    parts = []
    for s0 in (256, 0):
        kk = torch.cat([k[:, s0:s0 + 256]] * 2, 1).contiguous()
        vv = torch.cat([v[:, s0:s0 + 256]] * 2, 1).contiguous()
        o, l = lca.attn_fwd(q, kk, vv, causal=False, kv_chunk=128)
        # [B,S,H,d] -> rows ordered (b, s, h); lse [B,H,S] -> same row order
        parts.append((o.reshape(-1, 128).contiguous(),
                      (l.permute(0, 2, 1).reshape(-1) - math.log(2.0)).contiguous()))
    o, l = lca.lse_merge(parts[0][0], parts[0][1], parts[1][0], parts[1][1])
    torch.cuda.synchronize()
    ref_o, ref_l = oracle.attention_forward(q, k, v, False)
    np.testing.assert_allclose(host(o), ref_o.reshape(-1, 128), atol=1e-4)
    np.testing.assert_allclose(host(l), ref_l.transpose(0, 2, 1).reshape(-1), atol=1e-4)
