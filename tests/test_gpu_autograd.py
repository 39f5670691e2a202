"""The autograd wrappers give exactly what the C-ABI calls give (they are
plumbing over the same entry points)."""

import pytest
import torch

from long_context_exact_attention_b200 import lca
from long_context_exact_attention_b200.autograd import attention, feedforward, s2_attention
from long_context_exact_attention_b200.inputs import FFN_WORKLOADS, WORKLOADS, make_ffn_inputs, \
    shrink

from gpu_util import device_inputs

pytestmark = pytest.mark.gpu


def leaf(t):
    return t.detach().clone().requires_grad_(True)


def test_attention_autograd_matches_direct_calls():
    w = shrink(WORKLOADS["llama2_7b_s32k"], S=640, B=1, Hq=4, Hkv=2, rope=False, seed=21)
    x = device_inputs(w)
    q, k, v = leaf(x["q"]), leaf(x["k"]), leaf(x["v"])
    out = attention(q, k, v, causal=True, kv_chunk=256, order="ring")
    out.backward(x["dout"])
    ro, rl = lca.attn_fwd(x["q"], x["k"], x["v"], causal=True, kv_chunk=256, order="ring")
    dq, dk, dv = lca.attn_bwd(x["q"], x["k"], x["v"], ro, rl, x["dout"], causal=True)
    torch.cuda.synchronize()
    assert torch.equal(out.detach(), ro)
    # dK, dV are deterministic; dQ sums float32 partials in arrival order
    assert torch.equal(k.grad, dk) and torch.equal(v.grad, dv)
    assert (q.grad.float() - dq.float()).abs().max() < 1e-2


def test_s2_attention_autograd_runs_both_paths():
    for G in (512, 200):  # tile remap, and the rolled path
        w = shrink(WORKLOADS["longlora_s2_s8k"], S=1200 if G == 200 else 1024, B=1, Hq=2, Hkv=2,
                   group=G, shift_heads=1, seed=G)
        x = device_inputs(w)
        q, k, v = leaf(x["q"]), leaf(x["k"]), leaf(x["v"])
        out = s2_attention(q, k, v, G, 1)
        out.backward(x["dout"])
        ro, rl = lca.s2attn_fwd(x["q"], x["k"], x["v"], G, 1)
        _, dk, dv = lca.s2attn_bwd(x["q"], x["k"], x["v"], ro, rl, x["dout"], G, 1)
        torch.cuda.synchronize()
        assert torch.equal(out.detach(), ro)
        assert torch.equal(k.grad, dk) and torch.equal(v.grad, dv)


def test_feedforward_autograd_matches_direct_calls():
    import dataclasses
    fw = dataclasses.replace(FFN_WORKLOADS["tiny_ffn"], T=300, h=256, f=512, block=128)
    x = make_ffn_inputs(fw, "cuda")
    g = torch.Generator(device="cuda").manual_seed(3)
    dout = torch.randn((300, 256), generator=g, device="cuda").to(torch.bfloat16)
    xs = [leaf(x[n]) for n in ("x", "w_gate", "w_up", "w_down")]
    out = feedforward(*xs, block_tokens=128)
    out.backward(dout)
    ref = lca.ffn_fwd(x["x"], x["w_gate"], x["w_up"], x["w_down"], block_tokens=128)
    dx, dwg, dwu, dwd = lca.ffn_bwd(x["x"], x["w_gate"], x["w_up"], x["w_down"], dout,
                                    block_tokens=128)
    torch.cuda.synchronize()
    assert torch.equal(out.detach(), ref) and torch.equal(xs[0].grad, dx)
    for t, g32 in zip(xs[1:], (dwg, dwu, dwd)):
        assert torch.equal(t.grad, g32.to(torch.bfloat16))


def test_ring_attention_autograd_one_rank_matches_attention():
    """Without a process group the ring is one rank holding the whole
    sequence as its zig-zag block (chunks 0 and 1): the same results as the
    dense wrapper, up to the float32 order of the block merges."""
    from long_context_exact_attention_b200.autograd import ring_attention
    w = shrink(WORKLOADS["llama3_8b_gqa_s128k"], S=512, B=1, Hq=4, Hkv=2, seed=23)
    x = device_inputs(w)
    q, k, v = leaf(x["q"]), leaf(x["k"]), leaf(x["v"])
    out = ring_attention(q, k, v, causal=True)
    out.backward(x["dout"])
    q2, k2, v2 = leaf(x["q"]), leaf(x["k"]), leaf(x["v"])
    ref = attention(q2, k2, v2, causal=True)
    ref.backward(x["dout"])
    torch.cuda.synchronize()
    assert (out.detach().float() - ref.detach().float()).abs().max() < 2e-2
    for a, b in ((q.grad, q2.grad), (k.grad, k2.grad), (v.grad, v2.grad)):
        assert ((a.float() - b.float()).norm() / b.float().norm()).item() < 2e-2
