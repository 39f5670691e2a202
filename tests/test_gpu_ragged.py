"""Ragged tails: S not a multiple of the tile (the last query and key tiles
are partial), a last key/value chunk shorter than the others, and chunk
lengths that are not a multiple of the tile; forward and backward, bf16 and
fp32, against the fp64 oracle in full."""

import pytest
import torch

import oracle
from long_context_exact_attention_b200 import lca
from long_context_exact_attention_b200.inputs import WORKLOADS, chunk_permutation, shrink

from gpu_util import assert_fwd_close, assert_grads_close, device_inputs, host

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("S,B,Hq,Hkv,causal,kv_chunk,order", [
    (1000, 2, 4, 2, True, 256, "ring"),
    (300, 1, 2, 2, False, 128, "inorder"),
    (129, 1, 2, 1, True, 0, "inorder"),
    (65, 2, 2, 2, False, 0, "inorder"),
    (777, 1, 4, 4, True, 384, "custom"),
    (895, 1, 2, 2, False, 256, "ring"),
])
def test_bf16_ragged_fwd_bwd(S, B, Hq, Hkv, causal, kv_chunk, order):
    w = shrink(WORKLOADS["llama2_7b_s32k"], S=S, B=B, Hq=Hq, Hkv=Hkv, causal=causal,
               rope=False, seed=61 + S)
    x = device_inputs(w)
    n = -(-S // (kv_chunk or 128 * (-(-S // 128))))
    perm = chunk_permutation(n, 3) if order == "custom" else None
    out, lse = lca.attn_fwd(x["q"], x["k"], x["v"], causal=causal, kv_chunk=kv_chunk,
                            order=order, chunk_perm=perm)
    dq, dk, dv = lca.attn_bwd(x["q"], x["k"], x["v"], out, lse, x["dout"], causal=causal)
    torch.cuda.synchronize()
    lca.check()
    ro, rl = oracle.attention_forward(x["q"], x["k"], x["v"], causal)
    assert_fwd_close(host(out), host(lse), ro, rl)
    rg = oracle.attention_backward(x["q"], x["k"], x["v"], x["dout"], causal)
    assert_grads_close([host(dq), host(dk), host(dv)], rg)


@pytest.mark.parametrize("S,B,Hkv,causal,kv_chunk", [(100, 1, 2, True, 64),
                                                      (200, 2, 1, False, 128)])
def test_fp32_ragged_fwd_bwd(S, B, Hkv, causal, kv_chunk):
    w = shrink(WORKLOADS["tiny_fp32_s256"], S=S, B=B, Hq=2, Hkv=Hkv, causal=causal, seed=71)
    x = device_inputs(w)
    out, lse = lca.attn_fwd(x["q"], x["k"], x["v"], causal=causal, kv_chunk=kv_chunk,
                            order="ring")
    dq, dk, dv = lca.attn_bwd(x["q"], x["k"], x["v"], out, lse, x["dout"], causal=causal)
    torch.cuda.synchronize()
    ro, rl = oracle.attention_forward(x["q"], x["k"], x["v"], causal)
    assert_fwd_close(host(out), host(lse), ro, rl, fp32=True)
    rg = oracle.attention_backward(x["q"], x["k"], x["v"], x["dout"], causal)
    assert_grads_close([host(dq), host(dk), host(dv)], rg, fp32=True)


def test_ragged_outputs_leave_neighbours_untouched():
    # the last partial tile must not write past row S-1 of its own batch
    w = shrink(WORKLOADS["llama2_7b_s32k"], S=200, B=2, Hq=2, Hkv=2, rope=False, seed=81)
    x = device_inputs(w)
    big = torch.full((2 * 200 + 64, 2, 128), float("nan"), device="cuda", dtype=torch.bfloat16)
    out = big[:400].view(2, 200, 2, 128)
    lca.attn_fwd(x["q"], x["k"], x["v"], causal=True, out=out)
    torch.cuda.synchronize()
    assert torch.isfinite(out.float()).all()
    assert torch.isnan(big[400:].float()).all()


@pytest.mark.parametrize("S,causal,kv_chunk,order,q_block", [
    (1000, True, 300, "ring", 0),
    (1000, False, 300, "inorder", 0),
    (333, True, 50, "ring", 100),
    (130, True, 1, "ring", 0),          # one key per chunk: 130 visits per query tile
    (640, False, 129, "custom", 0),
])
def test_bf16_unaligned_chunks(S, causal, kv_chunk, order, q_block):
    """kv_chunk not a multiple of the tile: tiles straddling a chunk boundary
    are visited once per chunk, each visit masked to its chunk's keys."""
    w = shrink(WORKLOADS["llama2_7b_s32k"], S=S, B=1, Hq=2, Hkv=1, causal=causal, rope=False,
               seed=91 + kv_chunk)
    x = device_inputs(w, with_dout=False)
    perm = chunk_permutation(-(-S // kv_chunk), 5) if order == "custom" else None
    out, lse = lca.attn_fwd(x["q"], x["k"], x["v"], causal=causal, kv_chunk=kv_chunk,
                            order=order, chunk_perm=perm, q_block=q_block)
    torch.cuda.synchronize()
    lca.check()
    ro, rl = oracle.attention_forward(x["q"], x["k"], x["v"], causal)
    assert_fwd_close(host(out), host(lse), ro, rl)


@pytest.mark.parametrize("S,kv_chunk,order", [(200, 37, "ring"), (150, 64, "custom")])
def test_fp32_unaligned_chunks(S, kv_chunk, order):
    w = shrink(WORKLOADS["tiny_fp32_s256"], S=S, B=1, Hq=2, Hkv=2, causal=True, seed=97)
    x = device_inputs(w, with_dout=False)
    perm = chunk_permutation(-(-S // kv_chunk), 7) if order == "custom" else None
    out, lse = lca.attn_fwd(x["q"], x["k"], x["v"], causal=True, kv_chunk=kv_chunk,
                            order=order, chunk_perm=perm)
    torch.cuda.synchronize()
    ro, rl = oracle.attention_forward(x["q"], x["k"], x["v"], True)
    assert_fwd_close(host(out), host(lse), ro, rl, fp32=True)
