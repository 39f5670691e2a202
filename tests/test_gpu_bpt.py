"""The Blockwise Transformer sweep (lca_bpt_fwd / lca_bpt_bwd): per query
block, attention over the keys the block sees, then the gated-SiLU
feedforward of the block's rows (Ring Attention with Blockwise Transformers
for Near-Infinite Context, Summary and Key points), against the oracle's
composition: oracle.attention_forward, then oracle.ffn_forward of the
attention output; backward oracle.ffn_backward, then
oracle.attention_backward with the feedforward's input gradient as dO.

The feedforward leg is checked on the GPU's own attention output (the same
input for both sides), at the feedforward tests' tolerance; the attention
legs at the attention tests' tolerances."""

import dataclasses

import numpy as np
import pytest
import torch

import oracle
from long_context_exact_attention_b200 import lca
from long_context_exact_attention_b200.inputs import (FFN_WORKLOADS, WORKLOADS, make_ffn_inputs,
                                                      make_inputs, shrink)

from gpu_util import GRAD_REL, assert_fwd_close, host, rel_fro

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("S,qb,causal", [(1024, 256, True), (700, 256, True), (640, 384, False)])
def test_bpt_matches_oracle_composition(S, qb, causal):
    Hq, Hkv, f = 4, 2, 768
    h = Hq * 128
    w = shrink(WORKLOADS["llama3_8b_gqa_s128k"], B=1, S=S, Hq=Hq, Hkv=Hkv, seed=S + qb)
    x = make_inputs(w, "cuda", with_dout=False)
    q, k, v = (x[n][0] for n in ("q", "k", "v"))
    fw = make_ffn_inputs(dataclasses.replace(FFN_WORKLOADS["tiny_ffn"], T=S, h=h, f=f,
                                             seed=S), "cuda")
    wg, wu, wd = fw["w_gate"], fw["w_up"], fw["w_down"]
    attn_out, lse, out = lca.bpt_fwd(q, k, v, wg, wu, wd, causal=causal, q_block=qb)
    g = torch.Generator(device="cuda").manual_seed(S)
    dout = torch.randn((S, h), generator=g, device="cuda").to(torch.bfloat16)
    dq, dk, dv, dwg, dwu, dwd = lca.bpt_bwd(q, k, v, wg, wu, wd, attn_out, lse, dout,
                                            causal=causal, q_block=qb)
    torch.cuda.synchronize()
    lca.check()
    # attention leg
    ro, rl = oracle.attention_forward(q[None], k[None], v[None], causal)
    assert_fwd_close(host(attn_out)[None], host(lse)[None], ro, rl)
    # feedforward leg, on the GPU's attention output
    xa = attn_out.reshape(S, h)
    rf = oracle.ffn_forward(xa, wg, wu, wd)
    assert rel_fro(host(out), rf) <= 1e-2
    # backward: the feedforward's gradients, then attention with dO = dx
    dx_r, dwg_r, dwu_r, dwd_r = oracle.ffn_backward(xa, wg, wu, wd, dout)
    for got, want in ((dwg, dwg_r), (dwu, dwu_r), (dwd, dwd_r)):
        assert rel_fro(host(got), want) <= GRAD_REL
    dO = dx_r.reshape(1, S, Hq, 128)
    ga = oracle.attention_backward(q[None], k[None], v[None], dO, causal)
    for got, want, name in zip((dq, dk, dv), ga, ("dq", "dk", "dv")):
        assert np.isfinite(host(got)).all(), name
        assert rel_fro(host(got)[None], want) <= GRAD_REL, (name, rel_fro(host(got)[None], want))


def test_bpt_block_size_does_not_change_the_forward():
    """Blocks only bound what lives at once: the attention rows and the
    feedforward rows are computed the same way whatever the block."""
    S, Hq, Hkv, f = 768, 4, 4, 512
    w = shrink(WORKLOADS["llama2_7b_s32k"], B=1, S=S, Hq=Hq, Hkv=Hkv, rope=False, seed=5)
    x = make_inputs(w, "cuda", with_dout=False)
    q, k, v = (x[n][0] for n in ("q", "k", "v"))
    fw = make_ffn_inputs(dataclasses.replace(FFN_WORKLOADS["tiny_ffn"], T=S, h=Hq * 128, f=f,
                                             seed=6), "cuda")
    res = [lca.bpt_fwd(q, k, v, fw["w_gate"], fw["w_up"], fw["w_down"], q_block=qb)
           for qb in (128, 256, 768)]
    torch.cuda.synchronize()
    lca.check()
    for a, b in zip(res, res[1:]):
        # the attention of a row visits the same key tiles in the same order
        assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
        assert torch.equal(a[2], b[2])
