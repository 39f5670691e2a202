"""S2-Attn with groups whose half is not a whole number of tiles (LongLoRA's
100K context uses S = 100000, group 25000): the heads are rolled into the
workspace, the groups run as a packed batch and the results are rolled back.
Forward and backward against the oracle's literal shift / group / attend /
unshift, bf16 (with grouped-query heads) and fp32."""

import pytest
import torch

import oracle
from long_context_exact_attention_b200 import lca
from long_context_exact_attention_b200.inputs import WORKLOADS, shrink

from gpu_util import assert_fwd_close, assert_grads_close, device_inputs, host

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("S,G,B,Hq,Hkv,shift,causal", [
    (6000, 1500, 2, 4, 2, 2, True),     # half a group = 750 tokens, GQA
    (6000, 1500, 1, 2, 2, 1, False),
    (10000, 2500, 1, 2, 2, 1, True),    # LongLoRA's 100K proportions, scaled by 1/10
    (1200, 200, 1, 2, 2, 2, True),      # every head shifted, 6 groups
])
def test_bf16_s2_unaligned_group(S, G, B, Hq, Hkv, shift, causal):
    w = shrink(WORKLOADS["longlora_s2_s8k"], S=S, B=B, Hq=Hq, Hkv=Hkv, causal=causal,
               group=G, shift_heads=shift, seed=S + G)
    x = device_inputs(w)
    fws, bws = lca.s2attn_workspace_sizes(x["q"], x["k"], G, shift)
    assert fws > 0 and bws > lca.workspace_size(x["q"], x["k"])
    out, lse = lca.s2attn_fwd(x["q"], x["k"], x["v"], G, shift, causal=causal)
    dq, dk, dv = lca.s2attn_bwd(x["q"], x["k"], x["v"], out, lse, x["dout"], G, shift,
                                causal=causal)
    torch.cuda.synchronize()
    lca.check()
    ro, rl = oracle.s2attn_forward(x["q"], x["k"], x["v"], G, shift, causal)
    assert_fwd_close(host(out), host(lse), ro, rl)
    rg = oracle.s2attn_backward(x["q"], x["k"], x["v"], x["dout"], G, shift, causal)
    assert_grads_close([host(dq), host(dk), host(dv)], rg)


def test_fp32_s2_unaligned_group():
    # fp32 tiles are 64 tokens; half a group of 50 is not a whole tile
    w = shrink(WORKLOADS["tiny_fp32_s256"], S=400, B=1, Hq=2, Hkv=2, causal=True, group=100,
               shift_heads=1, seed=5)
    x = device_inputs(w)
    out, lse = lca.s2attn_fwd(x["q"], x["k"], x["v"], 100, 1, causal=True)
    dq, dk, dv = lca.s2attn_bwd(x["q"], x["k"], x["v"], out, lse, x["dout"], 100, 1, causal=True)
    torch.cuda.synchronize()
    ro, rl = oracle.s2attn_forward(x["q"], x["k"], x["v"], 100, 1, True)
    assert_fwd_close(host(out), host(lse), ro, rl, fp32=True)
    rg = oracle.s2attn_backward(x["q"], x["k"], x["v"], x["dout"], 100, 1, True)
    assert_grads_close([host(dq), host(dk), host(dv)], rg, fp32=True)


def test_s2_without_workspace_is_refused():
    w = shrink(WORKLOADS["longlora_s2_s8k"], S=1200, B=1, Hq=2, Hkv=2, group=200,
               shift_heads=1, seed=3)
    x = device_inputs(w, with_dout=False)
    out = torch.empty_like(x["q"])
    lse = torch.empty((1, 2, 1200), device="cuda")
    import ctypes
    sh = lca._shape(x["q"], x["k"], None)
    st = lca.lib().lca_s2attn_fwd(ctypes.byref(sh), lca._ptr(x["q"]), lca._ptr(x["k"]),
                                  lca._ptr(x["v"]), 1, 200, 1, lca._ptr(out), lca._ptr(lse),
                                  lca._stream(None))
    assert st == 5  # LCA_ERR_WORKSPACE
