"""lca_attn_bwd_noalloc: the backward pass for callers that cannot allocate
device memory (for example a plugin whose host framework owns every device
allocation, or a latency-critical caller that cannot take cudaMalloc's cost).
It takes its scratch from a fixed array inside the library instead of a
caller workspace.  These tests call it through the C ABI and check it against
lca_attn_bwd and against the fp64 oracle's gradients, on two calls in a row
(the second call finds the first call's leftovers in the shared scratch).
The file is named to run last."""

import ctypes

import pytest
import torch

import oracle
from long_context_exact_attention_b200 import lca
from long_context_exact_attention_b200.inputs import WORKLOADS, make_inputs, shrink

from gpu_util import GRAD_REL, F32_ABS, host, max_abs, rel_fro

SCRATCH_BYTES = 64 << 20


def _call_noalloc(x, out, lse, causal, grads):
    sh = lca._shape(x["q"], x["k"], None)
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    st = lca.lib().lca_attn_bwd_noalloc(
        ctypes.byref(sh), p(x["q"]), p(x["k"]), p(x["v"]), p(out), p(lse), p(x["dout"]),
        int(causal), p(grads[0]), p(grads[1]), p(grads[2]),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, lca.lib().lca_last_error()


def test_noalloc_rejects_shapes_beyond_its_scratch():
    # 32 heads x 32768 tokens need about 0.5 GiB of scratch: refused before
    # any device work (the pointers are never touched).
    sh = lca.Shape(1, 32, 32, 32768, 128, lca.LCA_BF16, 0.0)
    fake = ctypes.c_void_p(0x10000)
    st = lca.lib().lca_attn_bwd_noalloc(ctypes.byref(sh), *([fake] * 6), 1, fake, fake, fake,
                                        None)
    assert st == 5
    assert b"built-in scratch" in lca.lib().lca_last_error()
    assert lca.lib().lca_attn_bwd_workspace_size(ctypes.byref(sh)) > SCRATCH_BYTES


@pytest.mark.gpu
@pytest.mark.parametrize("name,kw,causal", [
    ("llama2_7b_s32k", dict(B=2, Hq=4, Hkv=2, S=512, rope=False, seed=41), True),
    ("llama2_7b_s32k", dict(B=1, Hq=2, Hkv=2, S=384, rope=False, seed=42), False),
    ("tiny_fp32_s256", dict(seed=43), True)])
def test_noalloc_matches_workspace_backward(name, kw, causal):
    w = shrink(WORKLOADS[name], **kw)
    x = make_inputs(w, "cuda")
    out, lse = lca.attn_fwd(x["q"], x["k"], x["v"], causal=causal)
    ref = lca.attn_bwd(x["q"], x["k"], x["v"], out, lse, x["dout"], causal=causal)
    torch.cuda.synchronize()
    ref = [host(t) for t in ref]
    want = oracle.attention_backward(x["q"], x["k"], x["v"], x["dout"], causal)
    for _ in range(2):
        grads = [torch.full_like(t, float("nan")) for t in (x["q"], x["k"], x["v"])]
        _call_noalloc(x, out, lse, causal, grads)
        torch.cuda.synchronize()
        lca.check()
        for g, r, o in zip(grads, ref, want):
            g = host(g)
            assert torch.isfinite(torch.from_numpy(g)).all()
            if w.dtype == "fp32":
                assert max_abs(g, r) <= F32_ABS
                assert max_abs(g, o) <= F32_ABS
            else:
                assert rel_fro(g, r) <= GRAD_REL
                assert rel_fro(g, o) <= GRAD_REL
