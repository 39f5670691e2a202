"""Blockwise feedforward (lca_ffn_fwd) against the fp64 oracle.

Tolerance, derived from the arithmetic: the GPU takes exact bf16 products
with float32 sums, rounds the gated intermediate H to bf16 (relative error
up to 2^-9 per element, independent across the f terms of a row) and the
output to bf16 (2^-9).  Both give a relative error of a few 1e-3 on the
output; the bound is 1e-2 relative Frobenius per row block and 2e-2 of the
largest |out| element-wise.  The intermediate is blocked by token rows and
each row's sums run in the same order whatever the block, so results are
bit-identical across block sizes."""

import numpy as np
import pytest
import torch

import oracle
from long_context_exact_attention_b200 import lca
from long_context_exact_attention_b200.inputs import FFN_WORKLOADS, make_ffn_inputs

from gpu_util import host, rel_fro

pytestmark = pytest.mark.gpu

REL = 1e-2
ABS_OF_MAX = 2e-2


def check(out, ref):
    out = np.asarray(out, np.float64)
    assert np.isfinite(out).all()
    assert rel_fro(out, ref) <= REL, rel_fro(out, ref)
    err = np.max(np.abs(out - ref))
    assert err <= ABS_OF_MAX * np.max(np.abs(ref)), (err, np.max(np.abs(ref)))


def inputs(name, **kw):
    import dataclasses
    w = dataclasses.replace(FFN_WORKLOADS[name], **kw)
    return w, make_ffn_inputs(w, "cuda")


@pytest.mark.parametrize("T,h,f,block", [
    (300, 256, 384, 128),    # three blocks, the last of 44 rows
    (128, 512, 256, 0),      # one full tile row
    (1, 256, 128, 0),        # a single token
    (1000, 512, 640, 256),
])
def test_ffn_matches_oracle(T, h, f, block):
    w, x = inputs("tiny_ffn", T=T, h=h, f=f, block=block, seed=T + h)
    out = lca.ffn_fwd(x["x"], x["w_gate"], x["w_up"], x["w_down"], block_tokens=block)
    torch.cuda.synchronize()
    lca.check()
    ref = oracle.ffn_forward(x["x"], x["w_gate"], x["w_up"], x["w_down"], block=block)
    check(host(out), ref)


def test_block_size_is_bit_exact():
    w, x = inputs("tiny_ffn", T=700, h=256, f=384, seed=3)
    outs = [lca.ffn_fwd(x["x"], x["w_gate"], x["w_up"], x["w_down"], block_tokens=b)
            for b in (128, 256, 384, 0)]
    torch.cuda.synchronize()
    for o in outs[1:]:
        assert torch.equal(o, outs[0])


def test_rows_past_T_untouched():
    w, x = inputs("tiny_ffn", T=200, h=256, f=128, seed=4)
    big = torch.full((264, 256), float("nan"), device="cuda", dtype=torch.bfloat16)
    lca.ffn_fwd(x["x"], x["w_gate"], x["w_up"], x["w_down"], block_tokens=128, out=big[:200])
    torch.cuda.synchronize()
    assert torch.isfinite(big[:200].float()).all()
    assert torch.isnan(big[200:].float()).all()


def test_llama2_7b_ffn_full_size_sampled_rows():
    """The bench configuration (T = 32768, h = 4096, f = 11008, 8192-token
    blocks) in the bench's launch configuration; sampled rows against the
    oracle, which computes each row on its own."""
    w = FFN_WORKLOADS["llama2_7b_ffn_s32k"]
    x = make_ffn_inputs(w, "cuda")
    out = lca.ffn_fwd(x["x"], x["w_gate"], x["w_up"], x["w_down"], block_tokens=w.block)
    torch.cuda.synchronize()
    lca.check()
    g = torch.Generator().manual_seed(5)
    rows = sorted(set([0, 127, 128, w.block - 1, w.block, w.T - 1] +
                      torch.randint(0, w.T, (10,), generator=g).tolist()))
    ref = oracle.ffn_rows(x["x"].cpu(), x["w_gate"].cpu(), x["w_up"].cpu(), x["w_down"].cpu(),
                          rows)
    check(host(out[rows]), ref)


# ---------------------------------------------------------------- backward
# dx and the weight gradients: relative Frobenius <= 2e-2 (the bar of the
# attention gradients; bf16 rounding of dH, dG, dU and H, float32 sums)
GRAD_REL = 2e-2


def grads(x, block, dw=None):
    g = torch.Generator(device="cuda").manual_seed(77)
    dout = torch.randn(x["x"].shape, generator=g, device="cuda").to(torch.bfloat16)
    kw = {} if dw is None else dict(dw_gate=dw[0], dw_up=dw[1], dw_down=dw[2])
    res = lca.ffn_bwd(x["x"], x["w_gate"], x["w_up"], x["w_down"], dout, block_tokens=block, **kw)
    torch.cuda.synchronize()
    lca.check()
    return dout, res


@pytest.mark.parametrize("T,h,f,block", [
    (300, 256, 512, 128),    # three blocks, the last of 44 rows (K steps past it)
    (1000, 512, 768, 256),
    (1, 256, 256, 0),
])
def test_ffn_backward_matches_oracle(T, h, f, block):
    w, x = inputs("tiny_ffn", T=T, h=h, f=f, block=block, seed=T + f)
    dout, got = grads(x, block)
    ref = oracle.ffn_backward(x["x"], x["w_gate"], x["w_up"], x["w_down"], dout, block=block)
    for name, a, b in zip(("dx", "dw_gate", "dw_up", "dw_down"), got, ref):
        a = host(a)
        assert np.isfinite(a).all(), name
        assert rel_fro(a, b) <= GRAD_REL, (name, rel_fro(a, b))


def test_ffn_backward_accumulates_and_dx_is_block_exact():
    w, x = inputs("tiny_ffn", T=600, h=256, f=512, seed=8)
    dout, (dx1, g1, u1, d1) = grads(x, 128)
    # a second call adds the same gradients again
    _, (dx2, g2, u2, d2) = grads(x, 128, dw=(g1.clone(), u1.clone(), d1.clone()))
    for a, b in ((g2, g1), (u2, u1), (d2, d1)):
        assert rel_fro(host(a), 2 * host(b)) < 1e-6
    # dx rows do not depend on the blocking
    _, (dx3, _, _, _) = grads(x, 256)
    assert torch.equal(dx1, dx2) and torch.equal(dx1, dx3)


def test_llama2_7b_ffn_backward_full_size_sampled():
    """The bench configuration; dx on sampled rows, the weight gradients on
    sampled feedforward columns (each exact in the oracle)."""
    w = FFN_WORKLOADS["llama2_7b_ffn_s32k"]
    x = make_ffn_inputs(w, "cuda")
    dout, (dx, dwg, dwu, dwd) = grads(x, w.block)
    xc = {k: v.cpu() for k, v in x.items()}
    doc = dout.cpu()
    rows = [0, 127, w.block - 1, w.block, w.T - 1, 12345]
    import oracle.ffn as F
    xs, wg, wu, wd, do = (F._f64(t) for t in (xc["x"], xc["w_gate"], xc["w_up"], xc["w_down"], doc))
    ref_dx = F.ffn_backward(xs[rows], wg, wu, wd, do[rows])[0]
    assert rel_fro(host(dx[rows]), ref_dx) <= GRAD_REL
    cols = [0, 1, 4095, 5000, 11007]
    a, b, c = oracle.ffn_backward_columns(xs, wg, wu, wd, do, cols)
    assert rel_fro(host(dwg[cols]), a) <= GRAD_REL
    assert rel_fro(host(dwu[cols]), b) <= GRAD_REL
    assert rel_fro(host(dwd[:, cols]), c) <= GRAD_REL
