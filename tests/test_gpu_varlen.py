"""Packed variable-length batches (lca_attn_fwd_varlen / lca_attn_bwd_varlen):
every sequence of a packed token axis attends only to itself.  Forward and
backward against the fp64 oracle on every covered row, for bf16 (tensor-core
path) and fp32, with empty, one-token, tile-multiple and ragged lengths;
rows outside every sequence stay untouched; a single sequence gives the
dense call's result bit for bit; invalid device offsets are reported by
lca_check without any out-of-range access."""

import numpy as np
import pytest
import torch

import oracle
from long_context_exact_attention_b200 import lca
from long_context_exact_attention_b200.inputs import (WORKLOADS, make_tensor, packed_lengths,
                                                      packed_offsets, shrink)

from gpu_util import assert_grads_close, host, max_abs, rel_fro, BF16_LSE_ABS, BF16_OUT_ABS, \
    BF16_OUT_REL, F32_ABS

pytestmark = pytest.mark.gpu


def packed_inputs(T, Hq, Hkv, dtype, seed):
    """q/dout [T,Hq,128|64], k/v [T,Hkv,d] drawn by the workload recipe on a
    single batch entry of T tokens."""
    base = WORKLOADS["llama2_7b_s32k"] if dtype == "bf16" else WORKLOADS["tiny_fp32_s256"]
    w = shrink(base, B=1, S=T, Hq=Hq, Hkv=Hkv, rope=False, seed=seed)
    return {n: make_tensor(w, n, "cuda")[0].contiguous() for n in ("q", "k", "v", "dout")}


def covered_rows(cu):
    return [t for c0, c1 in zip(cu, cu[1:]) for t in range(c0, c1)]


def check_packed_fwd(out, lse, ro, rl, cu, fp32):
    rows = covered_rows(cu)
    o, l = host(out)[rows], host(lse)[:, rows]
    assert np.isfinite(o).all() and np.isfinite(l).all()
    if fp32:
        assert max_abs(o, ro[rows]) <= F32_ABS
        assert max_abs(l, rl[:, rows]) <= F32_ABS
        return
    assert max_abs(o, ro[rows]) <= BF16_OUT_ABS
    assert max_abs(l, rl[:, rows]) <= BF16_LSE_ABS
    # the stricter relative bound per (sequence, head)
    for c0, c1 in zip(cu, cu[1:]):
        if c1 > c0:
            for h in range(o.shape[1]):
                assert rel_fro(host(out)[c0:c1, h], ro[c0:c1, h]) <= BF16_OUT_REL, (c0, h)


def run_packed(lengths, Hq, Hkv, causal, dtype="bf16", kv_chunk=0, order="inorder", seed=5,
               start=0, tail=0):
    cu = packed_offsets(lengths, start)
    T = cu[-1] + tail
    x = packed_inputs(T, Hq, Hkv, dtype, seed)
    cu_d = torch.tensor(cu, dtype=torch.int32, device="cuda")
    max_len = max(max(lengths), 1)
    out, lse = lca.attn_fwd_varlen(x["q"], x["k"], x["v"], cu_d, max_len, causal=causal,
                                   kv_chunk=kv_chunk, order=order)
    dq, dk, dv = lca.attn_bwd_varlen(x["q"], x["k"], x["v"], out, lse, x["dout"], cu_d, max_len,
                                     causal=causal)
    torch.cuda.synchronize()
    lca.check()
    return x, cu, out, lse, dq, dk, dv


@pytest.mark.parametrize("lengths,Hq,Hkv,causal,kv_chunk,order", [
    ([1000, 1, 0, 130, 257, 128, 640], 4, 2, True, 0, "inorder"),
    ([1000, 1, 0, 130, 257, 128, 640], 2, 2, False, 200, "ring"),
    ([384, 385, 383], 2, 1, True, 256, "ring"),
    (None, 2, 2, True, 0, "inorder"),            # seeded length mix
])
def test_bf16_packed_fwd_bwd(lengths, Hq, Hkv, causal, kv_chunk, order):
    if lengths is None:
        lengths = packed_lengths(9, 700, seed=1)
    x, cu, out, lse, dq, dk, dv = run_packed(lengths, Hq, Hkv, causal, kv_chunk=kv_chunk,
                                             order=order)
    ro, rl = oracle.packed_attention_forward(x["q"], x["k"], x["v"], cu, causal)
    check_packed_fwd(out, lse, ro, rl, cu, fp32=False)
    rg = oracle.packed_attention_backward(x["q"], x["k"], x["v"], x["dout"], cu, causal)
    rows = covered_rows(cu)
    assert_grads_close([host(dq)[rows], host(dk)[rows], host(dv)[rows]],
                       [g[rows] for g in rg])


@pytest.mark.parametrize("causal", [True, False])
def test_fp32_packed_fwd_bwd(causal):
    lengths = [100, 0, 64, 1, 129]
    x, cu, out, lse, dq, dk, dv = run_packed(lengths, 2, 1, causal, dtype="fp32",
                                             kv_chunk=48, order="ring")
    ro, rl = oracle.packed_attention_forward(x["q"], x["k"], x["v"], cu, causal)
    check_packed_fwd(out, lse, ro, rl, cu, fp32=True)
    rg = oracle.packed_attention_backward(x["q"], x["k"], x["v"], x["dout"], cu, causal)
    rows = covered_rows(cu)
    assert_grads_close([host(dq)[rows], host(dk)[rows], host(dv)[rows]],
                       [g[rows] for g in rg], fp32=True)


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_rows_outside_sequences_untouched(dtype):
    # sequences cover tokens [64, 700); rows 0..63 and 700..799 belong to none
    cu = [64, 300, 300, 700]
    T = 800
    x = packed_inputs(T, 2, 2, dtype, seed=9)
    cu_d = torch.tensor(cu, dtype=torch.int32, device="cuda")
    out = torch.full_like(x["q"], float("nan"))
    lse = torch.full((2, T), float("nan"), device="cuda")
    lca.attn_fwd_varlen(x["q"], x["k"], x["v"], cu_d, 400, causal=True, out=out, lse=lse)
    dk = torch.full_like(x["k"], float("nan"))
    dv = torch.full_like(x["v"], float("nan"))
    dq = torch.full_like(x["q"], float("nan"))
    lca.attn_bwd_varlen(x["q"], x["k"], x["v"], out, lse, x["dout"], cu_d, 400, causal=True,
                        dq=dq, dk=dk, dv=dv)
    torch.cuda.synchronize()
    lca.check()
    inside = torch.zeros(T, dtype=torch.bool)
    inside[64:700] = True
    for t in (out, dk, dv):
        assert torch.isfinite(t[inside].float()).all()
        assert torch.isnan(t[~inside].float()).all()
    assert torch.isfinite(lse[:, inside]).all() and torch.isnan(lse[:, ~inside]).all()
    assert (dq[~inside].float() == 0).all() and torch.isfinite(dq[inside].float()).all()


@pytest.mark.parametrize("dtype,S", [("bf16", 1000), ("fp32", 200)])
def test_single_sequence_equals_dense_bitwise(dtype, S):
    x = packed_inputs(S, 2, 1, dtype, seed=13)
    cu_d = torch.tensor([0, S], dtype=torch.int32, device="cuda")
    o1, l1 = lca.attn_fwd_varlen(x["q"], x["k"], x["v"], cu_d, S, causal=True, kv_chunk=256,
                                 order="ring")
    o2, l2 = lca.attn_fwd(x["q"][None], x["k"][None], x["v"][None], causal=True, kv_chunk=256,
                          order="ring")
    g1 = lca.attn_bwd_varlen(x["q"], x["k"], x["v"], o1, l1, x["dout"], cu_d, S, causal=True)
    g2 = lca.attn_bwd(x["q"][None], x["k"][None], x["v"][None], o2, l2, x["dout"][None],
                      causal=True)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2[0]) and torch.equal(l1, l2[0])
    # dK, dV are deterministic; dQ sums float32 partials in arrival order
    assert torch.equal(g1[1], g2[1][0]) and torch.equal(g1[2], g2[2][0])
    assert rel_fro(host(g1[0]), host(g2[0][0])) < 1e-3


@pytest.mark.parametrize("cu,max_len", [
    ([0, 300, 200, 500], 300),     # out of order
    ([0, 300, 600], 299),          # a sequence longer than max_seqlen
    ([0, 300, 900], 600),          # past the packed tokens
])
def test_invalid_offsets_reported(cu, max_len):
    # every kernel checks the offsets of its sequence before touching memory
    # and skips the sequence; lca_check then reports it
    T = 600
    x = packed_inputs(T, 2, 2, "bf16", seed=17)
    cu_d = torch.tensor(cu, dtype=torch.int32, device="cuda")
    out, lse = lca.attn_fwd_varlen(x["q"], x["k"], x["v"], cu_d, max_len)
    with pytest.raises(lca.LcaError) as e:
        lca.check()
    assert e.value.status == 1
    lca.attn_bwd_varlen(x["q"], x["k"], x["v"], out, lse, x["dout"], cu_d, max_len)
    with pytest.raises(lca.LcaError):
        lca.check()
    # the context stays usable
    good = torch.tensor([0, 300, 600], dtype=torch.int32, device="cuda")
    lca.attn_fwd_varlen(x["q"], x["k"], x["v"], good, 300)
    lca.check()
