"""torch.autograd wrappers over the C ABI, for training loops.

Plumbing only: each forward calls the library's forward entry point and
saves what its backward entry point needs (the inputs, the output and the
log-sum-exp -- never the attention matrix); each backward calls the
library's backward entry point.  Every step runs in the CUDA library.

    from long_context_exact_attention_b200.autograd import attention, s2_attention, feedforward
    out = attention(q, k, v, causal=True, kv_chunk=4096, order="ring")
    out.float().sum().backward()

Sequence parallel (every rank of the process group calls with its own block):
``ring_attention`` over zig-zag blocks (ring.shard), ``ulysses_attention``
over contiguous shards.

Errors inside a kernel (a wait that ran out, invalid packed offsets) are
recorded in the library's device error word, not raised by these calls,
because reading it synchronises the stream.  Call ``lca.check()`` at a point
where a synchronisation is acceptable (for example once per training step);
it raises if any kernel since the last check reported an error, and the
results of that step must then be discarded.
"""

from __future__ import annotations

import torch

from . import lca, ring, ulysses


class _Attention(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k, v, causal, kv_chunk, order, scale):
        out, lse = lca.attn_fwd(q, k, v, causal=causal, kv_chunk=kv_chunk, order=order,
                                scale=scale)
        ctx.save_for_backward(q, k, v, out, lse)
        ctx.causal, ctx.scale = causal, scale
        return out

    @staticmethod
    def backward(ctx, dout):
        q, k, v, out, lse = ctx.saved_tensors
        dq, dk, dv = lca.attn_bwd(q, k, v, out, lse, dout.contiguous(), causal=ctx.causal,
                                  scale=ctx.scale)
        return dq, dk, dv, None, None, None, None


class _S2Attention(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k, v, group, shift_heads, causal, scale):
        out, lse = lca.s2attn_fwd(q, k, v, group, shift_heads, causal=causal, scale=scale)
        ctx.save_for_backward(q, k, v, out, lse)
        ctx.args = (group, shift_heads, causal, scale)
        return out

    @staticmethod
    def backward(ctx, dout):
        q, k, v, out, lse = ctx.saved_tensors
        group, shift_heads, causal, scale = ctx.args
        dq, dk, dv = lca.s2attn_bwd(q, k, v, out, lse, dout.contiguous(), group, shift_heads,
                                    causal=causal, scale=scale)
        return dq, dk, dv, None, None, None, None


class _RingAttention(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k, v, causal, group, scale):
        out, lse = ring.ring_attn_fwd(q, k, v, causal=causal, group=group, scale=scale)
        ctx.save_for_backward(q, k, v, out, lse)
        ctx.args = (causal, group, scale)
        return out

    @staticmethod
    def backward(ctx, dout):
        q, k, v, out, lse = ctx.saved_tensors
        causal, group, scale = ctx.args
        dq, dk, dv = ring.ring_attn_bwd(q, k, v, out, lse, dout.contiguous(), causal=causal,
                                        group=group, scale=scale)
        return dq, dk, dv, None, None, None


class _UlyssesAttention(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k, v, causal, group, scale):
        out, lse_h = ulysses.ulysses_attn_fwd(q, k, v, causal=causal, group=group, scale=scale)
        ctx.save_for_backward(q, k, v, out, lse_h)
        ctx.args = (causal, group, scale)
        return out

    @staticmethod
    def backward(ctx, dout):
        q, k, v, out, lse_h = ctx.saved_tensors
        causal, group, scale = ctx.args
        dq, dk, dv = ulysses.ulysses_attn_bwd(q, k, v, out, lse_h, dout.contiguous(),
                                              causal=causal, group=group, scale=scale)
        return dq, dk, dv, None, None, None


class _Feedforward(torch.autograd.Function):
    @staticmethod
    def forward(ctx, x, w_gate, w_up, w_down, block_tokens):
        out = lca.ffn_fwd(x, w_gate, w_up, w_down, block_tokens=block_tokens)
        ctx.save_for_backward(x, w_gate, w_up, w_down)
        ctx.block_tokens = block_tokens
        return out

    @staticmethod
    def backward(ctx, dout):
        x, w_gate, w_up, w_down = ctx.saved_tensors
        dx, dwg, dwu, dwd = lca.ffn_bwd(x, w_gate, w_up, w_down, dout.contiguous(),
                                        block_tokens=ctx.block_tokens)
        return dx, dwg.to(w_gate.dtype), dwu.to(w_up.dtype), dwd.to(w_down.dtype), None


def attention(q, k, v, causal: bool = True, kv_chunk: int = 0, order: str = "inorder",
              scale=None):
    """Exact attention with autograd: q [B,S,Hq,d], k/v [B,S,Hkv,d]."""
    return _Attention.apply(q, k, v, causal, kv_chunk, order, scale)


def s2_attention(q, k, v, group: int, shift_heads: int, causal: bool = True, scale=None):
    """LongLoRA S2-Attn with autograd."""
    return _S2Attention.apply(q, k, v, group, shift_heads, causal, scale)


def feedforward(x, w_gate, w_up, w_down, block_tokens: int = 0):
    """Blockwise gated-SiLU feedforward with autograd: x [T,h]; weight
    gradients are accumulated in float32 by the library and returned in the
    weights' dtype."""
    return _Feedforward.apply(x, w_gate, w_up, w_down, block_tokens)


def ring_attention(q, k, v, causal: bool = True, group=None, scale=None):
    """Ring attention with autograd on this rank: q [B,2c,Hq,d], k/v
    [B,2c,Hkv,d] are the rank's zig-zag block (ring.shard); the output is
    the block's rows.  Every rank of `group` calls it together (without a
    process group it is one rank holding the whole sequence)."""
    return _RingAttention.apply(q, k, v, causal, group, scale)


def ulysses_attention(q, k, v, causal: bool = True, group=None, scale=None):
    """Ulysses sequence parallelism with autograd on this rank: q
    [B,S/W,Hq,d], k/v [B,S/W,Hkv,d] are the rank's contiguous shard."""
    return _UlyssesAttention.apply(q, k, v, causal, group, scale)
