"""C-ABI checks that need no GPU: the library loads, exports every entry point
the header declares, and rejects bad arguments synchronously (before any
CUDA call)."""

import ctypes
import os
import re

import pytest

from long_context_exact_attention_b200 import lca

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "lca.h")).read()
    return sorted(set(re.findall(r"LCA_API\s+[\w\s\*]+?\b(lca_\w+)\s*\(", text)))


def test_header_declares_the_binding_symbols():
    assert declared_symbols() == sorted(lca.SYMBOLS)


def test_library_exports_every_declared_symbol():
    L = lca.lib()
    for name in declared_symbols():
        assert hasattr(L, name), name


def test_status_strings_and_version():
    L = lca.lib()
    assert L.lca_status_string(0) == b"LCA_OK"
    assert L.lca_status_string(4) == b"LCA_ERR_TIMEOUT"
    assert L.lca_version() >> 16 == 1


def shape(**kw):
    base = dict(B=1, Hq=4, Hkv=2, S=256, d=128, dtype=lca.LCA_BF16, scale=0.0)
    base.update(kw)
    return lca.Shape(base["B"], base["Hq"], base["Hkv"], base["S"], base["d"],
                     base["dtype"], base["scale"])


FAKE = ctypes.c_void_p(0x10000)        # aligned, never dereferenced (call fails first)
MISALIGNED = ctypes.c_void_p(0x10008)


def fwd(sh, kv_chunk=0, opts=None, ptrs=None):
    p = ptrs or [FAKE] * 5
    return lca.lib().lca_attn_fwd(ctypes.byref(sh), p[0], p[1], p[2], 1, kv_chunk,
                                  ctypes.byref(opts) if opts else None, p[3], p[4], None)


@pytest.mark.parametrize("kw,code", [
    (dict(B=0), 1), (dict(Hq=3, Hkv=2), 1), (dict(d=64), 2), (dict(d=96, dtype=1), 2),
    (dict(S=0), 1), (dict(dtype=7), 1), (dict(scale=-1.0), 1),
])
def test_bad_shapes_rejected(kw, code):
    assert fwd(shape(**kw)) == code
    assert lca.lib().lca_last_error()


def test_bad_pointers_rejected():
    sh = shape()
    assert fwd(sh, ptrs=[FAKE, None, FAKE, FAKE, FAKE]) == 1
    assert fwd(sh, ptrs=[FAKE, FAKE, MISALIGNED, FAKE, FAKE]) == 1
    assert b"aligned" in lca.lib().lca_last_error()


@pytest.mark.parametrize("kv_chunk", [-1, -128])
def test_bad_chunks_rejected(kv_chunk):
    assert fwd(shape(S=512), kv_chunk=kv_chunk) == 1


def test_chunk_count_limit():
    # any chunk length is accepted (tiles straddling a boundary are split),
    # up to LCA_MAX_CHUNKS chunks
    assert fwd(shape(S=1025), kv_chunk=1) == 1
    assert b"LCA_MAX_CHUNKS" in lca.lib().lca_last_error()


def test_bad_permutation_rejected():
    perm = (ctypes.c_int32 * 4)(0, 1, 1, 3)
    o = lca.Opts(2, ctypes.cast(perm, ctypes.POINTER(ctypes.c_int32)), 0, 0)
    assert fwd(shape(S=512), kv_chunk=128, opts=o) == 1
    o2 = lca.Opts(2, None, 0, 0)
    assert fwd(shape(S=512), kv_chunk=128, opts=o2) == 1
    o3 = lca.Opts(9, None, 0, 0)
    assert fwd(shape(S=512), kv_chunk=128, opts=o3) == 1


def test_s2_arguments_rejected():
    L = lca.lib()
    sh = shape(S=1024, Hq=4, Hkv=4)
    call = lambda g, sh_, shp=sh: L.lca_s2attn_fwd(ctypes.byref(shp), FAKE, FAKE, FAKE, 1, g,
                                                   sh_, FAKE, FAKE, None)
    assert call(384, 2) == 1          # does not divide S
    assert call(127, 0, shape(S=127 * 8, Hq=4, Hkv=4)) == 1   # odd group
    assert call(512, 5) == 1          # more shifted heads than heads
    assert call(512, -1) == 1
    gqa = shape(S=1024, Hq=4, Hkv=2)
    assert call(512, 1, gqa) == 1     # shift boundary splits a query-head group
    # half a group that is not a whole number of tiles needs a workspace
    assert call(128, 2) == 5
    assert L.lca_s2attn_fwd_workspace_size(ctypes.byref(sh), 512, 2) == 0
    assert L.lca_s2attn_fwd_workspace_size(ctypes.byref(sh), 128, 2) > 0
    assert L.lca_s2attn_bwd_workspace_size(ctypes.byref(sh), 512, 2) == \
        L.lca_attn_bwd_workspace_size(ctypes.byref(sh))
    assert L.lca_s2attn_bwd_workspace_size(ctypes.byref(sh), 128, 2) > \
        L.lca_attn_bwd_workspace_size(ctypes.byref(sh))
    assert L.lca_s2attn_bwd_workspace_size(ctypes.byref(sh), 384, 2) == 0


def test_workspace_errors():
    L = lca.lib()
    sh = shape()
    need = L.lca_attn_bwd_workspace_size(ctypes.byref(sh))
    # D rows and the lse copy ([B,Hq,S rounded up to the tile]) + fp32 dq
    assert need == 2 * 4 * 1 * 4 * 256 + 4 * 256 * 4 * 128
    ragged = shape(S=300)
    assert L.lca_attn_bwd_workspace_size(ctypes.byref(ragged)) == \
        2 * 4 * 1 * 4 * 384 + 4 * 300 * 4 * 128
    assert L.lca_attn_bwd_workspace_size(ctypes.byref(shape(B=0))) == 0
    args = [ctypes.byref(sh)] + [FAKE] * 6 + [1] + [FAKE] * 3
    assert L.lca_attn_bwd(*args, None, need, None) == 5
    assert L.lca_attn_bwd(*args, FAKE, need - 1, None) == 5


def fwd_varlen(sh, cu=FAKE, max_seqlen=128, order=0, ptrs=None):
    p = ptrs or [FAKE] * 5
    o = lca.Opts(order, None, 0, 0)
    return lca.lib().lca_attn_fwd_varlen(ctypes.byref(sh), cu, max_seqlen, p[0], p[1], p[2], 1,
                                         0, ctypes.byref(o), p[3], p[4], None)


def test_varlen_arguments_rejected():
    sh = shape(B=3, S=1000)             # 3 packed sequences, 1000 tokens in all
    assert fwd_varlen(sh, cu=None) == 1
    assert fwd_varlen(sh, cu=ctypes.c_void_p(0x10002)) == 1   # not 4-byte aligned
    assert fwd_varlen(sh, max_seqlen=0) == 1
    assert fwd_varlen(sh, max_seqlen=1001) == 1
    perm = (ctypes.c_int32 * 1)(0)
    o = lca.Opts(2, ctypes.cast(perm, ctypes.POINTER(ctypes.c_int32)), 0, 0)
    assert lca.lib().lca_attn_fwd_varlen(ctypes.byref(sh), FAKE, 128, FAKE, FAKE, FAKE, 1, 0,
                                         ctypes.byref(o), FAKE, FAKE, None) == 1
    assert b"CUSTOM" in lca.lib().lca_last_error()
    assert fwd_varlen(shape(B=3, S=1000, d=64)) == 2


def test_varlen_many_sequences_accepted():
    # 2000 packed sequences over 3M tokens: sequences x tokens exceeds 2^31,
    # which bounds only dense batches.  Validation gets past the shape to
    # the (misaligned) output pointer, so nothing is launched.
    sh = shape(B=2000, S=3_000_000)
    assert fwd_varlen(sh, max_seqlen=4096,
                      ptrs=[FAKE, FAKE, FAKE, MISALIGNED, FAKE]) == 1
    assert b"pointer argument 3" in lca.lib().lca_last_error()


def test_varlen_workspace_size():
    L = lca.lib()
    sh = shape(B=3, S=1000)
    # D rows and lse copy [3, Hq, 384] each, fp32 dq accumulator [1000, Hq, 128]
    assert L.lca_attn_bwd_varlen_workspace_size(ctypes.byref(sh), 300) == \
        2 * 4 * 3 * 4 * 384 + 4 * 1000 * 4 * 128
    assert L.lca_attn_bwd_varlen_workspace_size(ctypes.byref(sh), 0) == 0
    assert L.lca_attn_bwd_varlen_workspace_size(ctypes.byref(sh), 1001) == 0
    args = [ctypes.byref(sh), FAKE, 300] + [FAKE] * 6 + [1] + [FAKE] * 3
    assert L.lca_attn_bwd_varlen(*args, None, 1 << 30, None) == 5


def test_ffn_arguments_rejected():
    L = lca.lib()

    def call(T=300, h=256, f=384, block=128, ws_bytes=1 << 30, ptrs=None, ws=FAKE):
        sh = lca.FfnShape(T, h, f)
        p = ptrs or [FAKE] * 5
        return L.lca_ffn_fwd(ctypes.byref(sh), p[0], p[1], p[2], p[3], block, p[4], ws, ws_bytes,
                             None)
    assert call(T=0) == 1
    assert call(block=100) == 1 and call(block=-128) == 1
    assert call(h=128) == 2 and call(f=200) == 2
    assert call(ptrs=[FAKE, None, FAKE, FAKE, FAKE]) == 1
    assert call(ptrs=[FAKE, FAKE, FAKE, MISALIGNED, FAKE]) == 1
    assert call(ws=None) == 5
    assert call(ws_bytes=128 * 384 * 2 - 1) == 5
    sh = lca.FfnShape(300, 256, 384)
    # block rows x f bf16; 0 -> the default block, capped at T rounded up to 128
    assert L.lca_ffn_workspace_size(ctypes.byref(sh), 128) == 128 * 384 * 2
    assert L.lca_ffn_workspace_size(ctypes.byref(sh), 0) == 384 * 384 * 2
    assert L.lca_ffn_workspace_size(ctypes.byref(lca.FfnShape(300, 100, 384)), 0) == 0


def test_ffn_bwd_arguments_rejected():
    L = lca.lib()

    def call(T=300, h=256, f=512, block=128, ws_bytes=1 << 30, ws=FAKE):
        sh = lca.FfnShape(T, h, f)
        return L.lca_ffn_bwd(ctypes.byref(sh), *([FAKE] * 5), block, *([FAKE] * 4), ws,
                             ws_bytes, None)
    assert call(T=0) == 1
    assert call(f=384) == 2          # the backward needs f % 256 == 0
    assert call(ws=None) == 5
    assert call(ws_bytes=4 * 128 * 512 * 2 - 1) == 5
    sh = lca.FfnShape(300, 256, 512)
    assert L.lca_ffn_bwd_workspace_size(ctypes.byref(sh), 128) == 4 * 128 * 512 * 2
    assert L.lca_ffn_bwd_workspace_size(ctypes.byref(lca.FfnShape(300, 256, 384)), 128) == 0


def test_merge_arguments_rejected():
    L = lca.lib()
    assert L.lca_lse_merge(0, 4, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None) == 1
    assert L.lca_lse_merge(4, 4, FAKE, None, FAKE, FAKE, FAKE, FAKE, None) == 1


def test_python_binding_refuses_cpu_tensors():
    import torch
    q = torch.zeros(1, 128, 1, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        lca.attn_fwd(q, q, q)


# ---------------------------------------------------------------- blocks

def bshape(**kw):
    base = dict(B=1, Hq=4, Hkv=2, Sq=256, Sk=256, d=128, dtype=lca.LCA_BF16, scale=0.0)
    base.update(kw)
    return lca.BlockShape(base["B"], base["Hq"], base["Hkv"], base["Sq"], base["Sk"], base["d"],
                          base["dtype"], base["scale"])


def fwd_block(sh, causal=1, q_pos0=0, k_pos0=0, accumulate=0, o_acc=FAKE, lse=FAKE, out=FAKE):
    return lca.lib().lca_attn_fwd_block(ctypes.byref(sh), FAKE, FAKE, FAKE, causal, q_pos0,
                                        k_pos0, accumulate, o_acc, lse, out, None)


@pytest.mark.parametrize("kw,code", [
    (dict(Sk=0), 1), (dict(Sq=0), 1), (dict(dtype=lca.LCA_FP32, d=64), 2), (dict(d=64), 2),
    (dict(Hq=3, Hkv=2), 1),
])
def test_block_shapes_rejected(kw, code):
    assert fwd_block(bshape(**kw)) == code


def test_block_positions_and_outputs_rejected():
    sh = bshape()
    assert fwd_block(sh, q_pos0=-1) == 1
    # the diagonal crosses the blocks 100 positions apart: not a whole tile
    assert fwd_block(sh, q_pos0=100, k_pos0=0) == 1
    assert b"multiple of 128" in lca.lib().lca_last_error()
    assert fwd_block(sh, o_acc=None, out=None) == 1
    assert fwd_block(sh, accumulate=1, o_acc=None) == 1
    assert fwd_block(sh, lse=None) == 1


def test_bwd_block_needs_exactly_one_output_pair():
    sh = bshape()
    n = lca.lib().lca_attn_bwd_block_workspace_size(ctypes.byref(sh))
    assert n > 0
    call = lambda dka, dva, dk, dv: lca.lib().lca_attn_bwd_block(
        ctypes.byref(sh), FAKE, FAKE, FAKE, FAKE, 1, 0, 0, FAKE, n, dka, dva, 1, dk, dv, None)
    assert call(None, None, None, None) == 1
    assert call(FAKE, FAKE, FAKE, FAKE) == 1
    assert lca.lib().lca_attn_bwd_block(ctypes.byref(sh), FAKE, FAKE, FAKE, FAKE, 1, 0, 0, FAKE,
                                        n - 16, FAKE, FAKE, 1, None, None, None) == 5


def test_finishing_ops_rejected():
    L = lca.lib()
    assert L.lca_cast_f32_bf16(0, FAKE, FAKE, None) == 1
    assert L.lca_cast_f32_bf16(8, FAKE, MISALIGNED, None) == 1
    assert L.lca_accumulate_f32(-1, FAKE, FAKE, None) == 1
    assert L.lca_accumulate_f32(8, None, FAKE, None) == 1


def test_bpt_arguments_rejected():
    L = lca.lib()
    def mk(**kw):
        base = dict(S=1024, Hq=4, Hkv=2, d=128, f=768, q_block=256, scale=0.0)
        base.update(kw)
        return lca.BptShape(*(base[n] for n in ("S", "Hq", "Hkv", "d", "f", "q_block", "scale")))

    ok = mk()
    assert L.lca_bpt_fwd_workspace_size(ctypes.byref(ok)) > 0
    assert L.lca_bpt_bwd_workspace_size(ctypes.byref(ok)) > 0
    assert L.lca_bpt_fwd_workspace_size(ctypes.byref(mk(q_block=100))) == 0
    assert L.lca_bpt_fwd_workspace_size(ctypes.byref(mk(Hq=3, Hkv=3))) == 0   # h % 256
    assert L.lca_bpt_bwd_workspace_size(ctypes.byref(mk(f=640))) == 0         # f % 256
    args = [FAKE] * 3 + [1] + [FAKE] * 6
    assert L.lca_bpt_fwd(ctypes.byref(mk(q_block=100)), *args, FAKE, 1 << 30, None) == 1
    assert L.lca_bpt_fwd(ctypes.byref(ok), *args, None, 0, None) == 5
