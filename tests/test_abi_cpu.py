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


@pytest.mark.parametrize("kv_chunk", [100, 200, -128])
def test_bad_chunks_rejected(kv_chunk):
    # a chunk must be a whole number of tiles (the last chunk of a sequence
    # may be partial, so it need not divide S)
    assert fwd(shape(S=512), kv_chunk=kv_chunk) == 1


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
    assert call(128, 2) == 1          # half group not a multiple of the tile
    assert call(512, 5) == 1          # more shifted heads than heads
    assert call(512, -1) == 1
    gqa = shape(S=1024, Hq=4, Hkv=2)
    assert call(512, 1, gqa) == 1     # shift boundary splits a query-head group


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


def test_merge_arguments_rejected():
    L = lca.lib()
    assert L.lca_lse_merge(0, 4, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None) == 1
    assert L.lca_lse_merge(4, 4, FAKE, None, FAKE, FAKE, FAKE, FAKE, None) == 1


def test_python_binding_refuses_cpu_tensors():
    import torch
    q = torch.zeros(1, 128, 1, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        lca.attn_fwd(q, q, q)
