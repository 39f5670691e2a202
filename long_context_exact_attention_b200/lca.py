"""Python binding of liblca (include/lca.h) over torch tensors.

Argument marshalling only: every step of the computation runs in the CUDA
library.  torch supplies device memory and the current stream.  There is no
fallback: if liblca.so is missing or the tensors are not CUDA tensors the
call raises.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import torch

# The in-tree build; the LCA_LIBRARY environment variable names another
# build of the same library to load instead.
LIB_PATH = os.environ.get("LCA_LIBRARY") or os.path.join(
    os.path.dirname(os.path.abspath(__file__)), "liblca.so")

LCA_BF16, LCA_FP32 = 0, 1
ORDERS = {"inorder": 0, "ring": 1, "custom": 2}
STATUS = {0: "LCA_OK", 1: "LCA_ERR_INVALID_ARG", 2: "LCA_ERR_UNSUPPORTED",
          3: "LCA_ERR_CUDA", 4: "LCA_ERR_TIMEOUT", 5: "LCA_ERR_WORKSPACE"}
SYMBOLS = ["lca_attn_fwd", "lca_attn_bwd_workspace_size", "lca_attn_bwd",
           "lca_attn_bwd_noalloc",
           "lca_attn_fwd_varlen", "lca_attn_bwd_varlen_workspace_size", "lca_attn_bwd_varlen",
           "lca_ffn_workspace_size", "lca_ffn_fwd", "lca_ffn_bwd_workspace_size", "lca_ffn_bwd",
           "lca_s2attn_fwd", "lca_s2attn_fwd_ws", "lca_s2attn_fwd_workspace_size",
           "lca_s2attn_bwd", "lca_s2attn_bwd_workspace_size", "lca_lse_merge",
           "lca_attn_fwd_block", "lca_attn_bwd_block_workspace_size", "lca_attn_bwd_block_prep",
           "lca_attn_bwd_block", "lca_attn_bwd_block_dq", "lca_cast_f32_bf16",
           "lca_accumulate_f32", "lca_bpt_fwd_workspace_size", "lca_bpt_fwd",
           "lca_bpt_bwd_workspace_size", "lca_bpt_bwd", "lca_check", "lca_status_string",
           "lca_last_error", "lca_version"]


class LcaError(RuntimeError):
    def __init__(self, status: int, detail: str):
        super().__init__(f"{STATUS.get(status, status)}: {detail}")
        self.status = status


class Shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int64), ("Hq", ctypes.c_int64), ("Hkv", ctypes.c_int64),
                ("S", ctypes.c_int64), ("d", ctypes.c_int64), ("dtype", ctypes.c_int32),
                ("scale", ctypes.c_float)]


class BlockShape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int64), ("Hq", ctypes.c_int64), ("Hkv", ctypes.c_int64),
                ("Sq", ctypes.c_int64), ("Sk", ctypes.c_int64), ("d", ctypes.c_int64),
                ("dtype", ctypes.c_int32), ("scale", ctypes.c_float)]


class BptShape(ctypes.Structure):
    _fields_ = [("S", ctypes.c_int64), ("Hq", ctypes.c_int64), ("Hkv", ctypes.c_int64),
                ("d", ctypes.c_int64), ("f", ctypes.c_int64), ("q_block", ctypes.c_int64),
                ("scale", ctypes.c_float)]


class FfnShape(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int64), ("h", ctypes.c_int64), ("f", ctypes.c_int64)]


class Opts(ctypes.Structure):
    _fields_ = [("order", ctypes.c_int32), ("chunk_perm", ctypes.POINTER(ctypes.c_int32)),
                ("q_block", ctypes.c_int64), ("timeout_cycles", ctypes.c_uint64)]


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded liblca.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"{LIB_PATH} is missing; build it with "
                "`python -m long_context_exact_attention_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, I64, I32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
        SP = ctypes.POINTER(Shape)
        L.lca_attn_fwd.argtypes = [SP, P, P, P, I32, I64, ctypes.POINTER(Opts), P, P, P]
        L.lca_attn_bwd_workspace_size.argtypes = [SP]
        L.lca_attn_bwd_workspace_size.restype = ctypes.c_size_t
        L.lca_attn_bwd.argtypes = [SP, P, P, P, P, P, P, I32, P, P, P, P, ctypes.c_size_t, P]
        L.lca_attn_bwd_noalloc.argtypes = [SP, P, P, P, P, P, P, I32, P, P, P, P]
        L.lca_attn_fwd_varlen.argtypes = [SP, P, I64, P, P, P, I32, I64, ctypes.POINTER(Opts),
                                          P, P, P]
        L.lca_attn_bwd_varlen_workspace_size.argtypes = [SP, I64]
        L.lca_attn_bwd_varlen_workspace_size.restype = ctypes.c_size_t
        L.lca_attn_bwd_varlen.argtypes = [SP, P, I64, P, P, P, P, P, P, I32, P, P, P, P,
                                          ctypes.c_size_t, P]
        L.lca_s2attn_fwd.argtypes = [SP, P, P, P, I32, I64, I64, P, P, P]
        L.lca_s2attn_fwd_ws.argtypes = [SP, P, P, P, I32, I64, I64, P, P, P, ctypes.c_size_t, P]
        for fn in ("lca_s2attn_fwd_workspace_size", "lca_s2attn_bwd_workspace_size"):
            getattr(L, fn).argtypes = [SP, I64, I64]
            getattr(L, fn).restype = ctypes.c_size_t
        L.lca_s2attn_bwd.argtypes = [SP, P, P, P, P, P, P, I32, I64, I64, P, P, P, P,
                                     ctypes.c_size_t, P]
        L.lca_lse_merge.argtypes = [I64, I64, P, P, P, P, P, P, P]
        BP = ctypes.POINTER(BlockShape)
        L.lca_attn_fwd_block.argtypes = [BP, P, P, P, I32, I64, I64, I32, P, P, P, P]
        L.lca_attn_bwd_block_workspace_size.argtypes = [BP]
        L.lca_attn_bwd_block_workspace_size.restype = ctypes.c_size_t
        L.lca_attn_bwd_block_prep.argtypes = [BP, P, P, P, P, ctypes.c_size_t, P]
        L.lca_attn_bwd_block.argtypes = [BP, P, P, P, P, I32, I64, I64, P, ctypes.c_size_t, P,
                                         P, I32, P, P, P]
        L.lca_attn_bwd_block_dq.argtypes = [BP, P, ctypes.c_size_t, P, P]
        L.lca_cast_f32_bf16.argtypes = [I64, P, P, P]
        L.lca_accumulate_f32.argtypes = [I64, P, P, P]
        TP = ctypes.POINTER(BptShape)
        for fn in ("lca_bpt_fwd_workspace_size", "lca_bpt_bwd_workspace_size"):
            getattr(L, fn).argtypes = [TP]
            getattr(L, fn).restype = ctypes.c_size_t
        L.lca_bpt_fwd.argtypes = [TP, P, P, P, I32, P, P, P, P, P, P, P, ctypes.c_size_t, P]
        L.lca_bpt_bwd.argtypes = [TP, P, P, P, I32, P, P, P, P, P, P, P, P, P, P, P, P, P,
                                  ctypes.c_size_t, P]
        FP = ctypes.POINTER(FfnShape)
        L.lca_ffn_workspace_size.argtypes = [FP, I64]
        L.lca_ffn_workspace_size.restype = ctypes.c_size_t
        L.lca_ffn_fwd.argtypes = [FP, P, P, P, P, I64, P, P, ctypes.c_size_t, P]
        L.lca_ffn_bwd_workspace_size.argtypes = [FP, I64]
        L.lca_ffn_bwd_workspace_size.restype = ctypes.c_size_t
        L.lca_ffn_bwd.argtypes = [FP, P, P, P, P, P, I64, P, P, P, P, P, ctypes.c_size_t, P]
        L.lca_check.argtypes = [P]
        L.lca_status_string.restype = ctypes.c_char_p
        L.lca_last_error.restype = ctypes.c_char_p
        for fn in ("lca_attn_fwd", "lca_attn_bwd", "lca_attn_bwd_noalloc", "lca_s2attn_fwd",
                   "lca_s2attn_fwd_ws",
                   "lca_s2attn_bwd", "lca_attn_fwd_varlen", "lca_attn_bwd_varlen", "lca_ffn_fwd", "lca_ffn_bwd",
                   "lca_lse_merge", "lca_attn_fwd_block", "lca_attn_bwd_block_prep",
                   "lca_attn_bwd_block", "lca_attn_bwd_block_dq", "lca_cast_f32_bf16",
                   "lca_accumulate_f32", "lca_bpt_fwd", "lca_bpt_bwd", "lca_check"):
            getattr(L, fn).restype = ctypes.c_int
        _lib = L
    return _lib


def _raise(st: int):
    if st != 0:
        raise LcaError(st, lib().lca_last_error().decode())


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _shape(q: torch.Tensor, k: torch.Tensor, scale) -> Shape:
    if not (q.is_cuda and k.is_cuda):
        raise ValueError("lca needs CUDA tensors")
    if q.dim() != 4 or k.dim() != 4:
        raise ValueError("q is [B,S,Hq,d], k/v are [B,S,Hkv,d]")
    B, S, Hq, d = q.shape
    if k.shape[0] != B or k.shape[1] != S or k.shape[3] != d:
        raise ValueError("k/v shape does not match q")
    if q.dtype == torch.bfloat16:
        dt = LCA_BF16
    elif q.dtype == torch.float32:
        dt = LCA_FP32
    else:
        raise ValueError(f"unsupported dtype {q.dtype}")
    return Shape(B, Hq, k.shape[2], S, d, dt, float(scale or 0.0))


def _check_tensors(dtype, *ts):
    for t in ts:
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError("tensors must be contiguous CUDA tensors")
        if t.dtype != dtype:
            raise ValueError(f"dtype mismatch: {t.dtype} vs {dtype}")


def _opts(order, chunk_perm, q_block, timeout_cycles):
    """lca_opts plus the host array it points to (keep both alive)."""
    opts = Opts(ORDERS[order], None, int(q_block), int(timeout_cycles))
    keep = None
    if chunk_perm is not None:
        keep = (ctypes.c_int32 * len(chunk_perm))(*[int(x) for x in chunk_perm])
        opts.chunk_perm = ctypes.cast(keep, ctypes.POINTER(ctypes.c_int32))
    return opts, keep


def attn_fwd(q, k, v, causal: bool = True, kv_chunk: int = 0, order: str = "inorder",
             chunk_perm: Optional[Sequence[int]] = None, q_block: int = 0, scale=None,
             out=None, lse=None, stream=None, timeout_cycles: int = 0):
    """Exact attention forward (lca_attn_fwd).  Returns (out, lse)."""
    sh = _shape(q, k, scale)
    _check_tensors(q.dtype, q, k, v)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((q.shape[0], q.shape[2], q.shape[1]), device=q.device,
                          dtype=torch.float32)
    opts, keep = _opts(order, chunk_perm, q_block, timeout_cycles)
    _raise(lib().lca_attn_fwd(ctypes.byref(sh), _ptr(q), _ptr(k), _ptr(v), int(causal),
                              int(kv_chunk), ctypes.byref(opts), _ptr(out), _ptr(lse),
                              _stream(stream)))
    del keep
    return out, lse


def _packed_shape(q, k, cu_seqlens, scale) -> Shape:
    """Shape of a packed batch: q [T,Hq,d], k/v [T,Hkv,d], cu_seqlens int32
    [n+1] on the device."""
    if q.dim() != 3 or k.dim() != 3:
        raise ValueError("packed q is [T,Hq,d], k/v are [T,Hkv,d]")
    if not (q.is_cuda and k.is_cuda and cu_seqlens.is_cuda):
        raise ValueError("lca needs CUDA tensors")
    if cu_seqlens.dtype != torch.int32 or cu_seqlens.dim() != 1 or cu_seqlens.numel() < 2:
        raise ValueError("cu_seqlens is an int32 tensor of n + 1 offsets")
    T, Hq, d = q.shape
    if k.shape[0] != T or k.shape[2] != d:
        raise ValueError("k/v shape does not match q")
    dt = {torch.bfloat16: LCA_BF16, torch.float32: LCA_FP32}.get(q.dtype)
    if dt is None:
        raise ValueError(f"unsupported dtype {q.dtype}")
    return Shape(cu_seqlens.numel() - 1, Hq, k.shape[1], T, d, dt, float(scale or 0.0))


def attn_fwd_varlen(q, k, v, cu_seqlens, max_seqlen: int, causal: bool = True,
                    kv_chunk: int = 0, order: str = "inorder", q_block: int = 0, scale=None,
                    out=None, lse=None, stream=None, timeout_cycles: int = 0):
    """Forward over a packed batch of sequences (lca_attn_fwd_varlen).
    q [T,Hq,d], k/v [T,Hkv,d]; sequence b is rows cu_seqlens[b]:cu_seqlens[b+1].
    Returns (out [T,Hq,d], lse [Hq,T])."""
    sh = _packed_shape(q, k, cu_seqlens, scale)
    _check_tensors(q.dtype, q, k, v)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((q.shape[1], q.shape[0]), device=q.device, dtype=torch.float32)
    opts, keep = _opts(order, None, q_block, timeout_cycles)
    _raise(lib().lca_attn_fwd_varlen(ctypes.byref(sh), _ptr(cu_seqlens), int(max_seqlen),
                                     _ptr(q), _ptr(k), _ptr(v), int(causal), int(kv_chunk),
                                     ctypes.byref(opts), _ptr(out), _ptr(lse), _stream(stream)))
    del keep
    return out, lse


def varlen_workspace_size(q, k, cu_seqlens, max_seqlen: int) -> int:
    sh = _packed_shape(q, k, cu_seqlens, None)
    return int(lib().lca_attn_bwd_varlen_workspace_size(ctypes.byref(sh), int(max_seqlen)))


def attn_bwd_varlen(q, k, v, out, lse, dout, cu_seqlens, max_seqlen: int, causal: bool = True,
                    scale=None, dq=None, dk=None, dv=None, workspace=None, stream=None):
    """Gradients over a packed batch (lca_attn_bwd_varlen).  Returns (dq, dk, dv)."""
    sh = _packed_shape(q, k, cu_seqlens, scale)
    _check_tensors(q.dtype, q, k, v, out, dout)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    if workspace is None:
        n = varlen_workspace_size(q, k, cu_seqlens, max_seqlen)
        workspace = torch.empty(max(n, 1), device=q.device, dtype=torch.uint8)
    _raise(lib().lca_attn_bwd_varlen(ctypes.byref(sh), _ptr(cu_seqlens), int(max_seqlen),
                                     _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse),
                                     _ptr(dout), int(causal), _ptr(dq), _ptr(dk), _ptr(dv),
                                     _ptr(workspace),
                                     workspace.numel() * workspace.element_size(),
                                     _stream(stream)))
    return dq, dk, dv


def workspace_size(q, k) -> int:
    sh = _shape(q, k, None)
    return int(lib().lca_attn_bwd_workspace_size(ctypes.byref(sh)))


def _alloc_grads(q, k, v, dq, dk, dv, workspace):
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    if workspace is None:
        workspace = torch.empty(workspace_size(q, k), device=q.device, dtype=torch.uint8)
    return dq, dk, dv, workspace


def attn_bwd(q, k, v, out, lse, dout, causal: bool = True, scale=None, dq=None, dk=None,
             dv=None, workspace=None, stream=None):
    """Gradients of sum(dout * out) (lca_attn_bwd).  Returns (dq, dk, dv)."""
    sh = _shape(q, k, scale)
    _check_tensors(q.dtype, q, k, v, out, dout)
    dq, dk, dv, workspace = _alloc_grads(q, k, v, dq, dk, dv, workspace)
    _raise(lib().lca_attn_bwd(ctypes.byref(sh), _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse),
                              _ptr(dout), int(causal), _ptr(dq), _ptr(dk), _ptr(dv),
                              _ptr(workspace), workspace.numel() * workspace.element_size(),
                              _stream(stream)))
    return dq, dk, dv


def attn_bwd_noalloc(q, k, v, out, lse, dout, causal: bool = True, scale=None, dq=None,
                     dk=None, dv=None, stream=None):
    """lca_attn_bwd_noalloc: the backward pass with the library's built-in
    scratch instead of a workspace, for callers that cannot allocate device
    memory.  Calls that overlap on the GPU share that scratch and race.
    Returns (dq, dk, dv)."""
    sh = _shape(q, k, scale)
    _check_tensors(q.dtype, q, k, v, out, dout)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    _raise(lib().lca_attn_bwd_noalloc(ctypes.byref(sh), _ptr(q), _ptr(k), _ptr(v), _ptr(out),
                                      _ptr(lse), _ptr(dout), int(causal), _ptr(dq), _ptr(dk),
                                      _ptr(dv), _stream(stream)))
    return dq, dk, dv


def s2attn_workspace_sizes(q, k, group: int, shift_heads: int):
    """(forward, backward) workspace bytes of S2-Attn with this group."""
    sh = _shape(q, k, None)
    L = lib()
    return (int(L.lca_s2attn_fwd_workspace_size(ctypes.byref(sh), int(group), int(shift_heads))),
            int(L.lca_s2attn_bwd_workspace_size(ctypes.byref(sh), int(group), int(shift_heads))))


def s2attn_fwd(q, k, v, group: int, shift_heads: int, causal: bool = True, scale=None,
               out=None, lse=None, workspace=None, stream=None):
    """LongLoRA S2-Attn forward (lca_s2attn_fwd_ws).  A workspace is only
    needed when group/2 is not a whole number of tiles.  Returns (out, lse)."""
    sh = _shape(q, k, scale)
    _check_tensors(q.dtype, q, k, v)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((q.shape[0], q.shape[2], q.shape[1]), device=q.device,
                          dtype=torch.float32)
    if workspace is None:
        n = s2attn_workspace_sizes(q, k, group, shift_heads)[0]
        workspace = torch.empty(n, device=q.device, dtype=torch.uint8) if n else None
    nbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _raise(lib().lca_s2attn_fwd_ws(ctypes.byref(sh), _ptr(q), _ptr(k), _ptr(v), int(causal),
                                   int(group), int(shift_heads), _ptr(out), _ptr(lse),
                                   _ptr(workspace), nbytes, _stream(stream)))
    return out, lse


def s2attn_bwd(q, k, v, out, lse, dout, group: int, shift_heads: int, causal: bool = True,
               scale=None, dq=None, dk=None, dv=None, workspace=None, stream=None):
    """LongLoRA S2-Attn backward (lca_s2attn_bwd).  Returns (dq, dk, dv)."""
    sh = _shape(q, k, scale)
    _check_tensors(q.dtype, q, k, v, out, dout)
    if workspace is None:
        n = s2attn_workspace_sizes(q, k, group, shift_heads)[1]
        workspace = torch.empty(max(n, 16), device=q.device, dtype=torch.uint8)
    dq, dk, dv, workspace = _alloc_grads(q, k, v, dq, dk, dv, workspace)
    _raise(lib().lca_s2attn_bwd(ctypes.byref(sh), _ptr(q), _ptr(k), _ptr(v), _ptr(out),
                                _ptr(lse), _ptr(dout), int(causal), int(group),
                                int(shift_heads), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(workspace),
                                workspace.numel() * workspace.element_size(), _stream(stream)))
    return dq, dk, dv


def ffn_workspace_size(T: int, h: int, f: int, block_tokens: int = 0) -> int:
    sh = FfnShape(int(T), int(h), int(f))
    return int(lib().lca_ffn_workspace_size(ctypes.byref(sh), int(block_tokens)))


def ffn_fwd(x, w_gate, w_up, w_down, block_tokens: int = 0, out=None, workspace=None,
            stream=None):
    """Blockwise gated-SiLU feedforward (lca_ffn_fwd): x [T,h], w_gate/w_up
    [f,h], w_down [h,f], all bf16.  Returns out [T,h]."""
    _check_tensors(torch.bfloat16, x, w_gate, w_up, w_down)
    if x.dim() != 2 or w_gate.dim() != 2 or w_down.dim() != 2:
        raise ValueError("x is [T,h], w_gate/w_up are [f,h], w_down is [h,f]")
    T, h = x.shape
    f = w_gate.shape[0]
    if w_gate.shape != (f, h) or w_up.shape != (f, h) or w_down.shape != (h, f):
        raise ValueError("weight shapes do not match x")
    sh = FfnShape(T, h, f)
    out = torch.empty_like(x) if out is None else out
    if workspace is None:
        n = ffn_workspace_size(T, h, f, block_tokens)
        workspace = torch.empty(max(n, 16), device=x.device, dtype=torch.uint8)
    _raise(lib().lca_ffn_fwd(ctypes.byref(sh), _ptr(x), _ptr(w_gate), _ptr(w_up), _ptr(w_down),
                             int(block_tokens), _ptr(out), _ptr(workspace),
                             workspace.numel() * workspace.element_size(), _stream(stream)))
    return out


def ffn_bwd_workspace_size(T: int, h: int, f: int, block_tokens: int = 0) -> int:
    sh = FfnShape(int(T), int(h), int(f))
    return int(lib().lca_ffn_bwd_workspace_size(ctypes.byref(sh), int(block_tokens)))


def ffn_bwd(x, w_gate, w_up, w_down, dout, block_tokens: int = 0, dx=None, dw_gate=None,
            dw_up=None, dw_down=None, workspace=None, stream=None):
    """Gradients of the blockwise feedforward (lca_ffn_bwd).  dx (bf16) is
    overwritten; dw_gate, dw_up, dw_down are float32 and the gradients are
    added to them (new zero tensors when not given).  Returns (dx, dw_gate,
    dw_up, dw_down)."""
    _check_tensors(torch.bfloat16, x, w_gate, w_up, w_down, dout)
    T, h = x.shape
    f = w_gate.shape[0]
    if dout.shape != x.shape:
        raise ValueError("dout must have x's shape")
    dx = torch.empty_like(x) if dx is None else dx
    z = lambda t: torch.zeros(t.shape, device=t.device, dtype=torch.float32)
    dw_gate = z(w_gate) if dw_gate is None else dw_gate
    dw_up = z(w_up) if dw_up is None else dw_up
    dw_down = z(w_down) if dw_down is None else dw_down
    _check_tensors(torch.float32, dw_gate, dw_up, dw_down)
    sh = FfnShape(T, h, f)
    if workspace is None:
        n = ffn_bwd_workspace_size(T, h, f, block_tokens)
        workspace = torch.empty(max(n, 16), device=x.device, dtype=torch.uint8)
    _raise(lib().lca_ffn_bwd(ctypes.byref(sh), _ptr(x), _ptr(w_gate), _ptr(w_up), _ptr(w_down),
                             _ptr(dout), int(block_tokens), _ptr(dx), _ptr(dw_gate), _ptr(dw_up),
                             _ptr(dw_down), _ptr(workspace),
                             workspace.numel() * workspace.element_size(), _stream(stream)))
    return dx, dw_gate, dw_up, dw_down


def lse_merge(o_a, lse_a, o_b, lse_b, o_out=None, lse_out=None, stream=None):
    """Merge two float32 partial results (lca_lse_merge).  o_*: [rows, d],
    lse_*: [rows].  Returns (o, lse)."""
    for t in (o_a, lse_a, o_b, lse_b):
        if not t.is_cuda or t.dtype != torch.float32 or not t.is_contiguous():
            raise ValueError("lse_merge takes contiguous float32 CUDA tensors")
    rows, d = o_a.shape[0], o_a.numel() // max(o_a.shape[0], 1)
    o_out = torch.empty_like(o_a) if o_out is None else o_out
    lse_out = torch.empty_like(lse_a) if lse_out is None else lse_out
    _raise(lib().lca_lse_merge(rows, d, _ptr(o_a), _ptr(lse_a), _ptr(o_b), _ptr(lse_b),
                               _ptr(o_out), _ptr(lse_out), _stream(stream)))
    return o_out, lse_out


# ---------------------------------------------------------------- blocks

def _block_shape(q, k, scale) -> BlockShape:
    """q [B,Sq,Hq,d] (bf16), k/v [B,Sk,Hkv,d]."""
    if not (q.is_cuda and k.is_cuda):
        raise ValueError("lca needs CUDA tensors")
    if q.dim() != 4 or k.dim() != 4 or k.shape[0] != q.shape[0] or k.shape[3] != q.shape[3]:
        raise ValueError("q is [B,Sq,Hq,d], k/v are [B,Sk,Hkv,d]")
    if q.dtype != torch.bfloat16:
        raise ValueError("block calls take bf16 tensors")
    B, Sq, Hq, d = q.shape
    return BlockShape(B, Hq, k.shape[2], Sq, k.shape[1], d, LCA_BF16, float(scale or 0.0))


def attn_fwd_block(q, k, v, q_pos0: int, k_pos0: int, causal: bool = True,
                   accumulate: bool = False, o_acc=None, lse_acc=None, out=None, scale=None,
                   stream=None):
    """One ring step of the forward (lca_attn_fwd_block): attend the query
    block (rows at positions q_pos0...) to the key/value block (keys at
    k_pos0...) and fold the result into the running float32 (o_acc, lse_acc)
    (or start it when accumulate is False).  out, when given, receives the
    merged output as bf16.  Returns (o_acc, lse_acc, out)."""
    sh = _block_shape(q, k, scale)
    _check_tensors(torch.bfloat16, q, k, v)
    B, Sq, Hq, d = q.shape
    if o_acc is None:
        o_acc = torch.empty((B, Sq, Hq, d), device=q.device, dtype=torch.float32)
    if lse_acc is None:
        lse_acc = torch.empty((B, Hq, Sq), device=q.device, dtype=torch.float32)
    _check_tensors(torch.float32, o_acc, lse_acc)
    _raise(lib().lca_attn_fwd_block(ctypes.byref(sh), _ptr(q), _ptr(k), _ptr(v), int(causal),
                                    int(q_pos0), int(k_pos0), int(bool(accumulate)), _ptr(o_acc),
                                    _ptr(lse_acc), _ptr(out), _stream(stream)))
    return o_acc, lse_acc, out


def bwd_block_workspace_size(q, k) -> int:
    sh = _block_shape(q, k, None)
    return int(lib().lca_attn_bwd_block_workspace_size(ctypes.byref(sh)))


def attn_bwd_block_prep(q, out, lse, dout, workspace=None, scale=None, stream=None):
    """Start a query block's backward (lca_attn_bwd_block_prep) from its
    final out and lse.  Returns the workspace (allocated when not given)."""
    sh = _block_shape(q, q, scale)
    _check_tensors(torch.bfloat16, out, dout)
    if workspace is None:
        workspace = torch.empty(bwd_block_workspace_size(q, q), device=q.device,
                                dtype=torch.uint8)
    _raise(lib().lca_attn_bwd_block_prep(ctypes.byref(sh), _ptr(out), _ptr(lse), _ptr(dout),
                                         _ptr(workspace),
                                         workspace.numel() * workspace.element_size(),
                                         _stream(stream)))
    return workspace


def attn_bwd_block(q, k, v, dout, q_pos0: int, k_pos0: int, workspace, causal: bool = True,
                   dk_acc=None, dv_acc=None, accumulate_kv: bool = True, dk=None, dv=None,
                   scale=None, stream=None):
    """One ring step of the backward (lca_attn_bwd_block): dQ into the
    workspace, dK/dV into the float32 accumulators dk_acc/dv_acc (added when
    accumulate_kv, else overwritten) or, when those are None, into bf16
    dk/dv (overwritten).  Returns (dk_acc, dv_acc) or (dk, dv)."""
    sh = _block_shape(q, k, scale)
    _check_tensors(torch.bfloat16, q, k, v, dout)
    if dk_acc is None and dk is None:
        dk, dv = torch.empty_like(k), torch.empty_like(v)
    _raise(lib().lca_attn_bwd_block(ctypes.byref(sh), _ptr(q), _ptr(k), _ptr(v), _ptr(dout),
                                    int(causal), int(q_pos0), int(k_pos0), _ptr(workspace),
                                    workspace.numel() * workspace.element_size(), _ptr(dk_acc),
                                    _ptr(dv_acc), int(bool(accumulate_kv)), _ptr(dk), _ptr(dv),
                                    _stream(stream)))
    return (dk_acc, dv_acc) if dk_acc is not None else (dk, dv)


def attn_bwd_block_dq(q, workspace, dq=None, scale=None, stream=None):
    """Finish a query block's backward (lca_attn_bwd_block_dq).  Returns dq."""
    sh = _block_shape(q, q, scale)
    dq = torch.empty_like(q) if dq is None else dq
    _raise(lib().lca_attn_bwd_block_dq(ctypes.byref(sh), _ptr(workspace),
                                       workspace.numel() * workspace.element_size(), _ptr(dq),
                                       _stream(stream)))
    return dq


def cast_bf16(src, dst=None, stream=None):
    """dst = bf16(src) for a contiguous float32 CUDA tensor (lca_cast_f32_bf16)."""
    _check_tensors(torch.float32, src)
    dst = torch.empty(src.shape, device=src.device, dtype=torch.bfloat16) if dst is None else dst
    _check_tensors(torch.bfloat16, dst)
    _raise(lib().lca_cast_f32_bf16(src.numel(), _ptr(src), _ptr(dst), _stream(stream)))
    return dst


def accumulate(src, dst, stream=None):
    """dst += src for contiguous float32 CUDA tensors (lca_accumulate_f32)."""
    _check_tensors(torch.float32, src, dst)
    if src.numel() != dst.numel():
        raise ValueError("accumulate: sizes differ")
    _raise(lib().lca_accumulate_f32(src.numel(), _ptr(src), _ptr(dst), _stream(stream)))
    return dst


# ---------------------------------------------------------------- blockwise transformer

def _bpt_shape(q, k, w_gate, q_block, scale) -> BptShape:
    """q [S, Hq, d], k/v [S, Hkv, d] (one sequence), w_gate [f, Hq*d]."""
    if q.dim() != 3 or k.dim() != 3 or k.shape[0] != q.shape[0] or k.shape[2] != q.shape[2]:
        raise ValueError("q is [S,Hq,d], k/v are [S,Hkv,d]")
    S, Hq, d = q.shape
    if w_gate.dim() != 2 or w_gate.shape[1] != Hq * d:
        raise ValueError("w_gate is [f, Hq*d]")
    return BptShape(S, Hq, k.shape[1], d, w_gate.shape[0], int(q_block), float(scale or 0.0))


def bpt_fwd(q, k, v, w_gate, w_up, w_down, causal: bool = True, q_block: int = 0, scale=None,
            attn_out=None, lse=None, out=None, workspace=None, stream=None):
    """Blockwise Transformer sweep (lca_bpt_fwd): per block of q_block query
    rows, attention over the keys they see, then the gated-SiLU feedforward
    of those rows.  Returns (attn_out [S,Hq,d], lse [Hq,S], out [S,Hq*d])."""
    _check_tensors(torch.bfloat16, q, k, v, w_gate, w_up, w_down)
    sh = _bpt_shape(q, k, w_gate, q_block, scale)
    S, Hq, d = q.shape
    attn_out = torch.empty_like(q) if attn_out is None else attn_out
    lse = torch.empty((Hq, S), device=q.device, dtype=torch.float32) if lse is None else lse
    out = torch.empty((S, Hq * d), device=q.device, dtype=torch.bfloat16) if out is None else out
    if workspace is None:
        n = int(lib().lca_bpt_fwd_workspace_size(ctypes.byref(sh)))
        workspace = torch.empty(max(n, 16), device=q.device, dtype=torch.uint8)
    _raise(lib().lca_bpt_fwd(ctypes.byref(sh), _ptr(q), _ptr(k), _ptr(v), int(causal),
                             _ptr(w_gate), _ptr(w_up), _ptr(w_down), _ptr(attn_out), _ptr(lse),
                             _ptr(out), _ptr(workspace),
                             workspace.numel() * workspace.element_size(), _stream(stream)))
    return attn_out, lse, out


def bpt_bwd(q, k, v, w_gate, w_up, w_down, attn_out, lse, dout, causal: bool = True,
            q_block: int = 0, scale=None, dq=None, dk=None, dv=None, dw_gate=None, dw_up=None,
            dw_down=None, workspace=None, stream=None):
    """Gradients of the sweep (lca_bpt_bwd).  dw_* are float32 and the
    gradients are added to them (new zero tensors when not given).  Returns
    (dq, dk, dv, dw_gate, dw_up, dw_down)."""
    _check_tensors(torch.bfloat16, q, k, v, w_gate, w_up, w_down, attn_out, dout)
    sh = _bpt_shape(q, k, w_gate, q_block, scale)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    z = lambda t: torch.zeros(t.shape, device=t.device, dtype=torch.float32)
    dw_gate = z(w_gate) if dw_gate is None else dw_gate
    dw_up = z(w_up) if dw_up is None else dw_up
    dw_down = z(w_down) if dw_down is None else dw_down
    if workspace is None:
        n = int(lib().lca_bpt_bwd_workspace_size(ctypes.byref(sh)))
        workspace = torch.empty(max(n, 16), device=q.device, dtype=torch.uint8)
    _raise(lib().lca_bpt_bwd(ctypes.byref(sh), _ptr(q), _ptr(k), _ptr(v), int(causal),
                             _ptr(w_gate), _ptr(w_up), _ptr(w_down), _ptr(attn_out), _ptr(lse),
                             _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dw_gate),
                             _ptr(dw_up), _ptr(dw_down), _ptr(workspace),
                             workspace.numel() * workspace.element_size(), _stream(stream)))
    return dq, dk, dv, dw_gate, dw_up, dw_down


def check(stream=None):
    """Synchronise and raise LcaError if a kernel wait ran out."""
    _raise(lib().lca_check(_stream(stream)))
