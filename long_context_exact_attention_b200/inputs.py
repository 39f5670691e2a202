"""Seeded synthetic inputs for exact long-context attention.

This module holds workload shapes and random-number recipes only: it contains
none of the attention arithmetic, and both the CUDA path's tests and the CPU
oracle's tests draw their inputs from it.  Nothing here imports the CUDA
binding or the oracle.

Recipe (the pages fix none of it beyond "Llama-shaped" sequences):
  * every tensor is drawn in slabs of ``SLAB_TOKENS`` tokens; slab ``i`` of
    tensor ``t`` uses a ``torch.Generator`` seeded with
    ``seed * 1_000_003 + t * 10_007 + i`` on the device that generates it
    (tensor ids: q=0, k=1, v=2, dout=3);
  * values are standard normal, scaled by the workload's ``std`` (1.0 for the
    fp32 check, 0.5 for the bf16 Llama-shaped workloads);
  * where the workload asks for it, rotary position embedding (base 10000,
    half-split pairing of dims i and i + d/2, positions 0..S-1) is applied to
    q and k in float64 before the single rounding to the storage dtype;
  * bf16 storage rounds to nearest even (torch's cast).

Values drawn on a CUDA device differ from values drawn on the CPU for the
same seed; a parity test always hands the oracle a host copy of the very
tensors the kernel saw.
"""

from __future__ import annotations

import dataclasses
from typing import Optional

import torch

SLAB_TOKENS = 65536
TENSOR_ID = {"q": 0, "k": 1, "v": 2, "dout": 3}


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape and input recipe of one attention workload.

    Layout: q/out/dout are [B, S, Hq, d]; k/v are [B, S, Hkv, d]; lse is
    [B, Hq, S].  ``kv_chunk`` is the KV chunk length of the simulated ring;
    ``group``/``shift_heads`` select LongLoRA's shifted sparse attention.
    ``lengths`` makes it a packed batch: B = 1, S = sum(lengths) tokens on
    one axis, sequence i holding the next lengths[i] of them.
    """

    name: str
    B: int
    Hq: int
    Hkv: int
    S: int
    d: int
    dtype: str  # "bf16" or "fp32"
    causal: bool
    seed: int
    std: float
    rope: bool = False
    kv_chunk: int = 0          # 0: one chunk spanning the sequence
    order: str = "inorder"     # "inorder" | "ring" | "custom"
    q_block: int = 0           # ring query-block length (0: kv_chunk)
    group: int = 0             # S2-Attn group size (0: not S2)
    shift_heads: int = 0       # S2-Attn: trailing heads shifted by group/2
    backward: bool = True
    lengths: tuple = ()        # packed batch: sequence lengths (sum = S)

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32

    @property
    def s2(self) -> bool:
        return self.group > 0

    @property
    def packed(self) -> bool:
        return len(self.lengths) > 0

    def fwd_flops(self) -> float:
        """Algorithmic forward FLOPs: 4*B*Hq*S*S_vis*d with S_vis the mean
        number of visible keys per row (S for dense, S/2 for causal, G or G/2
        for S2-Attn); a packed batch sums 4*Hq*L*L_vis*d over its sequences."""
        frac = 0.5 if self.causal else 1.0
        if self.packed:
            return 4.0 * self.Hq * frac * self.d * float(sum(n * n for n in self.lengths))
        span = self.group if self.s2 else self.S
        return 4.0 * self.B * self.Hq * self.S * span * frac * self.d

    def bwd_flops(self) -> float:
        """Backward counts five matmuls against the forward's two."""
        return 2.5 * self.fwd_flops()


WORKLOADS = {
    w.name: w
    for w in [
        Workload("tiny_fp32_s256", B=1, Hq=2, Hkv=2, S=256, d=64, dtype="fp32",
                 causal=True, seed=0, std=1.0, kv_chunk=64),
        Workload("llama2_7b_s32k", B=1, Hq=32, Hkv=32, S=32768, d=128,
                 dtype="bf16", causal=True, seed=1, std=0.5, rope=True,
                 kv_chunk=4096, order="ring"),
        Workload("longlora_s2_s8k", B=1, Hq=32, Hkv=32, S=8192, d=128,
                 dtype="bf16", causal=True, seed=2, std=0.5, group=2048,
                 shift_heads=16),
        Workload("llama3_8b_gqa_s128k", B=1, Hq=32, Hkv=8, S=131072, d=128,
                 dtype="bf16", causal=True, seed=3, std=0.5, kv_chunk=8192),
        Workload("llama2_13b_s1m", B=1, Hq=40, Hkv=40, S=1048576, d=128,
                 dtype="bf16", causal=True, seed=4, std=0.5, kv_chunk=16384,
                 q_block=16384, order="ring", backward=False),
        # LongLoRA's 100K context: half a group (12500 tokens) is not a
        # whole tile, so the rolled S2 path runs
        Workload("longlora_s2_s100k", B=1, Hq=32, Hkv=32, S=100000, d=128,
                 dtype="bf16", causal=True, seed=5, std=0.5, group=25000,
                 shift_heads=16),
        # the Llama-3-8B layer at 256K tokens: the sequence-parallel (ring)
        # workload, split over the ranks
        Workload("llama3_8b_gqa_s256k", B=1, Hq=32, Hkv=8, S=262144, d=128,
                 dtype="bf16", causal=True, seed=7, std=0.5),
        # a quarter of the 32K layer's heads: the case ncu captures in full
        # (inputs 4 x 64 MiB, still larger than L2 together)
        Workload("llama2_7b_s32k_h8", B=1, Hq=8, Hkv=8, S=32768, d=128,
                 dtype="bf16", causal=True, seed=1, std=0.5, rope=True,
                 kv_chunk=4096, order="ring"),
        # a quarter of the 128K GQA layer's heads (8 query, 2 key/value),
        # the same sequence and chunking: the case ncu captures in full for
        # that layer (inputs 2 x 256 + 2 x 64 MiB)
        Workload("llama3_8b_gqa_s128k_h8", B=1, Hq=8, Hkv=2, S=131072, d=128,
                 dtype="bf16", causal=True, seed=3, std=0.5, kv_chunk=8192),
    ]
}


def _packed_workload(name, n, max_len, seed, **kw):
    lengths = tuple(packed_lengths(n, max_len, seed))
    return Workload(name, B=1, S=sum(lengths), lengths=lengths, seed=seed, **kw)


def packed_lengths(n: int, max_len: int, seed: int) -> list:
    """Seeded lengths of ``n`` packed sequences: a mix of empty, one-token,
    tile-multiple and ragged lengths up to ``max_len`` (the recipe of the
    packed-batch cases; the pages fix no length distribution).  One sequence
    in four takes an edge value (0, 1, 128 or max_len), the rest are uniform
    in [1, max_len]."""
    g = torch.Generator().manual_seed(seed * 104729 + n)
    edges = [0, 1, min(128, max_len), max_len]
    out = []
    for i in range(n):
        if int(torch.randint(4, (1,), generator=g)) == 0:
            out.append(edges[int(torch.randint(len(edges), (1,), generator=g))])
        else:
            out.append(int(torch.randint(1, max_len + 1, (1,), generator=g)))
    return out


# Llama-3-8B attention shapes over a packed batch of documents up to 32K
# tokens (about 128K tokens in all): the ragged, variable-length case.
for _w in [_packed_workload("llama3_8b_gqa_packed_128k", n=8, max_len=32768, seed=6, Hq=32,
                            Hkv=8, d=128, dtype="bf16", causal=True, std=0.5)]:
    WORKLOADS[_w.name] = _w


@dataclasses.dataclass(frozen=True)
class FfnWorkload:
    """Shape and input recipe of one blockwise-feedforward workload: token
    rows x [T, h] (standard normal, as after an RMS norm), weights w_gate,
    w_up [f, h] and w_down [h, f] (normal with std ``w_std``, Llama's
    initialisation), all rounded once to bf16; ``block`` token rows at a
    time."""

    name: str
    T: int
    h: int
    f: int
    block: int
    seed: int
    w_std: float = 0.02

    def flops(self) -> float:
        """Forward: three products of 2*T*h*f each (gate, up, down)."""
        return 6.0 * self.T * self.h * self.f

    def bwd_flops(self) -> float:
        """Backward: eight products of 2*T*h*f (dH; gate and up recomputed;
        dx from dG and dU; three weight gradients)."""
        return 16.0 * self.T * self.h * self.f


FFN_WORKLOADS = {
    w.name: w
    for w in [
        # the Llama-2-7B feedforward over the 32K-token sequence, 8K tokens
        # per block
        FfnWorkload("llama2_7b_ffn_s32k", T=32768, h=4096, f=11008, block=8192, seed=11),
        FfnWorkload("tiny_ffn", T=300, h=256, f=384, block=128, seed=12),
    ]
}


def make_ffn_inputs(w: FfnWorkload, device="cpu") -> dict:
    """x, w_gate, w_up, w_down of workload w (one generator per tensor)."""
    shapes = {"x": (w.T, w.h), "w_gate": (w.f, w.h), "w_up": (w.f, w.h), "w_down": (w.h, w.f)}
    out = {}
    for i, (name, shp) in enumerate(shapes.items()):
        g = torch.Generator(device=device)
        g.manual_seed(w.seed * 1_000_003 + 20 + i)
        t = torch.randn(shp, generator=g, device=device, dtype=torch.float32)
        if name != "x":
            t.mul_(w.w_std)
        out[name] = t.to(torch.bfloat16)
        del t
    return out


def _slab_seed(seed: int, tensor_id: int, slab: int) -> int:
    return seed * 1_000_003 + tensor_id * 10_007 + slab


def rope_inplace_f64(x: torch.Tensor, pos0: int, base: float = 10000.0) -> None:
    """Rotary embedding on a float64 [B, T, H, d] slab whose first token sits
    at absolute position ``pos0``.  Pairs dim i with dim i + d/2, angle
    pos * base**(-2i/d)."""
    d = x.shape[-1]
    half = d // 2
    T = x.shape[1]
    i = torch.arange(half, dtype=torch.float64, device=x.device)
    inv_freq = base ** (-2.0 * i / d)
    pos = torch.arange(pos0, pos0 + T, dtype=torch.float64, device=x.device)
    ang = pos[:, None] * inv_freq[None, :]          # [T, half]
    c = torch.cos(ang)[None, :, None, :]
    s = torch.sin(ang)[None, :, None, :]
    a = x[..., :half].clone()
    b = x[..., half:].clone()
    x[..., :half] = a * c - b * s
    x[..., half:] = a * s + b * c


def make_tensor(w: Workload, which: str, device="cpu",
                tokens: Optional[tuple] = None) -> torch.Tensor:
    """Draw tensor ``which`` ("q", "k", "v" or "dout") of workload ``w``.

    ``tokens=(t0, t1)`` draws only that token range (slab-aligned generation
    keeps it identical to the matching slice of the full tensor)."""
    tid = TENSOR_ID[which]
    H = w.Hq if which in ("q", "dout") else w.Hkv
    t0, t1 = tokens if tokens is not None else (0, w.S)
    out = torch.empty((w.B, t1 - t0, H, w.d), dtype=w.torch_dtype, device=device)
    first_slab = t0 // SLAB_TOKENS
    last_slab = (t1 - 1) // SLAB_TOKENS
    for slab in range(first_slab, last_slab + 1):
        s0 = slab * SLAB_TOKENS
        s1 = min(s0 + SLAB_TOKENS, w.S)
        g = torch.Generator(device=device)
        g.manual_seed(_slab_seed(w.seed, tid, slab))
        x = torch.randn((w.B, s1 - s0, H, w.d), generator=g, device=device,
                        dtype=torch.float32)
        a0, a1 = max(s0, t0), min(s1, t1)
        x = x[:, a0 - s0:a1 - s0]
        if w.rope and which in ("q", "k"):
            x64 = x.to(torch.float64) * w.std
            rope_inplace_f64(x64, a0)
            out[:, a0 - t0:a1 - t0] = x64.to(w.torch_dtype)
            del x64
        else:
            out[:, a0 - t0:a1 - t0] = (x * w.std).to(w.torch_dtype)
        del x
    return out


def make_inputs(w: Workload, device="cpu", with_dout: Optional[bool] = None):
    """Return dict with q, k, v (and dout when the workload has a backward)."""
    if with_dout is None:
        with_dout = w.backward
    names = ["q", "k", "v"] + (["dout"] if with_dout else [])
    return {n: make_tensor(w, n, device) for n in names}


def packed_offsets(lengths, start: int = 0) -> list:
    """Offsets cu[0..n] of sequences of the given lengths packed from token
    ``start`` on."""
    cu = [start]
    for n in lengths:
        cu.append(cu[-1] + int(n))
    return cu


def chunk_permutation(n_chunks: int, seed: int) -> list:
    """Seeded random order of ``n_chunks`` KV chunks (for order-invariance
    runs)."""
    g = torch.Generator().manual_seed(seed * 7919 + n_chunks)
    return torch.randperm(n_chunks, generator=g).tolist()


def shrink(w: Workload, **kw) -> Workload:
    """Same recipe at other sizes (for parity cases the oracle finishes)."""
    return dataclasses.replace(w, **kw)
