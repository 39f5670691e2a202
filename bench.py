"""Benchmark: exact causal attention forward + backward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl lca|reference]

A step is one pass of the whole path over one batch: lca_attn_fwd over the
key/value chunks (with the (O, lse) merge) followed by the backward.  The
default workload is the largest single-GPU forward + backward configuration
of the metric, the Llama-3-8B GQA layer at 128K: B=1, 32 query / 8
key/value heads, d=128, S=131072, bf16, causal, 16 KV chunks of 8192.  The
same line also reports the Llama-2-7B 32K layer (B=1, H=32, S=32768, 8
chunks of 4096 in ring order, RoPE inputs) under "other_workloads", so the
line covers both ends of the 32K-128K range.

The dense backward is timed as its three launches (row-dot prep, the main
tensor-core kernel, dq finalize) through the block entry points, so the main
kernel has CUDA events of its own; the end-to-end leg calls lca_attn_fwd and
lca_attn_bwd with host buffers.

Under torchrun (N > 1) every rank runs an independent replica of the
workload on its own GPU; timing is the maximum over ranks.  Rank 0 prints
one JSON line.

--impl reference times the fp64 CPU oracle on a bounded sample of the same
workload on this host's cores (the oracle is the only other implementation
there is).

--workload llama2_7b_ffn_s32k measures the blockwise feedforward instead
(lca_ffn_fwd + lca_ffn_bwd over 32768 tokens of the Llama-2-7B feedforward
in blocks of 8192): its own line, metric "blockwise feedforward TFLOP/s".

--workload ring_<attention workload> (e.g. ring_llama3_8b_gqa_s256k) runs
ring attention across the N ranks instead of replicas: one sequence split
zig-zag over the ranks, every step one ring forward + backward with NCCL
transfers; strong scaling, value = the whole problem's FLOPs / step time.
--workload ulysses_<attention workload> does the same with Ulysses
(contiguous blocks, all-to-all between the sequence split and a head split;
N must divide the key/value heads).
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "causal attention TFLOP/s fwd+bwd (bf16, 1×B200) & fraction of dense BF16 peak"
FFN_METRIC = "blockwise feedforward TFLOP/s fwd+bwd (bf16, 1×B200) & fraction of dense BF16 peak"
NOMINAL_BF16_TFLOPS = 2250.0
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="llama3_8b_gqa_s128k")
    ap.add_argument("--impl", default="lca", choices=["lca", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the second attention workload of the line")
    return ap.parse_args()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def source_sha(files=None):
    """Hash of the kernel sources `files` (names in csrc/; all of them when
    None)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "long_context_exact_attention_b200", "csrc")
    for f in sorted(files or os.listdir(csrc)):
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(f.encode() + fh.read())
    return h.hexdigest()[:16]


def traffic_record(kernel, workload):
    """DRAM bytes per launch of `kernel` on `workload` from the committed ncu
    summaries, if they were taken on the current sources of that kernel (the
    files the record lists); else None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    rec = d.get(f"{kernel}@{workload}")
    if not rec or rec.get("source_sha") != source_sha(rec.get("sources")):
        return None
    return rec


class ClockSampler:
    """nvidia-smi clock/throttle samples during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.rows = []
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append([x.strip() for x in line.split(",")])

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = [r for r in self.rows if len(r) >= 9]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            for n, v in zip(names, r[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(rows)}


# ---------------------------------------------------------------- ranks

def max_over_ranks(value, device=None):
    """Maximum of a per-rank float over all ranks of the default process
    group (the value itself when there is no group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device or "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(flops_per_step, world, steps, max_ms):
    """Whole-job throughput: every rank runs `steps` steps of the same
    workload (replicas), timed by the slowest rank."""
    return flops_per_step * world * steps / (max_ms * 1e-3) / 1e12


def pipelined_e2e(torch, dev, sets, in_names, out_names, host_in, host_out, compute, n):
    """Time n end-to-end steps through pinned host memory: every step uploads
    its inputs (host_in -> set[in_names]), computes, and downloads its
    results (set[out_names] -> host_out).  Two device sets alternate, with
    uploads on one copy stream and downloads on another, so step i+1's upload
    and step i-1's download overlap step i's compute (a training input
    pipeline).  Returns the device time in ms from the first upload to the
    last download."""
    up, down, comp = (torch.cuda.Stream(dev) for _ in range(3))
    ev = lambda: torch.cuda.Event()
    in_ready, done, drained = [ev(), ev()], [ev(), ev()], [ev(), ev()]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    start.record(up)
    for i in range(n):
        b = i % 2
        S = sets[b]
        if i >= 2:
            up.wait_event(done[b])      # step i-2 no longer reads this set's inputs
        with torch.cuda.stream(up):
            for name, h in zip(in_names, host_in):
                S[name].copy_(h, non_blocking=True)
        in_ready[b].record(up)
        comp.wait_event(in_ready[b])
        if i >= 2:
            comp.wait_event(drained[b])  # step i-2's results have left this set
        compute(S, comp)
        done[b].record(comp)
        down.wait_event(done[b])
        with torch.cuda.stream(down):
            for h, name in zip(host_out, out_names):
                h.copy_(S[name], non_blocking=True)
        drained[b].record(down)
    up.wait_event(drained[(n - 1) % 2])  # the download stream runs in order
    end.record(up)
    end.synchronize()
    return start.elapsed_time(end)


# ---------------------------------------------------------------- CPU oracle

def oracle_sample(w, seconds_target=12.0, max_rows=None):
    """Time the fp64 oracle (as it stands) on the last R query rows of head 0
    of workload w: forward and backward of those rows.  R doubles until one
    run takes >= seconds_target / 4, then the timed run is repeated to about
    seconds_target.  Returns (tflops, rows, seconds, cores)."""
    import numpy as np
    import torch

    import oracle
    from long_context_exact_attention_b200.inputs import make_tensor

    tok = (0, w.S)
    if w.packed:
        # a packed batch: the longest sequence, as a dense problem of its own
        i = max(range(len(w.lengths)), key=lambda j: w.lengths[j])
        tok = (sum(w.lengths[:i]), sum(w.lengths[:i + 1]))
    elif w.s2:
        # S2-Attn: the last group of head 0 (an unshifted head, so the
        # group is a contiguous token range attended causally on its own)
        assert w.shift_heads < w.Hq
        tok = (w.S - w.group, w.S)
    S = tok[1] - tok[0]
    q = make_tensor(w, "q", "cpu", tok)[:, :, :w.Hq // w.Hkv]
    k = make_tensor(w, "k", "cpu", tok)[:, :, :1]
    v = make_tensor(w, "v", "cpu", tok)[:, :, :1]
    do = make_tensor(w, "dout", "cpu", tok)[:, :, :w.Hq // w.Hkv]
    q, k, v, do = (t.contiguous() for t in (q, k, v, do))

    def flops(rows):
        vis = np.asarray(rows) + 1 if w.causal else np.full(len(rows), S)
        return 3.5 * 4.0 * w.d * float(vis.sum()) * (w.Hq // w.Hkv)

    R = 64
    while True:
        rows = np.arange(S - R, S)
        t0 = time.perf_counter()
        oracle.attention_backward_rows(q, k, v, do, w.causal, 0, 0, rows)
        dt = time.perf_counter() - t0
        if dt >= seconds_target / 4 or R >= S or (max_rows and R >= max_rows):
            break
        R *= 2
    reps = max(1, int(round(seconds_target / max(dt, 1e-3))))
    t0 = time.perf_counter()
    for _ in range(reps):
        oracle.attention_backward_rows(q, k, v, do, w.causal, 0, 0, rows)
    dt = (time.perf_counter() - t0) / reps
    cores = len(os.sched_getaffinity(0))
    return flops(rows) / dt / 1e12, R, dt, cores, reps


# ---------------------------------------------------------------- feedforward

def ffn_oracle_sample(w, seconds_target=12.0, max_rows=None):
    """Time the fp64 oracle on R token rows of feedforward workload w (each
    row is independent); R doubles until one run takes >= seconds_target/4.
    Returns (tflops, rows, seconds, cores, reps)."""
    import oracle
    from long_context_exact_attention_b200.inputs import make_ffn_inputs

    x = make_ffn_inputs(w, "cpu")
    xs, wg, wu, wd = (t.to(__import__("torch").float64).numpy() for t in
                      (x["x"], x["w_gate"], x["w_up"], x["w_down"]))
    do = xs[::-1].copy()  # any dout of the right shape; the cost does not depend on it

    def run(R):
        oracle.ffn_forward(xs[:R], wg, wu, wd)
        oracle.ffn_backward(xs[:R], wg, wu, wd, do[:R])

    R = 8
    while True:
        t0 = time.perf_counter()
        run(R)
        dt = time.perf_counter() - t0
        if dt >= seconds_target / 4 or R >= w.T or (max_rows and R >= max_rows):
            break
        R *= 2
    reps = max(1, int(round(seconds_target / max(dt, 1e-3))))
    t0 = time.perf_counter()
    for _ in range(reps):
        run(R)
    dt = (time.perf_counter() - t0) / reps
    # the oracle's backward recomputes nothing it does not need: 6 + 12 T h f
    return 18.0 * R * w.h * w.f / dt / 1e12, R, dt, len(os.sched_getaffinity(0)), reps


def main_ffn(args, w):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    cfg = {"workload": w.name, "T": w.T, "h": w.h, "f": w.f, "block_tokens": w.block,
           "activation": "gated SiLU (Llama)"}
    if args.impl == "reference":
        if rank != 0:
            return
        for _ in range(args.warmup):
            ffn_oracle_sample(w, seconds_target=2.0, max_rows=64)
        vals, info = [], None
        for _ in range(args.steps):
            info = ffn_oracle_sample(w, seconds_target=5.0, max_rows=1024)
            vals.append(info[0])
        tf, R, dt, cores, reps = info
        val = statistics.median(vals)
        print(json.dumps({
            "impl": "reference", "metric": FFN_METRIC, "value": val, "unit": "TFLOP/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": dt * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": cfg,
            "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                             "sample": f"fp64 oracle feedforward forward + backward of {R} "
                                       "token rows"},
            "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}), flush=True)
        return

    import torch
    import torch.distributed as dist
    from long_context_exact_attention_b200 import lca
    from long_context_exact_attention_b200.inputs import make_ffn_inputs

    torch.cuda.set_device(local)  # before the process group, so NCCL binds this GPU
    if world > 1:
        dist.init_process_group("nccl", init_method="env://",
                                timeout=__import__("datetime").timedelta(seconds=120))
    dev = torch.device("cuda", local)
    stream = torch.cuda.Stream(dev)
    x = make_ffn_inputs(w, dev)
    out = torch.empty_like(x["x"])
    g = torch.Generator(device=dev).manual_seed(w.seed * 1_000_003 + 30)
    dout = torch.randn(x["x"].shape, generator=g, device=dev).to(torch.bfloat16)
    dx = torch.empty_like(x["x"])
    dws = [torch.zeros(x[n].shape, device=dev, dtype=torch.float32)
           for n in ("w_gate", "w_up", "w_down")]
    ws = torch.empty(max(lca.ffn_workspace_size(w.T, w.h, w.f, w.block),
                         lca.ffn_bwd_workspace_size(w.T, w.h, w.f, w.block)), device=dev,
                     dtype=torch.uint8)
    n_blocks = -(-w.T // w.block)
    fwd_flops, bwd_flops = w.flops(), w.bwd_flops()
    torch.cuda.synchronize()

    primary = {"x": x["x"], "dout": dout, "out": out, "dx": dx}

    def step(ev=None, S=None, st=None):
        S = S or primary
        st = st or stream
        if ev:
            ev[0].record(st)
        lca.ffn_fwd(S["x"], x["w_gate"], x["w_up"], x["w_down"], block_tokens=w.block,
                    out=S["out"], workspace=ws, stream=st)
        if ev:
            ev[1].record(st)
        lca.ffn_bwd(S["x"], x["w_gate"], x["w_up"], x["w_down"], S["dout"],
                    block_tokens=w.block, dx=S["dx"], dw_gate=dws[0], dw_up=dws[1],
                    dw_down=dws[2], workspace=ws, stream=st)
        if ev:
            ev[2].record(st)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            step()
    stream.synchronize()
    lca.check(stream)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    cvd = os.environ.get("CUDA_VISIBLE_DEVICES")
    clocks = ClockSampler(cvd.split(",")[local] if cvd else str(local))
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    with torch.cuda.stream(stream):
        for i in range(args.steps):
            step(evs[i])
    stream.synchronize()
    torch.cuda.synchronize()
    clk = clocks.stop()
    lca.check(stream)
    fwd_ms = [e[0].elapsed_time(e[1]) for e in evs]
    bwd_ms = [e[1].elapsed_time(e[2]) for e in evs]
    total_ms = max_over_ranks(evs[0][0].elapsed_time(evs[-1][2]), dev)
    value = whole_job_tflops(fwd_flops + bwd_flops, world, args.steps, total_ms)

    e2e = None
    if not args.no_e2e:
        in_names, out_names = ["x", "dout"], ["out", "dx"]
        host_in = [primary[n].cpu().pin_memory() for n in in_names]
        host_out = [torch.empty_like(primary[n], device="cpu").pin_memory() for n in out_names]
        sets = [primary, {n: torch.empty_like(t) for n, t in primary.items()}]
        compute = lambda S, st: step(S=S, st=st)
        pipelined_e2e(torch, dev, sets, in_names, out_names, host_in, host_out, compute, 2)
        n_e2e = max(3, min(args.steps, 6))
        if world > 1:
            dist.barrier()
        e_ms = max_over_ranks(pipelined_e2e(torch, dev, sets, in_names, out_names, host_in,
                                            host_out, compute, n_e2e), dev)
        e2e = {"value": whole_job_tflops(fwd_flops + bwd_flops, world, n_e2e, e_ms),
               "unit": "TFLOP/s",
               "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in host_in),
               "d2h_bytes_per_step": sum(t.numel() * t.element_size() for t in host_out),
               "ms_per_step": e_ms / n_e2e,
               "pipelining": "two device buffer sets; uploads and downloads on their own "
                             "streams overlap the neighbouring steps' compute"}
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    pk, pk_kind = peaks()
    sustained = pk.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    fwd_t, bwd_t = statistics.median(fwd_ms), statistics.median(bwd_ms)
    ach = bwd_flops / (bwd_t * 1e-3) / 1e12
    tr = traffic_record("ffn_gemm_sm100_bwd", w.name)
    in_bytes = sum(t.numel() * t.element_size() for t in list(x.values()) + [dout])
    cfg["l2"] = (f"inputs larger than L2 (x and weights {in_bytes / 2**20:.0f} MiB together, "
                 "L2 126 MB); no flush")
    line = {
        "metric": FFN_METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic", "impl": "lca", "config": cfg,
        "frac_of_peak": {"measured_burst": value / world / pk.get("bf16_tflops", 1590.0),
                         "measured_sustained": value / world / sustained,
                         "nominal_2250": value / world / NOMINAL_BF16_TFLOPS},
        "fwd_tflops": fwd_flops / (fwd_t * 1e-3) / 1e12, "fwd_ms": fwd_t,
        "bwd_tflops": ach, "bwd_ms": bwd_t,
        "roofline": {"bound": "tensor", "kernel": "ffn_gemm_sm100 (lca_ffn_bwd)", "achieved": ach,
                     "peak": sustained, "unit": "TFLOP/s", "frac": ach / sustained,
                     "peak_kind": f"{pk_kind} sustained bf16",
                     "traffic": tr["dram_bytes_per_launch"] if tr else None,
                     "frac_of_nominal_2250": ach / NOMINAL_BF16_TFLOPS,
                     "timing": "CUDA events around the whole lca_ffn_bwd call (five products "
                               "per block, 16 T h f FLOPs with the recompute), median over timed "
                               "steps"},
        "clocks": clk,
        # per block: 2 forward products and 5 backward products (dH, the gate/up
        # recompute, dx, [dW_gate; dW_up], dW_down)
        "gpu_launches": args.steps * 7 * n_blocks,
        "e2e": e2e,
    }
    if not args.no_cpu_baseline and world == 1:
        tf, R, dt, cores, reps = ffn_oracle_sample(w)
        line["cpu_baseline"] = {"value": tf, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                                "sample": f"fp64 oracle feedforward of {R} token rows, {reps} "
                                          f"runs, {dt:.2f} s each"}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- main

class AttnRun:
    """Device buffers and the timed step of one attention workload."""

    def __init__(self, w, dev, stream):
        import torch
        from long_context_exact_attention_b200 import lca
        from long_context_exact_attention_b200.inputs import make_inputs
        self.w, self.dev, self.stream, self.lca = w, dev, stream, lca
        x = make_inputs(w, dev)
        torch.cuda.synchronize()
        q, k, v = x["q"], x["k"], x["v"]
        dout = x.get("dout")
        self.cu = self.max_len = None
        if w.packed:
            # one token axis: [T, H, d] views of the single batch entry
            q, k, v = q[0], k[0], v[0]
            dout = dout[0] if dout is not None else None
            self.cu = torch.tensor([0] + list(__import__("itertools").accumulate(w.lengths)),
                                   dtype=torch.int32, device=dev)
            self.max_len = max(w.lengths)
        out = torch.empty_like(q)
        lse = torch.empty((w.Hq, w.S) if w.packed else (w.B, w.Hq, w.S), device=dev,
                          dtype=torch.float32)
        self.primary = {"q": q, "k": k, "v": v, "out": out, "lse": lse}
        self.ws = self.fws = None
        # the dense backward runs as its three phases (prep, main kernel, dq)
        # through the block entry points, so the main kernel has events of its
        # own; these are the launches lca_attn_bwd makes
        self.phased = w.backward and not w.packed and not w.s2
        if w.backward:
            self.primary.update(dout=dout, dq=torch.empty_like(q), dk=torch.empty_like(k),
                                dv=torch.empty_like(v))
            if w.packed:
                n = lca.varlen_workspace_size(q, k, self.cu, self.max_len)
            elif w.s2:
                n = lca.s2attn_workspace_sizes(q, k, w.group, w.shift_heads)[1]
            else:
                n = lca.workspace_size(q, k)
            self.ws = torch.empty(n, device=dev, dtype=torch.uint8)
        if w.s2:
            n = lca.s2attn_workspace_sizes(q, k, w.group, w.shift_heads)[0]
            self.fws = torch.empty(n, device=dev, dtype=torch.uint8) if n else None

    def step(self, ev=None, S=None, st=None, phased=None):
        """One fwd + bwd pass.  ev: 5 events (start, after fwd, after the
        backward's prep, after its main kernel, end) or None."""
        lca, w = self.lca, self.w
        S = S or self.primary
        st = st or self.stream
        phased = self.phased if phased is None else phased
        q, k, v, out, lse = S["q"], S["k"], S["v"], S["out"], S["lse"]
        rec = (lambda i: ev[i].record(st)) if ev else (lambda i: None)
        rec(0)
        if w.packed:
            lca.attn_fwd_varlen(q, k, v, self.cu, self.max_len, causal=w.causal,
                                kv_chunk=w.kv_chunk, order=w.order, q_block=w.q_block, out=out,
                                lse=lse, stream=st)
        elif w.s2:
            lca.s2attn_fwd(q, k, v, w.group, w.shift_heads, causal=w.causal, out=out, lse=lse,
                           workspace=self.fws, stream=st)
        else:
            lca.attn_fwd(q, k, v, causal=w.causal, kv_chunk=w.kv_chunk, order=w.order,
                         q_block=w.q_block, out=out, lse=lse, stream=st)
        rec(1)
        if not w.backward:
            rec(2), rec(3), rec(4)
            return
        g = dict(dq=S["dq"], dk=S["dk"], dv=S["dv"], workspace=self.ws, stream=st)
        if w.packed:
            lca.attn_bwd_varlen(q, k, v, out, lse, S["dout"], self.cu, self.max_len,
                                causal=w.causal, **g)
            rec(2), rec(3)
        elif w.s2:
            lca.s2attn_bwd(q, k, v, out, lse, S["dout"], w.group, w.shift_heads,
                           causal=w.causal, **g)
            rec(2), rec(3)
        elif phased:
            lca.attn_bwd_block_prep(q, out, lse, S["dout"], workspace=self.ws, stream=st)
            rec(2)
            lca.attn_bwd_block(q, k, v, S["dout"], 0, 0, self.ws, causal=w.causal, dk=S["dk"],
                               dv=S["dv"], stream=st)
            rec(3)
            lca.attn_bwd_block_dq(q, self.ws, dq=S["dq"], stream=st)
        else:
            lca.attn_bwd(q, k, v, out, lse, S["dout"], causal=w.causal, **g)
            rec(2), rec(3)
        rec(4)

    def time(self, steps, warmup, world=1, sample_clocks=False, local=0):
        """Warm up, then time `steps` steps on the device; returns a dict of
        per-phase medians and the whole-region time (max over ranks)."""
        import torch
        import torch.distributed as dist
        with torch.cuda.stream(self.stream):
            for _ in range(warmup):
                self.step()
        self.stream.synchronize()
        self.lca.check(self.stream)
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(steps)]
        start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        clocks = None
        if sample_clocks:
            cvd = os.environ.get("CUDA_VISIBLE_DEVICES")
            clocks = ClockSampler(cvd.split(",")[local] if cvd else str(local))
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        if clocks:
            clocks.start()
            time.sleep(0.3)
        start.record(self.stream)
        for i in range(steps):
            self.step(evs[i])
        stop.record(self.stream)
        stop.synchronize()
        torch.cuda.synchronize()
        clk = clocks.stop() if clocks else None
        if world > 1:
            dist.barrier()
        self.lca.check(self.stream)
        med = lambda a, b: statistics.median(e[a].elapsed_time(e[b]) for e in evs)
        total = max_over_ranks(start.elapsed_time(stop), self.dev)
        return {"total_ms": total, "fwd_ms": med(0, 1), "bwd_ms": med(1, 4),
                "bwd_main_ms": med(2, 3), "clocks": clk}


def attn_summary(w, t, pk):
    """Throughputs of one timed attention workload (single device)."""
    burst = pk.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    sustained = pk.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    ff, fb = w.fwd_flops(), (w.bwd_flops() if w.backward else 0.0)
    tf = lambda fl, ms: fl / (ms * 1e-3) / 1e12 if ms > 0 else None
    d = {"fwd_tflops": tf(ff, t["fwd_ms"]), "fwd_ms": t["fwd_ms"]}
    if w.backward:
        d.update(bwd_tflops=tf(fb, t["bwd_ms"]), bwd_ms=t["bwd_ms"],
                 fwd_bwd_tflops=tf(ff + fb, t["fwd_ms"] + t["bwd_ms"]))
        if run_phased(w):  # the main kernel has events of its own
            d.update(bwd_main_tflops=tf(fb, t["bwd_main_ms"]), bwd_main_ms=t["bwd_main_ms"])
    for key in ("fwd_tflops", "bwd_main_tflops"):
        if d.get(key):
            d[key.replace("_tflops", "_frac")] = {
                "measured_burst": d[key] / burst, "measured_sustained": d[key] / sustained,
                "nominal_2250": d[key] / NOMINAL_BF16_TFLOPS}
    return d


def main_seqpar(args, w, method):
    """Sequence-parallel attention over the ranks (strong scaling: one
    sequence of w.S tokens split over N ranks): ring attention (zig-zag
    blocks, key/value blocks rotating) or Ulysses (contiguous blocks, heads
    exchanged by all-to-all)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    flops_step = w.fwd_flops() + w.bwd_flops()
    label = ("ring x%d (zig-zag, sequence split)" if method == "ring"
             else "ulysses x%d (sequence split, heads exchanged by all-to-all)") % world
    cfg = {"workload": f"{method}_{w.name}", "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "S": w.S,
           "d": w.d, "causal": w.causal, "parallelism": label}
    if args.impl == "reference":
        if rank != 0:
            return
        vals, info = [], None
        for _ in range(args.warmup):
            oracle_sample(w, seconds_target=2.0, max_rows=512)
        for _ in range(args.steps):
            info = oracle_sample(w, seconds_target=5.0, max_rows=4096)
            vals.append(info[0])
        tf, R, dt, cores, reps = info
        val = statistics.median(vals)
        print(json.dumps({
            "impl": "reference", "metric": METRIC, "value": val, "unit": "TFLOP/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": dt * 1e3, "higher_is_better": True, "scaling": "strong",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": cfg,
            "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                             "sample": f"fp64 oracle fwd+bwd of the last {R} query rows of "
                                       f"the {w.Hq // w.Hkv} query heads of key/value head 0"},
            "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}), flush=True)
        return

    import torch
    import torch.distributed as dist
    from long_context_exact_attention_b200 import lca, ring, ulysses
    from long_context_exact_attention_b200.inputs import make_tensor

    torch.cuda.set_device(local)  # before the process group, so NCCL binds this GPU
    if world > 1:
        dist.init_process_group("nccl", init_method="env://",
                                timeout=__import__("datetime").timedelta(seconds=120))
    dev = torch.device("cuda", local)
    stream = torch.cuda.Stream(dev)
    if method == "ring":
        # this rank's zig-zag block: chunks r and 2N-1-r of 2N
        c = w.S // (2 * world)
        a, b = ring.zigzag_chunks(rank, world)
        blk = {n: torch.cat([make_tensor(w, n, dev, (a * c, (a + 1) * c)),
                             make_tensor(w, n, dev, (b * c, (b + 1) * c))], dim=1).contiguous()
               for n in ("q", "k", "v", "dout")}
        fwd, bwd = ring.ring_attn_fwd, ring.ring_attn_bwd
        launches = ring.launches_per_step(world, w.causal)
    else:
        # this rank's contiguous block of S / N tokens
        c = w.S // world
        blk = {n: make_tensor(w, n, dev, (rank * c, (rank + 1) * c)).contiguous()
               for n in ("q", "k", "v", "dout")}
        fwd, bwd = ulysses.ulysses_attn_fwd, ulysses.ulysses_attn_bwd
        launches = ulysses.launches_per_step(world)
    torch.cuda.synchronize()

    def step(S=None, st=None):
        S = S or blk
        with torch.cuda.stream(st or stream):
            o, l = fwd(S["q"], S["k"], S["v"], causal=w.causal)
            g = bwd(S["q"], S["k"], S["v"], o, l, S["dout"], causal=w.causal)
            S["out"], S["lse"] = o, l
            S["dq"], S["dk"], S["dv"] = g

    for _ in range(args.warmup):
        step()
    stream.synchronize()
    lca.check(stream)
    cvd = os.environ.get("CUDA_VISIBLE_DEVICES")
    clocks = ClockSampler(cvd.split(",")[local] if cvd else str(local))
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    start.record(stream)
    for _ in range(args.steps):
        step()
    stop.record(stream)
    stop.synchronize()
    torch.cuda.synchronize()
    clk = clocks.stop()
    if world > 1:
        dist.barrier()
    lca.check(stream)
    total_ms = max_over_ranks(start.elapsed_time(stop), dev)
    value = flops_step * args.steps / (total_ms * 1e-3) / 1e12

    e2e = None
    if not args.no_e2e:
        in_names, out_names = ["q", "k", "v", "dout"], ["out", "lse", "dq", "dk", "dv"]
        host_in = [blk[n].cpu().pin_memory() for n in in_names]
        host_out = [torch.empty_like(blk[n], device="cpu").pin_memory() for n in out_names]
        sets = [blk, {n: torch.empty_like(t) for n, t in blk.items()}]
        compute = lambda S, st: step(S, st)
        pipelined_e2e(torch, dev, sets, in_names, out_names, host_in, host_out, compute, 2)
        n_e2e = max(3, min(args.steps, 4))
        if world > 1:
            dist.barrier()
        e_ms = max_over_ranks(pipelined_e2e(torch, dev, sets, in_names, out_names, host_in,
                                            host_out, compute, n_e2e), dev)
        e2e = {"value": flops_step * n_e2e / (e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in host_in),
               "d2h_bytes_per_step": sum(t.numel() * t.element_size() for t in host_out),
               "per": "rank 0's block (every rank moves its own)", "ms_per_step": e_ms / n_e2e}
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    pk, pk_kind = peaks()
    burst = pk.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
        "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic", "impl": "lca", "config": cfg,
        "frac_of_peak": {"measured_burst": value / world / burst,
                         "nominal_2250": value / world / NOMINAL_BF16_TFLOPS},
        "roofline": {"bound": "tensor", "kernel": ("ring step (block forward and backward "
                     "kernels)" if method == "ring" else "Ulysses step (attention forward and "
                     "backward over the rank's heads)"), "achieved": value / world, "peak": burst,
                     "unit": "TFLOP/s",
                     "frac": value / world / burst,
                     "peak_kind": f"{pk_kind} burst bf16", "traffic": None,
                     "timing": f"CUDA events around whole {method} steps (kernels and "
                               "transfers), per GPU"},
        "clocks": clk,
        "gpu_launches": args.steps * launches,
        "e2e": e2e,
    }
    if not args.no_cpu_baseline and world == 1:
        tf, R, dt, cores, reps = oracle_sample(w)
        line["cpu_baseline"] = {"value": tf, "unit": "TFLOP/s", "cores": cores,
                                "kind": "oracle",
                                "sample": f"fp64 oracle fwd+bwd of the last {R} query rows of "
                                          f"the {w.Hq // w.Hkv} query heads of key/value head 0"
                                          f", {reps} runs, {dt:.2f} s each"}
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    from long_context_exact_attention_b200.inputs import FFN_WORKLOADS, WORKLOADS
    if args.workload in FFN_WORKLOADS:
        main_ffn(args, FFN_WORKLOADS[args.workload])
        return
    for method in ("ring", "ulysses"):
        if args.workload.startswith(method + "_"):
            main_seqpar(args, WORKLOADS[args.workload[len(method) + 1:]], method)
            return
    w = WORKLOADS[args.workload]
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    flops_step = w.fwd_flops() + (w.bwd_flops() if w.backward else 0.0)

    if args.impl == "reference":
        if rank != 0:
            return
        for _ in range(args.warmup):
            oracle_sample(w, seconds_target=2.0, max_rows=512)
        vals = []
        info = None
        for _ in range(args.steps):
            info = oracle_sample(w, seconds_target=5.0, max_rows=4096)
            vals.append(info[0])
        tf, R, dt, cores, reps = info
        val = statistics.median(vals)
        line = {
            "impl": "reference", "metric": METRIC, "value": val, "unit": "TFLOP/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": dt * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "S": w.S,
                       "d": w.d, "causal": w.causal},
            "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                             "sample": f"fp64 oracle fwd+bwd of the last {R} query rows of "
                                       f"the {w.Hq // w.Hkv} query head(s) of key/value head 0"
                                       + (" inside the last S2 group" if w.s2 else "")},
            "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
        }
        print(json.dumps(line), flush=True)
        return

    import torch
    import torch.distributed as dist

    torch.cuda.set_device(local)  # before the process group, so NCCL binds this GPU
    if world > 1:
        dist.init_process_group("nccl", init_method="env://",
                                timeout=__import__("datetime").timedelta(seconds=120))
    dev = torch.device("cuda", local)
    stream = torch.cuda.Stream(dev)
    run = AttnRun(w, dev, stream)
    t = run.time(args.steps, args.warmup, world, sample_clocks=True, local=local)
    total_ms = t["total_ms"]
    ms_step = total_ms / args.steps
    value = whole_job_tflops(flops_step, world, args.steps, total_ms)
    primary = run.primary

    # ---- end to end through the C ABI with pinned host buffers
    e2e = None
    if not args.no_e2e:
        in_names = ["q", "k", "v"] + (["dout"] if w.backward else [])
        out_names = ["out", "lse"] + (["dq", "dk", "dv"] if w.backward else [])
        host_in = [primary[n].cpu().pin_memory() for n in in_names]
        host_out = [torch.empty_like(primary[n], device="cpu").pin_memory() for n in out_names]
        sets = [primary, {n: torch.empty_like(x) for n, x in primary.items()}]
        # the user-facing calls (lca_attn_fwd + lca_attn_bwd)
        compute = lambda S, st: run.step(S=S, st=st, phased=False)
        pipelined_e2e(torch, dev, sets, in_names, out_names, host_in, host_out, compute, 2)
        n_e2e = max(3, min(args.steps, 6))
        if world > 1:
            dist.barrier()
        e_ms = max_over_ranks(pipelined_e2e(torch, dev, sets, in_names, out_names, host_in,
                                            host_out, compute, n_e2e), dev)
        e2e = {"value": whole_job_tflops(flops_step, world, n_e2e, e_ms), "unit": "TFLOP/s",
               "h2d_bytes_per_step": sum(x.numel() * x.element_size() for x in host_in),
               "d2h_bytes_per_step": sum(x.numel() * x.element_size() for x in host_out),
               "ms_per_step": e_ms / n_e2e,
               "pipelining": "two device buffer sets; uploads and downloads on their own "
                             "streams overlap the neighbouring steps' compute"}
        del sets, host_in, host_out

    pk, pk_kind = peaks()
    summary = attn_summary(w, t, pk)
    # the other workload of the metric's 32K-128K range, same process, device-timed
    others = {}
    if not args.no_extra and world == 1 and w.name in ("llama3_8b_gqa_s128k", "llama2_7b_s32k"):
        other = WORKLOADS["llama2_7b_s32k" if w.name != "llama2_7b_s32k"
                          else "llama3_8b_gqa_s128k"]
        del run
        torch.cuda.empty_cache()
        orun = AttnRun(other, dev, stream)
        ot = orun.time(max(3, min(args.steps, 10)), args.warmup)
        others[other.name] = dict(attn_summary(other, ot, pk), steps=max(3, min(args.steps, 10)),
                                  config={"B": other.B, "Hq": other.Hq, "Hkv": other.Hkv,
                                          "S": other.S, "kv_chunk": other.kv_chunk,
                                          "order": other.order})
        del orun

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return

    q, k, v, dout = (primary.get(n) for n in ("q", "k", "v", "dout"))
    in_bytes = sum(x.numel() * x.element_size() for x in (q, k, v, dout) if x is not None)
    l2_note = (f"inputs larger than L2 (q, k, v{', dout' if dout is not None else ''} "
               f"{in_bytes / 2**20:.0f} MiB together, L2 126 MB); no flush")
    burst = pk.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    sustained = pk.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    if w.backward and run_phased(w):
        kname = "attn_bwd_bf16_sm100"
        ach = summary["bwd_main_tflops"]
        timing = ("CUDA events on the launching stream around the main backward kernel alone "
                  "(row-dot and dq-finalize outside the bracket), median over timed steps")
    elif w.backward:
        kname = "attn_bwd_bf16_sm100"
        ach = summary["bwd_tflops"]
        timing = ("CUDA events around the whole backward call (its small kernels included, so "
                  "a lower bound for the main kernel), median over timed steps")
    else:
        kname = "attn_fwd_bf16_sm100"
        ach = summary["fwd_tflops"]
        timing = "CUDA events around lca_attn_fwd, median over timed steps"
    tr = traffic_record(kname, w.name)
    roof = {"bound": "tensor", "kernel": kname, "achieved": ach, "peak": burst,
            "unit": "TFLOP/s", "frac": ach / burst,
            "peak_kind": f"{pk_kind} burst bf16 (the kernel is timed per launch)",
            "frac_of_sustained": ach / sustained,
            "frac_of_nominal_2250": ach / NOMINAL_BF16_TFLOPS,
            "traffic": tr["dram_bytes_per_launch"] if tr else None,
            "timing": timing}
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic", "impl": "lca",
        "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "S": w.S, "d": w.d,
                   "causal": w.causal, "kv_chunk": w.kv_chunk, "order": w.order,
                   "s2_group": w.group or None, "s2_shift_heads": w.shift_heads or None,
                   "packed_lengths": list(w.lengths) or None,
                   "parallelism": f"replicas x{world}",
                   "l2": l2_note},
        **summary,
        "frac_of_peak": {"measured_burst": value / world / burst,
                         "measured_sustained": value / world / sustained,
                         "nominal_2250": value / world / NOMINAL_BF16_TFLOPS},
        "roofline": roof,
        "clocks": t["clocks"],
        "gpu_launches": args.steps * run_launches(w),
        "e2e": e2e,
    }
    if others:
        line["other_workloads"] = others
    if not args.no_cpu_baseline and world == 1:
        tf, R, dt, cores, reps = oracle_sample(w)
        line["cpu_baseline"] = {
            "value": tf, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "sample": f"fp64 oracle fwd+bwd of the last {R} query rows of the "
                      f"{w.Hq // w.Hkv} query head(s) of key/value head 0"
                      + (" inside the last S2 group" if w.s2 else "")
                      + f", {reps} runs, {dt:.2f} s each"}
    print(json.dumps(line), flush=True)


def run_phased(w):
    return w.backward and not w.packed and not w.s2


def run_launches(w):
    """This library's kernel launches per step (device-timed region)."""
    if not w.backward:
        return 1
    if w.s2 and (w.group // 2) % 128:
        return 7 + 12
    return 4  # forward; row-dot, main, dq-finalize


if __name__ == "__main__":
    main()
