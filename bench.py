#!/usr/bin/env python
"""Benchmark of the Hyper-Connections step on B200.

A step is one pass of the whole hot path over one batch: the fused mHC call
(per-token Sinkhorn projection of the 4x4 mixing logits, write mix, read-weight
softmax, read mix, pre-norm RMSNorm) on T = 16384 tokens, n = 4 streams,
d = 7168, bf16 storage, K = 20 -- one hc_write_then_read launch. Inputs are
synthetic (seeded, drawn on the device) and resident in HBM; the stream state
ping-pongs between two buffers, so every step reads and writes 2.35 GB, far
more than the 126 MB L2.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints ONE JSON line (rank 0). Multi-GPU runs (torchrun, one process per GPU)
are weak scaling: every rank runs its own batch; the step has no collective
(tokens are independent), NCCL is used only for the barrier and the max-over-
ranks timing.
"""
from __future__ import annotations

import argparse
import hashlib
import glob
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

WORKLOAD = dict(name="mhc_per_token_sinkhorn_fused", T=16384, n=4, d=7168, dtype="bf16", K=20,
                eps=1e-6, cfg=3)
METRIC = "HC step tokens/sec at n=4, d=7168 (bf16); achieved HBM GB/s vs ~8 TB/s peak"
UNIT = "tokens/s"
FALLBACK_HBM_GBS = 6650.0


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# Kernel sources each profiled traffic record depends on (the record is
# dropped as soon as one of them changes).
KERNEL_SOURCES = {
    "fused_mhc_n4_d7168_bf16_T16384": ["hc_pipe_kernels.cuh", "hc_device.cuh", "hc_sync.cuh",
                                       "hc_kernels_impl.cuh", "hc_k_bf16_fused.cu"],
    "mix_logits_n4_d7168_bf16_T16384": ["hc_logits.cu", "hc_tc.cuh", "hc_sync.cuh"],
    "collapse_n4_d7168_bf16_T16384": ["hc_stream_kernels.cuh", "hc_device.cuh",
                                      "hc_kernels_impl.cuh", "hc_k_bf16_ends.cu"],
    "expand_read_n4_d7168_bf16_T16384": ["hc_stream_kernels.cuh", "hc_device.cuh",
                                         "hc_kernels_impl.cuh", "hc_k_bf16_ends.cu"],
    "linear_write_n4_d7168_k7168_bf16_T16384": ["hc_linear_write.cu", "hc_tc.cuh", "hc_sync.cuh"],
    "backward_mhc_n4_d7168_bf16_T16384": ["hc_backward.cu", "hc_backward_pipe.cuh",
                                          "hc_backward_common.cuh", "hc_pipe_kernels.cuh",
                                          "hc_device.cuh", "hc_sync.cuh"],
    "backward_pipe_mhc_n4_d7168_bf16_T16384": ["hc_backward.cu", "hc_backward_pipe.cuh",
                                               "hc_backward_common.cuh", "hc_pipe_kernels.cuh",
                                               "hc_device.cuh", "hc_sync.cuh"],
    "reduce_write_r8_mhc_n4_d7168_bf16_T16384": ["hc_pipe_kernels.cuh", "hc_device.cuh",
                                                 "hc_sync.cuh", "hc_kernels_impl.cuh",
                                                 "hc_k_bf16_reduce.cu", "hc_reduce_write.cu"],
    "reduce_scatter_r8_mhc_n4_d7168_bf16_T16384": ["hc_pipe_kernels.cuh", "hc_device.cuh",
                                                   "hc_sync.cuh", "hc_kernels_impl.cuh",
                                                   "hc_k_bf16_reduce.cu", "hc_reduce_write.cu"],
}


def _source_hash(files=None):
    """Hash of the named kernel sources (all of csrc/ when files is None)."""
    csrc = os.path.join(ROOT, "hyper_connections_stream_b200", "csrc")
    paths = (sorted(glob.glob(os.path.join(csrc, "*"))) if files is None
             else [os.path.join(csrc, f) for f in sorted(files)])
    h = hashlib.sha256()
    for f in paths:
        with open(f, "rb") as fh:
            h.update(os.path.basename(f).encode())
            h.update(fh.read())
    return h.hexdigest()[:16]


def _profiled_traffic(kernel_key: str):
    """ncu DRAM bytes per launch committed under profiles/, if the kernel's
    sources have not changed since the capture."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            entry = json.load(f)[kernel_key]
    except Exception:
        return None
    if entry.get("source_sha") != _source_hash(KERNEL_SOURCES.get(kernel_key)):
        return None
    return entry.get("dram_bytes_per_launch")


# ----------------------------------------------------------------------------
# clocks during the timed region
# ----------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid: str | None):
        self.uuid = uuid
        self.proc = None
        self.path = None

    def __enter__(self):
        try:
            # the raw samples go to a temporary file; the JSON line carries the summary
            fd, self.path = tempfile.mkstemp(prefix="hc_clocks_", suffix=".csv")
            os.close(fd)
            cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                   "-lms", "100"]
            if self.uuid:
                cmd += ["-i", self.uuid]
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(cmd, stdout=self.fh, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.fh.close()

    def summary(self):
        if self.proc is None or not self.path or not os.path.exists(self.path):
            return None
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 8:
                    continue
                try:
                    rows.append((float(parts[0]), float(parts[1]), parts[4:8]))
                except ValueError:
                    continue
        try:
            os.remove(self.path)
        except OSError:
            pass
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, st in rows for i, s in enumerate(st)
                          if s.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in rows),
                "sm_max_mhz": max(r[1] for r in rows), "reasons": reasons,
                "samples": len(rows)}


BAD_REASONS = {"hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"}


# ----------------------------------------------------------------------------
# the GPU arm
# ----------------------------------------------------------------------------

def _dist_env():
    from hyper_connections_stream_b200 import dist as hd
    return hd.env()


def _max_over_ranks(value: float, ws: int, device) -> float:
    from hyper_connections_stream_b200 import dist as hd
    return hd.max_over_ranks(value, ws, device)


def _barrier(ws):
    from hyper_connections_stream_b200 import dist as hd
    hd.barrier(ws)


def _gpu_uuid(device):
    import torch
    try:
        return "GPU-" + str(torch.cuda.get_device_properties(device).uuid)
    except Exception:
        return None


def _set_path(args):
    from hyper_connections_stream_b200 import _lib as hc
    hc.set_path({"auto": hc.PATH_AUTO, "pipelined": hc.PATH_PIPELINED,
                 "register": hc.PATH_REGISTER}[args.path])


def make_inputs(w, rank, device):
    import torch
    import hc_inputs as gen
    from hyper_connections_stream_b200 import dist as hd
    T, n, d, cfg = w["T"], w["n"], w["d"], w["cfg"]
    sd = hd.seed_offset(rank)
    H = gen.device_normal(gen.SEED_H + cfg + sd, (T, n, d), torch.bfloat16, device)
    y = gen.device_normal(gen.SEED_Y + cfg + sd, (T, d), torch.bfloat16, device)
    L = gen.device_normal(gen.SEED_L + cfg + sd, (T, n, n), torch.float32, device)
    rl = gen.device_normal(gen.SEED_L + 100 + cfg + sd, (T, n), torch.float32, device)
    _, _, b = gen.static_params(cfg, n)
    return dict(H=H, y=y, L=L, rl=rl, b=torch.from_numpy(b).to(device),
                g=torch.ones(d, dtype=torch.float32, device=device))


def run_logits(args):
    """The input-dependent mixing logits (tensor-core GEMM with an RMS scale)
    on the workload's streams: T=16384 tokens, n=4, d=7168, P=24 logits.
    Kernel-only, device-timed; one launch per step."""
    import numpy as np
    import torch
    import hc_inputs as gen
    from hyper_connections_stream_b200 import _lib as hc
    ws, rank, local = _dist_env()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    w = dict(WORKLOAD)
    if args.tokens:
        w["T"] = args.tokens
    T, n, d = w["T"], w["n"], w["d"]
    P, K = n * n + 2 * n, n * d
    H = gen.device_normal(gen.SEED_H + w["cfg"], (T, n, d), torch.bfloat16, device)
    W = gen.device_normal(503, (P, K), torch.bfloat16, device, std=1.0 / np.sqrt(K))
    z = torch.empty((T, P), dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream(device)
    for _ in range(args.warmup):
        hc.mix_logits(H, W, eps=w["eps"], out=z)
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    for i in range(args.steps):
        ev[i][0].record(stream)
        hc.mix_logits(H, W, eps=w["eps"], out=z)
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    per = [s.elapsed_time(e) for s, e in ev]
    total_ms = ev[0][0].elapsed_time(ev[-1][1])
    kern_ms = statistics.mean(per)
    alg_bytes = T * K * 2 + P * K * 2 + T * P * 4
    flops = 2 * T * K * P
    peak, peak_kind = _peaks()
    achieved = alg_bytes / (kern_ms / 1e3) / 1e9
    return {
        "metric": "mixing-logits tokens/sec at n=4, d=7168 (bf16 streams, P=24, tensor cores)",
        "value": T * args.steps / (total_ms / 1e3), "unit": UNIT, "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": "mix_logits", "T": T, "n": n, "d": d, "P": P},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak,
                     "traffic": _profiled_traffic("mix_logits_n4_d7168_bf16_T16384") if T == 16384 else None,
                     "peak_source": peak_kind,
                     "algorithmic_bytes_per_launch": alg_bytes, "kernel_ms": kern_ms,
                     "tensor_tflops": flops / (kern_ms / 1e3) / 1e12},
        "gpu_launches": args.steps, "device_fault": hc.device_fault(),
    }


def run_ends(args):
    """The stack ends on the workload's shape (T=16384, n=4, d=7168, bf16):
    --op expand_read times hc_expand_then_read (one row in -> four copies and
    layer 0's RMS-normalised block input out); --op collapse times hc_collapse
    (four streams in -> one weighted row out). Kernel-only, device-timed, one
    launch per step; outputs ping-pong so consecutive launches do not share
    buffers in L2."""
    import numpy as np
    import torch
    import hc_inputs as gen
    from hyper_connections_stream_b200 import _lib as hc
    ws, rank, local = _dist_env()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    w = dict(WORKLOAD)
    if args.tokens:
        w["T"] = args.tokens
    T, n, d = w["T"], w["n"], w["d"]
    s = 2
    g = torch.from_numpy(gen.uniform(3500 + w["cfg"], (d,), 0.5, 1.5)).to(device)
    a = torch.full((n,), 1.0 / n, device=device)
    if args.op == "expand_read":
        xs = [gen.device_normal(gen.SEED_Y + w["cfg"] + i, (T, d), torch.bfloat16, device) for i in range(2)]
        Hs = [torch.empty((T, n, d), dtype=torch.bfloat16, device=device) for _ in range(2)]
        xr = [torch.empty((T, d), dtype=torch.bfloat16, device=device) for _ in range(2)]
        def launch(i):
            hc.expand_then_read(xs[i % 2], n, a, g, eps=w["eps"], out=Hs[i % 2], x_read=xr[i % 2])
        alg_bytes = T * d * s * (n + 2) + d * 4
        what = "expand + layer-0 read (hc_expand_then_read)"
    else:
        Hs = [gen.device_normal(gen.SEED_H + w["cfg"] + i, (T, n, d), torch.bfloat16, device) for i in range(2)]
        outs = [torch.empty((T, d), dtype=torch.bfloat16, device=device) for _ in range(2)]
        def launch(i):
            hc.collapse(Hs[i % 2], a, out=outs[i % 2])
        alg_bytes = T * d * s * (n + 1)
        what = "collapse (hc_collapse)"
    stream = torch.cuda.current_stream(device)
    for i in range(args.warmup):
        launch(i)
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    for i in range(args.steps):
        ev[i][0].record(stream)
        launch(i)
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    kern_ms = statistics.mean(s_.elapsed_time(e) for s_, e in ev)
    total_ms = ev[0][0].elapsed_time(ev[-1][1])
    peak, peak_kind = _peaks()
    achieved = alg_bytes / (kern_ms / 1e3) / 1e9
    return {
        "metric": f"stack-end tokens/sec at n=4, d=7168 (bf16): {what}",
        "value": T * args.steps / (total_ms / 1e3), "unit": UNIT, "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": args.op, "T": T, "n": n, "d": d, "l2": "inputs and outputs > L2"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak,
                     "traffic": _profiled_traffic(f"{args.op}_n4_d7168_bf16_T16384") if T == 16384 else None,
                     "peak_source": peak_kind,
                     "algorithmic_bytes_per_launch": alg_bytes, "kernel_ms": kern_ms},
        "gpu_launches": args.steps, "device_fault": hc.device_fault(),
    }


def run_reduce_write(args, scatter=False):
    """The write fused with the tensor-parallel all-reduce of y on the
    workload's streams: R partial block outputs (default 8, one per rank of a
    tensor-parallel group, all in this GPU's memory: the same kernels read
    them over NVLink when they are peer mappings), summed in rank order, then
    the fused mHC write + read. Device timed.

    One-shot form (--op reduce_write, hc_reduce_write_then_read): one launch
    per step over all T tokens. Unfused pair timed beside it: torch sum of the
    partials storing y, then hc_write_then_read.

    Reduce-scatter form (--op reduce_scatter, hc_reduce_scatter_write_then_read):
    the R ranks emulated on this GPU, one launch per rank per step, each over
    its token shard, storing its rows of x_next into all R ranks' x buffers.
    A step is all R launches (the whole group's work on one GPU). Unfused
    group work timed beside it: torch sum of the partials storing y, the
    fused step over all T tokens, and R - 1 copies of x_next (the
    all-gather)."""
    import torch
    import hc_inputs as gen
    from hyper_connections_stream_b200 import _lib as hc
    ws, rank, local = _dist_env()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    _set_path(args)
    w = dict(WORKLOAD)
    if args.tokens:
        w["T"] = args.tokens
    if args.streams:
        w["n"] = args.streams
    T, n, d, K, R = w["T"], w["n"], w["d"], w["K"], args.ranks
    cfg = w["cfg"]
    s = 2
    parts = [gen.device_normal(gen.SEED_Y + cfg + 10 * r, (T, d), torch.bfloat16, device)
             for r in range(R)]
    H = gen.device_normal(gen.SEED_H + cfg, (T, n, d), torch.bfloat16, device)
    L = gen.device_normal(gen.SEED_L + cfg, (T, n, n), torch.float32, device)
    l = gen.device_normal(gen.SEED_L + 100 + cfg, (T, n), torch.float32, device)
    b = torch.from_numpy(gen.normal(gen.SEED_P + cfg, (n,), mean=1.0, std=0.02)).to(device)
    g = torch.from_numpy(gen.uniform(3500 + cfg, (d,), 0.5, 1.5)).to(device)
    Hout = torch.empty_like(H)
    x = torch.empty((T, d), dtype=torch.bfloat16, device=device)
    kw = dict(eps=w["eps"], mix=hc.MIX_SINKHORN_LOGITS, K=K, read=hc.READ_SOFTMAX_LOGITS)
    y = torch.empty((T, d), dtype=torch.bfloat16, device=device)
    stacked = torch.stack(parts)

    if scatter:
        xs = [x] + [torch.empty((T, d), dtype=torch.bfloat16, device=device) for _ in range(R - 1)]
        shards = []
        for r in range(R):
            base, extra = divmod(T, R)
            t0 = r * base + min(r, extra)
            sl = slice(t0, t0 + base + (1 if r < extra else 0))
            shards.append((H[sl], L[sl], l[sl], Hout[sl]))

        def fused():
            for r, (Hr, Lr, lr, Ho) in enumerate(shards):
                hc.reduce_scatter_write_then_read(parts, xs, r, Hr, Lr, b, lr, g, out=Ho, **kw)

        def unfused():
            y.copy_(torch.sum(stacked, 0, dtype=torch.float32))
            hc.write_then_read(H, y, L, b, l, g, out=Hout, x_next=x, **kw)
            for q in range(1, R):
                xs[q].copy_(x)
        launches = R
        # per token: R partial rows and n stream rows read, n stream rows and
        # R x rows (one per rank) written; per launch the gain
        alg_bytes = T * (d * s * (2 * R + 2 * n) + 4 * (n * n + n)) + R * d * 4
    else:
        def fused():
            hc.reduce_write_then_read(parts, H, L, b, l, g, out=Hout, x_next=x, **kw)

        def unfused():
            y.copy_(torch.sum(stacked, 0, dtype=torch.float32))
            hc.write_then_read(H, y, L, b, l, g, out=Hout, x_next=x, **kw)
        launches = 1
        alg_bytes = T * (d * s * (R + 2 * n + 1) + 4 * (n * n + n)) + d * 4

    stream = torch.cuda.current_stream(device)

    def timed(fn, steps):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(steps)]
        for i in range(steps):
            ev[i][0].record(stream)
            fn()
            ev[i][1].record(stream)
        torch.cuda.synchronize()
        return (statistics.mean(a.elapsed_time(e) for a, e in ev), ev[0][0].elapsed_time(ev[-1][1]))

    with ClockSampler(_gpu_uuid(device)) as clk:
        kern_ms, total_ms = timed(fused, args.steps)
    unfused_ms, _ = timed(unfused, max(3, args.steps // 4))
    peak, peak_kind = _peaks()
    achieved = alg_bytes / (kern_ms / 1e3) / 1e9
    key = ("reduce_scatter" if scatter else "reduce_write") + "_r8_mhc_n4_d7168_bf16_T16384"
    form = "reduce-scatter form, R ranks emulated on one GPU" if scatter else "one-shot form"
    return {
        "metric": f"HC step on the all-reduced block output (R={R} partials, {form}) tokens/sec at "
                  f"n={n}, d={d} (bf16, mHC K={K})",
        "value": T * args.steps / (total_ms / 1e3), "unit": UNIT, "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": "reduce_scatter" if scatter else "reduce_write", "T": T, "n": n,
                   "d": d, "K": K, "ranks": R, "launches_per_step": launches,
                   "partials": "all in this GPU's memory",
                   "l2": "inputs > L2 (re-read from HBM every step)"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak,
                     "traffic": _profiled_traffic(key) if (T, n, R) == (16384, 4, 8) else None,
                     "peak_source": peak_kind,
                     "algorithmic_bytes_per_step": alg_bytes, "kernel_ms": kern_ms},
        "unfused_ms": unfused_ms,
        "clocks": clk.summary(),
        "gpu_launches": args.steps * launches, "device_fault": hc.device_fault(),
    }


def run_linear_write(args):
    """The block's output projection fused with the write mix
    (hc_linear_then_write) on the workload's streams: X [T, k=7168] times
    Wo^T [7168, d=7168] on the tensor cores, then the write of the n=4 streams
    with per-token Sinkhorn-projected A, y never stored. Device-timed, one
    launch per step. Also times the unfused pair it replaces (torch.matmul,
    i.e. cuBLAS, storing y, then hc_write_mix) for context."""
    import numpy as np
    import torch
    import hc_inputs as gen
    from hyper_connections_stream_b200 import _lib as hc
    ws, rank, local = _dist_env()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    w = dict(WORKLOAD)
    if args.tokens:
        w["T"] = args.tokens
    T, n, d = w["T"], w["n"], w["d"]
    k = d
    X = gen.device_normal(gen.SEED_Y + w["cfg"], (T, k), torch.bfloat16, device)
    Wo = gen.device_normal(505, (d, k), torch.bfloat16, device, std=1.0 / np.sqrt(k))
    Hs = [gen.device_normal(gen.SEED_H + w["cfg"], (T, n, d), torch.bfloat16, device),
          torch.empty((T, n, d), dtype=torch.bfloat16, device=device)]
    L = gen.device_normal(gen.SEED_L + w["cfg"], (T, n, n), torch.float32, device)
    A = hc.sinkhorn(L, w["K"])
    b = torch.from_numpy(gen.normal(gen.SEED_P + w["cfg"], (n,), mean=1.0, std=0.02)).to(device)
    y = torch.empty((T, d), dtype=torch.bfloat16, device=device)
    stream = torch.cuda.current_stream(device)

    def timed(fn, steps):
        for i in range(args.warmup):
            fn(i)
        torch.cuda.synchronize()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(steps)]
        for i in range(steps):
            ev[i][0].record(stream)
            fn(i)
            ev[i][1].record(stream)
        torch.cuda.synchronize()
        return (statistics.mean(s_.elapsed_time(e) for s_, e in ev),
                ev[0][0].elapsed_time(ev[-1][1]))

    def fused(i):
        hc.linear_then_write(X, Wo, Hs[i % 2], A, b, out=Hs[(i + 1) % 2])

    def unfused(i):
        torch.matmul(X, Wo.t(), out=y)
        hc.write_mix(Hs[i % 2], y, A, b, out=Hs[(i + 1) % 2])

    def cublas(i):
        torch.matmul(X, Wo.t(), out=y)

    kern_ms, total_ms = timed(fused, args.steps)
    ref_steps = max(3, min(args.steps, 50))
    unfused_ms, _ = timed(unfused, ref_steps)
    cublas_ms, _ = timed(cublas, ref_steps)
    flops = 2.0 * T * k * d
    tflops = flops / (kern_ms / 1e3) / 1e12
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            peak, peak_kind = float(json.load(f)["bf16_tflops"]), "measured (burst)"
    except Exception:
        peak, peak_kind = 1590.0, "fallback"
    hbm_bytes = T * k * 2 + d * k * 2 + T * n * d * 2 * 2 + T * n * n * 4
    return {
        "metric": "block output projection + HC write tokens/sec at n=4, d=k=7168 (bf16, tensor cores)",
        "value": T * args.steps / (total_ms / 1e3), "unit": UNIT, "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": "linear_write", "T": T, "n": n, "d": d, "k": k,
                   "mix": "per-token Sinkhorn-projected A (K=20)", "l2": "inputs and outputs > L2"},
        "roofline": {"bound": "tensor", "achieved": tflops, "peak": peak, "unit": "TFLOP/s",
                     "frac": tflops / peak,
                     "traffic": _profiled_traffic("linear_write_n4_d7168_k7168_bf16_T16384")
                     if T == 16384 else None,
                     "peak_source": peak_kind,
                     "flops_per_launch": flops, "kernel_ms": kern_ms,
                     "hbm_bytes_min": hbm_bytes,
                     "hbm_gbs_at_min_bytes": hbm_bytes / (kern_ms / 1e3) / 1e9},
        "unfused": {"ms": unfused_ms, "cublas_matmul_ms": cublas_ms,
                    "how": "torch.matmul(X, Wo.T, out=y) then hc_write_mix (y stored and re-read)"},
        "gpu_launches": args.steps, "device_fault": hc.device_fault(),
    }


def run_backward(args):
    """Backward of the fused mHC step (hc_write_then_read_backward) on the
    workload: T=16384, n=4, d=7168, bf16, per-token Sinkhorn (K=20) and softmax
    logits, gradients arriving at both H' and x_next, gain gradient summed over
    tokens. One step = the three launches (step kernel, parameter backward,
    gain reduction); device-timed per step."""
    import numpy as np
    import torch
    import hc_inputs as gen
    from hyper_connections_stream_b200 import _lib as hc
    ws, rank, local = _dist_env()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    _set_path(args)
    w = dict(WORKLOAD)
    if args.tokens:
        w["T"] = args.tokens
    if args.streams:
        w["n"] = args.streams
    T, n, d, K = w["T"], w["n"], w["d"], w["K"]
    cfg = w["cfg"]
    H = gen.device_normal(gen.SEED_H + cfg, (T, n, d), torch.bfloat16, device)
    y = gen.device_normal(gen.SEED_Y + cfg, (T, d), torch.bfloat16, device)
    L = gen.device_normal(gen.SEED_L + cfg, (T, n, n), torch.float32, device)
    l = gen.device_normal(gen.SEED_L + 100 + cfg, (T, n), torch.float32, device)
    b = torch.from_numpy(gen.normal(gen.SEED_P + cfg, (n,), mean=1.0, std=0.02)).to(device)
    g = torch.from_numpy(gen.uniform(3500 + cfg, (d,), 0.5, 1.5)).to(device)
    dHo = gen.device_normal(5000 + cfg, (T, n, d), torch.bfloat16, device)
    dx = gen.device_normal(5100 + cfg, (T, d), torch.bfloat16, device)
    need = int(hc.lib().hc_write_then_read_backward_workspace_bytes(hc.HC_BF16, T, n, d))
    work = torch.empty((max(need, 16),), dtype=torch.uint8, device=device)

    def step():
        return hc.write_then_read_backward(H, y, L, b, l, g, dHo, dx, eps=w["eps"],
                                           mix=hc.MIX_SINKHORN_LOGITS, K=K,
                                           read=hc.READ_SOFTMAX_LOGITS, workspace=work)

    stream = torch.cuda.current_stream(device)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    with ClockSampler(_gpu_uuid(device)) as clk:
        for i in range(args.steps):
            ev[i][0].record(stream)
            step()
            ev[i][1].record(stream)
        torch.cuda.synchronize()
    step_ms = statistics.mean(s_.elapsed_time(e) for s_, e in ev)
    total_ms = ev[0][0].elapsed_time(ev[-1][1])
    s = 2
    alg_bytes = (T * d * s * (3 * n + 3) + T * 4 * (n * n + n) + T * 4 * (n * n + 2 * n)
                 + d * 4 * 2)
    peak, peak_kind = _peaks()
    achieved = alg_bytes / (step_ms / 1e3) / 1e9
    return {
        "metric": f"HC step backward tokens/sec at n={n}, d={d} (bf16, mHC K={K})",
        "value": T * args.steps / (total_ms / 1e3), "unit": UNIT, "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": "backward", "T": T, "n": n, "d": d, "K": K,
                   "l2": "inputs and outputs > L2; the binding allocates the gradient outputs"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak,
                     "traffic": _profiled_traffic(("backward_pipe_mhc_n4_d7168_bf16_T16384"
                                                   if args.path == "pipelined" else
                                                   "backward_mhc_n4_d7168_bf16_T16384"))
                     if (T, n) == (16384, 4) else None,
                     "peak_source": peak_kind,
                     "algorithmic_bytes_per_step": alg_bytes, "step_ms": step_ms},
        "clocks": clk.summary(), "kernel_path": args.path,
        "gpu_launches": 3 * args.steps, "device_fault": hc.device_fault(),
    }


def run_decode(args):
    """Decode-sized calls of the fused mHC step (T = 1 by default, --tokens to
    change), n=4, d=7168, bf16, K=20: 200 calls captured in one CUDA graph and
    replayed, so the host's per-call overhead is out of the device time; the
    line reports microseconds per call (lower is better)."""
    import torch
    from hyper_connections_stream_b200 import _lib as hc
    ws, rank, local = _dist_env()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    w = dict(WORKLOAD)
    w["T"] = args.tokens or 1
    T, n, d, K = w["T"], w["n"], w["d"], w["K"]
    inp = make_inputs(w, rank, device)
    bufs = (inp["H"], torch.empty_like(inp["H"]))
    x = torch.empty((T, d), dtype=torch.bfloat16, device=device)
    calls = 200

    def step(i):
        hc.write_then_read(bufs[i % 2], inp["y"], inp["L"], inp["b"], inp["rl"], inp["g"],
                           eps=w["eps"], mix=hc.MIX_SINKHORN_LOGITS, K=K,
                           read=hc.READ_SOFTMAX_LOGITS, out=bufs[(i + 1) % 2], x_next=x)

    side = torch.cuda.Stream(device)
    side.wait_stream(torch.cuda.current_stream(device))
    with torch.cuda.stream(side):
        for i in range(max(args.warmup, 3)):
            step(i)
    torch.cuda.current_stream(device).wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for i in range(calls):
            step(i)
    graph.replay()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream(device)
    times = []
    for _ in range(args.steps):
        s_, e_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s_.record(stream)
        graph.replay()
        e_.record(stream)
        torch.cuda.synchronize()
        times.append(s_.elapsed_time(e_) * 1e3 / calls)
    del graph
    us = statistics.median(times)
    return {
        "metric": f"fused mHC step latency per call at T={T}, n=4, d=7168 (bf16, CUDA graph replay)",
        "value": us, "unit": "us/call", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": us / 1e3, "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": "decode", "T": T, "n": n, "d": d, "K": K,
                   "calls_per_graph": calls, "kernel_family": "auto (register-streaming)"},
        "gpu_launches": args.steps * calls, "device_fault": hc.device_fault(),
    }


SWEEP_T = (1, 64, 1024, 16384, 65536)
SWEEP_N = (2, 4, 8)
SWEEP_D = (4096, 7168)
L2_BYTES = 126 * 2 ** 20


def _slots(bytes_per_call):
    """Distinct buffer sets cycled through by consecutive calls, so that the
    calls between two uses of one set touch well over twice the L2."""
    return int(min(1024, max(1, -(-(3 * L2_BYTES) // max(1, bytes_per_call)))))


def _per_call_ms(fn, ncalls, device, warmup=3, graph=False, reps=5):
    """Mean device time per call of fn(i), i = 0 .. ncalls - 1, with CUDA
    events on the launching stream around the whole sequence (graph=True:
    captured once in a CUDA graph and replayed, the median of reps replays,
    so no host overhead lands between calls)."""
    import torch
    stream = torch.cuda.current_stream(device)
    side = torch.cuda.Stream(device)
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        for i in range(warmup):
            fn(i)
    stream.wait_stream(side)
    torch.cuda.synchronize()
    if graph:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(ncalls):
                fn(i)
        g.replay()
        torch.cuda.synchronize()
        times = []
        for _ in range(reps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            g.replay()
            b.record(stream)
            torch.cuda.synchronize()
            times.append(a.elapsed_time(b) / ncalls)
        del g
        return statistics.median(times)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for i in range(ncalls):
        fn(i)
    b.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b) / ncalls


def _oracle_point_rate(T, n, d, K, eps, seconds=0.25):
    """Oracle tokens/s (all host cores) on a sample of up to 32 tokens of
    the point's shape and distributions."""
    import numpy as np
    import hc_inputs as gen
    import oracle
    S = min(T, 32)
    H = gen.streams(5, S, n, d, "bf16")
    y = gen.block_out(5, S, d, "bf16")
    L = gen.mix_logits(5, S, n)
    rl = gen.read_logits(5, S, n)
    _, _, b = gen.static_params(5, n)
    g = np.ones(d, np.float32)
    reps, t0 = 0, time.perf_counter()
    while True:
        oracle.write_then_read(H, y, L, b, rl, g, eps, "bf16", K=K, mix_logits=True, read_logits=True)
        reps += 1
        dt = time.perf_counter() - t0
        if dt >= seconds:
            return S * reps / dt, S


def run_sweep(args):
    """Per-point throughput of the fused mHC step (per-token Sinkhorn K=20 and
    read softmax, bf16) over T x n x d, then the static layer at T=4096, n=4,
    d=4096 (read, write, the unfused pair and the fused call) and the 78-layer
    depth stack at T=8192, n=4, d=7168. One JSON line per point / op, device
    timed; consecutive calls cycle through distinct buffers so the working
    set between two uses of a buffer exceeds the L2 several times over; calls
    of T <= 4096 are replayed from a CUDA graph (no host time between them).
    Each sweep point also carries the oracle's tokens/s on a small sample."""
    import numpy as np
    import torch
    import hc_inputs as gen
    from hyper_connections_stream_b200 import _lib as hc
    from hyper_connections_stream_b200 import traffic
    ws, rank, local = _dist_env()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    _set_path(args)
    peak, peak_kind = _peaks()
    K, eps = WORKLOAD["K"], WORKLOAD["eps"]
    bf = torch.bfloat16
    lines = []

    def point_line(kind, T, n, d, ms, alg, extra):
        ach = alg / (ms / 1e3) / 1e9
        line = {"op": kind, "T": T, "n": n, "d": d, "us_per_call": ms * 1e3,
                "tokens_per_s": T / (ms / 1e3), "algorithmic_bytes_per_call": alg,
                "achieved_GBs": ach, "frac": ach / peak, "frac_of_8TBs": ach / 8000.0,
                "peak": peak, "peak_source": peak_kind}
        line.update(extra)
        print(json.dumps(line), flush=True)
        lines.append(line)

    Ts = [args.tokens] if args.tokens else SWEEP_T
    Ns = [args.streams] if args.streams else SWEEP_N
    Ds = [args.width] if args.width else SWEEP_D
    for d in Ds:
        for n in Ns:
            for T in Ts:
                alg = traffic.step_bytes("fused", T, n, d, "bf16", per_token_mix=True,
                                         per_token_read=True)
                P = _slots(alg)
                Hin = gen.device_normal(gen.SEED_H + 5, (P, T, n, d), bf, device)
                Hout = torch.empty_like(Hin)
                y = gen.device_normal(gen.SEED_Y + 5, (P, T, d), bf, device)
                L = gen.device_normal(gen.SEED_L + 5, (P, T, n, n), torch.float32, device)
                rl = gen.device_normal(gen.SEED_L + 105, (P, T, n), torch.float32, device)
                x = torch.empty((P, T, d), dtype=bf, device=device)
                b = torch.from_numpy(gen.static_params(5, n)[2]).to(device)
                g = torch.ones(d, dtype=torch.float32, device=device)

                def call(i):
                    j = i % P
                    hc.write_then_read(Hin[j], y[j], L[j], b, rl[j], g, eps=eps,
                                       mix=hc.MIX_SINKHORN_LOGITS, K=K,
                                       read=hc.READ_SOFTMAX_LOGITS, out=Hout[j], x_next=x[j])
                graph = T <= 4096
                ncalls = max(P, 64) if graph else max(P, 5 if T >= 65536 else 20)
                ms = _per_call_ms(call, ncalls, device, graph=graph)
                family = hc.step_path("fused", T, n, d)
                orate, S = _oracle_point_rate(T, n, d, K, eps)
                point_line("sweep_fused_mhc", T, n, d, ms, alg,
                           {"buffer_sets": P, "calls": ncalls, "graph": graph,
                            "kernel_family": "register" if family == hc.PATH_REGISTER else "pipelined",
                            "oracle_tokens_per_s": orate, "oracle_sample_tokens": S})
                del Hin, Hout, y, L, rl, x
                torch.cuda.empty_cache()

    if not (args.tokens or args.streams or args.width):
        # static HC layer: T=4096, n=4, d=4096, per-layer a, A, b = identity + N(0, 0.02)
        T, n, d = 4096, 4, 4096
        a, A, b = (torch.from_numpy(v).to(device) for v in gen.static_params(2, n))
        g = torch.ones(d, dtype=torch.float32, device=device)
        per = {k: traffic.step_bytes(k, T, n, d, "bf16") for k in ("read", "write", "fused")}
        P = _slots(per["read"])
        Hs = gen.device_normal(gen.SEED_H + 2, (P, T, n, d), bf, device)
        Ho = torch.empty_like(Hs)
        ys = gen.device_normal(gen.SEED_Y + 2, (P, T, d), bf, device)
        xs = torch.empty((P, T, d), dtype=bf, device=device)
        ops = {
            "read": (lambda i: hc.read_rmsnorm(Hs[i % P], a, g, eps=eps, x=xs[i % P]), per["read"]),
            "write": (lambda i: hc.write_mix(Hs[i % P], ys[i % P], A, b, out=Ho[i % P]),
                      per["write"]),
            "unfused_pair": (lambda i: (hc.write_mix(Hs[i % P], ys[i % P], A, b, out=Ho[i % P]),
                                        hc.read_rmsnorm(Ho[i % P], a, g, eps=eps, x=xs[i % P])),
                             per["write"] + per["read"]),
            "fused": (lambda i: hc.write_then_read(Hs[i % P], ys[i % P], A, b, a, g, eps=eps,
                                                   out=Ho[i % P], x_next=xs[i % P]), per["fused"]),
        }
        fam = {k: ("register" if hc.step_path(k, T, n, d) == hc.PATH_REGISTER else "pipelined")
               for k in ("read", "write", "fused")}
        fam["unfused_pair"] = f"write {fam['write']}, read {fam['read']}"
        for name, (fn, alg) in ops.items():
            ms = _per_call_ms(fn, max(P, 64), device, graph=True)
            point_line("static_layer_" + name, T, n, d, ms, alg,
                       {"buffer_sets": P, "kernel_family": fam[name]})
        del Hs, Ho, ys, xs
        torch.cuda.empty_cache()

        # depth stack: 78 layers, T=8192, n=4, d=7168; static per-layer mixing,
        # gains U(0.5, 1.5); block stand-in y = tanh(x) (torch, not timed as HC)
        T, n, d, layers = 8192, 4, 7168, 78
        prm = []
        for l in range(layers + 1):
            al, Al, bl = gen.static_params(4, n, layer=l)
            gl = gen.uniform(gen.SEED_P + 4 + 500 + l, (d,), 0.5, 1.5)
            prm.append(tuple(torch.from_numpy(v).to(device) for v in (al, Al, bl, gl)))
        H0 = gen.device_normal(gen.SEED_H + 4, (T, n, d), bf, device)
        Hb = (torch.empty_like(H0), torch.empty_like(H0))
        x = torch.empty((T, d), dtype=bf, device=device)
        yb = torch.empty((T, d), dtype=bf, device=device)
        stream = torch.cuda.current_stream(device)
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(layers + 1)]

        def stack(timed):
            e = ev[0]
            if timed:
                e[0].record(stream)
            hc.read_rmsnorm(H0, prm[1][0], prm[1][3], eps=eps, x=x)
            if timed:
                e[1].record(stream)
            src = H0
            for l in range(1, layers + 1):
                torch.tanh(x, out=yb)
                dst = Hb[l % 2]
                e = ev[l]
                if timed:
                    e[0].record(stream)
                if l < layers:
                    _, Al, bl, _ = prm[l]
                    an, _, _, gn = prm[l + 1]
                    hc.write_then_read(src, yb, Al, bl, an, gn, eps=eps, out=dst, x_next=x)
                else:
                    hc.write_mix(src, yb, prm[l][1], prm[l][2], out=dst)
                if timed:
                    e[1].record(stream)
                src = dst

        for _ in range(2):
            stack(False)
        torch.cuda.synchronize()
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s0.record(stream)
        stack(True)
        s1.record(stream)
        torch.cuda.synchronize()
        hc_ms = [a_.elapsed_time(b_) for a_, b_ in ev]
        stack_ms = s0.elapsed_time(s1)
        fused_ms = statistics.mean(hc_ms[1:layers])
        alg = traffic.step_bytes("fused", T, n, d, "bf16")
        point_line("depth_stack_fused_layer", T, n, d, fused_ms, alg,
                   {"layers": layers, "stack_hc_ms": sum(hc_ms), "stack_ms_with_tanh": stack_ms,
                    "stack_tokens_per_s": T / (stack_ms / 1e3),
                    "stack_hc_tokens_per_s": T / (sum(hc_ms) / 1e3),
                    "note": "per-layer mean of the 77 fused write->read launches; the stack "
                            "adds layer 1's read, layer 78's write and 78 torch tanh calls"})
    if rank == 0:
        return {"sweep_lines": len(lines), "device_fault": hc.device_fault(),
                "gpu_launches": None, "peak": peak, "peak_source": peak_kind}
    return None


def run_ours(args):
    import torch
    from hyper_connections_stream_b200 import _lib as hc
    from hyper_connections_stream_b200 import traffic

    ws, rank, local = _dist_env()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    hc.set_path({"auto": hc.PATH_AUTO, "pipelined": hc.PATH_PIPELINED,
                 "register": hc.PATH_REGISTER}[args.path])
    if ws > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=device)
    w = dict(WORKLOAD)
    if args.tokens:
        w["T"] = args.tokens
    if args.streams:
        w["n"] = args.streams
    if args.width:
        w["d"] = args.width
    T, n, d, K = w["T"], w["n"], w["d"], w["K"]
    inp = make_inputs(w, rank, device)
    H0 = inp["H"]
    H1 = torch.empty_like(H0)
    x = torch.empty((T, d), dtype=torch.bfloat16, device=device)
    stream = torch.cuda.current_stream(device)

    def step(src, dst):
        hc.write_then_read(src, inp["y"], inp["L"], inp["b"], inp["rl"], inp["g"], eps=w["eps"],
                           mix=hc.MIX_SINKHORN_LOGITS, K=K, read=hc.READ_SOFTMAX_LOGITS,
                           out=dst, x_next=x)

    bufs = (H0, H1)
    for i in range(args.warmup):
        step(bufs[i % 2], bufs[(i + 1) % 2])
    torch.cuda.synchronize()

    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(device).uuid)
    except Exception:
        pass

    # The timed steps are captured once in a CUDA graph (the way a layer loop
    # is deployed: no host time between launches) and replayed once untimed;
    # the timed region is one replay between two events. --stream-launch times
    # plain stream launches with events around every step instead.
    graph = None
    if not args.stream_launch:
        side = torch.cuda.Stream(device)
        side.wait_stream(stream)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=side):
            for i in range(args.steps):
                step(bufs[i % 2], bufs[(i + 1) % 2])
        graph.replay()
        torch.cuda.synchronize()

    def timed():
        _barrier(ws)
        torch.cuda.synchronize()
        if graph is not None:
            a_, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            with ClockSampler(uuid if rank == 0 else None) as clk:
                a_.record(stream)
                graph.replay()
                b_.record(stream)
                torch.cuda.synchronize()
            _barrier(ws)
            total_ms = a_.elapsed_time(b_)
            return total_ms, [total_ms / args.steps], clk.summary()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)]
        with ClockSampler(uuid if rank == 0 else None) as clk:
            for i in range(args.steps):
                ev[i][0].record(stream)
                step(bufs[i % 2], bufs[(i + 1) % 2])
                ev[i][1].record(stream)
            torch.cuda.synchronize()
        _barrier(ws)
        total_ms = ev[0][0].elapsed_time(ev[-1][1])
        per_launch = [s.elapsed_time(e) for s, e in ev]
        return total_ms, per_launch, clk.summary()

    total_ms, per_launch, clocks = timed()
    # rank 0 alone samples the clocks; every rank takes its decision through one
    # collective, so all ranks re-measure together (same collectives, same order)
    bad = 1.0 if clocks and BAD_REASONS & set(clocks["reasons"]) else 0.0
    if _max_over_ranks(bad, ws, device) > 0:
        total_ms, per_launch, clocks = timed()  # re-measured once
    total_ms = _max_over_ranks(total_ms, ws, device)
    ms_per_step = total_ms / args.steps
    value = ws * T * args.steps / (total_ms / 1e3)

    # dominant (only) kernel: algorithmic bytes per launch / mean launch time
    kern_ms = _max_over_ranks(statistics.mean(per_launch), ws, device)
    alg_bytes = traffic.step_bytes("fused", T, n, d, "bf16", per_token_mix=True,
                                   per_token_read=True)
    peak, peak_kind = _peaks()
    achieved = alg_bytes / (kern_ms / 1e3) / 1e9
    prof = (_profiled_traffic("fused_mhc_n4_d7168_bf16_T16384")
            if (T, n, d) == (WORKLOAD["T"], WORKLOAD["n"], WORKLOAD["d"]) else None)

    del graph
    # end to end through the public API with host buffers
    e2e = None if args.kernel_only else run_e2e(args, inp, w, device, ws)

    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    if rank != 0:
        return None
    line = {
        "metric": METRIC if (n, d) == (WORKLOAD["n"], WORKLOAD["d"])
        else f"HC step tokens/sec at n={n}, d={d} (bf16; sweep case)",
        "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": _step_config(w, ws),
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": prof, "peak_source": peak_kind,
                     "algorithmic_bytes_per_launch": alg_bytes, "kernel_ms": kern_ms,
                     "frac_of_8TBs": achieved / 8000.0},
        "e2e": e2e,
        "gpu_launches": args.steps * ws,
        "launch": "stream launches, events around every step" if args.stream_launch
        else f"CUDA graph of the {args.steps} timed steps, replayed once (one warm replay before); "
             "events around the replay",
        "kernel_path": args.path,
        "device_fault": hc.device_fault(),
        "clocks": clocks,
    }
    if ws == 1 and not (args.no_cpu_baseline or args.kernel_only):
        line["cpu_baseline"] = cpu_baseline(w, target_s=args.cpu_seconds)
    return line


def _step_config(w, ws):
    """The config dict of the step's line (both arms print the same one)."""
    from hyper_connections_stream_b200 import traffic
    T, n, d = w["T"], w["n"], w["d"]
    alg_bytes = traffic.step_bytes("fused", T, n, d, "bf16", per_token_mix=True, per_token_read=True)
    return {"workload": w["name"], "T": T, "n": n, "d": d, "K": w["K"], "storage": "bf16",
            "accumulate": "fp32", "tokens_per_gpu": T, "global_tokens": ws * T,
            "parallelism": f"token-sharded x{ws} (no collective)",
            "l2": f"inputs larger than L2: {alg_bytes / 1e9:.2f} GB read+written per step "
                  "vs 126 MB L2; stream state ping-pongs between two buffers"}


def run_e2e(args, inp, w, device, ws):
    """Same step through the public API with the stream state in pinned host
    memory: every step copies its inputs host->device, runs the fused kernel
    and copies H' and x back, chunked over three CUDA streams so both PCIe
    directions and the kernel overlap; all inside the timed region (CUDA
    events on the launching stream)."""
    import torch
    from hyper_connections_stream_b200 import _lib as hc
    from hyper_connections_stream_b200 import host
    T, n, d = w["T"], w["n"], w["d"]
    hH = inp["H"].cpu().pin_memory()
    hy = inp["y"].cpu().pin_memory()
    hL = inp["L"].cpu().pin_memory()
    hrl = inp["rl"].cpu().pin_memory()
    oH = torch.empty_like(hH).pin_memory()
    ox = torch.empty((T, d), dtype=torch.bfloat16).pin_memory()
    chunks = 16
    stepper = host.HostStepper((T + chunks - 1) // chunks, n, d, torch.bfloat16, device,
                               per_token_mix=True, per_token_read=True)
    stream = torch.cuda.current_stream(device)

    def step():
        host.write_then_read_from_host(hH, hy, hL, inp["b"], hrl, inp["g"], out_H=oH, out_x=ox,
                                       eps=w["eps"], mix=hc.MIX_SINKHORN_LOGITS, K=w["K"],
                                       read=hc.READ_SOFTMAX_LOGITS, stepper=stepper, chunks=chunks)

    steps = max(3, min(args.e2e_steps, args.steps))
    for _ in range(2):
        step()
    torch.cuda.synchronize()
    _barrier(ws)
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record(stream)
    for _ in range(steps):
        step()
    e.record(stream)
    torch.cuda.synchronize()
    ms = _max_over_ranks(s.elapsed_time(e), ws, device)
    h2d = hH.numel() * 2 + hy.numel() * 2 + hL.numel() * 4 + hrl.numel() * 4
    d2h = oH.numel() * 2 + ox.numel() * 2
    return {"value": ws * T * steps / (ms / 1e3), "unit": UNIT, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": steps, "ms_per_step": ms / steps,
            "how": f"pinned host buffers, {chunks} chunks over 3 CUDA streams"}


# ----------------------------------------------------------------------------
# the oracle (CPU baseline / reference arm)
# ----------------------------------------------------------------------------

def _oracle_sample(w, S, seed_shift=0):
    import numpy as np
    import hc_inputs as gen
    n, d, cfg = w["n"], w["d"], w["cfg"]
    H = gen.streams(cfg + seed_shift, S, n, d, "bf16")
    y = gen.block_out(cfg + seed_shift, S, d, "bf16")
    L = gen.mix_logits(cfg + seed_shift, S, n)
    rl = gen.read_logits(cfg + seed_shift, S, n)
    _, _, b = gen.static_params(cfg, n)
    return H, y, L, b, rl, np.ones(d, np.float32)


def _oracle_step(w, sample):
    import oracle
    H, y, L, b, rl, g = sample
    oracle.write_then_read(H, y, L, b, rl, g, w["eps"], "bf16", K=w["K"], mix_logits=True,
                           read_logits=True)


def _oracle_rate(w, S):
    sample = _oracle_sample(w, S)
    t0 = time.perf_counter()
    _oracle_step(w, sample)
    return S / (time.perf_counter() - t0)


def _oracle_timed(w, target_s):
    """(tokens/s, sample tokens, steps, seconds) of the oracle stepping a
    bounded token sample of the workload for about target_s seconds."""
    probe = 64
    rate = _oracle_rate(w, probe)
    S = int(max(probe, min(w["T"], rate * target_s)))
    sample = _oracle_sample(w, S)
    reps, t0 = 0, time.perf_counter()
    while True:
        _oracle_step(w, sample)
        reps += 1
        dt = time.perf_counter() - t0
        if dt >= target_s or reps >= 1000:
            break
    return S * reps / dt, S, reps, dt


def cpu_baseline(w, target_s=12.0):
    """The oracle, as it stands, on the host cores: a bounded token sample of
    the same workload, stepped repeatedly for about target_s seconds, with
    OpenMP over tokens on every core; then the same on one thread for a
    quarter of that time."""
    import oracle
    cores = oracle.max_threads()
    value, S, reps, dt = _oracle_timed(w, target_s)
    oracle.set_threads(1)
    try:
        v1, S1, reps1, dt1 = _oracle_timed(w, target_s / 4)
    finally:
        oracle.set_threads(cores)
    return {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{S} of the workload's {w['T']} tokens (same shapes and distributions, "
                      f"host-generated), {reps} fused step(s), {dt:.1f} s",
            "single_thread": {"value": v1, "unit": UNIT, "cores": 1,
                              "sample": f"{S1} tokens, {reps1} fused step(s), {dt1:.1f} s"}}


def run_reference(args):
    ws, rank, _ = _dist_env()
    if rank != 0:
        return None
    import oracle
    w = WORKLOAD
    rate = _oracle_rate(w, 32)
    budget_s = args.ref_seconds
    S = int(max(1, min(w["T"], rate * budget_s / max(1, args.steps + args.warmup))))
    sample = _oracle_sample(w, S)
    for _ in range(args.warmup):
        _oracle_step(w, sample)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        _oracle_step(w, sample)
    dt = time.perf_counter() - t0
    value = S * args.steps / dt
    cores = oracle.max_threads()
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": _step_config(w, ws),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"{S} tokens of the {w['T']}-token workload per step "
                                   "(same shapes and distributions, host-generated)"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--e2e-steps", type=int, default=8)
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--ref-seconds", type=float, default=90.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--kernel-only", action="store_true",
                    help="device-timed kernel only (no e2e, no CPU baseline): for profiling")
    ap.add_argument("--op", choices=["step", "logits", "expand_read", "collapse", "linear_write",
                                     "reduce_write", "reduce_scatter", "backward", "decode", "sweep"],
                    default="step",
                    help="step: the fused HC step (the metric); logits: the tensor-core "
                         "mixing-logits kernel on the same streams; expand_read / collapse: "
                         "the stack ends on the same shape; linear_write: the block's output "
                         "projection fused with the write; reduce_write: the write fused with "
                         "the tensor-parallel all-reduce of y (--ranks partials); reduce_scatter: "
                         "its reduce-scatter form (--ranks ranks emulated on one GPU); backward: the "
                         "step's backward pass; decode: per-call latency of small steps (CUDA graph); "
                         "sweep: tokens/s and HBM fraction per T x n x d point, the static layer "
                         "(read, write, unfused pair, fused) and the 78-layer depth stack")
    ap.add_argument("--stream-launch", action="store_true",
                    help="time the step with plain stream launches and events around every step "
                         "(default: the timed steps replayed from one CUDA graph)")
    ap.add_argument("--path", choices=["auto", "pipelined", "register"], default="auto",
                    help="kernel family (auto = pipelined wherever it applies)")
    ap.add_argument("--ranks", type=int, default=8,
                    help="partials summed by --op reduce_write (tensor-parallel group size)")
    ap.add_argument("--tokens", type=int, default=0,
                    help="override T (smaller cases for ncu captures)")
    ap.add_argument("--streams", type=int, default=0,
                    help="override n for --op step / backward (sweep cases; the metric's workload is n=4)")
    ap.add_argument("--width", type=int, default=0,
                    help="override d for --op step (sweep cases; the metric's workload is d=7168)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    if ws != args.gpus and not (ws == 1 and args.gpus == 1):
        if args.gpus > 1 and ws == 1:
            ap.error(f"--gpus {args.gpus} needs torchrun with {args.gpus} processes")
    if args.impl == "reference":
        line = run_reference(args)
    elif args.op == "logits":
        line = run_logits(args)
    elif args.op in ("expand_read", "collapse"):
        line = run_ends(args)
    elif args.op == "linear_write":
        line = run_linear_write(args)
    elif args.op == "reduce_write":
        line = run_reduce_write(args)
    elif args.op == "reduce_scatter":
        line = run_reduce_write(args, scatter=True)
    elif args.op == "backward":
        line = run_backward(args)
    elif args.op == "decode":
        line = run_decode(args)
    elif args.op == "sweep":
        line = run_sweep(args)
    else:
        line = run_ours(args)
    if line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
