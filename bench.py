#!/usr/bin/env python
"""Benchmark of the chunked SSD forward: tokens/s and TFLOP/s on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config c1] [--impl ours|reference]

One step is one ``ssd_fwd`` call over the whole workload (all chunked steps:
cumsum, intra-chunk output, chunk states, state passing, output correction)
with inputs already resident in HBM.  The default workload is the Mamba-2
2.7B-shaped layer (b8 L2048 H80 P64 N128 G1 Q64, bf16 in / fp32 accumulate).
Rank 0 prints one JSON line.

Timing: W untimed warm-up steps, then K steps bracketed by a barrier and a
device synchronize, timed with CUDA events on the launching stream; the
maximum over ranks is reported.  The inputs and outputs (hundreds of MB)
are larger than the 126 MB L2, so no flush is needed between steps.

With N > 1 (torchrun, one process per GPU) every rank runs its own replica
of the workload: the (batch, head) units are independent and need no
exchange, so there is no collective on the data path ("weak" scaling).

``--impl reference`` times the fp64 CPU oracle instead (host cores, bounded
samples of the same workload), as the comparison arm.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

import ssd_inputs as si  # noqa: E402

METRIC = "SSD fwd tokens/s and TFLOP/s (% of bf16 tensor roofline) at L=2K–16K, 1 B200"
DATASHEET_HBM_GBS = 8000.0
DATASHEET_BF16_TFLOPS = 2250.0
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_BYTES = 126 * 1024 * 1024
# fp32 FMA throughput of the CUDA cores: 148 SMs x 128 lanes x 2 FLOP x 1.965 GHz (max SM clock)
FP32_PEAK_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


# ----------------------------------------------------------------------------- helpers

def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    return dict(FALLBACK_PEAKS, source="fallback")


def work(shape: si.SSDShape, num_seqs):
    """Algorithmic FLOPs (full Q x Q tiles, C.B^T once per group; and the
    causal-half count) and minimum HBM bytes (each tensor touched once)."""
    s = shape
    b, L, H, P, N, G, Q = s.batch, s.seqlen, s.nheads, s.headdim, s.dstate, s.ngroups, s.chunk_size
    c = -(-L // Q)
    full = (2 * Q * Q * N * c * G * b + 2 * Q * Q * P * c * H * b + 4 * Q * N * P * c * H * b
            + 2 * N * P * c * H * b + 2 * P * b * L * H)
    causal = (Q * (Q + 1) * N * c * G * b + Q * (Q + 1) * P * c * H * b + 4 * Q * N * P * c * H * b
              + 2 * N * P * c * H * b + 2 * P * b * L * H)
    e = 2 if s.dtype == "bf16" else 4
    nbytes = 2 * b * L * H * P * e + 2 * b * L * G * N * e + 4 * b * L * H + 4 * H * (2 if s.has_D else 1)
    nbytes += 4 * H * P * N * (num_seqs if s.packed is not None else b)  # final states
    if s.h0_std > 0:
        nbytes += 4 * b * H * P * N
    if s.packed is not None:
        nbytes += 4 * b * L
    return {"flops": full, "flops_causal": causal, "bytes": nbytes}


def describe(shape: si.SSDShape) -> str:
    s = shape
    desc = (f"{s.name}: SSD fwd b{s.batch} L{s.seqlen} H{s.nheads} P{s.headdim} N{s.dstate} "
            f"G{s.ngroups} Q{s.chunk_size} {s.dtype}")
    if s.packed:
        desc += f" packed lengths~U{list(s.packed)}"
    if s.h0_std > 0:
        desc += f" h0~N(0,{s.h0_std}^2)"
    return desc


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""
    FIELDS = ("uuid,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid: str, period_ms: int = 50):
        self.uuid = uuid
        self.period_ms = period_ms
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
            os.close(fd)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", str(self.period_ms)], stdout=self.fh, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.1)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.close()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 10:
                continue
            if self.uuid and self.uuid not in parts[0]:
                continue
            rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        mx = [float(r[3]) for r in rows if r[3].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[6:10]) if v.lower() == "active"})
        loaded = [v for v in sm if mx and v >= 0.5 * max(mx)] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(rows)}


def gpu_uuid(dev) -> str:
    try:
        u = str(torch.cuda.get_device_properties(dev).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        return ""


def traffic_from_profiles(kernel_file: str, kernel: str, workload: str):
    """dram read+write bytes per launch from a committed ncu summary, if it was
    taken on the kernel source as it is now."""
    path = os.path.join(ROOT, "profiles", f"{workload}_{kernel}_dram.txt")
    if not os.path.exists(path):
        return None
    kv = {}
    for line in open(path):
        if ":" in line:
            k, v = line.split(":", 1)
            kv[k.strip()] = v.strip()
    src = os.path.join(ROOT, "mamba_ssd_chunked_03_b200", "csrc", kernel_file)
    if not os.path.exists(src):
        return None
    sha = hashlib.sha256(open(src, "rb").read()).hexdigest()
    if kv.get("source_sha256") != sha:
        return None
    try:
        return float(kv["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


def max_over_ranks(value: float, dist=None, device=None) -> float:
    """The largest of every rank's ``value`` (each rank times its own replica;
    the job takes as long as its slowest rank).  Without a process group the
    value is returned as is."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ----------------------------------------------------------------------------- CPU oracle timing

def oracle_sample(d, shape, target_s: float, max_units=None):
    """Time the fp64 oracle on the first U (batch, head) units of the workload,
    U chosen so the run takes about ``target_s`` seconds.  Returns
    (tokens/s, units, seconds, threads)."""
    import oracle  # test infrastructure: only this CPU-baseline leg uses it here
    f = {k: oracle.as_f32(d[k]) for k in ("x", "dt", "A", "B", "C", "D", "initial_states")}
    si_ = d.get("seq_idx")
    seq = None if si_ is None else oracle.as_i32(si_)
    threads = oracle.max_threads()
    total_units = shape.batch * shape.nheads
    t = time.perf_counter()
    oracle.ssd_fwd(f["x"], f["dt"], f["A"], f["B"], f["C"], f["D"], f["initial_states"], seq, d.get("num_seqs"),
                   units=list(range(min(threads, total_units))))
    t_wave = max(time.perf_counter() - t, 1e-3)
    waves = max(1, int(target_s / t_wave))
    U = min(total_units, waves * threads) if max_units is None else min(total_units, max_units)
    t = time.perf_counter()
    oracle.ssd_fwd(f["x"], f["dt"], f["A"], f["B"], f["C"], f["D"], f["initial_states"], seq, d.get("num_seqs"),
                   units=list(range(U)))
    el = time.perf_counter() - t
    tokens = U * shape.seqlen / shape.nheads
    return tokens / el, U, el, min(threads, U)


def run_reference_op(args):
    """``--impl reference`` for ``--op step`` / ``--op conv``: the oracle on the
    same workload as the GPU arm, timed on the host cores."""
    import oracle
    if args.op == "bwd":
        return run_reference_bwd(args)
    if args.op == "conv_bwd":
        return run_reference_conv_bwd(args)
    if args.op == "step":
        b, H, P, N, G = args.step_batch, 80, 64, 128, 1
        shape = si.SSDShape("decode", b, 1, H, P, N, G, 64, "bf16", h0_std=0.5, seed=11)
        d = si.make_inputs(shape)
        f = {k: oracle.as_f32(d[k]) for k in ("x", "dt", "A", "B", "C", "D", "initial_states")}
        run = lambda: oracle.ssd_fwd(f["x"], f["dt"], f["A"], f["B"], f["C"], f["D"], f["initial_states"])
        per_step, metric = b, "SSD decode step (one token per row), rows/s"
        workload = f"decode step: b{b} H{H} P{P} N{N} G{G} bf16, fp32 state"
        cores = oracle.max_threads()
    else:
        from oracle import block
        b, L, C, K = 8, 2048, 80 * 64 + 2 * 1 * 128, 4
        gen = torch.Generator().manual_seed(13)
        u = torch.randn(1, L, C, generator=gen).to(torch.bfloat16)  # one batch row per repetition
        w, bias = torch.randn(C, K, generator=gen) * 0.5, torch.randn(C, generator=gen) * 0.1
        run = lambda: block.conv1d_silu(u, w, bias)
        per_step, metric = L, "Mamba-2 block causal conv1d + SiLU tokens/s"
        workload = f"conv1d+SiLU: one batch row of b{b} L{L} channels {C} width {K} bf16"
        cores = 1
    for _ in range(args.warmup):
        run()
    t = time.perf_counter()
    for _ in range(args.steps):
        run()
    el = time.perf_counter() - t
    value = per_step * args.steps / el
    sample = f"{args.steps} repetitions of {workload}"
    line = {
        "impl": "reference", "metric": metric, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": el / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload, "sample": sample},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_reference_conv_bwd(args):
    """``--impl reference --op conv_bwd``: the conv backward oracle, one batch
    row of c1's xBC tensor per step, on the host."""
    from oracle import block
    b, L, C, K = 8, 2048, 80 * 64 + 2 * 1 * 128, 4
    gen = torch.Generator().manual_seed(13)
    u = torch.randn(1, L, C, generator=gen).to(torch.bfloat16)
    w, bias = torch.randn(C, K, generator=gen) * 0.5, torch.randn(C, generator=gen) * 0.1
    dout = torch.randn(1, L, C, generator=gen).to(torch.bfloat16)
    for _ in range(args.warmup):
        block.conv1d_silu_bwd(u, w, bias, dout)
    t = time.perf_counter()
    for _ in range(args.steps):
        block.conv1d_silu_bwd(u, w, bias, dout)
    el = time.perf_counter() - t
    value = L * args.steps / el
    sample = f"{args.steps} batch rows of b{b} L{L} channels {C} width {K} (numpy, one process)"
    line = {
        "impl": "reference", "metric": "Mamba-2 block causal conv1d + SiLU backward tokens/s", "value": value,
        "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": el / args.steps * 1e3, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic", "config": {"workload": "conv1d+SiLU backward, c1 xBC", "sample": sample},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_reference(args, shape):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    if args.op != "fwd":
        return run_reference_op(args)
    import oracle
    d = si.make_inputs(shape)
    f = {k: oracle.as_f32(d[k]) for k in ("x", "dt", "A", "B", "C", "D", "initial_states")}
    seq = None if d.get("seq_idx") is None else oracle.as_i32(d["seq_idx"])
    threads = oracle.max_threads()
    U = min(shape.batch * shape.nheads, threads)
    units = list(range(U))

    def step():
        oracle.ssd_fwd(f["x"], f["dt"], f["A"], f["B"], f["C"], f["D"], f["initial_states"], seq,
                       d.get("num_seqs"), units=units)

    for _ in range(args.warmup):
        step()
    t = time.perf_counter()
    for _ in range(args.steps):
        step()
    el = time.perf_counter() - t
    tokens = U * shape.seqlen / shape.nheads * args.steps
    value = tokens / el
    w = work(shape, d.get("num_seqs"))
    sample = (f"first {U} of {shape.batch * shape.nheads} (batch, head) units per step "
              f"= {U * shape.seqlen} head-tokens = {U * shape.seqlen / shape.nheads:.1f} tokens")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": el / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": describe(shape), "sample": sample},
        "tflops": value / shape.tokens * w["flops"] / 1e12,
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": min(threads, U), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- decode step

def run_step(args, dist, dev, world, rank):
    """``--op step``: the recurrent (decode) step ``ssd_step`` on one token per
    row for ``--step-batch`` rows of the c1 head layout (H 80, P 64, N 128,
    G 1, bf16), the fp32 state resident in HBM and updated in place.  Bound by
    HBM on the state: 8 b H P N bytes read and written per step."""
    import mamba_ssd_chunked_03_b200 as ssd
    b, H, P, N, G = args.step_batch, 80, 64, 128, 1
    shape = si.SSDShape("decode", b, 1, H, P, N, G, 64, "bf16", h0_std=0.5, seed=11 + rank)
    host = si.make_inputs(shape)
    inputs = {k: host[k][:, 0].contiguous() for k in ("x", "dt", "B", "C")}
    g = {k: v.to(dev) for k, v in inputs.items()}
    A, D = host["A"].to(dev), host["D"].to(dev)
    state = host["initial_states"].to(dev)
    y = torch.empty_like(g["x"])

    def step():
        ssd.step(g["x"], g["dt"], A, g["B"], g["C"], D, state, y=y)

    K = args.steps
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    clocks = ClockSampler(gpu_uuid(dev))
    clocks.start()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(K):
        step()
    e1.record()
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    clock_stats = clocks.stop()
    ms_step = max_over_ranks(e0.elapsed_time(e1), dist, dev) / K

    # end to end: this step's inputs from pinned host memory, y back; the state
    # stays on the device (it is the decode cache)
    pinned = {k: v.pin_memory() for k, v in inputs.items()}
    y_host = torch.empty(y.shape, dtype=y.dtype).pin_memory()
    h2d = sum(v.numel() * v.element_size() for v in pinned.values())
    d2h = y_host.numel() * y_host.element_size()

    def e2e_step():
        for k in pinned:
            g[k].copy_(pinned[k], non_blocking=True)
        step()
        y_host.copy_(y, non_blocking=True)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize()
    E = max(3, min(K, 50))
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a0.record()
    for _ in range(E):
        e2e_step()
    a1.record()
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(a0.elapsed_time(a1), dist, dev) / E

    state_bytes = b * H * P * N * 4
    nbytes = 2 * state_bytes + 2 * b * H * P * 2 + 2 * b * G * N * 2 + b * H * 4
    peaks = load_peaks()
    achieved = nbytes / (ms_step / 1e3) / 1e9
    line = {
        "metric": "SSD decode step (one token per row), rows/s", "value": b * world / (ms_step / 1e3),
        "unit": "tokens/s", "n_gpus": world, "steps": K, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"decode step: b{b} H{H} P{P} N{N} G{G} bf16, fp32 state in HBM "
                               f"({state_bytes / 1e6:.0f} MB)",
                   "l2": f"no flush: state {state_bytes / 1e6:.0f} MB > 126 MB L2",
                   "parallelism": "replicas" if world > 1 else "single GPU"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / peaks["hbm_gbs"], "peak_source": peaks["source"],
                     "frac_datasheet": achieved / DATASHEET_HBM_GBS, "kernel": "k_ssd_step",
                     "kernel_ms": ms_step, "traffic": None, "algorithmic_bytes": nbytes},
        "e2e": {"value": b * world / (e2e_ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": E},
        "gpu_launches": K,
        "clocks": clock_stats,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle  # test infrastructure: only this CPU-baseline leg uses it here
        f = {k: oracle.as_f32(host[k]) for k in ("x", "dt", "A", "B", "C", "D", "initial_states")}
        threads = oracle.max_threads()
        reps, t = 0, time.perf_counter()
        while True:
            oracle.ssd_fwd(f["x"], f["dt"], f["A"], f["B"], f["C"], f["D"], f["initial_states"])
            reps += 1
            el = time.perf_counter() - t
            if el >= min(args.cpu_seconds, 10.0):
                break
        line["cpu_baseline"] = {"value": reps * b / el, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                                "sample": f"{reps} whole steps of the workload (all {b} rows), {el:.1f} s"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist:
        dist.destroy_process_group()
    return 0


# ----------------------------------------------------------------------------- block piece: conv1d + SiLU

def run_conv(args, dist, dev, world, rank):
    """``--op conv``: the Mamba-2 block's causal depthwise conv1d + SiLU on c1's
    xBC tensor (b 8, L 2048, channels H P + 2 G N = 5376, width 4, bf16).
    Bound by HBM: u read and out written once."""
    import mamba_ssd_chunked_03_b200 as ssd
    b, L, C, K = 8, 2048, 80 * 64 + 2 * 1 * 128, 4
    gen = torch.Generator().manual_seed(13 + rank)
    u_h = torch.randn(b, L, C, generator=gen).to(torch.bfloat16)
    w_h = torch.randn(C, K, generator=gen) * 0.5
    bias_h = torch.randn(C, generator=gen) * 0.1
    u, w, bias = u_h.to(dev), w_h.to(dev), bias_h.to(dev)
    out = torch.empty_like(u)

    def step():
        ssd.conv1d_silu(u, w, bias, out=out)

    K_ = args.steps
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    clocks = ClockSampler(gpu_uuid(dev))
    clocks.start()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(K_):
        step()
    e1.record()
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    clock_stats = clocks.stop()
    ms_step = max_over_ranks(e0.elapsed_time(e1), dist, dev) / K_

    pinned, out_host = u_h.pin_memory(), torch.empty_like(u_h).pin_memory()

    def e2e_step():
        u.copy_(pinned, non_blocking=True)
        step()
        out_host.copy_(out, non_blocking=True)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize()
    E = max(3, min(K_, 50))
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a0.record()
    for _ in range(E):
        e2e_step()
    a1.record()
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(a0.elapsed_time(a1), dist, dev) / E

    nbytes = 2 * b * L * C * 2 + C * K * 4 + C * 4
    peaks = load_peaks()
    achieved = nbytes / (ms_step / 1e3) / 1e9
    tokens = b * L
    line = {
        "metric": "Mamba-2 block causal conv1d + SiLU tokens/s", "value": tokens * world / (ms_step / 1e3),
        "unit": "tokens/s", "n_gpus": world, "steps": K_, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"conv1d+SiLU: b{b} L{L} channels {C} (c1 xBC) width {K} bf16",
                   "l2": f"no flush: u + out {nbytes / 1e6:.0f} MB > 126 MB L2",
                   "parallelism": "replicas" if world > 1 else "single GPU"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / peaks["hbm_gbs"], "peak_source": peaks["source"],
                     "frac_datasheet": achieved / DATASHEET_HBM_GBS, "kernel": "k_conv1d_silu",
                     "kernel_ms": ms_step, "traffic": None, "algorithmic_bytes": nbytes},
        "e2e": {"value": tokens * world / (e2e_ms / 1e3), "unit": "tokens/s",
                "h2d_bytes_per_step": b * L * C * 2, "d2h_bytes_per_step": b * L * C * 2, "steps": E},
        "gpu_launches": K_,
        "clocks": clock_stats,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        from oracle import block  # test infrastructure: only this CPU-baseline leg uses it here
        reps, t = 0, time.perf_counter()
        while True:
            block.conv1d_silu(u_h[:1], w_h, bias_h)  # one batch row per repetition
            reps += 1
            el = time.perf_counter() - t
            if el >= min(args.cpu_seconds, 10.0):
                break
        line["cpu_baseline"] = {"value": reps * L / el, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                                "sample": f"{reps} batch rows of {L} tokens (numpy, one process), {el:.1f} s"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist:
        dist.destroy_process_group()
    return 0


def run_conv_bwd(args, dist, dev, world, rank):
    """``--op conv_bwd``: the conv1d + SiLU backward on c1's xBC tensor (b 8,
    L 2048, 5376 channels, width 4, bf16 in, fp32 gradients).  Bound by HBM:
    u and dout read once, du written once (fp32), plus the per-strip weight
    partials."""
    import mamba_ssd_chunked_03_b200 as ssd
    b, L, C, K = 8, 2048, 80 * 64 + 2 * 1 * 128, 4
    gen = torch.Generator().manual_seed(13 + rank)
    u_h = torch.randn(b, L, C, generator=gen).to(torch.bfloat16)
    w_h = torch.randn(C, K, generator=gen) * 0.5
    bias_h = torch.randn(C, generator=gen) * 0.1
    dout_h = torch.randn(b, L, C, generator=gen).to(torch.bfloat16)
    u, w, bias, dout = u_h.to(dev), w_h.to(dev), bias_h.to(dev), dout_h.to(dev)

    def step():
        return ssd.conv1d_silu_bwd(u, w, bias, dout)

    K_ = args.steps
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    clocks = ClockSampler(gpu_uuid(dev))
    clocks.start()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(K_):
        step()
    e1.record()
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    clock_stats = clocks.stop()
    ms_step = max_over_ranks(e0.elapsed_time(e1), dist, dev) / K_

    pinned_u, pinned_d = u_h.pin_memory(), dout_h.pin_memory()
    du_host = torch.empty(b, L, C, dtype=torch.float32).pin_memory()

    def e2e_step():
        u.copy_(pinned_u, non_blocking=True)
        dout.copy_(pinned_d, non_blocking=True)
        du_, _, _ = step()
        du_host.copy_(du_, non_blocking=True)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize()
    E = max(3, min(K_, 20))
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a0.record()
    for _ in range(E):
        e2e_step()
    a1.record()
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(a0.elapsed_time(a1), dist, dev) / E

    strips = -(-L // 32)
    nbytes = 2 * b * L * C * 2 + b * L * C * 4 + 2 * b * strips * C * (K + 1) * 4 + C * (K + 1) * 4
    peaks = load_peaks()
    achieved = nbytes / (ms_step / 1e3) / 1e9
    tokens = b * L
    line = {
        "metric": "Mamba-2 block causal conv1d + SiLU backward tokens/s", "value": tokens * world / (ms_step / 1e3),
        "unit": "tokens/s", "n_gpus": world, "steps": K_, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"conv1d+SiLU backward: b{b} L{L} channels {C} (c1 xBC) width {K}, bf16 in, "
                               f"fp32 gradients",
                   "l2": f"no flush: u + dout + du {nbytes / 1e6:.0f} MB > 126 MB L2",
                   "parallelism": "replicas" if world > 1 else "single GPU"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / peaks["hbm_gbs"], "peak_source": peaks["source"],
                     "frac_datasheet": achieved / DATASHEET_HBM_GBS, "kernel": "k_conv_bwd (with its reduce)",
                     "kernel_ms": ms_step, "traffic": None, "algorithmic_bytes": nbytes},
        "e2e": {"value": tokens * world / (e2e_ms / 1e3), "unit": "tokens/s",
                "h2d_bytes_per_step": 2 * b * L * C * 2, "d2h_bytes_per_step": b * L * C * 4, "steps": E},
        "gpu_launches": 2 * K_,
        "clocks": clock_stats,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        from oracle import block  # test infrastructure: only this CPU-baseline leg uses it here
        reps, t = 0, time.perf_counter()
        while True:
            block.conv1d_silu_bwd(u_h[:1], w_h, bias_h, dout_h[:1])  # one batch row per repetition
            reps += 1
            el = time.perf_counter() - t
            if el >= min(args.cpu_seconds, 10.0):
                break
        line["cpu_baseline"] = {"value": reps * L / el, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                                "sample": f"{reps} batch rows of {L} tokens (numpy, one process), {el:.1f} s"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist:
        dist.destroy_process_group()
    return 0


# ----------------------------------------------------------------------------- backward

BWD_SHAPE = si.SSDShape("c1_bwd", 8, 2048, 80, 64, 128, 1, 64, "bf16", seed=1001)
BWD_WORKLOAD = "SSD bwd on the c1 layout: b8 L2048 H80 P64 N128 G1 bf16, from dy, fp32 gradients"


def bwd_flops(b, L, H, P, N, Q, G=1):
    """Algorithmic FLOPs (2 per multiply-add) of the backward's per-chunk
    kernels, (k_bwd_chunk_states, k_bwd_chunk_cb, k_bwd_chunk), for chunk
    length Q.  Per chunk of Qc tokens, with T2 = Qc (Qc + 1) / 2
    lower-triangle pairs: k_bwd_chunk_states forms two P x N sums of Qc outer
    products (2 Qc P N per head); k_bwd_chunk_cb forms C B^T on the triangle
    (T2 N per group); k_bwd_chunk forms dy x^T on the triangle (T2 P), Lam B^T
    (Qc P N), the triangle products for dx, dB, dC (T2 (P + 2 N)), the state
    terms of dB and dC (2 Qc P N) and <Lam, h_in> (P N) per head."""
    states = cb = chunk = 0
    for c in range(-(-L // Q)):
        qc = min(Q, L - c * Q)
        t2 = qc * (qc + 1) // 2
        states += 2 * qc * P * N
        cb += t2 * N
        chunk += t2 * (2 * N + 2 * P) + 3 * qc * P * N + P * N
    return 2 * b * H * states, 2 * b * G * cb, 2 * b * H * chunk


def bwd_chunk_bytes(b, L, H, P, N, Q, G=1):
    """Algorithmic HBM bytes of the backward's per-chunk kernel (k_bwd_chunk_tc,
    or k_bwd_chunk on the CUDA cores), each tensor touched once: per (row,
    chunk, head) the entering state h_in and its adjoint Lam read (2 P N fp32),
    x and dy read (2 Qc P bf16), dt read and ddt written (2 Qc fp32), dx
    written (Qc P fp32) and the head's dB and dC written (2 Qc N fp32); per
    (row, chunk, group) B and C read (2 Qc N bf16)."""
    tot = 0
    for c in range(-(-L // Q)):
        qc = min(Q, L - c * Q)
        tot += H * (2 * P * N * 4 + 2 * qc * P * 2 + 2 * qc * 4 + qc * P * 4 + 2 * qc * N * 4) + G * 2 * qc * N * 2
    return b * tot


def bwd_inputs(shape, rank=0):
    host = si.make_inputs(shape, seed=shape.seed + rank)
    g = torch.Generator().manual_seed(shape.seed + 17 + rank)
    host["dy"] = torch.randn(*host["x"].shape, generator=g).to(host["x"].dtype)
    return host


def bwd_oracle_sample(host, shape, target_s: float):
    """The C backward oracle on batch row 0 and its first U heads, U grown
    by waves of the host's threads until a run takes about ``target_s``.
    Returns (tokens/s, U, seconds, threads)."""
    import oracle  # test infrastructure: only the CPU-baseline legs use it here
    threads = oracle.max_threads()

    def run(U):
        sl = {k: host[k][:1, :, :U].contiguous() for k in ("x", "dt", "dy")}
        A, D = host["A"][:U].contiguous(), host["D"][:U].contiguous()
        B, C = host["B"][:1], host["C"][:1]
        t = time.perf_counter()
        oracle.ssd_bwd(sl["x"], sl["dt"], A, B, C, D, None, sl["dy"], None, None)
        return time.perf_counter() - t

    U = min(shape.nheads, threads)
    el = run(U)
    while el < target_s / 2 and U < shape.nheads:
        U = min(shape.nheads, U * 2)
        el = run(U)
    return U * shape.seqlen / shape.nheads / el, U, el, min(threads, U)


def run_reference_bwd(args):
    """``--impl reference --op bwd``: the C backward oracle on a bounded sample
    (batch row 0, the first heads) of the backward workload."""
    shape = BWD_SHAPE
    host = bwd_inputs(shape)
    per_run = []
    for i in range(args.warmup + args.steps):
        v, U, el, cores = bwd_oracle_sample(host, shape, 2.0)
        if i >= args.warmup:
            per_run.append((v, U, el, cores))
    value = statistics.median(r[0] for r in per_run)
    U, cores = per_run[-1][1], per_run[-1][3]
    sample = f"batch row 0, heads 0..{U - 1} of {shape.nheads} ({U * shape.seqlen} head-tokens) per step"
    line = {
        "impl": "reference", "metric": "SSD bwd tokens/s", "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": statistics.median(r[2] for r in per_run) * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": BWD_WORKLOAD, "sample": sample},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_bwd(args, dist, dev, world, rank):
    """``--op bwd``: the backward ``ssd_bwd`` on c1's layout (b 8, L 2048,
    H 80, P 64, N 128, G 1, bf16) from a random dy, all gradients in fp32.
    Its dominant kernel, k_bwd_chunk_tc, forms every contraction with tcgen05
    MMAs; at speed of light it is bound by its HBM traffic (the chunk states
    and adjoints read, the gradients written), so the roofline is that
    traffic over its time against the measured HBM peak."""
    import mamba_ssd_chunked_03_b200 as ssd
    shape = BWD_SHAPE.with_(batch=args.bwd_rows, nheads=args.bwd_heads)
    b, L, H, P, N = shape.batch, shape.seqlen, shape.nheads, shape.headdim, shape.dstate
    host = bwd_inputs(shape, rank)
    names = ("x", "dt", "B", "C", "dy")
    if args.gated:  # the gate, like x: dy is then the gradient of y * SiLU(z)
        zg = torch.Generator().manual_seed(7919 + rank)
        host["z"] = torch.randn(host["x"].shape, generator=zg).to(host["x"].dtype)
        names = names + ("z",)
    g = {k: host[k].to(dev) for k in names}
    A, D = host["A"].to(dev), host["D"].to(dev)
    ws = torch.empty(ssd.bwd_workspace_size(g["x"], g["B"], z=g.get("z")), dtype=torch.uint8, device=dev)
    bpath = ssd.bwd_path(g["x"], g["dy"], g["B"], g["C"], z=g.get("z"))
    Q = ssd.bwd_chunk_size(g["x"], g["B"])  # the library's own choice
    K = args.steps
    events = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    for e0_, e1_ in events:  # torch creates an event on its first record
        e0_.record()
        e1_.record()
    out = {}

    def step(ev=None):
        out.update(ssd.bwd(g["x"], g["dt"], A, g["B"], g["C"], D, g["dy"], workspace=ws, timing_events=ev,
                           z=g.get("z")))

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    clocks = ClockSampler(gpu_uuid(dev))
    clocks.start()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(K):
        step(events[i])
    e1.record()
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    clock_stats = clocks.stop()
    ms_step = max_over_ranks(e0.elapsed_time(e1), dist, dev) / K
    per = sorted(a.elapsed_time(z) for a, z in events)
    kernel_ms = max_over_ranks(sum(per) / K, dist, dev)

    pinned = {k: host[k].pin_memory() for k in names}
    grads_host = {k: torch.empty(v.shape, dtype=v.dtype).pin_memory() for k, v in out.items() if v is not None}
    h2d = sum(v.numel() * v.element_size() for v in pinned.values())
    d2h = sum(v.numel() * v.element_size() for v in grads_host.values())

    def e2e_step():
        for k in names:
            g[k].copy_(pinned[k], non_blocking=True)
        step()
        for k, v in grads_host.items():
            v.copy_(out[k], non_blocking=True)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize()
    E = max(3, min(K, 20))
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a0.record()
    for _ in range(E):
        e2e_step()
    a1.record()
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(a0.elapsed_time(a1), dist, dev) / E

    f_states, f_cb, f_chunk = bwd_flops(b, L, H, P, N, Q, shape.ngroups)
    by_chunk = bwd_chunk_bytes(b, L, H, P, N, Q, shape.ngroups)
    achieved = by_chunk / (kernel_ms / 1e3) / 1e9
    peaks = load_peaks()
    tokens = b * L
    line = {
        "metric": "SSD bwd tokens/s", "value": tokens * world / (ms_step / 1e3), "unit": "tokens/s",
        "n_gpus": world, "steps": K, "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": (BWD_WORKLOAD if (b, H) == (8, 80) else
                                BWD_WORKLOAD.replace("b8 ", f"b{b} ").replace("H80 ", f"H{H} "))
                   + (", gated: dy is the gradient of y * SiLU(z), z ~ N(0,1); dz too" if args.gated else ""),
                   "path": bpath,
                   "l2": "no flush: inputs, gradients and the per-chunk states exceed the 126 MB L2"
                         if (b, H) == (8, 80) else "small case for profiling",
                   "parallelism": "replicas" if world > 1 else "single GPU", "bwd_chunk": Q},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / peaks["hbm_gbs"], "peak_source": peaks["source"],
                     "kernel": "k_bwd_chunk_tc (tcgen05)" if bpath == "tcgen05" else "k_bwd_chunk (CUDA cores)",
                     "kernel_ms": kernel_ms,
                     "kernel_ms_p10_p50_p90": [per[int(0.1 * (K - 1))], per[int(0.5 * (K - 1))],
                                               per[int(0.9 * (K - 1))]],
                     "traffic": traffic_from_profiles("ssd_bwd_tc.cuh", "k_bwd_chunk_tc", "c1_bwd")
                     if (b, H) == (8, 80) and bpath == "tcgen05" else None,
                     "algorithmic_bytes": by_chunk, "algorithmic_flops": f_chunk,
                     "tflops": f_chunk / (kernel_ms / 1e3) / 1e12, "states_kernel_flops": f_states,
                     "cb_flops_in_kernel": f_cb},
        "e2e": {"value": tokens * world / (e2e_ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": E},
        "gpu_launches": (4 if bpath == "tcgen05" else 6) * K,
        "clocks": clock_stats,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, U, el, cores = bwd_oracle_sample(host, shape, min(args.cpu_seconds, 10.0))
        line["cpu_baseline"] = {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                                "sample": f"batch row 0, heads 0..{U - 1} of {H}, {el:.1f} s"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist:
        dist.destroy_process_group()
    return 0


# ----------------------------------------------------------------------------- GPU arm

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--config", default="c1", choices=sorted(si.CONFIGS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--generic", action="store_true", help="force the generic CUDA-core kernels")
    ap.add_argument("--gated", action="store_true", help="the forward with the gate z (y * SiLU(z)), z ~ N(0,1)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--op", default="fwd", choices=["fwd", "step", "conv", "bwd", "conv_bwd"],
                    help="fwd: the chunked forward (default); step: the recurrent decode step; "
                         "conv: the block's causal conv1d + SiLU; bwd: the backward on c1's layout; "
                         "conv_bwd: the conv1d + SiLU backward")
    ap.add_argument("--step-batch", type=int, default=256, help="rows of the decode step (--op step)")
    ap.add_argument("--bwd-rows", type=int, default=8, help="batch rows of --op bwd (8: c1)")
    ap.add_argument("--bwd-heads", type=int, default=80, help="heads of --op bwd (80: c1)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    shape = si.CONFIGS[args.config]

    if args.impl == "reference":
        return run_reference(args, shape)

    import mamba_ssd_chunked_03_b200 as ssd

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    if args.op == "step":
        return run_step(args, dist, dev, world, rank)
    if args.op == "conv":
        return run_conv(args, dist, dev, world, rank)
    if args.op == "bwd":
        return run_bwd(args, dist, dev, world, rank)
    if args.op == "conv_bwd":
        return run_conv_bwd(args, dist, dev, world, rank)

    host = si.make_inputs(shape, seed=shape.seed + rank)
    if args.gated:  # the gate, like x
        zg = torch.Generator().manual_seed(shape.seed + 7919 + rank)
        host["z"] = torch.randn(host["x"].shape, generator=zg).to(host["x"].dtype)
    num_seqs = host.get("num_seqs")
    g = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in host.items()}
    b, L, H, P, N = shape.batch, shape.seqlen, shape.nheads, shape.headdim, shape.dstate
    y = torch.empty_like(g["x"])
    rows = num_seqs if shape.packed is not None else b
    final = torch.empty(rows, H, P, N, device=dev, dtype=torch.float32)
    ws_bytes = ssd.workspace_size(g["x"], g["B"], shape.chunk_size, g.get("seq_idx"), num_seqs, True,
                                  generic=args.generic)
    ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=dev)
    launches_per_call = ssd.launch_count(g["x"], g["B"], shape.chunk_size, g.get("seq_idx"), num_seqs, True,
                                         generic=args.generic, z=g.get("z"))
    path = ssd.kernel_path(g["x"], g["B"], shape.chunk_size, generic=args.generic, seq_idx=g.get("seq_idx"),
                           num_seqs=num_seqs)
    main_kernel = ssd.main_kernel(g["x"], g["dt"], g["B"], shape.chunk_size, generic=args.generic,
                                  seq_idx=g.get("seq_idx"), num_seqs=num_seqs, z=g.get("z"))

    K = args.steps
    # the fused kernel's own duration is timed in a separate loop: events
    # recorded between the kernels of a call would stop them overlapping
    KE = max(3, min(K, 50))
    kev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(KE)]

    def step(events=None):
        ssd.fwd(g["x"], g["dt"], g["A"], g["B"], g["C"], g["D"], chunk_size=shape.chunk_size,
                initial_states=g["initial_states"], seq_idx=g.get("seq_idx"), num_seqs=num_seqs,
                y=y, final_states=final, workspace=ws, generic=args.generic, timing_events=events, z=g.get("z"))

    for _ in range(args.warmup):
        step()
    for a_, c_ in kev:  # torch creates the underlying cudaEvent on first record
        a_.record()
        c_.record()
    torch.cuda.synchronize()

    clocks = ClockSampler(gpu_uuid(dev))
    clocks.start()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(K):
        step()
    e1.record()
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    clock_stats = clocks.stop()
    ms = e0.elapsed_time(e1)
    for i in range(KE):
        step(kev[i])
    torch.cuda.synchronize()
    kernel_each = sorted(a.elapsed_time(c) for a, c in kev)
    kernel_ms = sum(kernel_each) / KE

    def pct(q):  # nearest-rank percentile of the per-launch times
        return kernel_each[min(KE - 1, int(q * KE))]
    ms = max_over_ranks(ms, dist, dev)

    # end to end through the public API from host memory: ssd_fwd_host takes the
    # pinned host inputs, copies them in by row pieces on two streams, runs the
    # forward on each piece and copies y and the final states back, one piece's
    # copies in overlapping the previous piece's compute and copies out
    names = [k for k in ("x", "dt", "A", "B", "C", "D", "initial_states", "seq_idx", "z") if host.get(k) is not None]
    pinned = {k: host[k].pin_memory() for k in names}
    y_host = torch.empty(y.shape, dtype=y.dtype).pin_memory()
    f_host = torch.empty(final.shape, dtype=final.dtype).pin_memory()
    h2d = sum(pinned[k].numel() * pinned[k].element_size() for k in names)
    d2h = y_host.numel() * y_host.element_size() + f_host.numel() * f_host.element_size()
    gen_flag = ssd.SSD_FLAG_GENERIC if args.generic else 0
    hws = torch.empty(max(1, ssd.fwd_host_workspace_size(
        host["x"], host["B"], shape.chunk_size, 0, host.get("seq_idx"), num_seqs, True, host.get("D") is not None,
        host.get("z") is not None, host.get("initial_states") is not None, gen_flag)), dtype=torch.uint8, device=dev)
    stream2 = torch.cuda.Stream(dev)

    def e2e_step():
        ssd.fwd_host(pinned["x"], pinned["dt"], pinned["A"], pinned["B"], pinned["C"], pinned.get("D"),
                     shape.chunk_size, pinned.get("initial_states"), pinned.get("seq_idx"), num_seqs,
                     y=y_host, final_states=f_host, workspace=hws, device=dev, stream2=stream2, flags=gen_flag,
                     z=pinned.get("z"))

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    E = max(3, min(K, 50))
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a0.record()
    for _ in range(E):
        e2e_step()
    a1.record()
    torch.cuda.synchronize()
    e2e_ms = a0.elapsed_time(a1)
    e2e_ms = max_over_ranks(e2e_ms, dist, dev)
    if dist:
        dist.barrier()

    w = work(shape, num_seqs)
    if args.gated and main_kernel != "k_ssd_fwd_pair":  # the single-head kernel reads z in its epilogue
        w["bytes"] += host["z"].numel() * host["z"].element_size()
    peaks = load_peaks()
    ms_step = ms / K
    tokens_job = shape.tokens * world
    value = tokens_job / (ms_step / 1e3)
    t_hbm = w["bytes"] / (peaks["hbm_gbs"] * 1e9)
    t_tc = w["flops"] / (peaks["bf16_tflops"] * 1e12)
    if t_hbm >= t_tc:
        achieved = w["bytes"] / (kernel_ms / 1e3) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"], "peak_source": peaks["source"]}
    else:
        achieved = w["flops"] / (kernel_ms / 1e3) / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": achieved / peaks["bf16_tflops"], "peak_source": peaks["source"]}
    kfile = {"k_ssd_fwd_pair": "ssd_tc_pair.cu", "k_ssd_fwd_fast": "ssd_tc_fast.cu"}.get(main_kernel,
                                                                                      "ssd_generic.cu")
    roof["kernel"] = main_kernel if path == "tcgen05" else "generic (all kernels of the call)"
    roof["kernel_ms"] = kernel_ms
    roof["kernel_ms_p10_p50_p90"] = [pct(0.1), pct(0.5), pct(0.9)]
    # the same achieved figure against the datasheet peaks (8 TB/s HBM3e, 2.25 PFLOP/s dense bf16)
    roof["frac_datasheet"] = achieved / (DATASHEET_HBM_GBS if roof["bound"] == "hbm" else DATASHEET_BF16_TFLOPS)
    roof["traffic"] = traffic_from_profiles(kfile, main_kernel, shape.name)
    roof["algorithmic_bytes"] = w["bytes"]
    roof["algorithmic_flops"] = w["flops"]

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16" if shape.dtype == "bf16" else "f32", "data": "synthetic",
        "config": {"workload": describe(shape) + ((", gated: y * SiLU(z), z ~ N(0,1)" + (
                       "; the gate in k_gate_silu after the two-head kernel (the roofline is the two-head"
                       " kernel's)" if main_kernel == "k_ssd_fwd_pair" else "; the gate in the fused epilogue"))
                   if args.gated else ""),
                   "batch": b, "seqlen": L, "nheads": H, "headdim": P,
                   "dstate": N, "ngroups": shape.ngroups, "chunk_size": shape.chunk_size,
                   "l2": f"no flush: inputs+outputs {w['bytes'] / 1e6:.0f} MB per step > 126 MB L2",
                   "parallelism": "replicas" if world > 1 else "single GPU"},
        "tflops": {"full": w["flops"] * world / (ms_step / 1e3) / 1e12,
                   "causal": w["flops_causal"] * world / (ms_step / 1e3) / 1e12},
        "kernel_path": path,
        "roofline": roof,
        "e2e": {"value": tokens_job / (e2e_ms / E / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": E},
        "gpu_launches": launches_per_call * K,
        "clocks": clock_stats,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, U, el, cores = oracle_sample(host, shape, args.cpu_seconds)
        line["cpu_baseline"] = {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                                "sample": f"first {U} of {b * H} (batch, head) units of the workload, "
                                          f"{U * L / H:.1f} tokens, {el:.1f} s"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
