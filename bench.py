#!/usr/bin/env python
"""Benchmark of the Lattice compression-layer state recurrence on B200.

A step is one lattice_scan_fwd over one batch of the long-context workload
(B=1, H=16, T=65536, m=64, d=128, chunk 64, bf16 x/q, fp32 state carried over
1024 chunks): the whole hot path (projection, orthogonal write, forget gate,
unit-sphere projection, read-out, chunk state carry). It is the largest of the
single-GPU workloads (1.05 M token-heads, 1.2 GB of algorithmic traffic).
Inputs are resident in HBM before the timed region; they exceed the L2, which is
also flushed (a 256 MiB write) between timed steps. Each step is timed with CUDA
events on the launching stream.

The same JSON line also reports, under "extra", the small training shape and the
mid-size layer (each with its own roofline record), the exact recurrence, the
chunk-form variants, the backward pass and the decode step (1000 consecutive
steps of B=256, H=32, m=d=128).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun (N > 1) every rank runs its own batch (weak scaling, no
data-path collective); the reported time is the max over ranks.
"""
from __future__ import annotations

import argparse
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

import numpy as np

import lattice_inputs as LI

METRIC = "Lattice layer fwd tokens/s (1 B200) + % of roofline; decode step GB/s"
HEADLINE = "long_ctx"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20


# ---------------------------------------------------------------- arithmetic

def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def scan_alg_bytes(w: LI.Workload, B=None, T=None, H=None) -> int:
    """Algorithmic HBM bytes of one scan: every input read once, y and S written once."""
    B = w.B if B is None else B
    T = w.T if T is None else T
    H = w.H if H is None else H
    xb = 2 if w.x_dtype == "bf16" else 4
    qb = 2 if w.q_dtype == "bf16" else 4
    per_tok = w.d * xb + w.m * qb + 4 * w.m + 4 + 4 * w.d
    return B * T * H * per_tok + 2 * 4 * B * H * w.m * w.d


def bwd_alg_bytes(w: LI.Workload) -> int:
    """Algorithmic HBM bytes of one backward pass: the forward's inputs, dy and S0/dS_T
    read once, dx, dc, dq, dmu and dS0 written once (the workspace is scratch)."""
    xb = 2 if w.x_dtype == "bf16" else 4
    qb = 2 if w.q_dtype == "bf16" else 4
    per_tok = (w.d * xb + w.m * qb + 4 * w.m + 4 + 4 * w.d) + (4 * w.d + 8 * w.m + 4)
    return w.B * w.T * w.H * per_tok + 3 * 4 * w.B * w.H * w.m * w.d


def chunk_mma_flops(w: LI.Workload, C: int, B=None, T=None, H=None) -> int:
    """Tensor-core flops of the chunked form per token and head: 6md + C(m+d)
    (projection, inter-chunk read-out and state update: 2md each; causal score
    and intra-chunk read-out: C*m and C*d with the causal half counted once)."""
    B = w.B if B is None else B
    T = w.T if T is None else T
    H = w.H if H is None else H
    return B * T * H * (6 * w.m * w.d + C * (w.m + w.d))


def step_alg_bytes(w: LI.Workload, B=None, H=None) -> int:
    B = w.B if B is None else B
    H = w.H if H is None else H
    xb = 2 if w.x_dtype == "bf16" else 4
    qb = 2 if w.q_dtype == "bf16" else 4
    return B * H * (2 * 4 * w.m * w.d + w.d * xb + w.m * qb + 4 * w.m + 4 + 4 * w.d)


# ------------------------------------------------------------ multi-rank host

def rank_workload(w: LI.Workload, rank: int) -> LI.Workload:
    """Each rank scans its own batch: the same shapes and distributions, its own seed."""
    return w if rank == 0 else w.with_(seed=w.seed + 1000 * rank)


def max_over_ranks(torch, dist, value: float, device) -> float:
    """The slowest rank's time (every rank calls this, in the same order)."""
    if dist is None:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(world: int, w: LI.Workload, ms_per_step: float) -> float:
    """Whole-job throughput: every rank's B*T tokens in the slowest rank's step time."""
    return world * w.B * w.T / (ms_per_step * 1e-3)


def scan_config(w: LI.Workload, world: int) -> dict:
    """The `config` record of a scan line (both arms print the same one)."""
    big = scan_alg_bytes(w) > 2 * (126 << 20)
    return {"workload": w.name, "B": w.B, "H": w.H, "T": w.T, "m": w.m, "d": w.d, "chunk": w.chunk,
            "x_q_dtype": w.x_dtype, "state_dtype": "f32",
            "l2": ("inputs exceed the L2; also flushed between timed steps (256 MiB write)" if big
                   else "flushed between timed steps (256 MiB write)"),
            "parallelism": f"independent batches per GPU x{world}"}


# DRAM bytes (read + write) per launch from one ncu capture of each kernel on each
# workload. Each entry names the profile summary that holds the capture's command and
# figures, and the SHA-256 (first 12 hex digits) of the kernel's source file at the
# time of the capture: traffic_for() reports None once that file has changed, since
# the counters then describe a kernel that no longer exists.
CAPTURED_TRAFFIC = {
    ("chunk_split_kernel", "small_train"): dict(bytes=34.56e6, profile="profiles/chunk_split_kernel_full.md",
                                                source="csrc/chunk_split.cuh", sha="047d8e41962f"),
    ("chunk_split_kernel", "long_ctx"): dict(bytes=676.05e6 + 498.46e6, profile="profiles/chunk_split_kernel_full.md",
                                             source="csrc/chunk_split.cuh", sha="047d8e41962f"),
    ("chunk_tc_kernel", "mid_layer"): dict(bytes=550.70e6 + 237.14e6, profile="profiles/chunk_tc_kernel_full.md",
                                           source="csrc/chunk_tc.cuh", sha="488f569268b7"),
    ("scan_simt_kernel<exact>", "small_train"): dict(bytes=34.43e6 + 0.00e6,
                                                     profile="profiles/scan_simt_kernel_exact_small_train.md",
                                                     source="csrc/scan_simt.cuh", sha="9b2b98fd3aeb"),
    ("scan_bwd_kernel<chunked>", "small_train"): dict(bytes=71.41e6 + 54.81e6,
                                                      profile="profiles/scan_bwd_kernel_small_train.md",
                                                      source="csrc/scan_bwd.cuh", sha="3fa6eb987d11"),
    # the chunk-parallel backward, full-size launches, dram counters alone (one pass);
    # chunk_bwd.cuh changed since only in its header comment (captured on 3fb59cd3d40e)
    ("chunk_bwd_kernel", "small_train"): dict(bytes=62.00e6 + 26.59e6,
                                              profile="profiles/chunk_bwd_kernel_small_train.md",
                                              source="csrc/chunk_bwd.cuh", sha="d2425c5dc1fa"),
    ("chunk_bwd_kernel", "mid_layer"): dict(bytes=1.41e9 + 1.32e9,
                                            profile="profiles/chunk_bwd_kernel_small_train.md",
                                            source="csrc/chunk_bwd.cuh", sha="d2425c5dc1fa"),
    # full-size launches, dram counters alone (one pass); chunk_reg.cuh changed since only
    # in its header comment (captured on 4a519db1dbb5)
    ("chunk_reg_kernel<16 slots>", "long_ctx"): dict(bytes=676.59e6 + 501.80e6,
                                                    profile="profiles/chunk_reg_kernel_long_ctx.md",
                                                    source="csrc/chunk_reg.cuh", sha="d87ccc814da7"),
    ("chunk_reg_kernel<16 slots>", "small_train"): dict(bytes=34.40e6 + 0.07e6,
                                                       profile="profiles/chunk_reg_kernel_small_train.md",
                                                       source="csrc/chunk_reg.cuh", sha="d87ccc814da7"),
    # the persistent decode step, both objectives
    ("step_pf_kernel", "decode"): dict(bytes=545.33e6 + 480.69e6, profile="profiles/step_kernel_decode.md",
                                       source="csrc/step.cuh", sha="71553fca01a5"),
    ("step_pf_kernel<dec>", "decode"): dict(bytes=545.34e6 + 480.52e6, profile="profiles/step_kernel_decode.md",
                                            source="csrc/step.cuh", sha="71553fca01a5"),
}


def step_kernel_name(mode: str) -> str:
    """The decode-step kernel the library launches on the decode workload (8192 heads,
    more than the SMs: the persistent kernel, for either objective)."""
    return "step_pf_kernel" if mode == "sim" else "step_pf_kernel<dec>"


def source_sha(rel: str) -> str:
    import hashlib
    p = os.path.join(ROOT, "orthogonal_update_recurrent_b200", rel)
    with open(p, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:12]


def traffic_for(kernel: str, workload: str):
    """Captured DRAM bytes per launch of `kernel` on `workload`, or None when there is
    no capture or the kernel's source changed since it was taken."""
    e = CAPTURED_TRAFFIC.get((kernel, workload))
    if e is None or e["sha"] is None or source_sha(e["source"]) != e["sha"]:
        return None
    return e["bytes"]


# -------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during a timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def __enter__(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        if self.proc is None or not self.path or not os.path.exists(self.path):
            return None
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    rows.append((float(parts[1]), float(parts[2]), parts[5:9]))
                except ValueError:
                    continue
        os.unlink(self.path)
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, r in rows for i, v in enumerate(r) if v.lower() == "active"})
        top = max(r[0] for r in rows)
        loaded = [r[0] for r in rows if r[0] >= 0.5 * top] or [r[0] for r in rows]
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": rows[0][1], "reasons": reasons,
                "samples": len(rows)}


# --------------------------------------------------------------- GPU timing

def _dev_inputs(torch, inp, device):
    def vec(n):
        b = inp.get(n + "_bits")
        if b is not None:
            return torch.from_numpy(b.view(np.int16)).view(torch.bfloat16).to(device)
        return torch.from_numpy(np.ascontiguousarray(inp[n], np.float32)).to(device)
    return dict(x=vec("x"), q=vec("q"), c=torch.from_numpy(inp["c"]).to(device),
                mu=torch.from_numpy(inp["mu"]).to(device), S0=torch.from_numpy(inp["S0"]).to(device))


def time_scan(torch, L, t, chunk, steps, warmup, flush=None, impl="auto", mode="sim", lin=2, norm="token"):
    """Per-step device time (ms) of lattice_scan_fwd, CUDA events on its stream."""
    stream = torch.cuda.current_stream()
    y = torch.empty(t["x"].shape[:3] + (t["S0"].shape[-1],), dtype=torch.float32, device=t["x"].device)
    S = torch.empty_like(t["S0"])
    run = lambda: L.scan_fwd(t["x"], t["c"], t["q"], t["mu"], t["S0"], chunk=chunk, S_out=S, y=y,
                             impl=impl, stream=stream, mode=mode, lin=lin, norm=norm)
    for _ in range(warmup):
        run()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    for e0, e1 in ev:
        if flush is not None:
            flush.add_(1)
        e0.record(stream)
        run()
        e1.record(stream)
    torch.cuda.synchronize()
    L.device_status()
    return [e0.elapsed_time(e1) for e0, e1 in ev]


def time_bwd(torch, L, t, chunk, steps, warmup, flush=None):
    """Per-step device time (ms) of lattice_scan_bwd (unit cotangents), CUDA events
    on its stream; the workspace is allocated once, outside the timed region."""
    stream = torch.cuda.current_stream()
    B, T, H, d = t["x"].shape
    m = t["c"].shape[-1]
    dy = torch.ones((B, T, H, d), dtype=torch.float32, device=t["x"].device)
    ws = torch.empty(max(L.scan_bwd_workspace_bytes(B, T, H, m, d, chunk), 16), dtype=torch.uint8,
                     device=t["x"].device)
    run = lambda: L.scan_bwd(t["x"], t["c"], t["q"], t["mu"], t["S0"], dy, chunk=chunk,
                             workspace=ws, stream=stream)
    for _ in range(warmup):
        run()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    for e0, e1 in ev:
        if flush is not None:
            flush.add_(1)
        e0.record(stream)
        run()
        e1.record(stream)
    torch.cuda.synchronize()
    L.device_status()
    return [e0.elapsed_time(e1) for e0, e1 in ev]


def time_scan_e2e(torch, L, inp, chunk, steps, warmup, device):
    """End to end through the public call with host buffers, as a streaming user runs
    it: each step copies its inputs in from pinned host memory, runs the scan and
    copies y and the final state back. Steps are pipelined over three streams (copy
    in, compute, copy out) with two device buffer sets, so step k+1's upload and
    step k-1's download overlap step k's scan. Returns (ms per step, bytes in, bytes out)."""
    host = {}
    for n in ("x", "q"):
        b = inp.get(n + "_bits")
        host[n] = (torch.from_numpy(b.view(np.int16)).view(torch.bfloat16) if b is not None
                   else torch.from_numpy(inp[n])).pin_memory()
    for n in ("c", "mu", "S0"):
        host[n] = torch.from_numpy(inp[n]).pin_memory()
    B, T, H, d = host["x"].shape
    dev = [{k: torch.empty_like(v, device=device) for k, v in host.items()} for _ in range(2)]
    ys = [torch.empty((B, T, H, d), dtype=torch.float32, device=device) for _ in range(2)]
    Ss = [torch.empty_like(dev[0]["S0"]) for _ in range(2)]
    y_h = [torch.empty((B, T, H, d), dtype=torch.float32).pin_memory() for _ in range(2)]
    S_h = [torch.empty(Ss[0].shape, dtype=torch.float32).pin_memory() for _ in range(2)]
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = y_h[0].numel() * 4 + S_h[0].numel() * 4
    s_in, s_run, s_out = (torch.cuda.Stream(device=device) for _ in range(3))
    ev = lambda: torch.cuda.Event()
    done_in = [ev(), ev()]     # inputs of buffer set k%2 uploaded
    done_run = [ev(), ev()]    # scan of buffer set k%2 finished (inputs free, outputs ready)
    done_out = [ev(), ev()]    # outputs of buffer set k%2 downloaded (output buffers free)
    for e in done_run + done_out:
        e.record(torch.cuda.current_stream())

    def step(k):
        i = k & 1
        with torch.cuda.stream(s_in):
            s_in.wait_event(done_run[i])
            for key in host:
                dev[i][key].copy_(host[key], non_blocking=True)
            done_in[i].record(s_in)
        with torch.cuda.stream(s_run):
            s_run.wait_event(done_in[i])
            s_run.wait_event(done_out[i])
            L.scan_fwd(dev[i]["x"], dev[i]["c"], dev[i]["q"], dev[i]["mu"], dev[i]["S0"], chunk=chunk,
                       S_out=Ss[i], y=ys[i], stream=s_run)
            done_run[i].record(s_run)
        with torch.cuda.stream(s_out):
            s_out.wait_event(done_run[i])
            y_h[i].copy_(ys[i], non_blocking=True)
            S_h[i].copy_(Ss[i], non_blocking=True)
            done_out[i].record(s_out)

    for k in range(warmup):
        step(k)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for k in range(steps):
        step(k)
    s_in.wait_stream(s_out)
    e1.record(s_in)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / steps, h2d, d2h


def time_decode(torch, L, w, n_steps, ring, device, mode="sim"):
    """n_steps consecutive decode steps replayed from a CUDA graph over a ring of
    pre-drawn per-step inputs (the ring and the 512 MiB state exceed L2)."""
    S = torch.from_numpy(LI.make_decode_state(w)).to(device)
    st = LI.make_decode_steps(w, ring)
    xs = torch.from_numpy(st["x_bits"].view(np.int16)).view(torch.bfloat16).to(device)
    qs = torch.from_numpy(st["q_bits"].view(np.int16)).view(torch.bfloat16).to(device)
    cs = torch.from_numpy(st["c"]).to(device)
    mus = torch.from_numpy(st["mu"]).to(device)
    y = torch.empty((w.B, w.H, w.d), dtype=torch.float32, device=device)
    s = torch.cuda.Stream(device=device)
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for k in range(3):  # warm-up
            L.step(S, xs[k], cs[k], qs[k], mus[k], y=y, stream=s, mode=mode)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            for k in range(ring):
                L.step(S, xs[k], cs[k], qs[k], mus[k], y=y, stream=s, mode=mode)
    torch.cuda.synchronize()
    reps = max(1, n_steps // ring)
    with torch.cuda.stream(s):
        g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s)
        for _ in range(reps):
            g.replay()
        e1.record(s)
    torch.cuda.synchronize()
    L.device_status()
    del g
    return e0.elapsed_time(e1) / (reps * ring), reps * ring


# ---------------------------------------------------------------- CPU oracle

def oracle_sample_tokens(w: LI.Workload) -> int:
    """Tokens per sequence of one bounded oracle sample: the whole sequence for the
    shorter workloads, the first 8192 tokens (128 chunks) of every head for longer
    ones. The oracle's cost per token is the same all along a sequence, so tokens/s
    over the sample is the workload's rate."""
    return min(w.T, 8192)


def oracle_baseline(w: LI.Workload, chunk: int, min_seconds: float = 12.0, max_reps: int = 10000):
    """The fp64 oracle, as it stands, on the host cores: passes over a bounded sample of
    the workload (every sequence, oracle_sample_tokens tokens each) repeated until about
    min_seconds of CPU work. Returns (tokens/s, cores, sample)."""
    import oracle
    Ts = oracle_sample_tokens(w)
    inp = LI.make_inputs(w, T=Ts)
    cores = len(os.sched_getaffinity(0))
    t0 = time.perf_counter()
    reps = 0
    while True:
        oracle.scan(inp["x"], inp["c"], inp["q"], inp["mu"], inp["S0"], chunk=chunk, nthreads=cores)
        reps += 1
        el = time.perf_counter() - t0
        if el >= min_seconds or reps >= max_reps:
            break
    tok = w.B * Ts * reps
    what = "full pass(es)" if Ts == w.T else f"pass(es) over the first {Ts} of {w.T} tokens"
    sample = (f"{reps} {what} of {w.name} (B={w.B},H={w.H},T={w.T},m={w.m},d={w.d}), "
              f"{'exact' if chunk == 1 else f'chunked C={chunk}'}, fp64 oracle, {el:.1f} s")
    return tok / el, cores, sample


def oracle_legs(w: LI.Workload, seconds: float = 3.0) -> dict:
    """Further oracle timings on the host: the exact recurrence on all cores and the
    chunked form on one thread (each over the bounded sample, the one-thread leg over
    its first 1024 tokens), and decode steps of the decode workload (3 steps of the full
    512 MiB state, per step)."""
    import oracle
    cores = len(os.sched_getaffinity(0))

    def rate(chunk, threads, T):
        inp = LI.make_inputs(w, T=T)
        t0, reps = time.perf_counter(), 0
        while True:
            oracle.scan(inp["x"], inp["c"], inp["q"], inp["mu"], inp["S0"], chunk=chunk, nthreads=threads)
            reps += 1
            el = time.perf_counter() - t0
            if el >= seconds:
                return w.B * T * reps / el
    Ts = oracle_sample_tokens(w)
    out = {"exact_tokens_per_s": rate(1, cores, Ts),
           "chunked_tokens_per_s_1_thread": rate(w.chunk, 1, min(Ts, 1024))}
    wd = LI.WORKLOADS["decode"]
    S = LI.make_decode_state(wd).astype(np.float64)
    st = LI.make_decode_steps(wd, 3)
    t0 = time.perf_counter()
    for k in range(3):
        _, S, _ = oracle.step(S, st["x"][k], st["c"][k], st["q"][k], st["mu"][k], nthreads=cores)
    out["decode_us_per_step"] = 1e6 * (time.perf_counter() - t0) / 3
    out["decode_sample"] = f"3 steps of B={wd.B} H={wd.H} m={wd.m} d={wd.d}, fp64 oracle, {cores} threads"
    return out


# ---------------------------------------------------------------------- main

def kernel_name(L, w: LI.Workload, chunk: int, impl: str = "auto") -> str:
    """The kernel lattice_scan_fwd runs for this workload (the automatic choice by default)."""
    kimpl = L.chunk_impl(w.B, w.H, w.m, w.d, chunk) if impl == "auto" else impl
    return {"tcgen05": "chunk_tc_kernel", "tcgen05_split": "chunk_split_kernel",
            "split_reg": "chunk_reg_kernel<16 slots>", "split_reg8": "chunk_reg_kernel<8 slots>"}.get(
        kimpl, "scan_simt_kernel<chunked>" if chunk > 1 else "scan_simt_kernel<exact>")


def scan_roofline(L, w: LI.Workload, traffic_key: str, kern_ms: float, pk: dict, pk_src: str,
                  impl: str = "auto") -> dict:
    """Roofline record of one scan launch of `w` that took kern_ms (CUDA events):
    algorithmic HBM bytes / time against the measured copy bandwidth, and for the
    tensor-core kernels the algorithmic MMA flops / time against the bf16 peak."""
    kname = kernel_name(L, w, w.chunk, impl)
    alg_b = scan_alg_bytes(w)
    achieved = alg_b / (kern_ms * 1e-3) / 1e9
    roof = {"bound": "hbm", "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s",
            "frac": achieved / pk["hbm_gbs"], "traffic": traffic_for(kname, traffic_key),
            "kernel": kname, "ms_per_launch": kern_ms,
            "alg_bytes_per_launch": alg_b, "peak_source": f"{pk_src} (burst copy)"}
    t_roof_ms = 1e3 * alg_b / (pk["hbm_gbs"] * 1e9)
    if kname.startswith("chunk_"):
        fl = chunk_mma_flops(w, w.chunk)
        roof["tensor"] = {"achieved_tflops": fl / (kern_ms * 1e-3) / 1e12,
                          "peak_tflops": pk["bf16_tflops"],
                          "frac": fl / (kern_ms * 1e-3) / 1e12 / pk["bf16_tflops"],
                          "flops_per_launch": fl}
        t_roof_ms = max(t_roof_ms, 1e3 * fl / (pk["bf16_tflops"] * 1e12))
    roof["frac_of_binding_roofline"] = t_roof_ms / kern_ms
    return roof


def bench_step(args, torch, L, dist, world, rank, local, device, pk, pk_src):
    """--pass step: one step is one decode token for every (b,h) of the decode workload
    (lattice_step, state updated in place), steps replayed from a CUDA graph."""
    wd = rank_workload(LI.WORKLOADS["decode"], rank)
    ring = 40
    n = max(ring, (args.steps // ring) * ring)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        step_ms, n = time_decode(torch, L, wd, n, ring, device, mode=args.mode)
    torch.cuda.synchronize()
    step_ms = max_over_ranks(torch, dist, step_ms, device)
    if rank != 0:
        return 0
    sb = step_alg_bytes(wd)
    gbps = sb / (step_ms * 1e-3) / 1e9
    line = {"metric": "Lattice decode step GB/s (1 B200)", "value": gbps * world, "unit": "GB/s",
            "n_gpus": world, "steps": n, "warmup": 3, "ms_per_step": step_ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": wd.name, "pass": "step", "B": wd.B, "H": wd.H, "m": wd.m, "d": wd.d,
                       "objective": args.mode, "x_q_dtype": "bf16", "state_dtype": "f32",
                       "l2": "state (512 MiB) and input ring exceed L2",
                       "parallelism": f"independent batches per GPU x{world}"},
            "roofline": {"bound": "hbm", "achieved": gbps, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": gbps / pk["hbm_gbs"],
                         "traffic": traffic_for(step_kernel_name(args.mode), "decode"),
                         "kernel": step_kernel_name(args.mode),
                         "alg_bytes_per_launch": sb, "peak_source": f"{pk_src} (burst copy)"},
            "gpu_launches": n}
    cs = clk.summary()
    if cs is not None:
        line["clocks"] = cs
    print(json.dumps(line), flush=True)
    return 0


def bwd_kernel_name(chunk: int, d: int) -> str:
    """The kernel lattice_scan_bwd runs (16-byte-aligned buffers): the chunk-parallel
    kernel for chunks of 2..64 tokens at d >= 32, else the token-by-token kernel."""
    if 2 <= chunk <= 64 and d in (32, 64, 128):
        return "chunk_bwd_kernel"
    return "scan_bwd_kernel<chunked>" if chunk > 1 else "scan_bwd_kernel<exact>"


def bench_bwd(args, torch, L, dist, t, w, w0, world, rank, local, device, flush, pk, pk_src):
    """--pass bwd: one step is one lattice_scan_bwd of the workload (gradients of every
    input for unit dy), workspace allocated once outside the timed region."""
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        times = time_bwd(torch, L, t, w.chunk, args.steps, args.warmup, flush=flush)
    torch.cuda.synchronize()
    total_ms = max_over_ranks(torch, dist, sum(times), device)
    if dist is not None:
        dist.barrier()
    if rank != 0:
        return 0
    ms = total_ms / args.steps
    alg_b = bwd_alg_bytes(w)
    kern_ms = statistics.mean(times)
    achieved = alg_b / (kern_ms * 1e-3) / 1e9
    kname = bwd_kernel_name(w.chunk, w.d)
    line = {"metric": "Lattice layer bwd tokens/s (1 B200)", "value": job_tokens_per_s(world, w, ms),
            "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f32", "data": "synthetic",
            "config": {"workload": w.name, "pass": "bwd", "B": w.B, "H": w.H, "T": w.T, "m": w.m,
                       "d": w.d, "chunk": w.chunk, "x_q_dtype": "bf16",
                       "l2": "flushed between timed steps (256 MiB write)",
                       "parallelism": f"independent batches per GPU x{world}"},
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": achieved / pk["hbm_gbs"], "traffic": traffic_for(kname, w0.name),
                         "kernel": kname,
                         "alg_bytes_per_launch": alg_b, "peak_source": f"{pk_src} (burst copy)"},
            "gpu_launches": args.steps}
    cs = clk.summary()
    if cs is not None:
        line["clocks"] = cs
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-extra", action="store_true", help="skip the context workloads")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end timing")
    ap.add_argument("--workload", default=HEADLINE, choices=["small_train", "mid_layer", "long_ctx"],
                    help="chunked workload of the timed step (default: the long-context workload)")
    ap.add_argument("--pass", dest="which", default="fwd", choices=["fwd", "bwd", "step"],
                    help="bwd: time the backward pass (lattice_scan_bwd) of the workload instead; "
                         "step: time the decode step (lattice_step) on the decode workload")
    ap.add_argument("--kernel", default="auto", choices=["auto", "simt", "tcgen05", "tcgen05_split", "split_reg", "split_reg8"],
                    help="kernel choice of the timed scan (default: the library's automatic choice)")
    ap.add_argument("--tokens", type=int, default=None,
                    help="override the workload's sequence length T (for profiling a smaller case)")
    ap.add_argument("--mode", default="sim", choices=["sim", "dec"],
                    help="objective of the --pass step timing: similarity (default) or reconstruction")
    ap.add_argument("--chunk", type=int, default=None,
                    help="override the workload's chunk size (1: the exact recurrence)")
    args = ap.parse_args()
    assert args.warmup >= 3, "at least 3 warm-up steps"

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    w0 = LI.WORKLOADS[args.workload]
    if args.chunk is not None:
        w0 = w0.with_(chunk=args.chunk)
    if args.tokens is not None:
        w0 = w0.with_(T=args.tokens)
    w = rank_workload(w0, rank)

    if args.impl == "reference":
        if rank != 0:
            return 0
        steps = max(1, args.steps)
        import oracle
        Ts = oracle_sample_tokens(w)
        inp = LI.make_inputs(w, T=Ts)
        cores = len(os.sched_getaffinity(0))
        for _ in range(args.warmup):  # untimed passes
            oracle.scan(inp["x"], inp["c"], inp["q"], inp["mu"], inp["S0"], chunk=w.chunk, nthreads=cores)
        t0 = time.perf_counter()
        for _ in range(steps):
            oracle.scan(inp["x"], inp["c"], inp["q"], inp["mu"], inp["S0"], chunk=w.chunk, nthreads=cores)
        el = time.perf_counter() - t0
        v = w.B * Ts * steps / el
        what = "one full pass" if Ts == w.T else f"one pass over the first {Ts} of {w.T} tokens of every sequence"
        line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": args.gpus,
                "steps": steps, "warmup": args.warmup, "ms_per_step": 1e3 * el / steps,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic", "config": scan_config(w, args.gpus),
                "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                                 "sample": f"{what} of {w.name} per step, "
                                           f"{'exact' if w.chunk == 1 else f'chunked C={w.chunk}'}, "
                                           f"fp64 C oracle on {cores} threads"},
                "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return 0

    import torch
    import orthogonal_update_recurrent_b200 as L
    from orthogonal_update_recurrent_b200 import build as Bld
    if rank == 0 or not os.path.exists(Bld.LIB):
        Bld.build()
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    L.lib()

    pk, pk_src = peaks()
    inp = LI.make_inputs(w)
    t = _dev_inputs(torch, inp, device)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=device)

    if args.which == "bwd":
        return bench_bwd(args, torch, L, dist, t, w, w0, world, rank, local, device, flush, pk, pk_src)
    if args.which == "step":
        return bench_step(args, torch, L, dist, world, rank, local, device, pk, pk_src)

    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        times = time_scan(torch, L, t, w.chunk, args.steps, args.warmup, flush=flush, impl=args.kernel)
    torch.cuda.synchronize()
    total_ms = max_over_ranks(torch, dist, sum(times), device)
    if dist is not None:
        dist.barrier()
    ms = total_ms / args.steps
    value = job_tokens_per_s(world, w, ms)

    # roofline of the (single) kernel of the step
    roof = scan_roofline(L, w, w0.name, statistics.mean(times), pk, pk_src, impl=args.kernel)
    tc = "tensor" in roof

    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16" if tc else "f32", "data": "synthetic",
            "config": scan_config(w, world), "roofline": roof, "gpu_launches": args.steps}
    cs = clk.summary()
    if cs is not None:
        line["clocks"] = cs

    # end to end through the public call with host buffers (every rank; the slowest counts)
    if not args.no_e2e:
        e2e_ms, h2d, d2h = time_scan_e2e(torch, L, inp, w.chunk, max(8, args.steps), 3, device)
        e2e_ms = max_over_ranks(torch, dist, e2e_ms, device)
    if rank == 0:
        if not args.no_e2e:
            line["e2e"] = {"value": job_tokens_per_s(world, w, e2e_ms), "unit": "tokens/s",
                           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                           "pipelined": "copy-in / scan / copy-out on three streams, two buffer sets"}
        extra = {}
        if not args.no_extra:
            # the exact recurrence on the timed workload
            te = time_scan(torch, L, t, 1, 3, 3, flush=flush)
            extra[f"{w.name}_exact"] = {"ms": statistics.mean(te), "kernel": kernel_name(L, w, 1),
                                        "tokens_per_s": w.B * w.T / (statistics.mean(te) * 1e-3)}
            if w.m == 64 and w.chunk == 64:  # the earlier cluster kernel, for comparison
                extra[f"{w.name}_tcgen05_split_ms"] = statistics.mean(
                    time_scan(torch, L, t, w.chunk, 5, 3, flush=flush, impl="tcgen05_split"))
            # the backward pass on the timed workload
            tbw = statistics.mean(time_bwd(torch, L, t, w.chunk, 3, 2, flush=flush))
            extra[f"{w.name}_bwd"] = {"ms": tbw, "tokens_per_s": w.B * w.T / (tbw * 1e-3),
                                      "kernel": bwd_kernel_name(w.chunk, w.d)}
            del t
            torch.cuda.empty_cache()
            # the other chunked workloads, each with its own roofline record
            for name in [n for n in ("small_train", "mid_layer", "long_ctx") if n != w.name]:
                wn = LI.WORKLOADS[name]
                inn = LI.make_inputs(wn)
                tn = _dev_inputs(torch, inn, device)
                del inn
                tch = time_scan(torch, L, tn, wn.chunk, 10, 3, flush=flush)
                kms = statistics.mean(tch)
                ent = {"ms": kms, "tokens_per_s": wn.B * wn.T / (kms * 1e-3),
                       "roofline": scan_roofline(L, wn, name, kms, pk, pk_src)}
                if wn.m == 64:  # the earlier cluster kernel, for comparison
                    ent["tcgen05_split_ms"] = statistics.mean(
                        time_scan(torch, L, tn, wn.chunk, 5, 3, flush=flush, impl="tcgen05_split"))
                tex = time_scan(torch, L, tn, 1, 3, 3, flush=flush)
                ent["exact_ms"] = statistics.mean(tex)
                ent["exact_tokens_per_s"] = wn.B * wn.T / (ent["exact_ms"] * 1e-3)
                if name == "mid_layer":   # the backward pass (small_train's is timed below)
                    ent["bwd_ms"] = statistics.mean(time_bwd(torch, L, tn, wn.chunk, 3, 2, flush=flush))
                    ent["bwd_kernel"] = bwd_kernel_name(wn.chunk, wn.d)
                extra[name] = ent
                del tn
                torch.cuda.empty_cache()
            # chunk-form variants and the backward pass on the small training shape
            ws = LI.WORKLOADS["small_train"]
            ts = _dev_inputs(torch, LI.make_inputs(ws), device)
            tok = lambda ms: ws.B * ws.T / (ms * 1e-3)
            # the reconstruction objective (CUDA-core kernels), exact and chunked; the
            # chunked form takes intensities sigmoid(N(-4,1)), with which it stays bounded
            td = statistics.mean(time_scan(torch, L, ts, 1, 5, 3, flush=flush, mode="dec"))
            extra["small_train_dec_exact"] = {"ms": td, "tokens_per_s": tok(td),
                                              "kernel": "scan_simt_kernel<exact, dec>"}
            tdc = _dev_inputs(torch, LI.make_inputs(ws.with_(c_loc=-4.0)), device)
            td = statistics.mean(time_scan(torch, L, tdc, ws.chunk, 5, 3, flush=flush, mode="dec"))
            extra["small_train_dec_chunked"] = {"ms": td, "tokens_per_s": tok(td),
                                                "kernel": "scan_simt_kernel<chunked, dec>",
                                                "inputs": "c = sigmoid(N(-4,1))"}
            del tdc
            # chunk 16, the throughput figure's other chunk size: the register-chain kernel
            # (four chunks per 64-token stage) and the CUDA-core kernel
            t16 = statistics.mean(time_scan(torch, L, ts, 16, 5, 3, flush=flush))
            t16s = statistics.mean(time_scan(torch, L, ts, 16, 5, 3, flush=flush, impl="simt"))
            extra["small_train_chunk16"] = {"ms": t16, "tokens_per_s": tok(t16),
                                            "kernel": kernel_name(L, ws, 16),
                                            "simt_ms": t16s, "simt_tokens_per_s": tok(t16s)}
            # the normalisation ablation of Appendix C (CUDA-core kernel)
            tn = statistics.mean(time_scan(torch, L, ts, ws.chunk, 5, 3, flush=flush, norm="chunk"))
            extra["small_train_chunk_norm"] = {"ms": tn, "tokens_per_s": tok(tn),
                                               "kernel": "scan_simt_kernel<chunked, norm at chunk ends>"}
            # the other chunk linearisation (recurrence_linear1, CUDA-core kernel)
            tl = statistics.mean(time_scan(torch, L, ts, ws.chunk, 5, 3, flush=flush, lin=1))
            extra["small_train_lin1_chunked"] = {"ms": tl, "tokens_per_s": tok(tl),
                                                 "kernel": "scan_simt_kernel<chunked, recurrence_linear1>"}
            # backward pass, chunked (chunk-parallel kernel) and exact (token kernel)
            for cb, tag in ((ws.chunk, "chunked"), (1, "exact")):
                tb = statistics.mean(time_bwd(torch, L, ts, cb, 3, 2, flush=flush))
                extra[f"small_train_bwd_{tag}"] = {"ms": tb, "tokens_per_s": tok(tb),
                                                   "kernel": bwd_kernel_name(cb, ws.d),
                                                   "allocations": "outputs per call; workspace once"}
            del ts
            torch.cuda.empty_cache()
            wd = LI.WORKLOADS["decode"]
            us_ms, n = time_decode(torch, L, wd, 1000, 40, device)
            sb = step_alg_bytes(wd)
            extra["decode"] = {"us_per_step": us_ms * 1e3, "steps": n, "gbps": sb / (us_ms * 1e-3) / 1e9,
                               "hbm_frac": sb / (us_ms * 1e-3) / 1e9 / pk["hbm_gbs"],
                               "tokens_per_s": wd.B / (us_ms * 1e-3), "alg_bytes_per_step": sb,
                               "kernel": step_kernel_name("sim"),
                               "traffic": traffic_for(step_kernel_name("sim"), "decode")}
            us_ms, n = time_decode(torch, L, wd, 1000, 40, device, mode="dec")
            extra["decode_dec"] = {"us_per_step": us_ms * 1e3, "steps": n, "gbps": sb / (us_ms * 1e-3) / 1e9,
                                   "hbm_frac": sb / (us_ms * 1e-3) / 1e9 / pk["hbm_gbs"],
                                   "tokens_per_s": wd.B / (us_ms * 1e-3), "alg_bytes_per_step": sb,
                                   "kernel": step_kernel_name("dec"),
                                   "traffic": traffic_for(step_kernel_name("dec"), "decode")}
        line["extra"] = extra
        if not args.no_cpu:
            v, cores, sample = oracle_baseline(w, w.chunk)
            line["cpu_baseline"] = {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                                    "sample": sample, "legs": oracle_legs(w)}
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
