#!/usr/bin/env python
"""Benchmark of the exact-attention hot path on B200.

One step = one training pass of attention over one batch of the GQA workload
(B=1, Hq=32, Hkv=8, N=8192, d=128, causal): fa_fwd then fa_bwd, through the C
ABI, inputs resident in HBM, L2 flushed before every timed call.  "value" is
that step's TFLOP/s; "roofline" is fa_bwd (its bwd_main kernel is most of the
step) against the measured burst bf16 peak (each call is timed on its own,
after an L2 flush; the ratio to the sustained peak is given beside it); "e2e"
is the same step
with every step's inputs copied in from pinned host memory and its gradients
copied out, double-buffered on three streams (the serial figure too).  Timed in
the same run and reported under "parts": the step's forward and backward, the
same workload in fp16 and (forward) in e4m3, the long-MHA and d = 64
workloads, the decode workload (B=64, Hq=32, Hkv=8, Nq=1, Nk=8192) and the
same decode over a paged cache.  "cpu_baseline" (rank 0, one GPU) times the
fp64 oracle on a bounded sample on all host cores.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl libfa|reference]

Multi-GPU: one process per GPU.  Under torchrun (RANK / WORLD_SIZE set) each
process is one rank; otherwise --gpus N > 1 starts the N ranks itself through
torch.distributed.run on 127.0.0.1.  Every rank runs its own replica of the
workload on its own seeded batch (weak scaling, no collective on the data
path); the timed region is bracketed by a barrier and synchronize and the
reported time is the max over ranks.  Rank 0 prints one JSON line.

FLOP rule: fwd = 4 B Hq Nq Nk d (halved when causal), bwd = 2.5 x fwd.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synth  # noqa: E402

STEP_WORKLOAD = "gqa_8k"
METRIC = "attention fwd+bwd TFLOP/s (causal GQA, N=8192, d=128)"
DECODE_WORKLOAD = "gqa_decode"
L2_BYTES = 126 * 1024 * 1024


# ----------------------------------------------------------------------------
# distributed plumbing (host side; covered by CPU gloo tests)
# ----------------------------------------------------------------------------
def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def rank_seed(base_seed: int, rank: int) -> int:
    """Each rank draws its own batch: a distinct seed per rank."""
    return base_seed + 1000 * rank


def free_port() -> int:
    import socket
    sk = socket.socket()
    sk.bind(("127.0.0.1", 0))
    port = sk.getsockname()[1]
    sk.close()
    return port


def replica_command(n: int, argv, script=None, port=None) -> list:
    """The torch.distributed.run command that starts n ranks of `script` (this
    file by default) with `argv`, one process per GPU of this node."""
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
            "--master-addr", "127.0.0.1", "--master-port", str(port or free_port()),
            script or os.path.abspath(__file__), *argv]


def spawn_replicas(n: int, argv, script=None) -> int:
    """Runs n ranks and returns the launcher's exit status (rank 0's line
    reaches this process's stdout)."""
    import subprocess
    return subprocess.run(replica_command(n, argv, script)).returncode


def step_config(world: int) -> dict:
    """The step workload as both arms report it."""
    w = synth.WORKLOADS[STEP_WORKLOAD]
    return {"workload": f"{STEP_WORKLOAD}: B={w.B}, Hq={w.Hq}, Hkv={w.Hkv}, N={w.Nq}, d={w.d}, causal, "
                        f"bf16 N(0,1) inputs (seed {w.seed})",
            "global_batch": world * w.B, "seq_len": w.Nq, "parallelism": f"replicas x{world}",
            "l2": "flushed before every timed call (2 x 126 MiB write)"}


def max_over_ranks(value: float, world: int, device=None) -> float:
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ----------------------------------------------------------------------------
# measured peaks and clocks
# ----------------------------------------------------------------------------
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return dict(hbm_gbs=float(pk["hbm_gbs"]), bf16_tflops=float(pk["bf16_tflops"]),
                    bf16_tflops_sustained=float(pk.get("bf16_tflops_sustained", pk["bf16_tflops"])),
                    source="measured")
    except Exception:
        return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0,
                    source="fallback")


class ClockSampler:
    """Samples SM clock, max SM clock and throttle reasons through NVML every
    `period_s` seconds on a background thread while the timed region runs
    (read-only queries; nothing about the GPU is changed)."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("hw_power_brake_slowdown", "nvmlClocksEventReasonHwPowerBrakeSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"))

    def __init__(self, gpu_index: int, period_s: float = 0.005):
        self.gpu = gpu_index
        self.period = period_s
        self.samples = []
        self._stop = None
        self._thread = None

    def __enter__(self):
        import threading
        try:
            import pynvml
            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByIndex(self.gpu)
        except Exception:
            return self
        self._stop = threading.Event()

        def loop():
            while not self._stop.is_set():
                try:
                    sm = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
                    mx = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
                    rs = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                    mem = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_MEM)
                    self.samples.append((sm, mx, rs, mem))
                except Exception:
                    pass
                self._stop.wait(self.period)

        self._thread = threading.Thread(target=loop, daemon=True)
        self._thread.start()
        return self

    def __exit__(self, *exc):
        if self._thread is not None:
            self._stop.set()
            self._thread.join(timeout=2)
        return False

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        import pynvml
        reasons = set()
        for s_ in self.samples:
            for name, const in self.REASONS:
                if s_[2] & getattr(pynvml, const, 0):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(x[0] for x in self.samples),
                "sm_max_mhz": max(x[1] for x in self.samples), "reasons": sorted(reasons),
                "mem_mhz": statistics.median(x[3] for x in self.samples),
                "samples": len(self.samples)}


# ----------------------------------------------------------------------------
# CPU reference arm: the oracle on a bounded sample
# ----------------------------------------------------------------------------
def oracle_sample_workload():
    """One kv group (4 query heads) of the step workload at N = 2048: 15 GFLOP
    of fwd + bwd by the FLOP rule, a few seconds of oracle time per step."""
    w = synth.WORKLOADS[STEP_WORKLOAD]
    return w.with_(B=1, Hq=w.G, Hkv=1, Nq=2048, Nk=2048)


def time_oracle_step(w, nthreads=0):
    """Wall-clock seconds of the oracle's forward and backward on ``w``."""
    import oracle
    x = synth.make_inputs(w)
    t0 = time.perf_counter()
    oracle.fwd(x["q"], x["k"], x["v"], w.scale, w.causal, nthreads=nthreads)
    t1 = time.perf_counter()
    oracle.bwd(x["q"], x["k"], x["v"], x["dout"], w.scale, w.causal, nthreads=nthreads)
    return t1 - t0, time.perf_counter() - t1


def cpu_baseline_leg(reps=10):
    w = oracle_sample_workload()
    times = [time_oracle_step(w) for _ in range(reps)]
    t_fwd = sum(t[0] for t in times) / reps
    t_bwd = sum(t[1] for t in times) / reps
    flops = w.fwd_flops() + w.bwd_flops()
    # one thread on one (b, h) of the d = 64 MHA workload, for scaling context
    w1 = synth.WORKLOADS["mha_1k"].with_(B=1, Hq=1, Hkv=1)
    f1, b1 = time_oracle_step(w1, nthreads=1)
    return {"value": flops / (t_fwd + t_bwd) / 1e12, "unit": "TFLOP/s", "cores": os.cpu_count(),
            "kind": "oracle",
            "sample": (f"fwd+bwd of one kv group (B=1, Hq=4, Hkv=1, N=2048, d=128, causal) "
                       f"of the {STEP_WORKLOAD} workload, {flops / 1e9:.1f} GFLOP by the FLOP "
                       f"rule, mean of {reps} runs of {t_fwd + t_bwd:.1f} s, fp64 oracle on all host cores"),
            "fwd_gflops": w.fwd_flops() / t_fwd / 1e9, "bwd_gflops": w.bwd_flops() / t_bwd / 1e9,
            "one_thread": {"sample": "one (b, h) of mha_1k (N=1024, d=64, causal)",
                           "fwd_gflops": w1.fwd_flops() / f1 / 1e9, "bwd_gflops": w1.bwd_flops() / b1 / 1e9}}


def reference_config(w) -> dict:
    """The workload the reference arm times: a bounded sample of the step
    workload (its metric and unit are the GPU arm's)."""
    full = synth.WORKLOADS[STEP_WORKLOAD]
    return {"workload": f"sample of {STEP_WORKLOAD}: B={w.B}, Hq={w.Hq}, Hkv={w.Hkv}, N={w.Nq}, d={w.d}, "
                        f"causal, bf16 N(0,1) inputs (seed {w.seed}); one kv group at a quarter of the "
                        f"sequence of the full B={full.B}, Hq={full.Hq}, Hkv={full.Hkv}, N={full.Nq} workload",
            "global_batch": w.B, "seq_len": w.Nq, "parallelism": "none (host cores, rank 0)",
            "sample_of": STEP_WORKLOAD}


def run_reference(args, rank, world):
    if rank != 0:
        return 0
    w = oracle_sample_workload()
    flops = w.fwd_flops() + w.bwd_flops()
    for _ in range(args.warmup):
        time_oracle_step(w)      # untimed: loads the oracle library and pages in its buffers
    times = [time_oracle_step(w) for _ in range(args.steps)]
    dt = sum(sum(t) for t in times) / len(times)
    value = flops / dt / 1e12
    line = {
        "impl": "reference", "metric": METRIC,
        "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": reference_config(w),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": os.cpu_count(), "kind": "oracle",
                         "sample": (f"each step: fp64 oracle fwd+bwd of one kv group (B=1, Hq={w.Hq}, "
                                    f"Hkv=1, N={w.Nq}, d={w.d}, causal) of the step workload, "
                                    f"{flops / 1e9:.1f} GFLOP by the FLOP rule, on all host cores, "
                                    f"rank 0 only")},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------
# GPU arm
# ----------------------------------------------------------------------------
# Shared-memory bytes of one 64-row query step of bwd_main at d = 128 (the kernel's
# dataflow): MMA operand reads (S^T: K 32 KB + Q 16 KB, dP^T: V 32 KB + dO 16 KB, dV: dO
# 16 KB and dK: Q 16 KB with A in tensor memory, dQ^T: K 32 KB + dS^T 16 KB), TMA writes
# (Q, dO 16 KB each, -LSE / -D 512 B), dS^T stores 16 KB, and the fp32 dQ staging tile
# (32 KB stored by the drain warps, 32 KB read by the bulk reduce)
BWD_MAIN_SMEM_BYTES_PER_STEP = 180224 + 33280 + 16384 + 65536
SMEM_BYTES_PER_CLK_PER_SM = 128


def smem_roofline(w, bwd_ms, clocks):
    """bwd_main's shared-memory traffic by its dataflow (bytes per step x steps) over the
    fa_bwd call's mean time, against 148 SMs x 128 B/clk at the sampled SM clock."""
    steps = bwd_main_steps(w)
    mhz = clocks.get("sm_mhz") or 1965.0
    peak = 148 * SMEM_BYTES_PER_CLK_PER_SM * mhz * 1e6 / 1e12
    achieved = steps * BWD_MAIN_SMEM_BYTES_PER_STEP / (bwd_ms * 1e-3) / 1e12
    return {"unit": "TB/s", "achieved": achieved, "peak": peak, "frac": achieved / peak,
            "steps": steps, "bytes_per_step": BWD_MAIN_SMEM_BYTES_PER_STEP,
            "rule": "bytes per 64-row step of the kernel's dataflow x steps / mean fa_bwd call time "
                    "(pre / post included); peak 148 SMs x 128 B/clk at the sampled SM clock"}


def bwd_main_steps(w) -> int:
    """64-row query steps of one bwd_main launch: every (key block, kv head) unit walks
    G heads x the 64-row query blocks that can see its keys."""
    nqb_all = (w.Nq + 63) // 64
    total = 0
    for kb in range((w.Nk + 127) // 128):
        qb0 = 0
        if w.causal:
            first = kb * 128 - (w.Nk - w.Nq)
            qb0 = 0 if first <= 0 else first // 64
        total += max(0, nqb_all - qb0)
    return total * w.B * w.Hkv * (w.Hq // w.Hkv)


# DRAM bytes (read + write) of one bwd_main launch on this workload, from the ncu
# launch list of this bench command on the current kernel (dram__bytes_read.sum +
# dram__bytes_write.sum, mean of the six warm-up and timed-step launches); to be
# taken again whenever the kernel changes.
BWD_MAIN_DRAM_BYTES = 720.38e6 + 341.18e6


def run_libfa(args, rank, world, local):
    import torch
    import exact_attention_114_b200 as fa

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    peaks = load_peaks()

    w = synth.WORKLOADS[STEP_WORKLOAD]
    w = w.with_(seed=rank_seed(w.seed, rank))
    x = synth.make_inputs(w, pinned=True)
    xd = {k: v.to(dev, non_blocking=True) for k, v in x.items()}
    o = torch.empty_like(xd["q"])
    lse = torch.empty((w.B, w.Hq, w.Nq), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(xd["q"]), torch.empty_like(xd["k"]), torch.empty_like(xd["v"])
    ws = torch.empty(fa.fa_bwd_workspace_size(w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d), dtype=torch.uint8,
                     device=dev)
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    def fwd():
        fa.fa_fwd(xd["q"], xd["k"], xd["v"], o, lse, causal=True, scale=w.scale)

    def bwd():
        fa.fa_bwd(xd["q"], xd["k"], xd["v"], o, xd["dout"], lse, dq, dk, dv, causal=True,
                  scale=w.scale, workspace=ws)

    def timed(fn, k):
        """Per-call CUDA-event times (ms), L2 flushed before each call."""
        ts = []
        for _ in range(k):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            ts.append((a, b))
        torch.cuda.synchronize()
        return [a.elapsed_time(b) for a, b in ts]

    for _ in range(args.warmup):
        fwd()
        bwd()
    torch.cuda.synchronize()
    fa.fa_check_device_status()

    # ---- the timed steps
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        step_ms, fwd_ms, bwd_ms = [], [], []
        for _ in range(args.steps):
            flush.zero_()
            e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
            e[0].record(stream)
            fwd()
            e[1].record(stream)
            bwd()
            e[2].record(stream)
            step_ms.append(e)
        torch.cuda.synchronize()
    barrier(world)
    for e in step_ms:
        fwd_ms.append(e[0].elapsed_time(e[1]))
        bwd_ms.append(e[1].elapsed_time(e[2]))
    fa.fa_check_device_status()
    total_ms = sum(fwd_ms) + sum(bwd_ms)
    total_ms = max_over_ranks(total_ms, world, dev)
    ms_step = total_ms / args.steps
    flops_step = w.fwd_flops() + w.bwd_flops()
    value = world * flops_step / (ms_step * 1e-3) / 1e12
    fwd_med, bwd_med = statistics.median(fwd_ms), statistics.median(bwd_ms)
    fwd_tf = w.fwd_flops() / (fwd_med * 1e-3) / 1e12
    bwd_tf = w.bwd_flops() / (bwd_med * 1e-3) / 1e12
    # the roofline's achieved rate: algorithmic FLOPs per fa_bwd call over the
    # call's average duration in the timed region (max over ranks)
    bwd_mean = max_over_ranks(statistics.fmean(bwd_ms), world, dev)
    bwd_tf_mean = w.bwd_flops() / (bwd_mean * 1e-3) / 1e12

    # ---- end to end through the public API: pinned host in, gradients out.
    # Every step copies its own inputs host -> device and its three gradients
    # device -> host inside the timed region.  Steps are double-buffered on three
    # streams (copy in, compute, copy out) so that step i+1's inputs travel while
    # step i computes, as a training loop with a prefetching loader would run;
    # the serial figure (copy, compute, copy on one stream) is reported beside it.
    hx = x
    hdq = torch.empty_like(x["q"], pin_memory=True)
    hdk = torch.empty_like(x["k"], pin_memory=True)
    hdv = torch.empty_like(x["v"], pin_memory=True)
    h2d = sum(t.numel() * t.element_size() for t in hx.values())
    d2h = sum(t.numel() * t.element_size() for t in (hdq, hdk, hdv))

    def e2e_step():
        for kk in ("q", "k", "v", "dout"):
            xd[kk].copy_(hx[kk], non_blocking=True)
        fwd()
        bwd()
        hdq.copy_(dq, non_blocking=True)
        hdk.copy_(dk, non_blocking=True)
        hdv.copy_(dv, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize()
    e2e_serial_ms = statistics.median(timed(e2e_step, max(3, min(args.steps, 10))))

    # double-buffered device sets: inputs, o / lse, gradients
    bufs = [dict(xd=xd, o=o, lse=lse, g=(dq, dk, dv))]
    bufs.append(dict(xd={k_: torch.empty_like(v_) for k_, v_ in xd.items()}, o=torch.empty_like(o),
                     lse=torch.empty_like(lse), g=tuple(torch.empty_like(t) for t in (dq, dk, dv))))
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    for e_ in ev_comp + ev_out:
        e_.record(stream)

    def e2e_pipelined(n):
        for i in range(n):
            bf = bufs[i & 1]
            with torch.cuda.stream(s_in):          # inputs of step i (buffer free once step i-2 computed)
                s_in.wait_event(ev_comp[i & 1])
                for kk in ("q", "k", "v", "dout"):
                    bf["xd"][kk].copy_(hx[kk], non_blocking=True)
                ev_in[i & 1].record(s_in)
            stream.wait_event(ev_in[i & 1])         # compute step i (gradients free once step i-2 copied out)
            stream.wait_event(ev_out[i & 1])
            xb, (gq, gk, gv) = bf["xd"], bf["g"]
            fa.fa_fwd(xb["q"], xb["k"], xb["v"], bf["o"], bf["lse"], causal=True, scale=w.scale)
            fa.fa_bwd(xb["q"], xb["k"], xb["v"], bf["o"], xb["dout"], bf["lse"], gq, gk, gv, causal=True,
                      scale=w.scale, workspace=ws)
            ev_comp[i & 1].record(stream)
            with torch.cuda.stream(s_out):          # gradients of step i back to the host
                s_out.wait_event(ev_comp[i & 1])
                hdq.copy_(gq, non_blocking=True)
                hdk.copy_(gk, non_blocking=True)
                hdv.copy_(gv, non_blocking=True)
                ev_out[i & 1].record(s_out)

    e2e_pipelined(4)
    torch.cuda.synchronize()
    n_e2e = max(4, min(args.steps, 20))
    t_a, t_b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t_a.record(stream)
    s_in.wait_event(t_a)
    e2e_pipelined(n_e2e)
    s_out.wait_event(ev_comp[(n_e2e - 1) & 1])
    t_b.record(s_out)
    torch.cuda.synchronize()
    e2e_ms = t_a.elapsed_time(t_b) / n_e2e
    fa.fa_check_device_status()
    e2e_ms = max_over_ranks(e2e_ms, world, dev)
    e2e_serial_ms = max_over_ranks(e2e_serial_ms, world, dev)
    e2e_value = world * flops_step / (e2e_ms * 1e-3) / 1e12
    del bufs[1]

    # The end-to-end step's own bound: the same bytes moved by plain copies alone (the
    # step's four inputs host -> device, its three gradients device -> host), against
    # the compute time of the step.  Each direction is timed on its own and both at
    # once on two streams, as the double-buffered steps move them; the bound is the
    # slower of the concurrent copies and the compute.
    def copy_ms(fn, reps=5):
        fn()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(reps):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / reps

    def h2d_only():
        for kk in ("q", "k", "v", "dout"):
            xd[kk].copy_(hx[kk], non_blocking=True)

    def d2h_only():
        hdq.copy_(dq, non_blocking=True)
        hdk.copy_(dk, non_blocking=True)
        hdv.copy_(dv, non_blocking=True)

    h2d_ms, d2h_ms = copy_ms(h2d_only), copy_ms(d2h_only)

    def both_ms(reps=5):
        h2d_only()
        d2h_only()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        done_in = torch.cuda.Event()
        a.record(stream)
        s_in.wait_event(a)
        s_out.wait_event(a)
        with torch.cuda.stream(s_in):
            for _ in range(reps):
                h2d_only()
            done_in.record(s_in)
        with torch.cuda.stream(s_out):
            for _ in range(reps):
                d2h_only()
        s_out.wait_event(done_in)
        b.record(s_out)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / reps

    both = both_ms()
    e2e_bound_ms = max(h2d_ms, d2h_ms, both, ms_step)

    # ---- the other training-shape workloads, reported beside the step workload: the
    # long MHA one (B=2, H=32, N=4096, d=128, causal, every 64th query row x8) held
    # to the same bar, and the d = 64 MHA one (B=4, H=16, N=1024), causal and not
    other = {}
    # the step workload's shape at head size 256 (the feature-split backward), and
    # without the causal mask (the backward shares each unit between two CTAs there)
    # without the causal mask (the backward shares each unit between two CTAs there), and a
    # 512-row chunk appended to a 32K-key context (the forward cuts each work tile's keys into shares)
    extra = {"gqa_8k_d256": synth.WORKLOADS[STEP_WORKLOAD].with_(name="gqa_8k_d256", d=256),
             "gqa_8k_noncausal": synth.WORKLOADS[STEP_WORKLOAD].with_(name="gqa_8k_noncausal", causal=False),
             "append_512_32k": synth.WORKLOADS[STEP_WORKLOAD].with_(name="append_512_32k", Nq=512, Nk=32768)}
    for name in ("mha_4k_long", "mha_1k", "mha_1k_noncausal", "gqa_8k_d256", "gqa_8k_noncausal",
                 "append_512_32k"):
        base = extra.get(name) or synth.WORKLOADS[name]
        wo = base.with_(seed=rank_seed(base.seed, rank))
        xo = {k_: v_.to(dev) for k_, v_ in synth.make_inputs(wo).items()}
        oo = torch.empty_like(xo["q"])
        lo = torch.empty((wo.B, wo.Hq, wo.Nq), dtype=torch.float32, device=dev)
        go = [torch.empty_like(xo[k_]) for k_ in ("q", "k", "v")]
        wso = torch.empty(fa.fa_bwd_workspace_size(wo.B, wo.Hq, wo.Hkv, wo.Nq, wo.Nk, wo.d),
                          dtype=torch.uint8, device=dev)

        def fo():
            fa.fa_fwd(xo["q"], xo["k"], xo["v"], oo, lo, causal=wo.causal, scale=wo.scale)

        def bo():
            fa.fa_bwd(xo["q"], xo["k"], xo["v"], oo, xo["dout"], lo, *go, causal=wo.causal,
                      scale=wo.scale, workspace=wso)

        for _ in range(3):
            fo()
            bo()
        torch.cuda.synchronize()
        f_ms = statistics.median(timed(fo, max(10, args.steps)))
        b_ms = statistics.median(timed(bo, max(10, args.steps)))
        if wo.Nq == wo.Nk:
            shape, f_fl, b_fl, rule = f"N={wo.Nq}", wo.fwd_flops(), wo.bwd_flops(), "FLOP rule"
        else:
            # bottom-right mask with Nq << Nk: almost every (query, key) pair is visible, so
            # the rule's causal half would understate the work; count the visible pairs
            vis = sum(min(max(i + wo.Nk - wo.Nq + 1, 0), wo.Nk) for i in range(wo.Nq)) if wo.causal \
                else wo.Nq * wo.Nk
            shape = f"Nq={wo.Nq}, Nk={wo.Nk}"
            f_fl = 4.0 * wo.B * wo.Hq * vis * wo.d
            b_fl, rule = 2.5 * f_fl, "4 d per visible (query, key) pair and head, x2.5 for the backward"
        other[name] = {"workload": f"B={wo.B}, Hq={wo.Hq}, Hkv={wo.Hkv}, {shape}, d={wo.d}, "
                                   f"{'causal' if wo.causal else 'non-causal'}",
                       "fwd_kv_split": fa.fa_fwd_kv_split(wo.B, wo.Hq, wo.Hkv, wo.Nq, wo.Nk, wo.d, wo.causal),
                       "bwd_query_split": fa.fa_bwd_query_split(wo.B, wo.Hq, wo.Hkv, wo.Nq, wo.Nk, wo.d,
                                                                wo.causal),
                       "flops": rule,
                       "fwd_ms": f_ms, "fwd_tflops": f_fl / (f_ms * 1e-3) / 1e12,
                       "bwd_ms": b_ms, "bwd_tflops": b_fl / (b_ms * 1e-3) / 1e12}
        del xo, oo, lo, go, wso
    fa.fa_check_device_status()

    # ---- the same workload with fp16 inputs, and the e4m3 forward (kind::f8f6f4)
    x16 = {k: v.to(dev) for k, v in synth.make_inputs(w, dtype=torch.float16).items()}
    o16, dq16 = torch.empty_like(x16["q"]), torch.empty_like(x16["q"])
    dk16, dv16 = torch.empty_like(x16["k"]), torch.empty_like(x16["v"])

    def fwd16():
        fa.fa_fwd(x16["q"], x16["k"], x16["v"], o16, lse, causal=True, scale=w.scale)

    def bwd16():
        fa.fa_bwd(x16["q"], x16["k"], x16["v"], o16, x16["dout"], lse, dq16, dk16, dv16, causal=True,
                  scale=w.scale, workspace=ws)

    for _ in range(3):
        fwd16()
        bwd16()
    torch.cuda.synchronize()
    f16_ms = statistics.median(timed(fwd16, max(10, args.steps)))
    b16_ms = statistics.median(timed(bwd16, max(10, args.steps)))
    fa.fa_check_device_status()
    del x16, o16, dq16, dk16, dv16

    DS = synth.FP8_DESCALE
    x8 = {k: v.to(dev) for k, v in synth.make_inputs_fp8(w).items()}
    ws8 = torch.empty(fa.fa_fwd_fp8_workspace_size(w.B, w.Hkv, w.Nk, w.d), dtype=torch.uint8,
                      device=dev)

    def fwd8():
        fa.fa_fwd_fp8(x8["q"], x8["k"], x8["v"], DS["q"], DS["k"], DS["v"], o, lse, causal=True,
                      scale=w.scale, workspace=ws8)

    for _ in range(3):
        fwd8()
    torch.cuda.synchronize()
    f8_ms = statistics.median(timed(fwd8, max(10, args.steps)))
    f8_tf = w.fwd_flops() / (f8_ms * 1e-3) / 1e12
    fa.fa_check_device_status()
    del x8, ws8

    # ---- decode workload (HBM-bound path)
    wd = synth.WORKLOADS[DECODE_WORKLOAD]
    wd = wd.with_(seed=rank_seed(wd.seed, rank))
    dx = synth.make_inputs(wd)
    dxd = {k: v.to(dev) for k, v in dx.items()}
    del dx
    od = torch.empty_like(dxd["q"])
    lsed = torch.empty((wd.B, wd.Hq, 1), dtype=torch.float32, device=dev)

    def dec():
        fa.fa_fwd(dxd["q"], dxd["k"], dxd["v"], od, lsed, causal=False, scale=wd.scale)

    for _ in range(max(3, args.warmup)):
        dec()
    torch.cuda.synchronize()
    dec_ms = statistics.median(timed(dec, max(10, args.steps)))
    dec_bytes = (2 * wd.B * wd.Hkv * wd.Nk * wd.d * 2 + 2 * wd.B * wd.Hq * wd.d * 2
                 + wd.B * wd.Hq * 4)
    dec_gbs = dec_bytes / (dec_ms * 1e-3) / 1e9
    fa.fa_check_device_status()

    # ---- the same decode over a paged KV cache: 64-key pages handed out in a
    # seeded random order (same bytes, one block-table lookup per tile)
    ps = 64
    pages = wd.Nk // ps
    gen = torch.Generator().manual_seed(wd.seed)
    perm = torch.randperm(wd.B * pages, generator=gen).to(dev)
    pool_k = torch.empty((wd.B * pages, ps, wd.Hkv, wd.d), dtype=torch.bfloat16, device=dev)
    pool_v = torch.empty_like(pool_k)
    pool_k[perm] = dxd["k"].permute(0, 2, 1, 3).reshape(wd.B * pages, ps, wd.Hkv, wd.d)
    pool_v[perm] = dxd["v"].permute(0, 2, 1, 3).reshape(wd.B * pages, ps, wd.Hkv, wd.d)
    table = perm.to(torch.int32).reshape(wd.B, pages).contiguous()
    lens = torch.full((wd.B,), wd.Nk, dtype=torch.int32, device=dev)
    del dxd["k"], dxd["v"]
    torch.cuda.empty_cache()
    pws = torch.empty(max(1, fa.fa_fwd_paged_workspace_size(wd.B, wd.Hq, wd.Hkv, 1, ps, pages, wd.d)),
                      dtype=torch.uint8, device=dev)

    def dec_paged():
        fa.fa_fwd_paged(dxd["q"], pool_k, pool_v, table, lens, od, lsed, scale=wd.scale,
                        workspace=pws)

    for _ in range(3):
        dec_paged()
    torch.cuda.synchronize()
    pag_ms = statistics.median(timed(dec_paged, max(10, args.steps)))
    pag_gbs = dec_bytes / (pag_ms * 1e-3) / 1e9
    fa.fa_check_device_status()
    del pool_k, pool_v, pws, dxd
    torch.cuda.empty_cache()

    # ---- the decode shape at d = 256: beyond the split-KV kernels' width, so it runs the
    # tiled kernel with the 4 query heads of each kv head in one tile (group rows)
    w256 = wd.with_(d=256)
    d2 = {k: v.to(dev) for k, v in synth.make_inputs(w256).items()}
    o2 = torch.empty_like(d2["q"])
    l2 = torch.empty((w256.B, w256.Hq, 1), dtype=torch.float32, device=dev)

    def dec256():
        fa.fa_fwd(d2["q"], d2["k"], d2["v"], o2, l2, causal=False, scale=w256.scale)

    for _ in range(3):
        dec256()
    torch.cuda.synchronize()
    d256_ms = statistics.median(timed(dec256, max(10, args.steps)))
    d256_bytes = (2 * w256.B * w256.Hkv * w256.Nk * w256.d * 2 + 2 * w256.B * w256.Hq * w256.d * 2
                  + w256.B * w256.Hq * 4)
    d256_gbs = d256_bytes / (d256_ms * 1e-3) / 1e9
    fa.fa_check_device_status()
    del d2, o2, l2

    clocks = clk.summary()
    line = {
        "metric": METRIC,
        "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": step_config(world),
        "parts": {
            "fwd": {"ms": fwd_med, "tflops": fwd_tf, "frac_of_peak": fwd_tf / peaks["bf16_tflops"],
                    "frac_of_sustained_peak": fwd_tf / peaks["bf16_tflops_sustained"]},
            "bwd": {"ms": bwd_med, "tflops": bwd_tf, "frac_of_peak": bwd_tf / peaks["bf16_tflops"],
                    "frac_of_sustained_peak": bwd_tf / peaks["bf16_tflops_sustained"]},
            "fwd_fp16": {"ms": f16_ms, "tflops": w.fwd_flops() / (f16_ms * 1e-3) / 1e12},
            "bwd_fp16": {"ms": b16_ms, "tflops": w.bwd_flops() / (b16_ms * 1e-3) / 1e12},
            "fwd_fp8": {"ms": f8_ms, "tflops": f8_tf,
                        "peak": 2 * peaks["bf16_tflops"],
                        "frac_of_peak": f8_tf / (2 * peaks["bf16_tflops"]),
                        "peak_source": f"{peaks['source']} burst bf16 x 2 (nominal e4m3 / bf16 dense ratio)",
                        "includes": "V transpose kernel + forward kernel"},
            **other,
            "decode": {"workload": f"{DECODE_WORKLOAD}: B=64, Hq=32, Hkv=8, Nq=1, Nk=8192, d=128",
                       "ms": dec_ms, "gbs": dec_gbs, "frac_of_hbm": dec_gbs / peaks["hbm_gbs"],
                       "algorithmic_bytes": dec_bytes},
            "decode_paged": {"workload": f"{DECODE_WORKLOAD} over 64-key pages in random order",
                             "ms": pag_ms, "gbs": pag_gbs, "frac_of_hbm": pag_gbs / peaks["hbm_gbs"],
                             "algorithmic_bytes": dec_bytes},
            "decode_d256": {"workload": f"{DECODE_WORKLOAD} at d=256 (tiled kernel, group rows)",
                            "ms": d256_ms, "gbs": d256_gbs, "frac_of_hbm": d256_gbs / peaks["hbm_gbs"],
                            "algorithmic_bytes": d256_bytes},
        },
        "roofline": {"kernel": "fa_bwd (bwd_main dominant; pre/post included in the time)",
                     "bound": "tensor", "achieved": bwd_tf_mean,
                     "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": bwd_tf_mean / peaks["bf16_tflops"],
                     "frac_of_sustained_peak": bwd_tf_mean / peaks["bf16_tflops_sustained"],
                     "sustained_peak": peaks["bf16_tflops_sustained"],
                     "achieved_rule": f"{w.bwd_flops() / 1e9:.1f} GFLOP (FLOP rule) per fa_bwd call / mean "
                                      f"CUDA-event duration of the {args.steps} timed calls",
                     "traffic": BWD_MAIN_DRAM_BYTES, "traffic_kernel": "bwd_main (one launch at this workload, one-pass ncu)",
                     "peak_source": peaks["source"] + " burst bf16 cuBLAS (each call timed alone after an "
                                                      "L2 flush)",
                     # the resource that binds bwd_main: shared-memory bandwidth
                     "smem": smem_roofline(w, bwd_mean, clocks)},
        "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                "mode": "double-buffered: step i+1 inputs copied in and step i-1 gradients copied out "
                        "while step i computes (three streams)",
                "serial_ms_per_step": e2e_serial_ms,
                "serial_value": world * flops_step / (e2e_serial_ms * 1e-3) / 1e12,
                "copy_bound": {"h2d_ms": h2d_ms, "h2d_gbs": h2d / (h2d_ms * 1e-3) / 1e9,
                               "d2h_ms": d2h_ms, "d2h_gbs": d2h / (d2h_ms * 1e-3) / 1e9,
                               "both_ms": both, "both_gbs": (h2d + d2h) / (both * 1e-3) / 1e9,
                               "bound_ms_per_step": e2e_bound_ms,
                               "frac": e2e_bound_ms / e2e_ms,
                               "rule": "max(plain H2D copies, plain D2H copies, both at once on two streams, "
                                       "compute) of one step over the double-buffered step time"}},
        "gpu_launches": args.steps * 4,  # timed region: fwd (1) + bwd (pre, main, post) per step
        "gpu_name": torch.cuda.get_device_name(dev),
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_leg()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------
# profiling mode: a few launches of one call on a reduced shape (for ncu)
# ----------------------------------------------------------------------------
PROFILE_CASES = {
    # working sets above the 126 MB L2, a few hundred MB on the device
    "fwd": ("gqa_8k", dict(Nq=4096, Nk=4096)),
    "bwd": ("gqa_8k", dict(Nq=4096, Nk=4096)),
    "decode": ("gqa_decode", dict(B=16)),
    "fwd_fp8": ("gqa_8k", dict(Nq=4096, Nk=4096)),
    # head size 256: Q and O 64 MiB each, K and V 16 MiB each
    "fwd_d256": ("gqa_8k", dict(Nq=4096, Nk=4096, d=256)),
    "bwd_d256": ("gqa_8k", dict(Nq=4096, Nk=4096, d=256)),
    # a 512-row chunk appended to 32K keys: the forward's key split (K and V 64 MiB each)
    "fwd_append": ("gqa_8k", dict(Nq=512, Nk=32768)),
}


def run_profile(which: str, launches: int = 3) -> int:
    """Runs `launches` calls of fa_fwd / fa_bwd / decode on the reduced shape in
    PROFILE_CASES (the first ones are warm-up for an ncu -s skip)."""
    import torch
    import exact_attention_114_b200 as fa
    name, over = PROFILE_CASES[which]
    w = synth.WORKLOADS[name].with_(**over)
    x = {k: v.cuda() for k, v in synth.make_inputs(w).items()}
    o, lse = fa.fa_fwd(x["q"], x["k"], x["v"], causal=w.causal, scale=w.scale)
    if which == "fwd_fp8":
        DS = synth.FP8_DESCALE
        x = {k: v.cuda() for k, v in synth.make_inputs_fp8(w).items()}
    for _ in range(launches):
        if which in ("bwd", "bwd_d256"):
            fa.fa_bwd(x["q"], x["k"], x["v"], o, x["dout"], lse, causal=w.causal, scale=w.scale)
        elif which == "fwd_fp8":
            fa.fa_fwd_fp8(x["q"], x["k"], x["v"], DS["q"], DS["k"], DS["v"], o, lse, causal=w.causal,
                          scale=w.scale)
        else:
            fa.fa_fwd(x["q"], x["k"], x["v"], o, lse, causal=w.causal, scale=w.scale)
    torch.cuda.synchronize()
    fa.fa_check_device_status()
    print(json.dumps({"profile": which, "workload": name, **over, "launches": launches}))
    return 0


# (B, Hq, Hkv, Nq, Nk, d, causal): sequence lengths, masks and head sizes around the step
# workload, short-query shapes (chunked prefill against a long context) and small launches
SWEEP_SHAPES = [
    (1, 32, 8, n, n, 128, c) for n in (1024, 2048, 4096, 8192, 16384) for c in (True, False)
] + [
    (1, 32, 8, 8192, 8192, 64, True), (1, 32, 8, 8192, 8192, 256, True),
    (4, 16, 16, 1024, 1024, 64, True), (2, 32, 32, 4096, 4096, 128, True),
    (1, 32, 8, 512, 32768, 128, True), (1, 32, 8, 2048, 32768, 128, True),
    (1, 32, 8, 4096, 32768, 128, True), (1, 4, 1, 2048, 2048, 128, True),
]


def run_sweep(steps: int) -> int:
    """fa_fwd and fa_bwd on SWEEP_SHAPES: median CUDA-event time per call (L2 flushed
    before each), TFLOP/s over the visible (query, key) pairs (4 d per pair and head,
    x2.5 for the backward), the key / query splits each call takes and the SM clocks
    sampled while the shape ran.  One JSON line per shape."""
    import torch
    import exact_attention_114_b200 as fa
    dev = torch.device("cuda", 0)
    flush = torch.empty(2 * 126 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)

    def med(fn):
        ts = []
        for i in range(steps + 3):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            torch.cuda.synchronize()
            if i >= 3:
                ts.append(a.elapsed_time(b))
        return statistics.median(ts)

    for i, (B, Hq, Hkv, Nq, Nk, d, causal) in enumerate(SWEEP_SHAPES):
        w = synth.Workload("sweep", B, Hq, Hkv, Nq, Nk, d, causal, 5000 + i)
        x = {k: v.to(dev) for k, v in synth.make_inputs(w).items()}
        o = torch.empty_like(x["q"])
        lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=dev)
        g = [torch.empty_like(x[k]) for k in ("q", "k", "v")]
        ws = torch.empty(fa.fa_bwd_workspace_size(B, Hq, Hkv, Nq, Nk, d), dtype=torch.uint8, device=dev)
        with ClockSampler(0) as clk:
            f_ms = med(lambda: fa.fa_fwd(x["q"], x["k"], x["v"], o, lse, causal=causal, scale=w.scale))
            b_ms = med(lambda: fa.fa_bwd(x["q"], x["k"], x["v"], o, x["dout"], lse, *g, causal=causal,
                                         scale=w.scale, workspace=ws))
        fa.fa_check_device_status()
        vis = (sum(min(max(r + Nk - Nq + 1, 0), Nk) for r in range(Nq)) if causal else Nq * Nk)
        fl = 4.0 * B * Hq * vis * d
        print(json.dumps({"sweep": {"B": B, "Hq": Hq, "Hkv": Hkv, "Nq": Nq, "Nk": Nk, "d": d, "causal": causal},
                          "fwd_ms": f_ms, "fwd_tflops": fl / (f_ms * 1e-3) / 1e12,
                          "bwd_ms": b_ms, "bwd_tflops": 2.5 * fl / (b_ms * 1e-3) / 1e12,
                          "fwd_kv_split": fa.fa_fwd_kv_split(B, Hq, Hkv, Nq, Nk, d, causal),
                          "bwd_query_split": fa.fa_bwd_query_split(B, Hq, Hkv, Nq, Nk, d, causal),
                          "clocks": clk.summary()}),
              flush=True)
        del x, o, lse, g, ws
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["libfa", "reference"], default="libfa")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile", choices=sorted(PROFILE_CASES),
                    help="run a few launches of one call on a reduced shape (for ncu) and exit")
    ap.add_argument("--sweep", action="store_true",
                    help="time fa_fwd / fa_bwd over a grid of shapes (one JSON line each) and exit")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        args.warmup = 3
    if args.profile:
        return run_profile(args.profile)
    if args.sweep:
        return run_sweep(max(5, args.steps // 2))
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        # one process per GPU: start the ranks here and let rank 0 print the line
        return spawn_replicas(args.gpus, sys.argv[1:] if argv is None else list(argv))
    rank, world, local = dist_env()
    if args.impl == "reference":
        # the CPU oracle: rank 0 alone measures it; other ranks have no work
        return run_reference(args, rank, world)
    if world > 1:
        import datetime
        import torch.distributed as dist
        import torch
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        return run_libfa(args, rank, world, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
