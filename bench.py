#!/usr/bin/env python
"""Benchmark of the packed 1-bit / balanced-ternary matmul on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl bnn|reference]
                    [--config 1,2,3,4,5] [--seeds 1,2,3] [--extras sparse,stack,probe]
                    [--cpu-budget S] [--csv PATH]

Headline (the JSON line's value): the large compute-bound binary GEMM,
M = N = K = 8192, fair-coin +-1 activations and weights pre-packed to uint64,
per-channel alpha ~ U(0.5, 1.5); one step = one bnn_binary_gemm call writing
int32 dots and float32 alpha-scaled outputs; metric = GMAC/s (M*N*K / time).
Every step reads its own copy of the packed operands (copies totalling more
than 2x the L2 size, so each step starts cold) and writes 512 MiB of outputs.

Every config of the workload list (1: GEMV 1x1024x1000; 2: sign-pack of
256x4096 fp32 activations + GEMM 256x4096x4096; 3: FFN GEMV 1x28672x8192 with
its activation pack; 4: the headline; 5: the balanced-ternary 11008x4096 layer
at M = 1 and M = 64) also gets a record of its own under "configs" -- GPU
figures for each seed, the roofline of its dominant kernel, and the CPU
baselines -- and one CSV row per config and seed (--csv).

CPU baselines (rank 0, N = 1 only; each a bounded sample, --cpu-budget
seconds): the oracle (the plain unpack-and-sum definition the GPU is checked
against) and K1 (the pages' row-by-row XOR + 64-bit popcount, restated), each
on one core and on all host cores.

Under torchrun (N > 1) every rank runs its own independent copy of the
headline (weak scaling, no data-path collective); the job's time is the max
over ranks and value = all ranks' MACs / that time.

--impl reference times the CPU oracle on bounded samples of the headline
workload on the host cores (rank 0 only).
"""
from __future__ import annotations

import argparse
import csv
import ctypes as C
import hashlib
import json
import math
import os
import sys
import threading
import time
from concurrent.futures import ThreadPoolExecutor

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

from ternary_neural_net_b200 import synth  # noqa: E402

METRIC = "binary GEMM GMAC/s (M·N·K) and batch-1 GEMV HBM GB/s vs B200 peak"
L2_BYTES = 126 * 1024 * 1024
POPC32_PER_CLK_PER_SM = 16  # 32-bit population counts per clock per SM (integer pipe)
HBM_SPEC_GBS = 8000.0       # B200 HBM3e specification (~8 TB/s)
HEADLINE = ("binary GEMM M=N=K=8192: fair-coin +-1 activations and weights pre-packed to uint64, per-channel "
            "alpha ~ U(0.5,1.5); int32 dots + fp32 alpha-scaled outputs")


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def parse_args(argv=None):
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["bnn", "reference"], default="bnn")
    p.add_argument("--config", default="1,2,3,4,5",
                   help="comma list of the configs that get a record of their own (1..5), or 'none'")
    p.add_argument("--seeds", default="1,2,3", help="seeds the per-config GPU figures are taken for")
    p.add_argument("--extras", default="sparse,stack,probe",
                   help="comma list of extra measurements: sparse, stack, probe (or 'none')")
    p.add_argument("--cpu-budget", type=float, default=2.0,
                   help="seconds of CPU work per CPU-baseline sample (0 = no CPU baselines)")
    p.add_argument("--csv", default=None, help="write one CSV row per config and seed to this path")
    p.add_argument("--no-headline", action="store_true", help="skip the headline (profiling runs)")
    p.add_argument("--seed", type=int, default=1, help="seed of the headline's inputs")
    p.add_argument("--gemm-shape", default=None,
                   help="M,N,K of config 4's binary GEMM in its per-seed records (profiling of smaller cases; the "
                        "headline keeps 8192^3)")
    a = p.parse_args(argv)
    a.gemm_shape = tuple(int(v) for v in a.gemm_shape.split(",")) if a.gemm_shape else None
    a.configs = [] if a.config == "none" else sorted({int(c) for c in a.config.split(",") if c})
    a.seed_list = [int(s) for s in a.seeds.split(",") if s]
    a.extra_set = set() if a.extras == "none" else set(a.extras.split(","))
    return a


# ----------------------------------------------------------------------------
# distributed plumbing (one process per GPU; no data-path collective)
# ----------------------------------------------------------------------------
class Dist:
    def __init__(self):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = None

    def init(self, backend):
        if self.world > 1:
            import datetime

            import torch.distributed as dist
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
            self.pg = dist

    def barrier(self, device=None):
        if self.pg:
            if device is not None:
                self.pg.barrier(device_ids=[device.index])
            else:
                self.pg.barrier()

    def max(self, value: float, device) -> float:
        """Max of a per-rank value over all ranks (the job's time is the slowest rank's)."""
        if not self.pg:
            return value
        import torch
        t = torch.tensor([value], dtype=torch.float64, device=device)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg:
            self.pg.destroy_process_group()


# ----------------------------------------------------------------------------
# clocks during the timed region (NVML, sampled from a thread)
# ----------------------------------------------------------------------------
_REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
            0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
            0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}


class ClockSampler:
    def __init__(self, device_index: int, period_s: float = 0.002):
        self.ok = False
        self.samples = []
        self.reasons = 0
        self.period = period_s
        try:
            import pynvml
            pynvml.nvmlInit()
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            idx = int(vis.split(",")[device_index]) if vis else device_index
            self.h = pynvml.nvmlDeviceGetHandleByIndex(idx)
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # NVML missing: clocks are reported as unavailable
            log(f"clock sampler unavailable: {e}")
            self.max_mhz = None

    def _reasons(self):
        f = getattr(self.nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            self.nv.nvmlDeviceGetCurrentClocksThrottleReasons
        return f(self.h)

    def _run(self):
        i = 0
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                if i % 4 == 0:  # the reasons query is the slower one: every fourth sample (and the last)
                    self.reasons |= int(self._reasons())
            except Exception:
                pass
            i += 1
            time.sleep(self.period)
        try:
            self.reasons |= int(self._reasons())
        except Exception:
            pass

    def __enter__(self):
        if self.ok:
            self._stop = threading.Event()
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *exc):
        if self.ok:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unsampled"], "samples": 0}
        names = [v for k, v in _REASONS.items() if self.reasons & k and v != "gpu_idle"]
        return {"sm_mhz": float(np.median(self.samples)), "sm_max_mhz": self.max_mhz, "reasons": names,
                "samples": len(self.samples)}


# ----------------------------------------------------------------------------
# helpers
# ----------------------------------------------------------------------------
def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f), "measured"
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "sm_max_mhz": 1965.0}, "fallback"


def traffic_for(kernel_key: str, source: str):
    """dram bytes per launch from the committed ncu summary, if the kernel's
    source file is unchanged since the capture (else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    try:
        digest = hashlib.sha256(open(os.path.join(ROOT, source), "rb").read()).hexdigest()[:16]
        for line in open(path):
            f = line.split()
            if len(f) >= 3 and not line.startswith("#") and f[0] == kernel_key and f[2] == digest:
                return float(f[1])
    except OSError:
        pass
    return None


class Cuda:
    """Raw C-ABI access with cached pointers (keeps the host side of a step to
    a few microseconds so that the GPU, not Python, sets the pace)."""

    def __init__(self, torch, device):
        from ternary_neural_net_b200 import bnn
        self.torch, self.device, self.bnn = torch, device, bnn
        self.lib = bnn.lib()
        self.stream = torch.cuda.current_stream(device)
        self.s = C.c_void_p(self.stream.cuda_stream)
        self.lib.bnn_probe_popc.argtypes = [C.c_int, C.c_int64, C.c_int64, C.c_void_p, C.POINTER(C.c_double),
                                            C.c_void_p]
        self.lib.bnn_probe_popc.restype = C.c_int

    def check(self, st, what):
        if st != 0:
            raise self.bnn.BnnError(st, what)

    def events(self, n):
        return [self.torch.cuda.Event(enable_timing=True) for _ in range(n)]


def job_throughput(units_per_rank: float, world: int, ms_max: float) -> float:
    """Whole-job rate: every rank processed units_per_rank in its own timed
    region; the job took the slowest rank's time (ms_max)."""
    return world * units_per_rank / (ms_max * 1e-3)


def rotation_copies(bytes_per_set: int) -> int:
    return max(2, min(256, math.ceil(2 * L2_BYTES / max(1, bytes_per_set)) + 1))


# ----------------------------------------------------------------------------
# the headline: binary GEMM M = N = K = 8192 (pre-packed operands)
# ----------------------------------------------------------------------------
def run_headline(cu: Cuda, args, dist: Dist):
    torch, dev, lib = cu.torch, cu.device, cu.lib
    c = synth.gemm_large(args.seed + dist.rank)
    m, n, k = c["m"], c["n"], c["k"]
    kw = synth.words_per_row(k)
    R = rotation_copies((m + n) * kw * 8)
    xp_h = torch.from_numpy(c["xp"].view(np.int64))
    wp_h = torch.from_numpy(c["wp"].view(np.int64))
    XP = [xp_h.to(dev) for _ in range(R)]
    WP = [wp_h.to(dev) for _ in range(R)]
    al = torch.from_numpy(c["alpha"]).to(dev)
    D = [torch.empty((m, n), dtype=torch.int32, device=dev) for _ in range(2)]
    O = [torch.empty((m, n), dtype=torch.float32, device=dev) for _ in range(2)]
    torch.cuda.synchronize(dev)     # weights complete before any matmul is enqueued
    cap = torch.cuda.Stream(dev)
    cs = C.c_void_p(cap.cuda_stream)
    P = lambda t: C.c_void_p(t.data_ptr())  # noqa: E731
    gemm_args = [(P(XP[r]), P(WP[r]), P(al), m, n, k, P(D[r % 2]), P(O[r % 2]), cs) for r in range(R)]

    def step(i):
        st = lib.bnn_binary_gemm(*gemm_args[i % R])
        if st:
            cu.check(st, "headline step")

    cap.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(cap):
        for i in range(args.warmup):
            step(i)
    torch.cuda.synchronize(dev)
    K = args.steps
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=cap):
        for i in range(K):
            step(args.warmup + i)
    g.replay()                                   # upload the graph (untimed)
    t0, t1 = cu.events(2)
    torch.cuda.synchronize(dev)
    dist.barrier(dev)
    torch.cuda.synchronize(dev)
    with ClockSampler(dev.index, 0.0005) as clocks:  # every 0.5 ms: several samples in a region of K steps
        t0.record(cu.stream)
        g.replay()
        t1.record(cu.stream)
        torch.cuda.synchronize(dev)
    dist.barrier(dev)
    torch.cuda.synchronize(dev)
    ms = dist.max(t0.elapsed_time(t1), dev)
    del g
    macs = float(m) * n * k
    res = dict(m=m, n=n, k=k, R=R, ms_total=ms, ms_per_step=ms / K, macs=macs, clocks=clocks.summary(),
               kernel_ms=ms / K)
    # per-launch events around a few eager launches (a cross-check of the
    # graph-averaged kernel time; each launch is one kernel of ~0.6 ms)
    evs = [cu.events(2) for _ in range(4)]
    with torch.cuda.stream(cap):
        for i, (a, b) in enumerate(evs):
            a.record(cap)
            step(i)
            b.record(cap)
    torch.cuda.synchronize(dev)
    res["kernel_ms_events"] = float(np.median([a.elapsed_time(b) for a, b in evs]))
    # the popcount kernel family on the same operands (its own roofline)
    with ClockSampler(dev.index) as clk:
        res["popc_ms"] = graph_time(cu, lambda i: lib.bnn_binary_gemm_algo(*gemm_args[i % R][:-1], 1, cs), 3, cap)
    res["popc_clocks"] = clk.summary()

    # end to end through the public API: pinned host activations in, dots and
    # outputs back to pinned host, pipelined over two buffer slots and three
    # streams (copy in / compute / copy out).  Every step moves its own 8 MiB
    # of packed activations in and its own 512 MiB of results out.
    xh = xp_h.pin_memory()
    DH = [torch.empty((m, n), dtype=torch.int32).pin_memory() for _ in range(2)]
    OH = [torch.empty((m, n), dtype=torch.float32).pin_memory() for _ in range(2)]
    Ke = max(3, min(K, 12))
    s_in, s_comp, s_out = (torch.cuda.Stream(dev) for _ in range(3))
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    for e in ev_comp + ev_out:
        e.record(cu.stream)
    torch.cuda.synchronize(dev)

    def e2e_step(i):
        sl = i % 2
        with torch.cuda.stream(s_in):
            s_in.wait_event(ev_comp[sl])            # step i-2's GEMM has read this slot's activations
            XP[sl].copy_(xh, non_blocking=True)
            ev_in[sl].record(s_in)
        with torch.cuda.stream(s_comp):
            s_comp.wait_event(ev_in[sl])
            s_comp.wait_event(ev_out[sl])           # step i-2's results have left this slot
            cu.bnn.bnn_binary_gemm(XP[sl], WP[0], al, k, dots=D[sl], out=O[sl])
            ev_comp[sl].record(s_comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_comp[sl])
            DH[sl].copy_(D[sl], non_blocking=True)
            OH[sl].copy_(O[sl], non_blocking=True)
            ev_out[sl].record(s_out)

    for i in range(2):
        e2e_step(i)
    e0, e1 = cu.events(2)
    torch.cuda.synchronize(dev)
    dist.barrier(dev)
    e0.record(cu.stream)
    for st_ in (s_in, s_comp, s_out):
        st_.wait_event(e0)
    for i in range(Ke):
        e2e_step(2 + i)
    for st_ in (s_in, s_comp, s_out):
        cu.stream.wait_stream(st_)
    e1.record(cu.stream)
    torch.cuda.synchronize(dev)
    e2e_ms = dist.max(e0.elapsed_time(e1), dev) / Ke
    res["e2e"] = dict(ms_per_step=e2e_ms, steps=Ke, h2d=m * kw * 8, d2h=m * n * 8,
                      pipelining="2 buffer slots, 3 streams (copy in / compute / copy out)")
    # the last step's results on the host, checked against the CPU baseline
    # on a few rows (a consistency check of the measured run, not the parity test)
    torch.cuda.synchronize(dev)
    res["host_result"] = (DH[(Ke + 1) % 2], OH[(Ke + 1) % 2])
    for lst in (XP, WP, D, O):
        lst.clear()
    return res


# ----------------------------------------------------------------------------
# per-config GPU figures
# ----------------------------------------------------------------------------
def roofline(bound, achieved, peak, unit, kernel, basis, traffic=None, **extra):
    d = {"bound": bound, "kernel": kernel, "achieved": achieved, "peak": peak, "unit": unit,
         "frac": achieved / peak if peak else None, "traffic": traffic, "peak_basis": basis}
    d.update(extra)
    return d


def check_within(kernel_ms, step_ms, what):
    """A kernel's time cannot exceed the step it is part of."""
    if kernel_ms > step_ms * 1.02:
        raise RuntimeError(f"{what}: kernel time {kernel_ms:.4f} ms exceeds its step's {step_ms:.4f} ms")


def gpu_cfg1(cu, seed, P, st, s, pk):
    torch, dev, lib = cu.torch, cu.device, cu.lib
    c = synth.gemv_small(seed)
    n, k = c["n"], c["k"]
    xp = torch.from_numpy(c["xp"].view(np.int64)).to(dev)
    wp = torch.from_numpy(c["wp"].view(np.int64)).to(dev)
    al = torch.from_numpy(c["alpha"]).to(dev)
    d = torch.empty((1, n), dtype=torch.int32, device=dev)
    o = torch.empty((1, n), dtype=torch.float32, device=dev)
    torch.cuda.synchronize(dev)
    ms_eager = time_calls(cu, lambda i: lib.bnn_binary_gemm(P(xp), P(wp), P(al), 1, n, k, P(d), P(o), cu.s), 2000)
    ms_graph = graph_time(cu, lambda i: lib.bnn_binary_gemm(P(xp), P(wp), P(al), 1, n, k, P(d), P(o), s), 400, st)
    alg = n * 16 * 8 + 16 * 8 + n * 4 * 3
    gbs = alg / (ms_graph * 1e-3) / 1e9
    return dict(value=ms_graph * 1e3, unit="us per call (graph)", us_eager=ms_eager * 1e3, gbs=gbs,
                macs=float(n) * k, roofline=roofline(
                    "hbm", gbs, pk["hbm_gbs"], "GB/s", "binary_gemv_kernel (m = 1)",
                    f"HBM copy {pk['hbm_gbs']} GB/s ({pk['src']}); 143 KB per call: launch-latency bound",
                    note="a 2 us call moves 143 KB; the fraction only shows that the call is latency bound"))


def gpu_cfg2(cu, seed, P, st, s, pk):
    torch, dev, lib = cu.torch, cu.device, cu.lib
    c = synth.gemm_fused_pack(seed)
    m, n, k = c["m"], c["n"], c["k"]
    kw = synth.words_per_row(k)
    w = torch.from_numpy(c["w"]).to(dev)
    wp0 = cu.bnn.bnn_pack_signs(w)
    del w
    R = rotation_copies(m * k * 4 + n * kw * 8 + m * kw * 8 + m * n * 8)
    x0 = torch.from_numpy(c["x"]).to(dev)
    X = [x0.clone() for _ in range(R)]
    WP = [wp0.clone() for _ in range(R)]
    XP = [torch.empty((m, kw), dtype=torch.int64, device=dev) for _ in range(R)]
    D = [torch.empty((m, n), dtype=torch.int32, device=dev) for _ in range(R)]
    O = [torch.empty((m, n), dtype=torch.float32, device=dev) for _ in range(R)]
    al = torch.from_numpy(c["alpha"]).to(dev)
    torch.cuda.synchronize(dev)

    def step(i):
        r = i % R
        return lib.bnn_pack_signs(P(X[r]), m, k, P(XP[r]), s) or \
            lib.bnn_binary_gemm(P(XP[r]), P(WP[r]), P(al), m, n, k, P(D[r]), P(O[r]), s)
    step_ms = graph_time(cu, step, 200, st)
    gemm_ms = graph_time(cu, lambda i: lib.bnn_binary_gemm(P(XP[i % R]), P(WP[i % R]), P(al), m, n, k, P(D[i % R]),
                                                           P(O[i % R]), s), 200, st)
    pack_ms = graph_time(cu, lambda i: lib.bnn_pack_signs(P(X[i % R]), m, k, P(XP[i % R]), s), 200, st)
    check_within(gemm_ms, step_ms, "config 2 GEMM")
    macs = float(m) * n * k
    mma_ms = graph_time(cu, lambda i: lib.bnn_binary_gemm_algo(P(XP[i % R]), P(WP[i % R]), P(al), m, n, k,
                                                               P(D[i % R]), P(O[i % R]), 2, s), 100, st)
    popc_ms = graph_time(cu, lambda i: lib.bnn_binary_gemm_algo(P(XP[i % R]), P(WP[i % R]), P(al), m, n, k,
                                                                P(D[i % R]), P(O[i % R]), 1, s), 50, st)
    fp4 = 4.0 * pk["bf16_tflops"]
    return dict(value=macs / (step_ms * 1e-3) / 1e9, unit="GMAC/s", us_step=step_ms * 1e3, us_gemm=gemm_ms * 1e3,
                us_pack=pack_ms * 1e3, us_gemm_mma_s8=mma_ms * 1e3, us_gemm_popc=popc_ms * 1e3, macs=macs,
                roofline=roofline(
                    "tensor", 2 * macs / (gemm_ms * 1e-3) / 1e12, fp4, "TOP/s",
                    "binary_gemm_tc_kernel (AUTO for m >= 64): bits as e2m1 nibbles, tcgen05.mma kind::mxf4 "
                    "(unit block scales) into tensor memory",
                    f"fp4 dense = 4 x bf16 {pk['bf16_tflops']} TFLOP/s ({pk['src']}; nominal fp4:bf16 = 9:2.25)",
                    traffic_for("binary_gemm_tc_128x2", "ternary_neural_net_b200/csrc/binary_gemm_tc.cu"),
                    achieved_basis="kernel alone, back to back in a CUDA graph (inside the step: pack + GEMM)"),
                rotation=R)


def gpu_cfg3(cu, seed, P, st, s, pk):
    torch, dev, lib = cu.torch, cu.device, cu.lib
    c = synth.gemv_ffn(seed)
    n, k = c["n"], c["k"]
    kw = synth.words_per_row(k)
    wp_bytes = n * kw * 8
    R = rotation_copies(wp_bytes)
    WP = [torch.from_numpy(c["wp"].view(np.int64)).to(dev)]
    WP += [WP[0].clone() for _ in range(R - 1)]
    x = torch.from_numpy(c["x"]).to(dev)
    xp = torch.empty((1, kw), dtype=torch.int64, device=dev)
    al = torch.from_numpy(c["alpha"]).to(dev)
    o = torch.empty((1, n), dtype=torch.float32, device=dev)
    lib.bnn_pack_signs(P(x), 1, k, P(xp), cu.s)
    torch.cuda.synchronize(dev)
    ms_gemv = graph_time(cu, lambda i: lib.bnn_binary_gemm(P(xp), P(WP[i % R]), P(al), 1, n, k, None, P(o), s),
                         300, st)

    def step(i):
        return lib.bnn_pack_signs(P(x), 1, k, P(xp), s) or \
            lib.bnn_binary_gemm(P(xp), P(WP[i % R]), P(al), 1, n, k, None, P(o), s)
    ms_step = graph_time(cu, step, 300, st)
    check_within(ms_gemv, ms_step, "config 3 GEMV")
    alg = wp_bytes + kw * 8 + n * 4 + n * 4
    gbs = alg / (ms_gemv * 1e-3) / 1e9
    return dict(value=gbs, unit="GB/s", us_gemv=ms_gemv * 1e3, us_step=ms_step * 1e3,
                step_gbs=(alg + k * 4 + kw * 8) / (ms_step * 1e-3) / 1e9, macs=float(n) * k,
                frac_of_spec_8tbs=gbs / HBM_SPEC_GBS,
                frac_of_read_stream=gbs / pk["read_gbs"] if pk.get("read_gbs") else None,
                roofline=roofline("hbm", gbs, pk["hbm_gbs"], "GB/s", "binary_gemv_kernel (m = 1)",
                                  f"HBM copy {pk['hbm_gbs']} GB/s ({pk['src']})",
                                  traffic_for("binary_gemv", "ternary_neural_net_b200/csrc/binary_gemm.cu")),
                rotation=R)


def gpu_cfg4(cu, seed, P, st, s, pk, head=None, shape=None):
    """Seed 1 is the headline's own measurement; other seeds time the kernel in
    a short graph on their own operands."""
    torch, dev, lib = cu.torch, cu.device, cu.lib
    fp4 = 4.0 * pk["bf16_tflops"]
    if head is not None:
        ms, macs = head["kernel_ms"], head["macs"]
    else:
        c = synth.gemm_large(seed, *shape) if shape else synth.gemm_large(seed)
        m, n, k = c["m"], c["n"], c["k"]
        xp = torch.from_numpy(c["xp"].view(np.int64)).to(dev)
        wp = torch.from_numpy(c["wp"].view(np.int64)).to(dev)
        al = torch.from_numpy(c["alpha"]).to(dev)
        d = torch.empty((m, n), dtype=torch.int32, device=dev)
        o = torch.empty((m, n), dtype=torch.float32, device=dev)
        torch.cuda.synchronize(dev)
        ms = graph_time(cu, lambda i: lib.bnn_binary_gemm(P(xp), P(wp), P(al), m, n, k, P(d), P(o), s), 8, st)
        macs = float(m) * n * k
        del d, o
    return dict(value=macs / (ms * 1e-3) / 1e9, unit="GMAC/s", ms_kernel=ms, macs=macs,
                shape=list(shape) if shape else [8192, 8192, 8192],
                roofline=roofline("tensor", 2 * macs / (ms * 1e-3) / 1e12, fp4, "TOP/s",
                                  "binary_gemm_pair_kernel (persistent CTA pairs, 256x224 tiles, tcgen05 kind::mxf4)",
                                  f"fp4 dense = 4 x bf16 {pk['bf16_tflops']} TFLOP/s ({pk['src']}; nominal fp4:bf16 "
                                  f"= 9:2.25 PFLOP/s)",
                                  None if shape else
                                  traffic_for("binary_gemm_pair_m8192", "ternary_neural_net_b200/csrc/binary_gemm_tc.cu")))


def gpu_cfg5(cu, seed, P, st, s, pk):
    torch, dev, lib = cu.torch, cu.device, cu.lib
    c = synth.ternary(seed, m=256)
    n, k = c["n"], c["k"]
    kt = synth.trit_words_per_row(k)
    w = torch.from_numpy(c["w"]).to(dev)
    packed = torch.empty((n, kt), dtype=torch.int16, device=dev)
    scale = torch.empty((n,), dtype=torch.float32, device=dev)
    delta = torch.empty((1,), dtype=torch.float32, device=dev)
    ms_pack = time_calls(cu, lambda i: lib.bnn_ternary_pack(P(w), n, k, P(packed), P(scale), P(delta), cu.s), 10)
    ms_pack_na = time_calls(cu, lambda i: lib.bnn_ternary_pack_noalloc(P(w), n, k, P(packed), P(scale), P(delta),
                                                                        cu.s), 10)
    ms_modes = {}
    for mode, name, thr in ((1, "absmean", 0.0), (2, "delta", 0.5)):
        ms_modes[name] = time_calls(cu, lambda i: lib.bnn_ternary_pack_mode(P(w), n, k, mode, thr, P(packed),
                                                                            P(scale), P(delta), cu.s), 5, warm=2)
    lib.bnn_ternary_pack(P(w), n, k, P(packed), P(scale), P(delta), cu.s)   # TWN: what the layer uses
    del w
    torch.cuda.synchronize(dev)
    pbytes = n * kt * 2
    R = rotation_copies(pbytes)
    PK = [packed] + [packed.clone() for _ in range(R - 1)]
    xb = torch.from_numpy(c["x_bf16"].view(np.int16)).to(dev).view(torch.bfloat16)
    o = torch.empty((256, n), dtype=torch.float32, device=dev)
    torch.cuda.synchronize(dev)

    def t(m, iters, algo=0):
        return graph_time(cu, lambda i: lib.bnn_ternary_gemm_algo(P(xb), P(PK[i % R]), P(scale), m, n, k, P(o), algo,
                                                                  s), iters, st)
    ms1, ms64, ms256 = t(1, 300), t(64, 100), t(256, 30)
    ms64_mma = t(64, 50, 2)
    alg1 = pbytes + k * 2 + n * 4 + n * 4
    gbs1 = alg1 / (ms1 * 1e-3) / 1e9
    fl64, fl256 = 2.0 * 64 * n * k, 2.0 * 256 * n * k
    bf16 = pk["bf16_tflops"]
    return dict(value=gbs1, unit="GB/s (M=1)", us_m1=ms1 * 1e3,
                us_m64=ms64 * 1e3, us_m256=ms256 * 1e3,
                us_m64_mma_sync=ms64_mma * 1e3, m64_tflops=fl64 / (ms64 * 1e-3) / 1e12,
                m256_tflops=fl256 / (ms256 * 1e-3) / 1e12, macs=float(n) * k,
                pack_ms=ms_pack, pack_noalloc_ms=ms_pack_na, pack_mode_ms=ms_modes,
                pack_gbs=(2 * n * k * 4 + pbytes) / (ms_pack * 1e-3) / 1e9,
                roofline=roofline("hbm", gbs1, pk["hbm_gbs"], "GB/s",
                                  "ternary_gemv_c5_kernel (m = 1, 5 + 5-trit tables over 5-CTA clusters)",
                                  f"HBM copy {pk['hbm_gbs']} GB/s ({pk['src']})",
                                  traffic_for("ternary_gemv_c5", "ternary_neural_net_b200/csrc/ternary.cu"),
                                  frac_of_read_stream=gbs1 / pk["read_gbs"] if pk.get("read_gbs") else None),
                roofline_m64=roofline("tensor", fl64 / (ms64 * 1e-3) / 1e12, bf16, "TFLOP/s",
                                      "ternary GEMM m = 64 (tcgen05 kind::f16)",
                                      f"bf16 dense {bf16} TFLOP/s ({pk['src']})",
                                      traffic_for("ternary_gemm_tmem_m64",
                                                  "ternary_neural_net_b200/csrc/ternary_gemm_tc.cu")),
                rotation=R)


GPU_CFG = {1: gpu_cfg1, 2: gpu_cfg2, 3: gpu_cfg3, 4: gpu_cfg4, 5: gpu_cfg5}
CFG_NAME = {1: "gemv_small_m1_n1024_k1000", 2: "gemm_fused_pack_m256_n4096_k4096", 3: "gemv_ffn_m1_n28672_k8192",
            4: "gemm_large_m8192_n8192_k8192", 5: "ternary_n11008_k4096"}


def read_stream_peak(cu):
    """Read-only HBM stream rate on this device (bnn_probe_stream_read over a
    4 GiB buffer, far above the L2 size), best of a few launches."""
    torch, dev, lib = cu.torch, cu.device, cu.lib
    nbytes = 4 << 30
    buf = torch.empty(nbytes // 4, dtype=torch.int32, device=dev)
    buf.fill_(1)
    sink = torch.zeros(1, dtype=torch.int32, device=dev)
    lib.bnn_probe_stream_read.argtypes = [C.c_void_p, C.c_int64, C.c_int64, C.c_void_p, C.c_void_p]
    lib.bnn_probe_stream_read.restype = C.c_int
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    best = 0.0
    for blocks in (sms * 4, sms * 8):
        for _ in range(4):
            a, b = cu.events(2)
            a.record(cu.stream)
            cu.check(lib.bnn_probe_stream_read(C.c_void_p(buf.data_ptr()), nbytes, blocks,
                                               C.c_void_p(sink.data_ptr()), cu.s), "stream read probe")
            b.record(cu.stream)
            torch.cuda.synchronize(dev)
            best = max(best, nbytes / (a.elapsed_time(b) * 1e-3) / 1e9)
    del buf
    return best


def run_configs(cu, args, pk, head):
    torch, dev = cu.torch, cu.device
    st = torch.cuda.Stream(dev)
    s = C.c_void_p(st.cuda_stream)
    P = lambda t: C.c_void_p(t.data_ptr()) if t is not None else None  # noqa: E731
    out = {}
    for cfg in args.configs:
        per_seed = {}
        for seed in args.seed_list:
            if cfg == 4:
                r = gpu_cfg4(cu, seed, P, st, s, pk,
                             head if (head and seed == args.seed and not args.gemm_shape) else None,
                             args.gemm_shape)
            else:
                r = GPU_CFG[cfg](cu, seed, P, st, s, pk)
            per_seed[seed] = r
            torch.cuda.synchronize(dev)
            torch.cuda.empty_cache()
        vals = [r["value"] for r in per_seed.values()]
        out[cfg] = dict(name=CFG_NAME[cfg], seeds=per_seed, value_median=float(np.median(vals)),
                        value_min=float(min(vals)), value_max=float(max(vals)), unit=per_seed[args.seed_list[0]]["unit"])
    return out


def graph_time(cu: Cuda, fn, iters: int, stream=None) -> float:
    """ms per call of fn(i) (fn launches on `stream`), from a CUDA graph of
    `iters` calls replayed once untimed and once between events."""
    torch = cu.torch
    dev = cu.device
    stream = stream or torch.cuda.Stream(dev)
    stream.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(stream):
        for i in range(3):
            st = fn(i)
            if st:
                cu.check(st, "warm-up")
    torch.cuda.synchronize(dev)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(iters):
            fn(3 + i)
    g.replay()
    a, b = cu.events(2)
    torch.cuda.synchronize(dev)
    a.record(cu.stream)
    g.replay()
    b.record(cu.stream)
    torch.cuda.synchronize(dev)
    del g
    return a.elapsed_time(b) / iters


def popc_probe(cu: Cuda, dev):
    """Integer-pipe rate on this device: popcount-only and the matmul's word
    step (2 XOR + 2 POPC + 1 IADD3), as counted ops per SM per clock."""
    torch = cu.torch
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    blocks = sms * 8
    sink = torch.empty(blocks * 256, dtype=torch.int32, device=dev)
    out = {}
    for mode in (0, 1):
        ops = C.c_double()
        iters = 20000
        cu.check(cu.lib.bnn_probe_popc(mode, blocks, 200, C.c_void_p(sink.data_ptr()), C.byref(ops), cu.s), "probe")
        a, b = cu.events(2)
        with ClockSampler(dev.index, 0.001) as clk:
            a.record(cu.stream)
            cu.check(cu.lib.bnn_probe_popc(mode, blocks, iters, C.c_void_p(sink.data_ptr()), C.byref(ops), cu.s),
                     "probe")
            b.record(cu.stream)
            torch.cuda.synchronize(dev)
        ms = a.elapsed_time(b)
        cs = clk.summary()
        mhz = cs["sm_mhz"] or cs["sm_max_mhz"] or 1965.0
        rate = ops.value / (ms * 1e-3)
        out["popc32" if mode == 0 else "word_step"] = dict(
            per_sm_per_clk=rate / (sms * mhz * 1e6), ops_per_s=rate, ms=ms, sm_mhz=mhz)
    return out


def time_calls(cu, fn, iters, warm=3):
    """ms per call of eager launches on the current stream (host launch cost included)."""
    torch = cu.torch
    for i in range(warm):
        fn(i)
    a, b = cu.events(2)
    torch.cuda.synchronize(cu.device)
    a.record(cu.stream)
    for i in range(iters):
        fn(warm + i)
    b.record(cu.stream)
    torch.cuda.synchronize(cu.device)
    return a.elapsed_time(b) / iters


def wl_sparse(cu, args, P, st, s, hbm):
    """The 11008 x 4096 ternary layer at high sparsity (fixed threshold F = 1.6449:
    ~10% non-zero trits for N(0,1) weights) in the index + sign form: sparse
    GEMV (M = 1) against the dense base-3 GEMV on the same trits."""
    torch, dev, lib = cu.torch, cu.device, cu.lib
    from ternary_neural_net_b200 import bnn
    c = synth.ternary(args.seed, m=1)
    n, k = c["n"], c["k"]
    w = torch.from_numpy(c["w"]).to(dev)
    packed, scale, _ = bnn.bnn_ternary_pack_mode(w, bnn.TERNARY_DELTA, 1.6449)
    del w
    row_ptr, ent = bnn.bnn_ternary_sparse_encode(packed, k)
    nnz = int(ent.numel())
    sparse_bytes = 2 * nnz + 8 * (n + 1)
    R = rotation_copies(sparse_bytes)
    ENT = [ent] + [ent.clone() for _ in range(R - 1)]
    RP = [row_ptr] + [row_ptr.clone() for _ in range(R - 1)]
    PK = [packed] + [packed.clone() for _ in range(R - 1)]
    xb = torch.from_numpy(c["x_bf16"].view(np.int16)).to(dev).view(torch.bfloat16)
    o = torch.empty((1, n), dtype=torch.float32, device=dev)
    ms_sp = graph_time(cu, lambda i: lib.bnn_ternary_sparse_gemm(P(xb), P(RP[i % R]), P(ENT[i % R]), P(scale), None,
                                                                1, n, k, P(o), s), 300, st)
    ms_dense = graph_time(cu, lambda i: lib.bnn_ternary_gemm(P(xb), P(PK[i % R]), P(scale), 1, n, k, P(o), s), 300, st)
    alg = sparse_bytes + 2 * k + 4 * n + 4 * n
    ms_enc = time_calls(cu, lambda i: lib.bnn_ternary_sparse_count(P(packed), n, k, P(RP[0]), cu.s) or
                        lib.bnn_ternary_sparse_encode(P(packed), n, k, P(RP[0]), P(ENT[0]), cu.s), 20)
    return {"ternary_sparse_n11008_k4096": dict(
        density=nnz / (n * k), entries_bytes=2 * nnz, base3_bytes=2 * n * ((k + 9) // 10),
        m1_us_sparse=ms_sp * 1e3, m1_us_dense_same_trits=ms_dense * 1e3,
        m1_sparse_gbs=alg / (ms_sp * 1e-3) / 1e9, m1_sparse_frac_of_hbm=alg / (ms_sp * 1e-3) / 1e9 / hbm,
        encode_us=ms_enc * 1e3, rotation=R)}


def wl_stack(cu, args, P, st, s):
    """Two binarised 4096 -> 4096 layers on a 256-row batch (the headline layer
    twice): fused (bnn_binary_linear: bias + the next layer's sign pack in the
    first layer's epilogue) against unfused (GEMM, then bnn_pack_signs of its
    float32 output, then the second GEMM)."""
    torch, dev, lib = cu.torch, cu.device, cu.lib
    m, n, k = 256, 4096, 4096
    kw = synth.words_per_row(k)
    c = synth.gemm_fused_pack(args.seed)
    x = torch.from_numpy(c["x"]).to(dev)
    w1 = torch.empty((n, kw), dtype=torch.int64, device=dev)
    lib.bnn_pack_signs(P(torch.from_numpy(c["w"]).to(dev)), n, k, P(w1), cu.s)
    w2 = torch.from_numpy(synth.fair_coin_words(args.seed + 7, 2, n, n).view(np.int64)).to(dev)
    a1 = torch.from_numpy(c["alpha"]).to(dev)
    a2 = torch.from_numpy(synth.uniform_f32(args.seed + 7, 3, (n,), 0.5, 1.5)).to(dev)
    b1 = torch.from_numpy(synth.normal_f32(args.seed + 7, 4, (n,))).to(dev)
    xp = torch.empty((m, kw), dtype=torch.int64, device=dev)
    h = torch.empty((m, kw), dtype=torch.int64, device=dev)
    y1 = torch.empty((m, n), dtype=torch.float32, device=dev)
    y2 = torch.empty((m, n), dtype=torch.float32, device=dev)
    torch.cuda.synchronize(dev)

    def fused(i):
        return lib.bnn_pack_signs(P(x), m, k, P(xp), s) or \
            lib.bnn_binary_linear(P(xp), P(w1), P(a1), P(b1), m, n, k, None, None, P(h), s) or \
            lib.bnn_binary_linear(P(h), P(w2), P(a2), None, m, n, n, None, P(y2), None, s)

    def unfused(i):
        return lib.bnn_pack_signs(P(x), m, k, P(xp), s) or \
            lib.bnn_binary_gemm(P(xp), P(w1), P(a1), m, n, k, None, P(y1), s) or \
            lib.bnn_pack_signs(P(y1), m, n, P(h), s) or \
            lib.bnn_binary_gemm(P(h), P(w2), P(a2), m, n, n, None, P(y2), s)
    ms_f = graph_time(cu, fused, 200, st)
    ms_u = graph_time(cu, unfused, 200, st)
    macs = 2.0 * m * n * k
    return {"stack_2x_m256_n4096_k4096": dict(
        us_fused=ms_f * 1e3, us_unfused=ms_u * 1e3, tmacs_fused=macs / (ms_f * 1e-3) / 1e12,
        tmacs_unfused=macs / (ms_u * 1e-3) / 1e12,
        note="fused: pack x, layer 1 with bias and the sign pack of its output in the epilogue, layer 2 "
             "(float32 out); unfused: pack x, GEMM, pack of the float32 layer-1 output, GEMM (no bias)")}


# ----------------------------------------------------------------------------
# CPU baselines: the oracle (as it stands) and K1 (the pages' XOR + popcount
# loop, restated), each on one core and on all host cores, bounded samples
# ----------------------------------------------------------------------------
def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def _timed_units(run_units, total, budget, threads):
    """Calibrate on one unit, then run as many units as fit `budget` seconds
    (at least one per thread, at most `total`), split into `threads`
    contiguous chunks run concurrently (ctypes releases the GIL, so the
    chunks run on separate cores).  Returns (units, seconds)."""
    t = time.perf_counter()
    run_units(0, 1)
    t1 = max(time.perf_counter() - t, 1e-6)
    units = int(max(threads, min(total, threads * budget / t1)))
    units = min(units, total)
    bounds = [(units * i // threads, units * (i + 1) // threads) for i in range(threads)]
    t = time.perf_counter()
    if threads == 1:
        run_units(0, units)
    else:
        with ThreadPoolExecutor(max_workers=threads) as ex:
            list(ex.map(lambda b: run_units(*b) if b[1] > b[0] else None, bounds))
    return units, time.perf_counter() - t


def cpu_baselines(cfg, budget, cores):
    """Oracle and K1 rates for one config, GMAC/s, on 1 core and on `cores`.
    The oracle (single-threaded code) runs on all cores as contiguous chunks of
    units on a pool of threads; K1 runs each sample as one call that spreads
    its (row, column) pairs over OpenMP threads."""
    import oracle
    res = {}
    k1 = None
    if cfg == 1:         # unit: one whole 1 x 1024 x 1000 call, repeated
        c = synth.gemv_small(1)
        n, k, xp, wp, al = c["n"], c["k"], c["xp"], c["wp"], c["alpha"]
        total, unit_macs = 1 << 30, float(n) * k

        def orc(a, b):
            for _ in range(a, b):
                oracle.binary_gemm(xp, wp, al, 1, n, k)

        def k1(a, b, th):
            for _ in range(a, b):
                oracle.k1_binary_gemm(xp, wp, al, 1, n, k, th)
    elif cfg == 3:       # unit: 256 output channels of the GEMV, with the activation pack
        c = synth.gemv_ffn(1)
        n, k, wp, al = c["n"], c["k"], c["wp"], c["alpha"]
        xp = oracle.pack_signs(c["x"])
        blk = 256
        total, unit_macs = n // blk, float(blk) * k

        def orc(a, b):
            for u in range(a, b):
                oracle.binary_gemm(oracle.pack_signs(c["x"]), wp[u * blk:(u + 1) * blk], al[u * blk:(u + 1) * blk],
                                   1, blk, k)

        def k1(a, b, th):
            oracle.k1_binary_gemm(xp, wp[a * blk:b * blk], al[a * blk:b * blk], 1, (b - a) * blk, k, th)
    elif cfg in (2, 4):  # unit: one activation row against all weight rows (cfg 2: with its sign-pack)
        if cfg == 2:
            c = synth.gemm_fused_pack(1)
            x, wp = c["x"], oracle.pack_signs(c["w"])
            xp = oracle.pack_signs(x)
        else:
            c = synth.gemm_large(1)
            x, xp, wp = None, c["xp"], c["wp"]
        m, n, k, al = c["m"], c["n"], c["k"], c["alpha"]
        total, unit_macs = m, float(n) * k

        def orc(a, b):
            oracle.binary_gemm(oracle.pack_signs(x[a:b]) if x is not None else xp[a:b], wp, al, b - a, n, k)

        def k1(a, b, th):
            oracle.k1_binary_gemm(xp[a:b], wp, al, b - a, n, k, th)
    else:                # ternary layer: M = 1 GEMV by blocks of 256 weight rows; M = 64 by activation rows
        c = synth.ternary(1, m=64)
        n, k = c["n"], c["k"]
        trits, sc, _ = oracle.twn_ternarize(c["w"])
        packed = oracle.base3_pack(trits)
        xb = c["x_bf16"]
        blk = 256
        total, unit_macs = n // blk, float(blk) * k

        def orc(a, b):
            oracle.ternary_gemm(xb[:1], packed[a * blk:b * blk], sc[a * blk:b * blk], 1, (b - a) * blk, k)

        def orc64(a, b):
            oracle.ternary_gemm(xb[a:b], packed, sc, b - a, n, k)
        for th, key in ((1, "1core"), (cores, "allcores")):
            u, dt = _timed_units(orc64, 64, budget, th)
            res[f"oracle_m64_{key}"] = dict(gmacs=u * float(n) * k / dt / 1e9, units=u, of=64, seconds=dt, threads=th)
    for th, key in ((1, "1core"), (cores, "allcores")):
        u, dt = _timed_units(orc, total, budget, th)
        res[f"oracle_{key}"] = dict(gmacs=u * unit_macs / dt / 1e9, units=u, of=total, seconds=dt, threads=th)
        if k1 is not None:
            used = oracle.k1_threads_used(th)
            t = time.perf_counter()
            k1(0, 1, used)
            t1 = max(time.perf_counter() - t, 1e-6)
            u = int(max(1, min(total, budget / t1)))
            t = time.perf_counter()
            k1(0, u, used)
            dt = time.perf_counter() - t
            res[f"k1_{key}"] = dict(gmacs=u * unit_macs / dt / 1e9, units=u, of=total, seconds=dt, threads=used)
    res["unit"] = {1: "one call (1 x 1024 x 1000)", 2: "one activation row: sign-pack + its 4096 x 4096 dots",
                   3: "256 output channels of the GEMV (with the 8192-element activation pack)",
                   4: "one activation row against all 8192 weight rows",
                   5: "256 weight rows of the M = 1 ternary GEMV (bf16 x, base-3 words, float64 sums); "
                      "m64: one activation row of the M = 64 layer"}[cfg]
    if cfg in (2, 3):
        res["k1_note"] = "K1 times the matmul on operands packed beforehand (the pages' kernel takes packed words)"
    return res


def oracle_headline_baseline(budget, cores):
    """cpu_baseline of the JSON line: the oracle on all host cores over a
    bounded sample of the headline workload (activation rows of the 8192^3
    GEMM against all weight rows)."""
    import oracle
    c = synth.gemm_large(1)
    m, n, k = c["m"], c["n"], c["k"]

    def orc(a, b):
        oracle.binary_gemm(c["xp"][a:b], c["wp"], c["alpha"], b - a, n, k)
    u, dt = _timed_units(orc, m, budget, cores)
    macs = u * float(n) * k
    return dict(value=macs / dt / 1e9, unit="GMAC/s", cores=cores, kind="oracle",
                sample=f"{u} of the {m} activation rows of the M=N=K=8192 GEMM, each against all {n} weight rows "
                       f"(unpack-and-sum, int64; {macs:.3g} MAC in {dt:.1f} s on {cores} threads)")


def e2e_consistency(head, rows=4):
    """The last end-to-end step's host results against K1 on a few rows."""
    import oracle
    c = synth.gemm_large(1)
    n, k = c["n"], c["k"]
    d, o = head["host_result"]
    d, o = d.numpy(), o.numpy()
    idx = np.linspace(0, c["m"] - 1, rows).astype(np.int64)
    kd, ko = oracle.k1_binary_gemm(c["xp"][idx], c["wp"], c["alpha"], rows, n, k, host_cores())
    return dict(rows=idx.tolist(), dots_equal=bool(np.array_equal(d[idx], kd)),
                out_equal=bool(np.array_equal(o[idx].view(np.uint32), ko.view(np.uint32))))


def run_reference(args, dist: Dist):
    if dist.rank != 0:
        return 0
    import oracle
    c = synth.gemm_large(args.seed)
    m, n, k = c["m"], c["n"], c["k"]
    cores = host_cores()
    # calibrate: one activation row against `cols` weight rows per thread per
    # step, so the whole --steps/--warmup run stays within about two minutes
    t = time.perf_counter()
    oracle.binary_gemm(c["xp"][:1], c["wp"][:256], c["alpha"][:256], 1, 256, k)
    per_col = (time.perf_counter() - t) / 256
    budget = 90.0 / max(1, args.steps + args.warmup)
    cols = int(max(1, min(n, budget / max(per_col, 1e-9))))

    def chunk(r, c0, cc):
        oracle.binary_gemm(c["xp"][r:r + 1], c["wp"][c0:c0 + cc], c["alpha"][c0:c0 + cc], 1, cc, k)

    def step(i, ex):
        jobs = []
        for t_ in range(cores):
            r = (i * cores + t_) % m
            c0 = ((i * cores + t_) * cols) % n
            jobs.append((r, c0, min(cols, n - c0)))
        list(ex.map(lambda j: chunk(*j), jobs))
        return sum(j[2] for j in jobs)

    with ThreadPoolExecutor(max_workers=cores) as ex:
        for i in range(args.warmup):
            step(i, ex)
        t = time.perf_counter()
        macs = 0.0
        for i in range(args.steps):
            macs += step(args.warmup + i, ex) * float(k)
        dt = time.perf_counter() - t
    value = macs / dt / 1e9
    sample = (f"per step and per host thread ({cores} threads): one activation row of the M=N=K=8192 workload "
              f"against {cols} of its {n} weight rows, unpack-and-sum in int64 (the oracle as it stands)")
    line = {
        "metric": METRIC, "value": value, "unit": "GMAC/s", "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": dt * 1e3 / max(1, args.steps), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "u64", "data": "synthetic", "impl": "reference",
        "config": {"workload": HEADLINE + " (oracle on a bounded sample)", "m": m, "n": n, "k": k},
        "cpu_baseline": {"value": value, "unit": "GMAC/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "GMAC/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------
def write_csv(path, configs, cpu):
    cols = ["config", "name", "seed", "value", "unit", "roofline_bound", "roofline_achieved", "roofline_peak",
            "roofline_unit", "roofline_frac", "cpu_oracle_1core_gmacs", "cpu_oracle_allcores_gmacs",
            "cpu_k1_1core_gmacs", "cpu_k1_allcores_gmacs", "cpu_threads"]
    with open(path, "w", newline="") as f:
        wr = csv.writer(f)
        wr.writerow(cols)
        for cfg, rec in configs.items():
            cb = cpu.get(cfg, {}) if cpu else {}
            for seed, r in rec["seeds"].items():
                rf = r["roofline"]
                wr.writerow([cfg, rec["name"], seed, r["value"], r["unit"], rf["bound"], rf["achieved"], rf["peak"],
                             rf["unit"], rf["frac"], cb.get("oracle_1core", {}).get("gmacs"),
                             cb.get("oracle_allcores", {}).get("gmacs"), cb.get("k1_1core", {}).get("gmacs"),
                             cb.get("k1_allcores", {}).get("gmacs"), cb.get("oracle_allcores", {}).get("threads")])


def main(argv=None):
    args = parse_args(argv)
    dist = Dist()
    if args.impl == "reference":
        return run_reference(args, dist)
    import torch
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    dev = torch.device("cuda", dist.local)
    torch.cuda.set_device(dev)
    dist.init("nccl")
    cu = Cuda(torch, dev)
    peaks, peak_src = measured_peaks()
    pk = dict(peaks, src=peak_src)
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    N, K, W = dist.world, args.steps, args.warmup
    lead = dist.rank == 0 and N == 1

    head = None if args.no_headline else run_headline(cu, args, dist)
    extras = {}
    if lead and "probe" in args.extra_set:
        pk["read_gbs"] = read_stream_peak(cu)
        extras["popc_probe"] = popc_probe(cu, dev)
    configs = run_configs(cu, args, pk, head) if lead else {}
    if lead:
        st = torch.cuda.Stream(dev)
        s = C.c_void_p(st.cuda_stream)
        P = lambda t: C.c_void_p(t.data_ptr()) if t is not None else None  # noqa: E731
        if "sparse" in args.extra_set:
            extras.update(wl_sparse(cu, args, P, st, s, pk["hbm_gbs"]))
        if "stack" in args.extra_set:
            extras.update(wl_stack(cu, args, P, st, s))
    torch.cuda.synchronize(dev)
    cores = host_cores()
    cpu = {}
    if lead and args.cpu_budget > 0:
        for cfg in args.configs:
            cpu[cfg] = cpu_baselines(cfg, args.cpu_budget, cores)
    for cfg, rec in configs.items():
        rec["cpu"] = cpu.get(cfg)
    if args.csv and lead:
        write_csv(args.csv, configs, cpu)
    if head is None:
        if dist.rank == 0:
            print(json.dumps({"configs": configs, "extras": extras, "peaks": pk}), flush=True)
        dist.close()
        return 0

    ms_step = head["ms_per_step"]
    value = job_throughput(head["macs"], N, ms_step) / 1e9
    fp4_peak = 4.0 * peaks["bf16_tflops"]                      # TOP/s (1 MAC = 2 ops)
    achieved = 2 * head["macs"] / (head["kernel_ms"] * 1e-3) / 1e12
    max_mhz = head["clocks"]["sm_max_mhz"] or peaks.get("sm_max_mhz", 1965.0)
    popc_peak = sms * POPC32_PER_CLK_PER_SM * 32 * max_mhz * 1e6 / 1e12   # TMAC/s at the max clock
    popc_ach = head["macs"] / (head["popc_ms"] * 1e-3) / 1e12
    e2e = head["e2e"]
    cpu_line = oracle_headline_baseline(args.cpu_budget * 2, cores) if (lead and args.cpu_budget > 0) else None
    line = {
        "metric": METRIC, "value": value, "unit": "GMAC/s", "n_gpus": N, "steps": K, "warmup": W,
        "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "u64", "data": "synthetic",
        "config": {"workload": HEADLINE, "m": head["m"], "n": head["n"], "k": head["k"],
                   "l2": f"packed operands rotate through {head['R']} copies (> 2x L2) and each step writes "
                         f"512 MiB of outputs, so every step starts cold",
                   "parallelism": f"replicas x{N} (independent problems per GPU)"},
        "roofline": {"bound": "tensor",
                     "kernel": "binary_gemm_pair_kernel (bnn_binary_gemm AUTO at two waves of 256x224 CTA-pair "
                               "tiles or more): persistent 2-CTA clusters, TMA-fed packed chunks -> e2m1 nibbles "
                               "(1.0 or 0) in swizzled smem by four producer groups, "
                               "tcgen05.mma.cta_group::2.kind::mxf4.block_scale (unit scale factors; the AND count "
                               "is exact in the float32 accumulator) into a double-buffered tensor-memory "
                               "accumulator, eight epilogue warps overlapping the next tile (+ row_popcount_kernel, "
                               "~1% of the step)",
                     "achieved": achieved, "peak": fp4_peak, "unit": "TOP/s", "frac": achieved / fp4_peak,
                     "achieved_basis": "2 ops x M*N*K per launch / the timed region's duration / K (the step is "
                                       "this one kernel; CUDA events on the launching stream)",
                     "kernel_ms": head["kernel_ms"], "kernel_ms_events": head["kernel_ms_events"],
                     "traffic": traffic_for("binary_gemm_pair_m8192", "ternary_neural_net_b200/csrc/binary_gemm_tc.cu"),
                     "peak_basis": f"fp4 dense tensor peak (the MMA kind the kernel runs) = bf16 "
                                   f"{peaks['bf16_tflops']} TFLOP/s x 4 (nominal fp4:bf16 ratio 9:2.25 PFLOP/s), "
                                   f"{peak_src} (burst figure: a kernel timed alone)"},
        "roofline_popc": {"bound": "alu", "kernel": "binary_gemm_tiled_kernel (bnn_binary_gemm_algo POPC)",
                          "achieved": popc_ach, "peak": popc_peak, "unit": "TMAC/s", "frac": popc_ach / popc_peak,
                          "ms": head["popc_ms"], "clocks": head["popc_clocks"],
                          "peak_basis": f"{sms} SMs x {POPC32_PER_CLK_PER_SM} popc32/clk x 32 bit-MACs x {max_mhz} "
                                        f"MHz (max SM clock)"},
        "cpu_baseline": cpu_line,
        "e2e": {"value": N * head["macs"] / (e2e["ms_per_step"] * 1e-3) / 1e9, "unit": "GMAC/s",
                "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"],
                "ms_per_step": e2e["ms_per_step"], "pipelining": e2e["pipelining"],
                "check": e2e_consistency(head) if lead else None},
        "gpu_launches": 2 * K,  # per step: row_popcount_kernel + binary_gemm_pair_kernel
        "timing": "W eager warm-up steps, then K steps captured in one CUDA graph, replayed once untimed and once "
                  "between CUDA events on the launching stream (barrier + synchronize on both sides)",
        "clocks": head["clocks"],
        "peaks": pk,
        "configs": configs,
        "extras": extras,
    }
    if dist.rank == 0:
        print(json.dumps(line), flush=True)
    dist.close()
    return 0


if __name__ == "__main__":
    sys.exit(main())
