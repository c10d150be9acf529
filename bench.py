#!/usr/bin/env python
"""Benchmark of the packed 1-bit / balanced-ternary matmul on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl bnn|reference] [--workloads all|headline]

Headline (the JSON line's value): binary GEMM with fused activation packing,
M=256 x K=4096 activations (float32, N(0,1), sign-packed on the device every
step) against N=4096 x K=4096 packed weights (packed once, before timing) with
per-channel alpha.  One step = bnn_pack_signs + bnn_binary_gemm (int32 dots and
float32 scaled outputs); metric = GMAC/s (M*N*K / time).  The step's inputs
and outputs rotate through enough copies that every step starts with a cold L2
(copies totalling more than 2x the L2 size).

The other workloads (batch-1 GEMVs, the 8192^3 GEMM, the ternary layer) are
reported under "workloads" on the same line; they are measured after the
headline's timed region.

Under torchrun (N > 1) every rank runs its own independent copy of the
workload (weak scaling, no data-path collective); the job's time is the max
over ranks and value = all ranks' MACs / that time.

--impl reference times the CPU oracle (the plain definition the GPU path is
checked against) on bounded samples of the same workload, on rank 0 only.
"""
from __future__ import annotations

import argparse
import ctypes as C
import hashlib
import json
import math
import os
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

from ternary_neural_net_b200 import synth  # noqa: E402

METRIC = "binary GEMM GMAC/s (M·N·K) and batch-1 GEMV HBM GB/s vs B200 peak"
L2_BYTES = 126 * 1024 * 1024
POPC32_PER_CLK_PER_SM = 16  # 32-bit population counts per clock per SM (integer pipe)


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=2000)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--impl", choices=["bnn", "reference"], default="bnn")
    p.add_argument("--workloads", default="all",
                   help="all, or a comma list of: headline, gemv_small, gemv_ffn, gemm_large, ternary "
                        "(without 'headline' no JSON headline is measured: for profiling runs)")
    p.add_argument("--seed", type=int, default=1)
    return p.parse_args()


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
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                self.reasons |= int(self._reasons())
            except Exception:
                pass
            time.sleep(self.period)

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
# the headline: binary GEMM with fused activation packing (M=256, N=K=4096)
# ----------------------------------------------------------------------------
def run_headline(cu: Cuda, args, dist: Dist):
    torch = cu.torch
    dev = cu.device
    c = synth.gemm_fused_pack(args.seed + dist.rank)
    m, n, k = c["m"], c["n"], c["k"]
    kw = synth.words_per_row(k)
    x_host = torch.from_numpy(c["x"])
    alpha = torch.from_numpy(c["alpha"]).to(dev)
    w_dev = torch.from_numpy(c["w"]).to(dev)
    wp0 = cu.bnn.bnn_pack_signs(w_dev)          # offline weight packing (not timed)
    del w_dev
    set_bytes = m * k * 4 + n * kw * 8 + m * kw * 8 + m * n * 8
    R = rotation_copies(set_bytes)
    X = [x_host.to(dev) for _ in range(R)]
    WP = [wp0.clone() for _ in range(R)]
    XP = [torch.empty((m, kw), dtype=torch.int64, device=dev) for _ in range(R)]
    D = [torch.empty((m, n), dtype=torch.int32, device=dev) for _ in range(R)]
    O = [torch.empty((m, n), dtype=torch.float32, device=dev) for _ in range(R)]
    lib = cu.lib
    cap = torch.cuda.Stream(dev)
    cs = C.c_void_p(cap.cuda_stream)
    pack_args = [(C.c_void_p(X[r].data_ptr()), m, k, C.c_void_p(XP[r].data_ptr()), cs) for r in range(R)]
    gemm_args = [(C.c_void_p(XP[r].data_ptr()), C.c_void_p(WP[r].data_ptr()), C.c_void_p(alpha.data_ptr()),
                  m, n, k, C.c_void_p(D[r].data_ptr()), C.c_void_p(O[r].data_ptr()), cs) for r in range(R)]

    def step(i, ev=None):
        r = i % R
        if ev:
            ev[0].record(cap)
        st1 = lib.bnn_pack_signs(*pack_args[r])
        if ev:
            ev[1].record(cap)
        st2 = lib.bnn_binary_gemm(*gemm_args[r])
        if ev:
            ev[2].record(cap)
        if st1 or st2:
            cu.check(st1 or st2, "headline step")

    # W eager warm-up steps, then the K timed steps captured once into a CUDA
    # graph (so host launch overhead cannot leave gaps between kernels).  One
    # step in EVERY carries external timing events around its two kernels:
    # event nodes serialise the graph around them, so instrumenting every step
    # would slow the whole timed region.
    cap.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(cap):
        for i in range(args.warmup):
            step(i)
    torch.cuda.synchronize(dev)
    K = args.steps
    EVERY = 16
    inst = list(range(0, K, EVERY))
    evs = {i: [torch.cuda.Event(enable_timing=True, external=True) for _ in range(3)] for i in inst}
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=cap):
        for i in range(K):
            step(args.warmup + i, evs.get(i))
    g.replay()                                   # upload the graph (untimed)
    t0, t1 = cu.events(2)
    torch.cuda.synchronize(dev)
    dist.barrier(dev)
    torch.cuda.synchronize(dev)
    with ClockSampler(dev.index) as clocks:
        t0.record(cu.stream)
        g.replay()
        t1.record(cu.stream)
        torch.cuda.synchronize(dev)
    dist.barrier(dev)
    torch.cuda.synchronize(dev)
    ms_local = t0.elapsed_time(t1)
    ms = dist.max(ms_local, dev)
    pack_ms = float(np.mean([evs[i][0].elapsed_time(evs[i][1]) for i in inst]))
    gemm_ms = float(np.mean([evs[i][1].elapsed_time(evs[i][2]) for i in inst]))
    del g
    macs = float(m) * n * k
    res = dict(m=m, n=n, k=k, R=R, ms_total=ms, ms_per_step=ms / K, pack_ms=pack_ms, gemm_ms=gemm_ms,
               macs=macs, clocks=clocks.summary())

    # the same GEMM with the popcount kernel family (for its own roofline)
    popc_args = [a[:-1] + (C.c_int(1), a[-1]) for a in gemm_args]
    res["gemm_popc_ms"] = graph_time(cu, lambda i: lib.bnn_binary_gemm_algo(*popc_args[i % R]), 200, cap)
    tc_args = [a[:-1] + (C.c_int(3), a[-1]) for a in gemm_args]
    res["gemm_tc_ms"] = graph_time(cu, lambda i: lib.bnn_binary_gemm_algo(*tc_args[i % R]), 200, cap)
    mma_args = [a[:-1] + (C.c_int(2), a[-1]) for a in gemm_args]
    res["gemm_mma_ms"] = graph_time(cu, lambda i: lib.bnn_binary_gemm_algo(*mma_args[i % R]), 200, cap)
    # each kernel alone, back to back in a graph without events in between
    res["pack_graph_ms"] = graph_time(cu, lambda i: lib.bnn_pack_signs(*pack_args[i % R]), 200, cap)
    res["gemm_graph_ms"] = graph_time(cu, lambda i: lib.bnn_binary_gemm(*gemm_args[i % R]), 200, cap)

    # end to end through the public API: pinned host activations in, dots and
    # outputs back to pinned host.  Steps are pipelined over two buffer slots
    # and three streams (copy in, compute, copy out), so that one step's
    # host->device copy, another's kernels and a third's device->host copies
    # overlap (PCIe carries both directions at once); every step still moves
    # its own inputs in and its own results out.
    xh = x_host.pin_memory()
    DH = [torch.empty((m, n), dtype=torch.int32).pin_memory() for _ in range(2)]
    OH = [torch.empty((m, n), dtype=torch.float32).pin_memory() for _ in range(2)]
    Ke = max(3, min(K, 200))
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
            s_in.wait_event(ev_comp[sl])            # step i-2 has packed this slot's activations
            X[sl].copy_(xh, non_blocking=True)
            ev_in[sl].record(s_in)
        with torch.cuda.stream(s_comp):
            s_comp.wait_event(ev_in[sl])
            s_comp.wait_event(ev_out[sl])           # step i-2's results have left this slot
            cu.bnn.bnn_pack_signs(X[sl], out=XP[sl])
            cu.bnn.bnn_binary_gemm(XP[sl], WP[0], alpha, k, dots=D[sl], out=O[sl])
            ev_comp[sl].record(s_comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_comp[sl])
            DH[sl].copy_(D[sl], non_blocking=True)
            OH[sl].copy_(O[sl], non_blocking=True)
            ev_out[sl].record(s_out)

    for i in range(3):
        e2e_step(i)
    e0, e1 = cu.events(2)
    torch.cuda.synchronize(dev)
    dist.barrier(dev)
    e0.record(cu.stream)
    for st_ in (s_in, s_comp, s_out):
        st_.wait_event(e0)
    for i in range(Ke):
        e2e_step(3 + i)
    for st_ in (s_in, s_comp, s_out):
        cu.stream.wait_stream(st_)
    e1.record(cu.stream)
    torch.cuda.synchronize(dev)
    e2e_ms = dist.max(e0.elapsed_time(e1), dev) / Ke
    res["e2e"] = dict(ms_per_step=e2e_ms, steps=Ke, h2d=m * k * 4, d2h=m * n * 8,
                      pipelining="2 buffer slots, 3 streams (copy in / compute / copy out)")
    for lst in (X, WP, XP, D, O):
        lst.clear()
    return res


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


# ----------------------------------------------------------------------------
# the other workloads (after the headline's timed region)
# ----------------------------------------------------------------------------
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


def run_workloads(cu: Cuda, args, peaks, popc_peak_macs):
    torch, dev, lib = cu.torch, cu.device, cu.lib
    P = lambda t: C.c_void_p(t.data_ptr()) if t is not None else None  # noqa: E731
    hbm = peaks["hbm_gbs"]
    st = torch.cuda.Stream(dev)
    s = C.c_void_p(st.cuda_stream)
    out = {}

    want = set(args.workloads.split(",")) if args.workloads != "all" else {"gemv_small", "gemv_ffn", "gemm_large",
                                                                           "ternary", "stack", "sparse"}
    if "gemv_small" in want:
        out.update(wl_gemv_small(cu, args, P, st, s))
    if "gemv_ffn" in want:
        out.update(wl_gemv_ffn(cu, args, P, st, s, hbm))
    if "gemm_large" in want:
        out.update(wl_gemm_large(cu, args, P, st, s, popc_peak_macs, peaks))
    if "ternary" in want:
        out.update(wl_ternary(cu, args, P, st, s, hbm, peaks))
    if "stack" in want:
        out.update(wl_stack(cu, args, P, st, s))
    if "sparse" in want:
        out.update(wl_sparse(cu, args, P, st, s, hbm))
    return out


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


def wl_gemv_small(cu, args, P, st, s):
    torch, dev, lib = cu.torch, cu.device, cu.lib
    out = {}
    # 1. GEMV small: M=1, K=1000, N=1024 (launch-latency bound)
    c = synth.gemv_small(args.seed)
    xp = torch.from_numpy(c["xp"].view(np.int64)).to(dev)
    wp = torch.from_numpy(c["wp"].view(np.int64)).to(dev)
    al = torch.from_numpy(c["alpha"]).to(dev)
    d = torch.empty((1, c["n"]), dtype=torch.int32, device=dev)
    o = torch.empty((1, c["n"]), dtype=torch.float32, device=dev)
    ms_eager = time_calls(cu, lambda i: lib.bnn_binary_gemm(P(xp), P(wp), P(al), 1, c["n"], c["k"], P(d), P(o),
                                                            cu.s), 2000)
    ms_graph = graph_time(cu, lambda i: lib.bnn_binary_gemm(P(xp), P(wp), P(al), 1, c["n"], c["k"], P(d), P(o), s),
                          200, st)
    bytes1 = c["n"] * 16 * 8 + 16 * 8 + c["n"] * 4 * 3
    out["gemv_small_m1_n1024_k1000"] = dict(us_per_call_eager=ms_eager * 1e3, us_per_call_graph=ms_graph * 1e3,
                                            gbs_graph=bytes1 / (ms_graph * 1e-3) / 1e9)
    return out


def wl_gemv_ffn(cu, args, P, st, s, hbm):
    torch, dev, lib = cu.torch, cu.device, cu.lib
    out = {}

    # 3. GEMV FFN: M=1, K=8192, N=28672 (HBM-bound weight stream), x packed on device
    c = synth.gemv_ffn(args.seed)
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
    ms_gemv = graph_time(cu, lambda i: lib.bnn_binary_gemm(P(xp), P(WP[i % R]), P(al), 1, n, k, None, P(o), s),
                         300, st)

    def step3(i):
        return lib.bnn_pack_signs(P(x), 1, k, P(xp), s) or \
            lib.bnn_binary_gemm(P(xp), P(WP[i % R]), P(al), 1, n, k, None, P(o), s)
    ms_step = graph_time(cu, step3, 300, st)
    alg_kernel = wp_bytes + kw * 8 + n * 4 + n * 4
    alg_step = alg_kernel + k * 4 + kw * 8
    out["gemv_ffn_m1_n28672_k8192"] = dict(
        us_gemv=ms_gemv * 1e3, gemv_gbs=alg_kernel / (ms_gemv * 1e-3) / 1e9,
        gemv_frac_of_hbm=alg_kernel / (ms_gemv * 1e-3) / 1e9 / hbm,
        us_step=ms_step * 1e3, step_gbs=alg_step / (ms_step * 1e-3) / 1e9, rotation=R,
        gemv_traffic_bytes=traffic_for("binary_gemv", "ternary_neural_net_b200/csrc/binary_gemm.cu"))
    del WP
    return out


def wl_gemm_large(cu, args, P, st, s, popc_peak_macs, peaks):
    torch, dev, lib = cu.torch, cu.device, cu.lib
    out = {}

    # 4. GEMM large: M=N=K=8192 pre-packed, both kernel families
    c = synth.gemm_large(args.seed)
    m, n, k = c["m"], c["n"], c["k"]
    xp = torch.from_numpy(c["xp"].view(np.int64)).to(dev)
    wp = torch.from_numpy(c["wp"].view(np.int64)).to(dev)
    al = torch.from_numpy(c["alpha"]).to(dev)
    d = torch.empty((m, n), dtype=torch.int32, device=dev)
    o = torch.empty((m, n), dtype=torch.float32, device=dev)
    macs = float(m) * n * k
    res4 = {}
    for algo, name in ((3, "tc"), (2, "mma_s8"), (1, "popc")):
        with ClockSampler(dev.index) as clk:
            ms = graph_time(cu, lambda i: lib.bnn_binary_gemm_algo(P(xp), P(wp), P(al), m, n, k, P(d), P(o), algo, s),
                            10 if algo == 2 else 5, st)
        res4[name] = dict(ms=ms, gmacs=macs / (ms * 1e-3) / 1e9, clocks=clk.summary())
    res4["popc"]["frac_of_popc_peak"] = res4["popc"]["gmacs"] / 1e3 / popc_peak_macs
    res4["mma_s8"]["x_popc_peak"] = res4["mma_s8"]["gmacs"] / 1e3 / popc_peak_macs
    res4["tc"]["x_popc_peak"] = res4["tc"]["gmacs"] / 1e3 / popc_peak_macs
    int8_peak = 2.0 * peaks["bf16_tflops"]  # TOP/s: nominal int8:bf16 ratio 2 x the measured bf16 rate
    res4["tc"]["frac_of_int8_peak"] = 2.0 * res4["tc"]["gmacs"] / 1e3 / int8_peak
    res4["tc"]["traffic_bytes"] = traffic_for("binary_gemm_tc_256x1", "ternary_neural_net_b200/csrc/binary_gemm_tc.cu")
    out["gemm_large_8192"] = res4
    del d, o, xp, wp
    return out


def wl_ternary(cu, args, P, st, s, hbm, peaks):
    torch, dev, lib = cu.torch, cu.device, cu.lib
    out = {}

    # 5. Ternary: TWN pack of N=11008 x K=4096 (offline), then M=1 and M=64
    c = synth.ternary(args.seed, m=64)
    n, k = c["n"], c["k"]
    kt = synth.trit_words_per_row(k)
    w = torch.from_numpy(c["w"]).to(dev)
    packed = torch.empty((n, kt), dtype=torch.int16, device=dev)
    scale = torch.empty((n,), dtype=torch.float32, device=dev)
    delta = torch.empty((1,), dtype=torch.float32, device=dev)
    ms_pack = time_calls(cu, lambda i: lib.bnn_ternary_pack(P(w), n, k, P(packed), P(scale), P(delta), cu.s), 20,
                         warm=3)
    lib.bnn_ternary_pack_noalloc.argtypes = [C.c_void_p, C.c_int64, C.c_int64, C.c_void_p, C.c_void_p, C.c_void_p,
                                             C.c_void_p]
    ms_pack_na = time_calls(cu, lambda i: lib.bnn_ternary_pack_noalloc(P(w), n, k, P(packed), P(scale), P(delta),
                                                                        cu.s), 20, warm=3)
    lib.bnn_ternary_pack_mode.argtypes = [C.c_void_p, C.c_int64, C.c_int64, C.c_int, C.c_float, C.c_void_p,
                                          C.c_void_p, C.c_void_p, C.c_void_p]
    ms_modes = {}
    for mode, name, thr in ((1, "absmean", 0.0), (2, "delta", 0.5)):
        ms_modes[name] = time_calls(cu, lambda i: lib.bnn_ternary_pack_mode(P(w), n, k, mode, thr, P(packed), P(scale),
                                                                            P(delta), cu.s), 10, warm=2)
    # the TWN pack is what the layer below uses
    lib.bnn_ternary_pack_noalloc(P(w), n, k, P(packed), P(scale), P(delta), cu.s)
    del w
    pbytes = n * kt * 2
    R = rotation_copies(pbytes)
    PK = [packed] + [packed.clone() for _ in range(R - 1)]
    xb = torch.from_numpy(c["x_bf16"].view(np.int16)).to(dev).view(torch.bfloat16)
    o1 = torch.empty((1, n), dtype=torch.float32, device=dev)
    o64 = torch.empty((64, n), dtype=torch.float32, device=dev)
    ms1 = graph_time(cu, lambda i: lib.bnn_ternary_gemm(P(xb), P(PK[i % R]), P(scale), 1, n, k, P(o1), s), 300, st)
    ms64 = graph_time(cu, lambda i: lib.bnn_ternary_gemm(P(xb), P(PK[i % R]), P(scale), 64, n, k, P(o64), s), 100,
                      st)
    lib.bnn_ternary_gemm_algo.argtypes = [C.c_void_p, C.c_void_p, C.c_void_p, C.c_int64, C.c_int64, C.c_int64,
                                          C.c_void_p, C.c_int, C.c_void_p]
    ms64_alg = {}
    for algo, name in ((2, "mma"), (3, "tc")):
        ms64_alg[name] = graph_time(
            cu, lambda i: lib.bnn_ternary_gemm_algo(P(xb), P(PK[i % R]), P(scale), 64, n, k, P(o64), algo, s), 100, st)
    alg1 = pbytes + k * 2 + n * 4 + n * 4
    flops64 = 2.0 * 64 * n * k
    out["ternary_n11008_k4096"] = dict(
        pack_ms=ms_pack, pack_noalloc_ms=ms_pack_na, pack_mode_ms=ms_modes, pack_gbs=(2 * n * k * 4 + pbytes) / (ms_pack_na * 1e-3) / 1e9,
        m1_us=ms1 * 1e3, m1_gbs=alg1 / (ms1 * 1e-3) / 1e9,
        m1_frac_of_hbm=alg1 / (ms1 * 1e-3) / 1e9 / hbm,
        m64_us=ms64 * 1e3, m64_tflops=flops64 / (ms64 * 1e-3) / 1e12,
        m64_us_by_algo={a: v * 1e3 for a, v in ms64_alg.items()},
        m64_tflops_by_algo={a: flops64 / (v * 1e-3) / 1e12 for a, v in ms64_alg.items()},
        m64_frac_of_bf16=flops64 / (ms64 * 1e-3) / 1e12 / peaks["bf16_tflops"], rotation=R)
    return out


# ----------------------------------------------------------------------------
# CPU baseline: the oracle, timed on a bounded sample of the headline workload
# ----------------------------------------------------------------------------
def oracle_sample_rate(seed: int, budget_s: float):
    import oracle
    c = synth.gemm_fused_pack(seed)
    m, n, k = c["m"], c["n"], c["k"]
    wp = oracle.pack_signs(c["w"])
    rows = 1
    t = time.perf_counter()
    xp = oracle.pack_signs(c["x"][:rows])
    oracle.binary_gemm(xp, wp, c["alpha"], rows, n, k)
    t1 = time.perf_counter() - t
    rows = int(max(1, min(m, budget_s / max(t1, 1e-6))))
    t = time.perf_counter()
    xp = oracle.pack_signs(c["x"][:rows])
    oracle.binary_gemm(xp, wp, c["alpha"], rows, n, k)
    dt = time.perf_counter() - t
    macs = float(rows) * n * k
    return dict(value=macs / dt / 1e9, unit="GMAC/s", cores=1, kind="oracle",
                sample=f"sign-pack of {rows} of {m} activation rows (fp32, K={k}) + unpack-and-sum "
                       f"binary matmul of those rows against all N={n} packed weight rows "
                       f"({macs:.3g} MAC, {dt:.1f} s, single thread)")


def run_reference(args, dist: Dist):
    if dist.rank != 0:
        return 0
    import oracle
    c = synth.gemm_fused_pack(args.seed)
    m, n, k = c["m"], c["n"], c["k"]
    wp = oracle.pack_signs(c["w"])
    # calibrate: one activation row against `cols` weight rows per step, so the
    # whole --steps/--warmup run stays within about two minutes
    t = time.perf_counter()
    xp = oracle.pack_signs(c["x"][:1])
    oracle.binary_gemm(xp, wp[:256], c["alpha"][:256], 1, 256, k)
    per_col = (time.perf_counter() - t) / 256
    budget = 90.0 / max(1, args.steps + args.warmup)
    cols = int(max(1, min(n, budget / max(per_col, 1e-9))))

    def step(i):
        r = i % m
        xp = oracle.pack_signs(c["x"][r:r + 1])
        c0 = (i * cols) % n
        cc = min(cols, n - c0)
        oracle.binary_gemm(xp, wp[c0:c0 + cc], c["alpha"][c0:c0 + cc], 1, cc, k)
        return cc

    for i in range(args.warmup):
        step(i)
    t = time.perf_counter()
    macs = 0.0
    for i in range(args.steps):
        macs += step(args.warmup + i) * float(k)
    dt = time.perf_counter() - t
    value = macs / dt / 1e9
    sample = (f"per step: sign-pack of 1 activation row (fp32, K={k}) and its unpack-and-sum binary matmul "
              f"against {cols} of the N={n} weight rows of the M={m} x N={n} x K={k} workload; single thread")
    line = {
        "metric": METRIC, "value": value, "unit": "GMAC/s", "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": dt * 1e3 / max(1, args.steps), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "u64", "data": "synthetic", "impl": "reference",
        "config": {"workload": "binary GEMM with fused activation sign-packing, M=256 N=4096 K=4096 "
                               "(oracle on a bounded sample)", "m": m, "n": n, "k": k},
        "cpu_baseline": {"value": value, "unit": "GMAC/s", "cores": 1, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "GMAC/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------
def main():
    args = parse_args()
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

    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    with_headline = args.workloads == "all" or "headline" in args.workloads.split(",")
    if not with_headline:   # profiling runs of single workloads: no headline line
        popc_peak_macs = sms * POPC32_PER_CLK_PER_SM * 32 * peaks.get("sm_max_mhz", 1965.0) * 1e6 / 1e12
        print(json.dumps({"workloads": run_workloads(cu, args, peaks, popc_peak_macs)}), flush=True)
        dist.close()
        return 0
    res = run_headline(cu, args, dist)
    probe = popc_probe(cu, dev)
    max_mhz = res["clocks"]["sm_max_mhz"] or peaks.get("sm_max_mhz", 1965.0)
    popc_peak_macs = sms * POPC32_PER_CLK_PER_SM * 32 * max_mhz * 1e6 / 1e12  # TMAC/s at max clock
    int8_peak = 2.0 * peaks["bf16_tflops"]                                     # TOP/s (1 MAC = 2 ops)
    workloads = run_workloads(cu, args, peaks, popc_peak_macs) if args.workloads != "headline" else {}
    torch.cuda.synchronize(dev)

    K, W, N = args.steps, args.warmup, dist.world
    ms_step = res["ms_per_step"]
    value = job_throughput(res["macs"], N, ms_step) / 1e9
    gemm_achieved = res["macs"] / (res["gemm_ms"] * 1e-3) / 1e12           # TMAC/s
    popc_achieved = res["macs"] / (res["gemm_popc_ms"] * 1e-3) / 1e12
    cpu = oracle_sample_rate(args.seed, 10.0) if (dist.rank == 0 and N == 1) else None
    e2e = res["e2e"]
    line = {
        "metric": METRIC, "value": value, "unit": "GMAC/s", "n_gpus": N, "steps": K, "warmup": W,
        "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "u64", "data": "synthetic",
        "config": {"workload": "binary GEMM with fused activation sign-packing: fp32 N(0,1) activations "
                               "M=256 x K=4096 packed on device each step, packed N=4096 x K=4096 weights, "
                               "per-channel alpha; int32 dots + fp32 scaled outputs",
                   "m": res["m"], "n": res["n"], "k": res["k"],
                   "l2": f"inputs and outputs rotate through {res['R']} copies (> 2x L2) so each step starts cold",
                   "parallelism": f"replicas x{N} (independent problems per GPU)"},
        "roofline": {"bound": "tensor", "kernel": "binary_gemm_tc_kernel<128,2,TMA,deep> (bnn_binary_gemm, m >= 64: "
                                                  "TMA-fed packed chunks -> 0/1 bytes in swizzled smem, tcgen05.mma "
                                                  "kind::i8 into TMEM, 2-CTA cluster split-K)",
                     "achieved": 2 * gemm_achieved, "peak": int8_peak, "unit": "TOP/s",
                     "frac": 2 * gemm_achieved / int8_peak,
                     "achieved_back_to_back": 2 * res["macs"] / (res["gemm_graph_ms"] * 1e-3) / 1e12,
                     "achieved_basis": "achieved: CUDA events around the kernel on every 16th step of the timed "
                                       "graph (includes the event nodes' serialisation); achieved_back_to_back: "
                                       "a graph of the kernel alone launched back to back",
                     "traffic": traffic_for("binary_gemm_tc_128x2", "ternary_neural_net_b200/csrc/binary_gemm_tc.cu"),
                     "peak_basis": f"int8 dense tensor peak = measured bf16 {peaks['bf16_tflops']} TFLOP/s x 2 "
                                   f"(nominal int8:bf16 ratio 4.5:2.25 PFLOP/s), {peak_src}"},
        "roofline_popc": {"bound": "alu", "kernel": "binary_gemm_tiled_kernel (bnn_binary_gemm_algo POPC)",
                          "achieved": popc_achieved, "peak": popc_peak_macs, "unit": "TMAC/s",
                          "frac": popc_achieved / popc_peak_macs,
                          "traffic": traffic_for("binary_gemm_tiled_4x4",
                                                 "ternary_neural_net_b200/csrc/binary_gemm.cu"),
                          "peak_basis": f"{sms} SMs x {POPC32_PER_CLK_PER_SM} popc32/clk x 32 bit-MAC x {max_mhz} MHz "
                                        f"(max SM clock); probe measured {probe['popc32']['per_sm_per_clk']:.2f} "
                                        f"popc32/clk/SM and {probe['word_step']['per_sm_per_clk']:.2f} "
                                        f"word-steps/clk/SM"},
        "kernels_ms": {"bnn_pack_signs": res["pack_ms"], "bnn_binary_gemm": res["gemm_ms"],
                       "bnn_binary_gemm_algo(POPC)": res["gemm_popc_ms"],
                       "bnn_binary_gemm_algo(TC)": res["gemm_tc_ms"],
                       "bnn_binary_gemm_algo(MMA_S8)": res["gemm_mma_ms"],
                       "bnn_pack_signs(graph, alone)": res["pack_graph_ms"],
                       "bnn_binary_gemm(graph, alone)": res["gemm_graph_ms"]},
        "cpu_baseline": cpu,
        "e2e": {"value": N * res["macs"] / (e2e["ms_per_step"] * 1e-3) / 1e9, "unit": "GMAC/s",
                "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"],
                "ms_per_step": e2e["ms_per_step"], "pipelining": e2e["pipelining"]},
        "gpu_launches": 2 * K,
        "timing": "K steps captured in one CUDA graph, replayed once untimed to upload, then once between events; "
                  "every 16th step carries external events around its two kernels (kernels_ms)",
        "clocks": res["clocks"],
        "peaks": {"source": peak_src, "hbm_gbs": peaks["hbm_gbs"], "bf16_tflops": peaks["bf16_tflops"]},
        "popc_probe": probe,
        "workloads": workloads,
    }
    if dist.rank == 0:
        print(json.dumps(line), flush=True)
    dist.close()
    return 0


if __name__ == "__main__":
    sys.exit(main())
