"""Benchmark of the Q4_0 dequant-matmul hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One JSON line on rank 0.  A *step* is one pass of the hot path over one batch
of synthetic input.  The default workload is one synthetic decoder layer of
the Voxtral 4B decoder at M=1 (fused QKV N=5120, O N=3072, fused gate/up
N=16384, all K=3072, and down K=8192, N=3072): the four Q4_0 GEMMs of a token
step, issued as one grouped launch.  Five independently seeded copies of the
layer's weights (283 MB, more than twice the 126 MB L2) rotate from step to
step, so every step streams its weights from HBM.

The metric is effective HBM bandwidth: algorithmic bytes (every Q4_0 weight
byte once + X and Y once) / time.  Other workloads (--workload): gemv, layer,
cfg_decode (M=2, 26 layers), concurrent (M=32, 26 layers), flow_head (M=2,
one Euler step of the 3-layer flow head) in GB/s; embed, quantize (the row
gather and the quantizer) in GB/s; adapter,
qkv_prefill (M=4096) in TFLOP/s.

N > 1 (torchrun, one process per GPU): every rank runs an independent
replica of the workload (the path has no exchange step); time is the max over
ranks and the value is the work of all ranks over that time (weak scaling).

--impl reference times the float64 CPU oracle on the same workload (a
bounded sample of each step, scaled to the metric's unit) on rank 0 only.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time
from typing import Optional

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "Q4_0 dequant-matmul HBM GB/s (M=1,2) and TFLOP/s (M>=64), % of B200 roofline"
L2_BYTES = 126 * 2**20
DEFAULT_WORKLOAD = "cfg_decode"

# kernel that dominates each workload, and the source file it lives in
DOMINANT = {
    "gemv": ("narrow_kernel", "q4_0_decode_m8.cu"),
    "layer": ("decode_m8_kernel", "q4_0_decode_m8.cu"),
    "cfg_decode": ("decode_m8_kernel", "q4_0_decode_m8.cu"),
    "concurrent": ("decode_mma_kernel", "q4_0_decode_mma.cu"),
    "flow_head": ("decode_m8_kernel", "q4_0_decode_m8.cu"),
    "layer_fused": ("decode_m8_kernel", "q4_0_decode_m8.cu"),
    "adapter": ("prefill_kernel", "q4_0_prefill.cu"),
    "qkv_prefill": ("prefill_kernel", "q4_0_prefill.cu"),
}
TENSOR_WORKLOADS = ("adapter", "qkv_prefill")
UTIL_KERNELS = {"embed": ("gather_kernel", "q4_0_embed.cu"), "quantize": ("quantize_kernel", "q4_0_embed.cu")}


def log(*a):
    print(*a, file=sys.stderr, flush=True)


# --------------------------------------------------------------------------- helpers

def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def source_sha(fname: str) -> str:
    with open(os.path.join(ROOT, "bit_weight_only_matmul_b200", "csrc", fname), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()


def recorded_traffic(workload: str):
    """DRAM bytes per launch of the dominant kernel from the committed ncu
    summary (the mean over a step's launches where a step has several), or
    None when absent or when the kernel source changed since."""
    kernel, src = DOMINANT[workload] if workload in DOMINANT else UTIL_KERNELS[workload]
    path = os.path.join(ROOT, "profiles", f"{kernel}_{workload}.traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    if d.get("source_sha256") != source_sha(src):
        return None
    return d.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled every 100 ms."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.rows = []
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                self.rows.append(parts)

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.thread.join(timeout=2)

    def summary(self):
        if not self.rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        sm = [float(r[1]) for r in self.rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in self.rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in self.rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(self.rows)}


# --------------------------------------------------------------------------- our implementation

class GpuWorkload:
    """A workload resident in HBM: packed Q4_0 weights (packed on the GPU by
    q4_0_pack from seeded codes and scales), activations and outputs, in
    `copies` replicas at distinct addresses; the first SEEDS are seeded
    independently, later ones repeat their values."""

    SEEDS = 8

    def __init__(self, q4, wl: workloads.Workload, copies: int, seed: int, wcache: Optional[dict] = None):
        import torch
        self.wl = wl
        self.sets = []
        # a step's X (and Y) tensors are views of one contiguous buffer per
        # copy, so that the end-to-end step moves them with one copy each way
        def offsets(sizes):
            out, at = [], 0
            for n in sizes:
                out.append(at)
                at += -(-n // 64) * 64   # 64-element steps keep every view 16-byte aligned
            return out, at
        x_off, x_total = offsets([l.M * l.K for l in wl.linears])
        y_off, y_total = offsets([l.M * l.N for l in wl.linears])
        self.x_off, self.y_off = x_off, y_off
        self.xbufs, self.ybufs = [], []
        for c in range(copies):
            probs = []
            xbuf = torch.zeros(x_total, dtype=torch.int16, device="cuda")
            ybuf = torch.empty(y_total, dtype=torch.float32, device="cuda")
            for li, (lin, xo, yo) in enumerate(zip(wl.linears, x_off, y_off)):
                X = xbuf[xo:xo + lin.M * lin.K].view(lin.M, lin.K)
                Y = ybuf[yo:yo + lin.M * lin.N].view(lin.M, lin.N)
                if c >= self.SEEDS:   # same values as copy c % SEEDS, in fresh buffers
                    W0, X0 = self.sets[c % self.SEEDS][0][li][:2]
                    W = W0.clone()
                    X.copy_(X0)
                    probs.append((W, X, Y, lin.M, lin.N, lin.K))
                    continue
                s = seed + 7919 * c
                key = (s, lin.layer, lin.linear, lin.N, lin.K)
                W = wcache.get(key) if wcache is not None else None
                if W is None:   # weights with the same seed streams are shared between workloads
                    codes = torch.from_numpy(lin.codes(s)).cuda()
                    scales = torch.from_numpy(lin.scales(s).view(np.int16)).cuda()
                    W = torch.empty(q4.q4_0_bytes(lin.N, lin.K), dtype=torch.uint8, device="cuda")
                    q4.q4_0_pack(codes, scales, W, lin.N, lin.K)
                    del codes, scales
                    if wcache is not None:
                        wcache[key] = W
                X.copy_(torch.from_numpy(lin.x(s).view(np.int16)))
                probs.append((W, X, Y, lin.M, lin.N, lin.K))
            self.sets.append((probs, q4.make_problems(probs)))
            self.xbufs.append(xbuf)
            self.ybufs.append(ybuf)
        # the M > 32 GEMMs run through q4_0_gemm_ws with one shared workspace
        # (X converted to fp16 once per GEMM); the M <= 32 ones in one grouped launch
        self.small = [i for i, l in enumerate(wl.linears) if l.M <= 32]
        self.large = [i for i, l in enumerate(wl.linears) if l.M > 32]
        ws = max([q4.q4_0_gemm_workspace_size(l.M, l.N, l.K) for l in wl.linears] + [0])
        self.ws = torch.empty(max(ws, 16), dtype=torch.uint8, device="cuda")
        # pipelined tensor-core steps: each M > 32 GEMM's X is converted on a
        # side stream (q4_0_prepare_x) into one of two buffers while the
        # previous step's GEMM (q4_0_gemm_prepared) runs on the launching stream
        self.pipelined = bool(self.large) and not wl.fused
        if self.pipelined:
            self.side = torch.cuda.Stream()
            self.xh = [[torch.empty(q4.q4_0_prepared_x_bytes(wl.linears[i].M, wl.linears[i].K), dtype=torch.uint8,
                                    device="cuda") for i in self.large] for _ in range(2)]
            self.prep_done = [torch.cuda.Event(), torch.cuda.Event()]
            self.gemm_done = [torch.cuda.Event(), torch.cuda.Event()]
            self.fork = torch.cuda.Event()
            self.begun = [False, False]
        self.small_arrs = [q4.make_problems([probs[i] for i in self.small]) for probs, _ in self.sets]
        self.fused_arrs = []
        if wl.fused:
            # the same weights with the epilogues fused: gate/up re-laid out
            # row-interleaved (gate rows 0..F-1, up rows F..2F-1 of the
            # concatenated weight), Y of width F; O and down add a residual
            self.keep = []
            self.fused_ys = []
            for probs, _ in self.sets:
                ex, ys = [], []
                for (W, X, Y, M, N, K), lin in zip(probs, wl.linears):
                    if lin.name == "gate_up":
                        F = N // 2
                        half = F * (K // 32) * 18
                        Wgu = torch.empty_like(W)
                        q4.q4_0_interleave_gate_up(W[:half], W[half:], Wgu, F, K)
                        Yf = torch.empty((M, F), dtype=torch.float32, device="cuda")
                        self.keep += [Wgu, Yf]
                        ys.append(Yf)
                        ex.append((Wgu, X, Yf, M, N, K, None, q4.Q4_0_EPI_SWIGLU))
                    elif lin.name in ("o", "down"):
                        R = torch.randn((M, N), device="cuda")
                        self.keep.append(R)
                        ys.append(Y)
                        ex.append((W, X, Y, M, N, K, R, q4.Q4_0_EPI_RESIDUAL))
                    else:
                        ys.append(Y)
                        ex.append((W, X, Y, M, N, K, None, q4.Q4_0_EPI_NONE))
                self.fused_arrs.append(q4.make_problems_ex(ex))
                self.fused_ys.append(ys)
        self.operand_bytes = sum(W.numel() + X.numel() * 2 + Y.numel() * 4 for W, X, Y, *_ in self.sets[0][0])
        torch.cuda.synchronize()

    def views(self, xbuf, ybuf):
        """The per-GEMM X and Y views of a step-sized pair of buffers."""
        xs = [xbuf[o:o + l.M * l.K].view(l.M, l.K) for l, o in zip(self.wl.linears, self.x_off)]
        ys = [ybuf[o:o + l.M * l.N].view(l.M, l.N) for l, o in zip(self.wl.linears, self.y_off)]
        return xs, ys

    def outputs(self, step: int):
        """The Y tensors a step writes."""
        k = step % len(self.sets)
        return self.fused_ys[k] if self.fused_arrs else [p[2] for p in self.sets[k][0]]

    def launch(self, q4, step: int):
        k = step % len(self.sets)
        probs, _ = self.sets[k]
        if self.fused_arrs:
            q4.q4_0_gemm_grouped_ex(self.fused_arrs[k], len(probs))
            return
        if self.small:
            q4.q4_0_gemm_grouped(self.small_arrs[k], len(self.small))
        for i in self.large:
            W, X, Y, M, N, K = probs[i]
            q4.q4_0_gemm_ws(W, X, Y, M, N, K, self.ws)

    def begin_pipeline(self):
        """Start a sequence of pipelined steps (a graph capture or an eager
        run): the side stream joins the launching stream here."""
        import torch
        main = torch.cuda.current_stream()
        self.fork.record(main)
        self.side.wait_event(self.fork)
        self.begun = [False, False]

    def launch_pipelined(self, q4, step: int):
        """One step with its X conversion on the side stream: buffer step % 2,
        free once the GEMM two steps back (which read it) is done; the GEMM
        waits for its conversion.  The conversion of step k+1 thus overlaps
        the GEMM of step k."""
        import torch
        k, b = step % len(self.sets), step % 2
        probs, _ = self.sets[k]
        main = torch.cuda.current_stream()
        if self.begun[b]:
            self.side.wait_event(self.gemm_done[b])
        with torch.cuda.stream(self.side):
            for j, i in enumerate(self.large):
                W, X, Y, M, N, K = probs[i]
                q4.q4_0_prepare_x(X, M, K, self.xh[b][j])
            self.prep_done[b].record(self.side)
        if self.small:
            q4.q4_0_gemm_grouped(self.small_arrs[k], len(self.small))
        main.wait_event(self.prep_done[b])
        for j, i in enumerate(self.large):
            W, X, Y, M, N, K = probs[i]
            q4.q4_0_gemm_prepared(W, self.xh[b][j], Y, M, N, K)
        self.gemm_done[b].record(main)
        self.begun[b] = True


def rotating_copies(wl: workloads.Workload) -> int:
    """Copies of a step's operands that together exceed twice the L2, so
    that every step's operands come from HBM, not L2 (one decoder layer: 5; a
    3072 x 3072 GEMV: 50)."""
    step = wl.weight_bytes + sum(l.act_bytes for l in wl.linears)
    return max(1, -(-2 * L2_BYTES // max(1, step)))


# B200 datasheet figures (context for the measured denominators): HBM3e 8 TB/s,
# dense bf16 tensor 2.25 PFLOP/s
SPEC = {"hbm_gbs": 8000.0, "bf16_tflops": 2250.0}
# the five configurations of the metric (config 5 as its two GEMMs), measured
# in one process: the headline workload with its end-to-end and CPU legs,
# the others as records of the same line
CONFIG_SET = ("gemv", "layer", "cfg_decode", "concurrent", "adapter", "qkv_prefill")
# layers of a 26-layer workload whose outputs the oracle samples
ORACLE_LAYERS = (0, 12, 25)


class Timed:
    """One workload measured on this rank: device time of `steps` back-to-back
    steps, clocks, and (headline only) the end-to-end time."""

    def __init__(self, **kw):
        self.__dict__.update(kw)


def _barrier(world):
    import torch
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()


def time_workload(q4, G, tensor: bool, steps: int, warmup: int, soak: float, world: int, no_graphs: bool,
                  min_ms: float = 0.0):
    """Warm up, soak for `soak` seconds, then time `steps` steps (at least
    enough for `min_ms` of device time when min_ms > 0) back to back between
    one pair of CUDA events on the launching stream.  Returns (ms_total,
    steps, clocks summary, launch description)."""
    import torch
    stream = torch.cuda.current_stream()
    with ClockSampler(torch.cuda.current_device()) as clocks:
        for i in range(warmup):
            G.launch(q4, i)
        _barrier(world)
        t_end = time.time() + soak
        i = 0
        while time.time() < t_end:
            for _ in range(16):
                G.launch(q4, i)
                i += 1
            torch.cuda.synchronize()
        _barrier(world)
        # the steps replay CUDA graphs of a whole cycle of operand copies (the
        # library's own launches captured: the X conversion and GEMM of a
        # tensor-core step, the one grouped launch of a decode step, whose
        # programmatic dependent launch edges the graph keeps), so that the
        # host's enqueue cost stays off the device's critical path
        # tensor-core steps run pipelined (each step's X conversion on a side
        # stream beside the previous step's GEMM), captured at least 12 steps
        # to a graph so that few conversions fall on a replay boundary
        cycle = len(G.sets) * (max(1, -(-12 // len(G.sets))) if G.pipelined else 1)
        step_fn = G.launch_pipelined if G.pipelined else G.launch
        graph = None
        if not no_graphs:
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                if G.pipelined:
                    G.begin_pipeline()
                for k in range(cycle):
                    step_fn(q4, k)
            torch.cuda.synchronize()

        def run_steps(n):
            k = 0
            while graph is not None and k + cycle <= n:
                graph.replay()
                k += cycle
            if k < n and G.pipelined:
                G.begin_pipeline()
            for j in range(k, n):
                step_fn(q4, j)

        run_steps(max(warmup, cycle if graph is not None else 0))
        _barrier(world)
        if min_ms > 0:
            # the same step count on every rank: from a short trial, maxed over ranks
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            run_steps(cycle if graph is not None else 8)
            e1.record(stream)
            _barrier(world)
            per = max_over_ranks([e0.elapsed_time(e1) / (cycle if graph is not None else 8)], world, "cuda")[0]
            steps = max(steps, int(min_ms / max(per, 1e-4)) + 1)
            if graph is not None:
                steps = -(-steps // cycle) * cycle
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        _barrier(world)
        t0.record(stream)
        run_steps(steps)
        t1.record(stream)
        _barrier(world)
    launch = (f"CUDA graph replay of cycles of {cycle} steps (the library's own launches inside)"
              if graph is not None else "eager, programmatic dependent launch")
    if G.pipelined:
        launch += ("; each step's X converted to fp16 (q4_0_prepare_x) on a second stream while the previous "
                   "step's tensor-core GEMM (q4_0_gemm_prepared) runs, two conversion buffers")
    del graph
    return t0.elapsed_time(t1), steps, clocks.summary(), launch


def e2e_overlapped(q4, G, steps: int, warmup: int, world: int):
    """End to end through the public API: every step copies its X from pinned
    host memory to the device, runs the step's grouped / workspace GEMMs and
    copies its Y back to pinned host memory.  The copies run on two copy
    streams and the GEMMs on the launching stream, with X and Y double
    buffered on the device, so that the H2D of step k+1 and the D2H of step
    k-1 overlap the GEMMs of step k (one cudaMemcpyAsync per buffer and
    direction).  Returns (ms for `steps` steps, h2d bytes, d2h bytes)."""
    import torch
    main = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    xb = [torch.empty_like(G.xbufs[0]) for _ in range(2)]
    yb = [torch.empty_like(G.ybufs[0]) for _ in range(2)]
    hx = torch.empty(G.xbufs[0].shape, dtype=G.xbufs[0].dtype, pin_memory=True).copy_(G.xbufs[0].cpu())
    hy = [torch.empty(G.ybufs[0].shape, dtype=G.ybufs[0].dtype, pin_memory=True) for _ in range(2)]
    # problem arrays of (operand copy c, buffer slot b): the weights rotate
    # as in the device-timed steps, X and Y live in the slot's buffers
    arrays = {}
    for c, (probs, _) in enumerate(G.sets):
        for b in range(2):
            xs, ys = G.views(xb[b], yb[b])
            arrays[c, b] = [(W, xs[i], ys[i], M, N, K) for i, (W, X, Y, M, N, K) in enumerate(probs)]
    small_arrs = {key: q4.make_problems([p[i] for i in G.small]) for key, p in arrays.items()}
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    recorded = [False, False]

    def step(k):
        c, b = k % len(G.sets), k & 1
        with torch.cuda.stream(s_in):
            if recorded[b]:
                s_in.wait_event(ev_done[b])      # step k-2 has read X[b]
            xb[b].copy_(hx, non_blocking=True)
            ev_in[b].record(s_in)
        main.wait_event(ev_in[b])
        if recorded[b]:
            main.wait_event(ev_out[b])           # step k-2's Y[b] has reached the host
        if G.small:
            q4.q4_0_gemm_grouped(small_arrs[c, b], len(G.small))
        for i in G.large:
            W, X, Y, M, N, K = arrays[c, b][i]
            q4.q4_0_gemm_ws(W, X, Y, M, N, K, G.ws)
        ev_done[b].record(main)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_done[b])
            hy[b].copy_(yb[b], non_blocking=True)
            ev_out[b].record(s_out)
        recorded[b] = True

    for k in range(warmup):
        step(k)
    _barrier(world)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(main)
    s_in.wait_event(e0)
    for k in range(steps):
        step(k)
    for b in range(2):
        main.wait_event(ev_out[b])
    e1.record(main)
    _barrier(world)
    return e0.elapsed_time(e1), hx.numel() * hx.element_size(), hy[0].numel() * hy[0].element_size()


def e2e_serial(q4, G, steps: int, warmup: int, world: int):
    """End to end for the fused-epilogue workload (its outputs are not the
    plain Y buffers): X in, the step, Y out, all on the launching stream."""
    import torch
    main = torch.cuda.current_stream()
    hx = torch.empty(G.xbufs[0].shape, dtype=G.xbufs[0].dtype, pin_memory=True).copy_(G.xbufs[0].cpu())
    hy = [torch.empty(y.shape, dtype=y.dtype, pin_memory=True) for y in G.outputs(0)]

    def step(k):
        G.xbufs[k % len(G.sets)].copy_(hx, non_blocking=True)
        G.launch(q4, k)
        for Y, h in zip(G.outputs(k), hy):
            h.copy_(Y, non_blocking=True)

    for k in range(warmup):
        step(k)
    _barrier(world)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(main)
    for k in range(steps):
        step(k)
    e1.record(main)
    _barrier(world)
    return e0.elapsed_time(e1), hx.numel() * hx.element_size(), sum(h.numel() * h.element_size() for h in hy)


def sampled_linears(wl):
    """Indices of the linears the oracle samples: all of them, or those of
    layers ORACLE_LAYERS for the 26-layer workloads."""
    if len(wl.linears) > 16:
        return [i for i, l in enumerate(wl.linears) if l.layer in ORACLE_LAYERS]
    return list(range(len(wl.linears)))


def pack_on_host(wl, seed, which=None):
    """The oracle's own packing of the seeded codes and scales of the linears
    `which` (default all): [(index, W_host, X_host)]."""
    import oracle
    o = oracle.get()
    which = range(len(wl.linears)) if which is None else which
    return o, [(i, o.pack(wl.linears[i].codes(seed), wl.linears[i].scales(seed)), wl.linears[i].x(seed))
               for i in which]


def oracle_error(q4, G, wl, host, samples: int = 48, seed: int = 7):
    """max |Y_gpu - Y_oracle| / (1e-3 * sum_k |x w| + 1e-6) over `samples`
    seeded output positions (the last row and column always among them) of
    each sampled linear, on operand copy 0 after one more step."""
    import torch
    if G.fused_arrs:
        return None, "fused epilogues: checked by the GPU tests, not here"
    o, packed = host
    if G.pipelined:   # the path the timed steps take
        G.begin_pipeline()
        G.launch_pipelined(q4, 0)
    else:
        G.launch(q4, 0)
    torch.cuda.synchronize()
    outs = G.outputs(0)
    rng = np.random.default_rng(seed)
    worst, n = 0.0, 0
    for i, W_host, X_host in packed:
        lin = wl.linears[i]
        ms = rng.integers(0, lin.M, size=samples)
        ns = rng.integers(0, lin.N, size=samples)
        ms[0], ns[0] = lin.M - 1, lin.N - 1
        Y_or, B_or = o.gemm_sampled(W_host, X_host, lin.M, lin.N, lin.K, ms, ns)
        got = outs[i].cpu().numpy().astype(np.float64)[ms, ns]
        worst = max(worst, float(np.max(np.abs(got - Y_or) / (1e-3 * B_or + 1e-6))))
        n += samples
    return worst, f"{n} outputs of {len(packed)} GEMM(s) (operand copy 0)"


def build_record(name, wl, tensor, ms_total, steps, world, clock, launch, peaks, G):
    kernel, src = DOMINANT[name]
    launch_avg_ms = ms_total / steps
    if tensor:
        unit, per_step = "TFLOP/s", wl.flops
        value = whole_job_rate(per_step, steps, world, ms_total) / 1e12
        achieved = per_step / (launch_avg_ms * 1e-3) / 1e12
        # the steps run back to back after a soak, under the power cap: the
        # sustained GEMM figure is the matching denominator
        peak, spec, bound = peaks["bf16_tflops_sustained"], SPEC["bf16_tflops"], "tensor"
        peak_src = peaks["source"] + " (sustained bf16 GEMM, same rate as fp16)"
    else:
        unit, per_step = "GB/s", wl.hbm_bytes
        value = whole_job_rate(per_step, steps, world, ms_total) / 1e9
        achieved = per_step / (launch_avg_ms * 1e-3) / 1e9
        peak, spec, bound = peaks["hbm_gbs"], SPEC["hbm_gbs"], "hbm"
        peak_src = peaks["source"] + " (STREAM-style copy)"
    return {
        "value": round(value, 2), "unit": unit, "ms_per_step": round(launch_avg_ms, 5), "steps": steps,
        "gpu_launches": steps * launches_per_step(name, wl),
        "config": {"workload": f"{wl.name}: {wl.description}", "gemms_per_step": len(wl.linears),
                   "bytes_per_step": wl.hbm_bytes, "flops_per_step": wl.flops,
                   "l2": (f"inputs larger than L2: {len(G.sets)} rotating copies of the step's operands = "
                          f"{len(G.sets) * G.operand_bytes / 1e6:.0f} MB > L2 ({L2_BYTES / 2**20:.0f} MiB)"),
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
        "launch": launch,
        "roofline": {"bound": bound, "kernel": kernel, "achieved": round(achieved, 2), "peak": peak, "unit": unit,
                     "frac": round(achieved / peak, 4), "peak_source": peak_src,
                     "spec_peak": spec, "frac_of_spec": round(achieved / spec, 4),
                     "traffic": recorded_traffic(name), "algorithmic_per_step": per_step,
                     "dominant_launches_per_step": dominant_launches_per_step(wl),
                     "algorithmic_per_launch": round(per_step / dominant_launches_per_step(wl))},
        "clocks": clock,
    }


def stream_ceiling(q4, world: int, reps: int = 10):
    """The read-only ceiling of the decode kernels' weight stream on this GPU:
    q4_0_stream_read (the same TMA boxes and per-SM ring, no arithmetic)
    over a 1 GiB Q4_0 matrix (K = 3072), `reps` reads back to back, timed
    with CUDA events.  Returns GB/s of weight bytes."""
    import torch
    K = 3072
    row = K // 32 * 18
    N = ((1 << 30) // row) // 128 * 128
    W = torch.zeros(N * row, dtype=torch.uint8, device="cuda")
    cs = torch.zeros(1, dtype=torch.int32, device="cuda")
    for _ in range(3):
        q4.q4_0_stream_read(W, N, K, cs)
    _barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        q4.q4_0_stream_read(W, N, K, cs)
    e1.record()
    _barrier(world)
    ms = max_over_ranks([e0.elapsed_time(e1)], world, "cuda")[0]
    del W
    return {"value": round(N * row * reps / (ms * 1e-3) / 1e9, 1), "unit": "GB/s", "bytes_per_read": N * row,
            "what": f"q4_0_stream_read of a {N} x {K} Q4_0 matrix ({N * row / 2**30:.2f} GiB), {reps} reads "
                    "back to back: the decode kernels' TMA weight stream with no arithmetic"}


def run_ours(args, rank: int, world: int):
    import torch
    import bit_weight_only_matmul_b200 as q4

    peaks = measured_peaks()
    names = [args.workload] + ([n for n in CONFIG_SET if n != args.workload] if not args.only else [])
    wcache = {}
    records = {}
    line = None
    q4.q4_0_device_error(clear=True)
    for name in names:
        headline = name == args.workload
        if args.layers and headline:
            wl = workloads.workload(name, layers=list(range(args.layers)))
            wl.description += f" -- first {args.layers} layer(s) only, a profiling case"
        else:
            wl = workloads.workload(name)
        tensor = name in TENSOR_WORKLOADS
        copies = rotating_copies(wl)
        log(f"[rank {rank}] building {wl.name}: {len(wl.linears)} GEMMs x {copies} copies, "
            f"{wl.hbm_bytes / 1e6:.1f} MB per step")
        G = GpuWorkload(q4, wl, copies, workloads.SEED + 1000 * rank, wcache)
        if headline:
            ms_total, steps, clock, launch = time_workload(q4, G, tensor, args.steps, args.warmup, args.soak, world,
                                                           args.no_graphs)
        else:
            # enough steps for at least 20 ms of device time (a GEMV step is ~5 us)
            ms_total, steps, clock, launch = time_workload(q4, G, tensor, args.steps, args.warmup,
                                                           min(args.soak, 0.5), world, args.no_graphs, min_ms=20.0)
        dev_err = q4.q4_0_device_error(clear=True)
        if dev_err:
            raise RuntimeError(f"device error word {dev_err:#x} after the timed region of {name}")
        ms_total = max_over_ranks([ms_total], world, "cuda")[0]
        rec = build_record(name, wl, tensor, ms_total, steps, world, clock, launch, peaks, G)
        if headline:
            if G.fused_arrs:
                e2e_ms, h2d, d2h = e2e_serial(q4, G, args.steps, args.warmup, world)
            else:
                e2e_ms, h2d, d2h = e2e_overlapped(q4, G, args.steps, args.warmup, world)
            e2e_ms = max_over_ranks([e2e_ms], world, "cuda")[0]
            per = wl.flops if tensor else wl.hbm_bytes
            e2e_value = whole_job_rate(per, args.steps, world, e2e_ms) / (1e12 if tensor else 1e9)
            rec["e2e"] = {"value": round(e2e_value, 2), "unit": rec["unit"], "h2d_bytes_per_step": h2d,
                          "d2h_bytes_per_step": d2h,
                          "copies": "H2D and D2H on two copy streams, X and Y double-buffered on the device"
                                    if not G.fused_arrs else "serial on the launching stream"}
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            # the oracle leg: a bounded, timed sample of the same workload on
            # the host (the CPU baseline), whose values also give the GPU
            # result's worst error over the method's tolerance
            host = pack_on_host(wl, workloads.SEED, sampled_linears(wl))
            rec["max_err_over_bound"], rec["oracle_sample"] = oracle_error(q4, G, wl, host)
            budget = args.cpu_seconds if headline else args.cpu_seconds / 6
            rec["cpu_baseline"] = cpu_baseline(wl, tensor, budget_s=budget, host=host)
            if headline:
                rec["cpu_baseline_all_cores"] = cpu_baseline_all_cores(wl, tensor, budget_s=budget / 2, host=host)
        records[name] = rec
        if headline:
            line = rec
        del G
        torch.cuda.empty_cache()
    del wcache
    ceiling = stream_ceiling(q4, world)
    for r in records.values():
        if r["roofline"]["bound"] == "hbm":
            r["roofline"]["frac_of_stream_ceiling"] = round(r["roofline"]["achieved"] / ceiling["value"], 4)
    if rank != 0:
        return None
    out = {
        "metric": METRIC,
        "value": line["value"],
        "unit": line["unit"],
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": line["ms_per_step"],
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": ("bf16 x q4_0 -> fp32" if args.workload not in TENSOR_WORKLOADS
                  else "fp16 x fp16(q4_0) -> fp32"),
        "data": "synthetic (seeded Philox; codes U{0..15}, d = fp16(|N(0,1)|*0.002+1e-4), X bf16 N(0,1))",
        "config": line["config"],
        "launch": line["launch"],
        "roofline": line["roofline"],
        "e2e": line["e2e"],
        "gpu_launches": line["gpu_launches"],
        "clocks": line["clocks"],
        "stream_ceiling": ceiling,
    }
    for key in ("max_err_over_bound", "oracle_sample", "cpu_baseline", "cpu_baseline_all_cores"):
        if key in line:
            out[key] = line[key]
    if len(records) > 1:
        out["configs"] = {n: {k: v for k, v in r.items() if k not in ("cpu_baseline_all_cores",)}
                          for n, r in records.items()}
    return out


# --------------------------------------------------------------------------- the utilities

def util_setup(q4, name: str, seed: int):
    """Device buffers of one utility workload and a launch per step.  Returns
    (launch(k), bytes per step, e2e step(k), h2d bytes, d2h bytes)."""
    import torch
    if name == "embed":
        V, D, T = workloads.EMBED_VOCAB, workloads.EMBED_DIM, workloads.EMBED_TOKENS
        W = torch.empty(q4.q4_0_bytes(V, D), dtype=torch.uint8, device="cuda")
        rows = 8192
        for r0 in range(0, V, rows):   # the table, packed on the GPU from seeded codes and scales, in slices
            codes = torch.from_numpy(workloads.gen_codes(rows, D, seed, layer=r0 // rows)).cuda()
            scales = torch.from_numpy(workloads.gen_scales(rows, D, seed, layer=r0 // rows).view(np.int16)).cuda()
            q4.q4_0_pack(codes, scales, W[r0 * (D // 32) * 18:(r0 + rows) * (D // 32) * 18], rows, D)
        # 32 id sets: a set's rows come back after 31 other steps (1.8 GB of traffic), not from L2
        ids = [torch.from_numpy(workloads.gen_ids(T, V, seed, stream=i)).cuda() for i in range(32)]
        outs = [torch.empty((T, D), device="cuda") for _ in range(2)]
        hid = torch.empty(T, dtype=torch.int32, pin_memory=True).copy_(ids[0].cpu())
        hout = torch.empty((T, D), dtype=torch.float32, pin_memory=True)

        def launch(k):
            q4.q4_0_gather(W, ids[k % len(ids)], outs[k % 2], T, V, D)

        def e2e(k):
            ids[k % len(ids)].copy_(hid, non_blocking=True)
            launch(k)
            hout.copy_(outs[k % 2], non_blocking=True)

        return launch, T * (D // 32 * 18 + 4 + 4 * D), e2e, T * 4, T * D * 4
    N, K = workloads.QUANT_N, workloads.QUANT_K
    Xs = [torch.from_numpy(workloads.gen_weights(N, K, seed, stream=i)).cuda() for i in range(2)]
    Ws = [torch.empty(q4.q4_0_bytes(N, K), dtype=torch.uint8, device="cuda") for _ in range(2)]
    hx = torch.empty((N, K), dtype=torch.float32, pin_memory=True).copy_(Xs[0].cpu())
    hw = torch.empty(q4.q4_0_bytes(N, K), dtype=torch.uint8, pin_memory=True)

    def launch(k):
        q4.q4_0_quantize(Xs[k % 2], Ws[k % 2], N, K)

    def e2e(k):
        Xs[k % 2].copy_(hx, non_blocking=True)
        launch(k)
        hw.copy_(Ws[k % 2], non_blocking=True)

    return launch, N * K * 4 + q4.q4_0_bytes(N, K), e2e, N * K * 4, q4.q4_0_bytes(N, K)


def util_cpu_sample(name: str, budget_s: float):
    """The oracle on a host-generated sample of the same workload; returns
    (GB/s, sample description)."""
    import oracle
    o = oracle.get()
    if name == "embed":
        V, D = 2048, workloads.EMBED_DIM
        W = o.pack(workloads.gen_codes(V, D), workloads.gen_scales(V, D))
        ids = workloads.gen_ids(256, V)
        per = len(ids) * (D // 32 * 18 + 4 + 4 * D)
        fn = lambda: o.gather_f32(W, ids, V, D)   # noqa: E731
        what = f"gather of 256 random rows of a {V} x {D} table per pass"
    else:
        X = workloads.gen_weights(64, workloads.QUANT_K)
        per = X.size * 4 + X.size // 32 * 18
        fn = lambda: o.quantize(X)   # noqa: E731
        what = f"quantize of a 64 x {workloads.QUANT_K} slice per pass"
    t0, reps = time.perf_counter(), 0
    while True:
        fn()
        reps += 1
        if time.perf_counter() - t0 > budget_s or reps >= 2000:
            break
    dt = time.perf_counter() - t0
    return per * reps / dt / 1e9, f"{reps} passes: {what}, {dt:.1f} s, scaled by bytes"


def run_util(args, rank: int, world: int):
    import torch
    import bit_weight_only_matmul_b200 as q4
    launch, step_bytes, e2e, h2d, d2h = util_setup(q4, args.workload, workloads.SEED + 1000 * rank)
    stream = torch.cuda.current_stream()

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
        torch.cuda.synchronize()

    q4.q4_0_device_error(clear=True)
    with ClockSampler(torch.cuda.current_device()) as clocks:
        for k in range(args.warmup):
            launch(k)
        barrier()
        t_end, k = time.time() + args.soak, 0
        while time.time() < t_end:
            for _ in range(8):
                launch(k)
                k += 1
            torch.cuda.synchronize()
        barrier()
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for k in range(args.steps):
            launch(k)
        t1.record(stream)
        barrier()
    ms_total = t0.elapsed_time(t1)
    if q4.q4_0_device_error(clear=True):
        raise RuntimeError("device error word set after the timed region")
    for k in range(args.warmup):
        e2e(k)
    barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for k in range(args.steps):
        e2e(k)
    e1.record(stream)
    barrier()
    e2e_ms = e0.elapsed_time(e1)
    ms_total, e2e_ms = max_over_ranks([ms_total, e2e_ms], world, "cuda")
    if rank != 0:
        return None
    peaks = measured_peaks()
    kernel, _ = UTIL_KERNELS[args.workload]
    value = whole_job_rate(step_bytes, args.steps, world, ms_total) / 1e9
    line = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_total / args.steps, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "q4_0 -> fp32" if args.workload == "embed" else "fp32 -> q4_0",
        "data": "synthetic (seeded Philox)",
        "config": {"workload": f"{args.workload}: {workloads.UTIL_WORKLOADS[args.workload]}",
                   "bytes_per_step": step_bytes,
                   "l2": ("inputs larger than L2: the 216 MiB table gathered through 32 rotating id sets"
                          if args.workload == "embed" else
                          "inputs larger than L2: 2 rotating 201 MB fp32 weight buffers"),
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU", "launch": "eager"},
        "roofline": {"bound": "hbm", "kernel": kernel, "achieved": round(value / world, 2),
                     "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": round(value / world / peaks["hbm_gbs"], 4),
                     "peak_source": peaks["source"] + " (STREAM-style copy)",
                     "traffic": recorded_traffic(args.workload), "algorithmic_per_launch": step_bytes},
        "e2e": {"value": round(whole_job_rate(step_bytes, args.steps, world, e2e_ms) / 1e9, 2), "unit": "GB/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": args.steps,
        "clocks": clocks.summary(),
    }
    if not args.no_cpu_baseline and world == 1:
        v, what = util_cpu_sample(args.workload, args.cpu_seconds)
        line["cpu_baseline"] = {"value": v, "unit": "GB/s", "cores": 1, "kind": "oracle", "sample": what}
    return line


def run_util_reference(args, rank: int):
    if rank != 0:
        return None
    for _ in range(args.warmup):
        util_cpu_sample(args.workload, 0.0)
    t0 = time.perf_counter()
    vals = [util_cpu_sample(args.workload, 0.0) for _ in range(args.steps)]
    dt = time.perf_counter() - t0
    value = statistics.mean(v for v, _ in vals)
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic (seeded Philox)",
            "config": {"workload": f"{args.workload}: {workloads.UTIL_WORKLOADS[args.workload]}",
                       "parallelism": "one host core"},
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": 1, "kind": "oracle", "sample": vals[0][1]},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def max_over_ranks(values, world: int, device: str):
    """Element-wise max of per-rank timings (every rank gets the result)."""
    if world <= 1:
        return [float(v) for v in values]
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def whole_job_rate(units_per_rank_step: float, steps: int, world: int, max_ms: float) -> float:
    """Work of all ranks (weak scaling: every rank does the same work) over
    the slowest rank's time, per second."""
    return world * steps * units_per_rank_step / (max_ms * 1e-3)


def dominant_launches_per_step(wl) -> int:
    """Launches of the step's dominant kernel: the decode launches of a
    decode step (see launches_per_step), or one tensor-core GEMM per M > 32
    problem.  `achieved` is the step's algorithmic work over the step's
    time, i.e. the mean over these launches, which run back to back."""
    big = sum(1 for l in wl.linears if l.M > 32)
    if big:
        return big
    n8 = sum(1 for l in wl.linears if l.M <= 8)
    n32 = sum(1 for l in wl.linears if 8 < l.M <= 32)
    return -(-n8 // 128) + -(-n32 // 64)


LAYERED_WORKLOADS = ("cfg_decode", "concurrent", "flow_head")


def launches_per_step(name, wl) -> int:
    """Kernel launches of one step.  A grouped call runs its M <= 8 problems
    in launches of up to 128 (one alone: the one-problem kernel) and its
    8 < M <= 32 problems in launches of up to 64 (their X tensor maps fill
    the kernel parameters); each M > 32 problem is two launches (the fp16
    conversion of X, then the tensor-core GEMM)."""
    n8 = sum(1 for l in wl.linears if l.M <= 8)
    n32 = sum(1 for l in wl.linears if 8 < l.M <= 32)
    return -(-n8 // 128) + -(-n32 // 64) + 2 * sum(1 for l in wl.linears if l.M > 32)


# --------------------------------------------------------------------------- the oracle as a baseline

def oracle_step_sample(o, wl, packed, row_stride: int):
    """The oracle on every `row_stride`-th output column (all rows of X) of
    the sampled GEMMs `packed` = [(index, W_host, X_host)].  Returns the
    fraction of the whole step's multiply-adds covered."""
    covered = 0
    for i, W, X in packed:
        lin = wl.linears[i]
        ns = np.arange(0, lin.N, row_stride)
        ms = np.repeat(np.arange(lin.M), len(ns))
        o.gemm_sampled(W, X, lin.M, lin.N, lin.K, ms, np.tile(ns, lin.M))
        covered += len(ns) * lin.M * lin.K
    return covered / sum(l.M * l.N * l.K for l in wl.linears)


def _sample_macs(wl, packed):
    return sum(wl.linears[i].M * wl.linears[i].N * wl.linears[i].K for i, _, _ in packed)


def _what(wl, packed):
    if len(packed) == len(wl.linears):
        return f"all {len(wl.linears)} GEMMs"
    return f"the {len(packed)} GEMMs of layers {', '.join(map(str, ORACLE_LAYERS))}"


def cpu_baseline(wl, tensor: bool, budget_s: float, host=None):
    o, packed = host or pack_on_host(wl, workloads.SEED, sampled_linears(wl))
    # choose a column stride so one sampled pass is about budget/3 seconds (46 M MAC/s measured on one core)
    stride = max(1, int(round(_sample_macs(wl, packed) / (4.5e7 * budget_s / 3))))
    frac_total, t0 = 0.0, time.perf_counter()
    reps = 0
    while True:
        frac_total += oracle_step_sample(o, wl, packed, stride)
        reps += 1
        if time.perf_counter() - t0 > budget_s * 0.66 or reps >= 50:
            break
    dt = time.perf_counter() - t0
    if tensor:
        value, unit = frac_total * wl.flops / dt / 1e12, "TFLOP/s"
    else:
        value, unit = frac_total * wl.hbm_bytes / dt / 1e9, "GB/s"
    return {"value": value, "unit": unit, "cores": 1, "kind": "oracle",
            "sample": f"{reps} pass(es) over every {stride}th output column of {_what(wl, packed)} "
                      f"({frac_total / reps:.4f} of a step each), {dt:.1f} s, scaled to whole steps"}


def oracle_step_sample_threads(o, wl, packed, row_stride: int, pool, threads: int):
    """oracle_step_sample with the sampled columns dealt round-robin to
    `threads` host threads of `pool` (the oracle's C routine releases the
    GIL).  Returns the fraction of the whole step covered."""
    def part(t):
        covered = 0
        for i, W, X in packed:
            lin = wl.linears[i]
            ns = np.arange(0, lin.N, row_stride)[t::threads]
            if len(ns):
                o.gemm_sampled(W, X, lin.M, lin.N, lin.K, np.repeat(np.arange(lin.M), len(ns)), np.tile(ns, lin.M))
            covered += len(ns) * lin.M * lin.K
        return covered

    return sum(pool.map(part, range(threads))) / sum(l.M * l.N * l.K for l in wl.linears)


def cpu_baseline_all_cores(wl, tensor: bool, budget_s: float, threads: int = 0, host=None):
    """The same oracle, partitioned over the output columns across all host
    cores: one host thread per core."""
    import concurrent.futures
    threads = threads or os.cpu_count() or 1
    o, packed = host or pack_on_host(wl, workloads.SEED, sampled_linears(wl))
    stride = max(1, int(round(_sample_macs(wl, packed) / (4.5e7 * threads * budget_s / 3))))
    frac_total, reps, t0 = 0.0, 0, time.perf_counter()
    with concurrent.futures.ThreadPoolExecutor(max_workers=threads) as pool:
        while True:
            frac_total += oracle_step_sample_threads(o, wl, packed, stride, pool, threads)
            reps += 1
            if time.perf_counter() - t0 > budget_s * 0.66 or reps >= 50:
                break
    dt = time.perf_counter() - t0
    if tensor:
        value, unit = frac_total * wl.flops / dt / 1e12, "TFLOP/s"
    else:
        value, unit = frac_total * wl.hbm_bytes / dt / 1e9, "GB/s"
    return {"value": value, "unit": unit, "cores": threads, "kind": "oracle",
            "sample": f"{reps} pass(es) over every {stride}th output column of {_what(wl, packed)}, "
                      f"columns dealt round-robin to {threads} threads ({frac_total / reps:.4f} of a step "
                      f"each), {dt:.1f} s, scaled to whole steps"}


def run_reference(args, rank: int, world: int):
    if rank != 0:
        return None
    wl = workloads.workload(args.workload)
    tensor = args.workload in TENSOR_WORKLOADS
    import concurrent.futures
    o, packed = pack_on_host(wl, workloads.SEED, sampled_linears(wl))
    threads = os.cpu_count() or 1
    # each step: a sample of about 1 s of oracle work on every host core
    stride = max(1, int(round(_sample_macs(wl, packed) / (4.5e7 * threads))))
    with concurrent.futures.ThreadPoolExecutor(max_workers=threads) as pool:
        for _ in range(args.warmup):
            oracle_step_sample_threads(o, wl, packed, stride, pool, threads)
        t0 = time.perf_counter()
        frac = 0.0
        for _ in range(args.steps):
            frac += oracle_step_sample_threads(o, wl, packed, stride, pool, threads)
        dt = time.perf_counter() - t0
    if tensor:
        value, unit = frac * wl.flops / dt / 1e12, "TFLOP/s"
    else:
        value, unit = frac * wl.hbm_bytes / dt / 1e9, "GB/s"
    sample = (f"each step = every {stride}th output column of {_what(wl, packed)} "
              f"({frac / args.steps:.4f} of a step), columns dealt round-robin to {threads} host threads, "
              f"scaled to whole steps")
    return {
        "impl": "reference",
        "metric": METRIC,
        "value": value,
        "unit": unit,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic (seeded Philox, same workload recipe)",
        # the same keys as the GPU arm's config; l2 and parallelism say what this arm does
        "config": {"workload": f"{wl.name}: {wl.description}", "gemms_per_step": len(wl.linears),
                   "bytes_per_step": wl.hbm_bytes, "flops_per_step": wl.flops,
                   "l2": "host run: the oracle reads its operands from host memory",
                   "parallelism": f"{threads} host threads"},
        "cpu_baseline": {"value": value, "unit": unit, "cores": threads, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# --------------------------------------------------------------------------- main

def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=workloads.WORKLOADS + list(UTIL_KERNELS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="CPU-baseline budget (rank 0, N=1)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graphs", action="store_true",
                    help="launch each timed step eagerly instead of replaying its captured CUDA graph")
    ap.add_argument("--only", action="store_true",
                    help="measure the named workload alone (no records of the other configurations)")
    ap.add_argument("--soak", type=float, default=1.0,
                    help="seconds of untimed load after warm-up, so the clock sampler sees the GPU busy "
                         "(0 for short profiling runs)")
    ap.add_argument("--layers", type=int, default=0,
                    help="with --only: keep the first N layers of a 26-layer workload (small cases for ncu "
                         "captures; the line then describes that case, not the configuration)")
    args = ap.parse_args(argv)
    if args.layers and (not args.only or args.workload not in LAYERED_WORKLOADS):
        ap.error("--layers needs --only and one of " + ", ".join(LAYERED_WORKLOADS))
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        log(f"note: --gpus {args.gpus} but WORLD_SIZE={world}; using WORLD_SIZE")

    if args.impl == "reference":
        if args.workload in UTIL_KERNELS:
            line = run_util_reference(args, rank)
        else:
            line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return 0

    import torch
    torch.cuda.set_device(local)
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    try:
        line = run_util(args, rank, world) if args.workload in UTIL_KERNELS else run_ours(args, rank, world)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    if line is not None:
        print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
