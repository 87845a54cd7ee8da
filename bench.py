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

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "Q4_0 dequant-matmul HBM GB/s (M=1,2) and TFLOP/s (M>=64), % of B200 roofline"
L2_BYTES = 126 * 2**20
DEFAULT_WORKLOAD = "layer"

# kernel that dominates each workload, and the source file it lives in
DOMINANT = {
    "gemv": ("decode_mma_kernel", "q4_0_decode_mma.cu"),
    "layer": ("decode_mma_kernel", "q4_0_decode_mma.cu"),
    "cfg_decode": ("decode_mma_kernel", "q4_0_decode_mma.cu"),
    "concurrent": ("decode_mma_kernel", "q4_0_decode_mma.cu"),
    "flow_head": ("decode_mma_kernel", "q4_0_decode_mma.cu"),
    "layer_fused": ("decode_mma_kernel", "q4_0_decode_mma.cu"),
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
    summary, or None when absent or when the kernel source changed since."""
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

    def __init__(self, q4, wl: workloads.Workload, copies: int, seed: int):
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
                codes = torch.from_numpy(lin.codes(s)).cuda()
                scales = torch.from_numpy(lin.scales(s).view(np.int16)).cuda()
                W = torch.empty(q4.q4_0_bytes(lin.N, lin.K), dtype=torch.uint8, device="cuda")
                q4.q4_0_pack(codes, scales, W, lin.N, lin.K)
                del codes, scales
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


def rotating_copies(wl: workloads.Workload) -> int:
    """Copies of a step's operands that together exceed twice the L2, so
    that every step's operands come from HBM, not L2 (one decoder layer: 5; a
    3072 x 3072 GEMV: 50)."""
    step = wl.weight_bytes + sum(l.act_bytes for l in wl.linears)
    return max(1, -(-2 * L2_BYTES // max(1, step)))


def run_ours(args, rank: int, world: int):
    import torch
    import torch.distributed as dist
    import bit_weight_only_matmul_b200 as q4

    wl = workloads.workload(args.workload)
    tensor = args.workload in TENSOR_WORKLOADS
    step_bytes = wl.hbm_bytes
    step_flops = wl.flops
    copies = rotating_copies(wl)
    log(f"[rank {rank}] building {wl.name}: {len(wl.linears)} GEMMs x {copies} copies, "
        f"{step_bytes / 1e6:.1f} MB per step")
    G = GpuWorkload(q4, wl, copies, workloads.SEED + 1000 * rank)
    stream = torch.cuda.current_stream()

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    q4.q4_0_device_error(clear=True)
    with ClockSampler(torch.cuda.current_device()) as clocks:
        # warm-up: W untimed steps, then an untimed soak of about a second so
        # that the clock sampler sees the GPU under this load
        for i in range(args.warmup):
            G.launch(q4, i)
        barrier()
        t_end = time.time() + args.soak
        i = 0
        while time.time() < t_end:
            for _ in range(16):
                G.launch(q4, i)
                i += 1
            torch.cuda.synchronize()
        barrier()
        # one CUDA graph holding a whole cycle of steps (one per operand copy,
        # in order), captured after the warm-up so that the library's one-time
        # set-up has run: host launch overhead does not gate the device, and
        # consecutive kernels keep their programmatic-launch overlap
        cycle = len(G.sets)
        graph = None
        # a decode step is one launch, which the host enqueues well ahead of
        # the device and which overlaps its predecessor's tail through
        # programmatic dependent launch; graphs pay off for the tensor-core
        # steps (two launches each: X conversion, then the GEMM)
        use_graph = tensor and not args.no_graphs
        if use_graph:
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                for k in range(cycle):
                    G.launch(q4, k)
            torch.cuda.synchronize()

        def run_steps(n):
            k = 0
            while graph is not None and k + cycle <= n:
                graph.replay()
                k += cycle
            for j in range(k, n):
                G.launch(q4, j)

        run_steps(args.warmup)
        barrier()
        # timed region: exactly K steps back to back between one pair of
        # events on the launching stream (events between the steps would put
        # gaps between the kernels that a real token loop does not have)
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        barrier()
        t0.record(stream)
        run_steps(args.steps)
        t1.record(stream)
        barrier()
    ms_total = t0.elapsed_time(t1)
    dev_err = q4.q4_0_device_error(clear=True)
    if dev_err:
        raise RuntimeError(f"device error word {dev_err:#x} after the timed region")

    # end to end through the public API: host X -> device, grouped GEMM, Y -> host
    # (one pinned copy each way: a step's X and Y live in one buffer each)
    hx = [torch.empty(G.xbufs[0].shape, dtype=G.xbufs[0].dtype, pin_memory=True).copy_(G.xbufs[0].cpu())]
    outs0 = [G.ybufs[0]] if not G.fused_arrs else G.outputs(0)
    hy = [torch.empty(y.shape, dtype=y.dtype, pin_memory=True) for y in outs0]
    h2d = sum(t.numel() * t.element_size() for t in hx)
    d2h = sum(t.numel() * t.element_size() for t in hy)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)

    def e2e_step(k):
        c = k % len(G.sets)
        G.xbufs[c].copy_(hx[0], non_blocking=True)
        G.launch(q4, k)
        for Y, h in zip([G.ybufs[c]] if not G.fused_arrs else G.outputs(k), hy):
            h.copy_(Y, non_blocking=True)

    for i in range(args.warmup):
        e2e_step(i)
    barrier()
    e0.record(stream)
    for k in range(args.steps):
        e2e_step(k)
    e1.record(stream)
    barrier()
    e2e_ms = e0.elapsed_time(e1)

    ms_total, e2e_ms = max_over_ranks([ms_total, e2e_ms], world, "cuda")
    # every step is the dominant kernel's launch (plus, for M > 32, the X
    # conversion pass before it): its average duration is the step time
    launch_avg_ms = ms_total / args.steps
    clock = clocks.summary()

    if rank != 0:
        return None
    peaks = measured_peaks()
    kernel, src = DOMINANT[args.workload]
    if tensor:
        unit = "TFLOP/s"
        value = whole_job_rate(step_flops, args.steps, world, ms_total) / 1e12
        e2e_value = whole_job_rate(step_flops, args.steps, world, e2e_ms) / 1e12
        achieved = step_flops / (launch_avg_ms * 1e-3) / 1e12
        # the steps run back to back after a soak, under the power cap: the
        # sustained GEMM figure is the matching denominator
        peak = peaks["bf16_tflops_sustained"]
        bound = "tensor"
    else:
        unit = "GB/s"
        value = whole_job_rate(step_bytes, args.steps, world, ms_total) / 1e9
        e2e_value = whole_job_rate(step_bytes, args.steps, world, e2e_ms) / 1e9
        achieved = step_bytes / (launch_avg_ms * 1e-3) / 1e9
        peak = peaks["hbm_gbs"]
        bound = "hbm"
    line = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": unit,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_total / args.steps, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16 x q4_0 -> fp32" if not tensor else "fp16 x fp16(q4_0) -> fp32",
        "data": "synthetic (seeded Philox; codes U{0..15}, d = fp16(|N(0,1)|*0.002+1e-4), X bf16 N(0,1))",
        "config": {
            "workload": f"{wl.name}: {wl.description}",
            "gemms_per_step": len(wl.linears),
            "bytes_per_step": step_bytes,
            "flops_per_step": step_flops,
            "weight_copies": len(G.sets),
            "l2": (f"inputs larger than L2: {len(G.sets)} rotating copies of the step's operands = "
                   f"{len(G.sets) * G.operand_bytes / 1e6:.0f} MB > L2 ({L2_BYTES / 2**20:.0f} MiB)"),
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
            "launch": (f"CUDA graph replay of cycles of {len(G.sets)} steps (the library's own launches "
                       "inside)") if (tensor and not args.no_graphs) else "eager, programmatic dependent launch",
        },
        "roofline": {
            "bound": bound,
            "kernel": kernel,
            "achieved": round(achieved, 2),
            "peak": peak,
            "unit": unit,
            "frac": round(achieved / peak, 4),
            "peak_source": peaks["source"] + (" (sustained bf16 GEMM, same rate as fp16)" if tensor else
                                              " (STREAM-style copy)"),
            "traffic": recorded_traffic(args.workload),
            "algorithmic_per_launch": step_flops if tensor else step_bytes,
        },
        "e2e": {"value": round(e2e_value, 2), "unit": unit, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": args.steps * launches_per_step(args.workload, wl),
        "clocks": clock,
    }
    if not args.no_cpu_baseline and world == 1:
        host = pack_on_host(wl, workloads.SEED)
        line["cpu_baseline"] = cpu_baseline(wl, tensor, budget_s=args.cpu_seconds, host=host)
        line["cpu_baseline_all_cores"] = cpu_baseline_all_cores(wl, tensor, budget_s=args.cpu_seconds / 2, host=host)
    return line


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


def launches_per_step(name, wl) -> int:
    # all M <= 32 problems of a step share one launch; each M > 32 problem is
    # two (the fp16 conversion of X, then the tensor-core GEMM)
    small = any(l.M <= 32 for l in wl.linears)
    return int(small) + 2 * sum(1 for l in wl.linears if l.M > 32)


# --------------------------------------------------------------------------- the oracle as a baseline

def oracle_step_sample(o, wl, packed, row_stride: int):
    """The oracle on every `row_stride`-th output column of every GEMM of
    the step (all rows of X).  Returns the fraction of the step covered."""
    covered = 0
    for lin, (W, X) in zip(wl.linears, packed):
        ns = np.arange(0, lin.N, row_stride)
        ms = np.repeat(np.arange(lin.M), len(ns))
        o.gemm_sampled(W, X, lin.M, lin.N, lin.K, ms, np.tile(ns, lin.M))
        covered += len(ns) * lin.M * lin.K
    total = sum(l.M * l.N * l.K for l in wl.linears)
    return covered / total


def pack_on_host(wl, seed):
    import oracle
    o = oracle.get()
    return o, [(o.pack(l.codes(seed), l.scales(seed)), l.x(seed)) for l in wl.linears]


def cpu_baseline(wl, tensor: bool, budget_s: float, host=None):
    o, packed = host or pack_on_host(wl, workloads.SEED)
    total_macs = sum(l.M * l.N * l.K for l in wl.linears)
    # choose a column stride so one sampled pass is about budget/3 seconds (46 M MAC/s measured on one core)
    est_rate = 4.5e7
    stride = max(1, int(round(total_macs / (est_rate * budget_s / 3))))
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
            "sample": f"{reps} pass(es) over every {stride}th output column of all {len(wl.linears)} GEMMs "
                      f"({frac_total / reps:.4f} of a step each), {dt:.1f} s, scaled to whole steps"}


def oracle_step_sample_threads(o, wl, packed, row_stride: int, pool, threads: int):
    """oracle_step_sample with the sampled columns dealt round-robin to
    `threads` host threads of `pool` (the oracle's C routine releases the
    GIL).  Returns the fraction of the step covered."""
    def part(i):
        covered = 0
        for lin, (W, X) in zip(wl.linears, packed):
            ns = np.arange(0, lin.N, row_stride)[i::threads]
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
    o, packed = host or pack_on_host(wl, workloads.SEED)
    total_macs = sum(l.M * l.N * l.K for l in wl.linears)
    stride = max(1, int(round(total_macs / (4.5e7 * threads * budget_s / 3))))
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
            "sample": f"{reps} pass(es) over every {stride}th output column of all {len(wl.linears)} GEMMs, "
                      f"columns dealt round-robin to {threads} threads ({frac_total / reps:.4f} of a step "
                      f"each), {dt:.1f} s, scaled to whole steps"}


def run_reference(args, rank: int, world: int):
    if rank != 0:
        return None
    wl = workloads.workload(args.workload)
    tensor = args.workload in TENSOR_WORKLOADS
    import concurrent.futures
    o, packed = pack_on_host(wl, workloads.SEED)
    threads = os.cpu_count() or 1
    total_macs = sum(l.M * l.N * l.K for l in wl.linears)
    # each step: a sample of about 1 s of oracle work on every host core
    stride = max(1, int(round(total_macs / (4.5e7 * threads))))
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
    sample = (f"each step = every {stride}th output column of all {len(wl.linears)} GEMMs "
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
        "config": {"workload": f"{wl.name}: {wl.description}", "bytes_per_step": wl.hbm_bytes,
                   "flops_per_step": wl.flops, "parallelism": f"{threads} host threads"},
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
    ap.add_argument("--soak", type=float, default=1.0,
                    help="seconds of untimed load after warm-up, so the clock sampler sees the GPU busy "
                         "(0 for short profiling runs)")
    args = ap.parse_args(argv)
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
