"""The N > 1 plumbing of bench.py on CPU: two gloo ranks (the path runs
replicas, so the only cross-rank steps are the barrier and the max-over-ranks
reduction of the timings)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        # rank r is slower by r ms; the reduction must return the slowest
        local = [10.0 + rank, 20.0 + 2 * rank, 0.5 + rank]
        dist.barrier()
        got = bench.max_over_ranks(local, world, "cpu")
        out[rank] = got
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert res[0] == res[1] == [11.0, 22.0, 1.5]


def test_whole_job_rate_is_weak_scaling():
    import bench
    # 2 ranks x 10 steps x 1e9 bytes in 20 ms (slowest rank) = 1e12 B/s
    assert bench.whole_job_rate(1e9, 10, 2, 20.0) == pytest.approx(1e12)
    assert bench.max_over_ranks([1.0, 2.0], 1, "cpu") == [1.0, 2.0]


def test_workload_byte_accounting():
    """The bench's algorithmic bytes: every weight byte once plus X and Y once;
    the fused layer writes half of the gate/up output and reads two residuals."""
    import workloads
    layer = workloads.workload("layer")
    W = sum(l.N * (l.K // 32) * 18 for l in layer.linears)
    XY = sum(l.M * l.K * 2 + l.M * l.N * 4 for l in layer.linears)
    assert layer.hbm_bytes == W + XY == 56768512
    fused = workloads.workload("layer_fused")
    assert fused.hbm_bytes == layer.hbm_bytes - 1 * 8192 * 4 + 2 * 1 * 3072 * 4
    cfg = workloads.workload("cfg_decode")
    assert cfg.hbm_bytes == 1479761920
    assert workloads.workload("adapter").flops == 2 * 4096 * 3072 * 5120


def test_rotating_copies_exceed_l2():
    """Every bench workload rotates enough copies of its step's operands that
    they come from HBM: more than twice the 126 MiB L2 in all, as the bench
    line's `l2` field states (a 3072 x 3072 GEMV needs 50 copies)."""
    import bench
    import workloads
    for name in workloads.WORKLOADS:
        wl = workloads.workload(name)
        step = wl.weight_bytes + sum(l.act_bytes for l in wl.linears)
        c = bench.rotating_copies(wl)
        assert c * step >= 2 * bench.L2_BYTES, name
        assert c == 1 or (c - 1) * step < 2 * bench.L2_BYTES, name   # no more than needed
    assert bench.rotating_copies(workloads.workload("gemv")) == 50
    assert bench.rotating_copies(workloads.workload("layer")) == 5


def test_cpu_baselines_single_and_all_cores():
    """The bench's two oracle baselines on a GEMV sample: one host core, and
    the columns dealt to two threads (the oracle call releases the GIL)."""
    import bench
    import workloads
    wl = workloads.workload("gemv")
    host = bench.pack_on_host(wl, workloads.SEED)
    one = bench.cpu_baseline(wl, False, 0.5, host=host)
    two = bench.cpu_baseline_all_cores(wl, False, 0.5, threads=2, host=host)
    assert one["cores"] == 1 and two["cores"] == 2
    assert one["unit"] == two["unit"] == "GB/s"
    assert one["value"] > 0 and two["value"] > 0
    assert one["kind"] == two["kind"] == "oracle"


def test_launch_counts_follow_the_library_chunks():
    """gpu_launches: a grouped call runs its M <= 8 problems in launches of up
    to 128 and its 8 < M <= 32 problems in launches of up to 64 (the X tensor
    maps fill the kernel parameters); an M > 32 problem is the X conversion
    plus the tensor-core GEMM.  The M = 32 decode step (104 GEMMs) is two
    launches, and `achieved` is the mean over them."""
    import bench
    import workloads
    want = {"gemv": (1, 1), "layer": (1, 1), "layer_fused": (1, 1), "cfg_decode": (1, 1),
            "concurrent": (2, 2), "flow_head": (1, 1), "adapter": (2, 1), "qkv_prefill": (2, 1)}
    for name, (launches, dominant) in want.items():
        wl = workloads.workload(name)
        assert bench.launches_per_step(name, wl) == launches, name
        assert bench.dominant_launches_per_step(wl) == dominant, name
    # mixed shapes: 130 problems at M = 2 and 65 at M = 16 -> 2 + 2 launches
    mixed = workloads.Workload("mixed", "test", [workloads.Linear("a", 256, 256, 0, 0, 2)] * 130 +
                               [workloads.Linear("b", 256, 256, 0, 1, 16)] * 65)
    assert bench.launches_per_step("mixed", mixed) == 4


def test_layers_option_needs_a_layered_workload():
    import bench
    with pytest.raises(SystemExit):
        bench.main(["--workload", "gemv", "--only", "--layers", "2"])
    with pytest.raises(SystemExit):
        bench.main(["--workload", "concurrent", "--layers", "2"])
