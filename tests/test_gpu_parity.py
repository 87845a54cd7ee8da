"""GPU parity: the CUDA library, called through its C ABI, against the
float64 oracle on the same seeded inputs.

Bars: pack and dequant bit-exact; GEMM within |Y - Y_exact| <= 1e-3 *
sum_k |x_k w_k| + 1e-6 per element (the method's stated tolerance)."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.gpu_helpers import (build_workload, check_built, check_gemm, dev, host_u16, no_device_error,
                               pack_on_gpu)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q4():
    import bit_weight_only_matmul_b200 as q4
    torch.cuda.init()
    q4.q4_0_force_path(0)
    yield q4
    q4.q4_0_force_path(0)


@pytest.fixture(autouse=True)
def _clean_error_word(q4):
    q4.q4_0_device_error(clear=True)
    yield
    no_device_error(q4)


def rand_inputs(rng, M, N, K, x_sigma=1.0):
    codes = rng.integers(0, 16, size=(N, K), dtype=np.uint8)
    scales = (np.abs(rng.standard_normal(size=(N, K // 32))) * 0.002 + 1e-4).astype(np.float16).view(np.uint16)
    X = workloads.fp32_to_bf16_bits(rng.standard_normal(size=(M, K)).astype(np.float32) * np.float32(x_sigma))
    return codes, scales, X


# --------------------------------------------------------------------------- pack / dequant

@pytest.mark.parametrize("N,K", [(1, 32), (3, 64), (5, 96), (64, 3072), (17, 8192), (33, 5120), (7, 288)])
def test_pack_bit_exact(q4, N, K):
    rng = np.random.default_rng(N * 131 + K)
    codes = rng.integers(0, 256, size=(N, K), dtype=np.uint8)     # high nibble must be ignored
    scales = rng.integers(0, 65536, size=(N, K // 32), dtype=np.uint16)
    W = pack_on_gpu(q4, codes, scales).cpu().numpy()
    assert np.array_equal(W, oracle.get().pack(codes & 15, scales).reshape(-1))


@pytest.mark.parametrize("N,K", [(1, 32), (4, 64), (9, 160), (64, 3072), (5, 8192)])
def test_dequant_bit_exact(q4, N, K):
    rng = np.random.default_rng(N * 7 + K)
    W = rng.integers(0, 256, size=(N, K // 32 * 18), dtype=np.uint8)   # every scale bit pattern, NaN/Inf too
    out = torch.empty((N, K), dtype=torch.float32, device="cuda")
    q4.q4_0_dequant(dev(W), out, N, K)
    got = out.cpu().numpy()
    ref = oracle.get().dequant_f32(W, N, K)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan].view(np.uint32), ref[~nan].view(np.uint32))


def test_pack_dequant_roundtrip_config_shape(q4):
    lin = workloads.workload("gemv").linears[0]
    codes, scales = lin.codes(), lin.scales()
    W = pack_on_gpu(q4, codes, scales)
    out = torch.empty((lin.N, lin.K), dtype=torch.float32, device="cuda")
    q4.q4_0_dequant(W, out, lin.N, lin.K)
    ref = oracle.get().dequant_f32(oracle.get().pack(codes, scales), lin.N, lin.K)
    assert np.array_equal(out.cpu().numpy().view(np.uint32), ref.view(np.uint32))


# --------------------------------------------------------------------------- GEMM, small shapes

def run_gemm(q4, M, N, K, seed=0, path=0, x_sigma=1.0):
    rng = np.random.default_rng(seed * 1000003 + M * 10007 + N * 101 + K)
    codes, scales, X = rand_inputs(rng, M, N, K, x_sigma)
    W = pack_on_gpu(q4, codes, scales)
    Y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    q4.q4_0_force_path(path)
    try:
        q4.q4_0_gemm(W, dev(X), Y, M, N, K)
    finally:
        q4.q4_0_force_path(0)
    Y_or, B_or = oracle.get().gemm(oracle.get().pack(codes, scales), X, M, N, K)
    return check_gemm(Y.cpu().numpy(), Y_or, B_or, f"M={M} N={N} K={K} path={path}")


@pytest.mark.parametrize("M", [1, 2, 3, 7, 8, 9, 16, 17, 31, 32])
@pytest.mark.parametrize("N,K", [(17, 256), (100, 1280), (129, 3072)])
def test_decode_path(q4, M, N, K):
    run_gemm(q4, M, N, K)


@pytest.mark.parametrize("M,N,K", [(1, 1, 256), (2, 16, 512), (1, 3, 8192), (32, 33, 2048), (5, 257, 768)])
def test_decode_path_ragged(q4, M, N, K):
    run_gemm(q4, M, N, K)


@pytest.mark.parametrize("M,N,K", [(1, 5, 32), (3, 9, 96), (2, 31, 160), (8, 64, 288), (33, 40, 64),
                                   (64, 17, 256), (100, 24, 320)])
def test_generic_shapes(q4, M, N, K):
    run_gemm(q4, M, N, K)


@pytest.mark.parametrize("M,N,K", [(1, 100, 1024), (4, 65, 3072), (32, 48, 512)])
def test_forced_generic_matches(q4, M, N, K):
    run_gemm(q4, M, N, K, path=q4.PATH_GENERIC)


@pytest.mark.parametrize("M,N,K", [(33, 64, 512), (64, 128, 1024), (128, 256, 3072), (200, 96, 320)])
def test_prefill_shapes(q4, M, N, K):
    run_gemm(q4, M, N, K, x_sigma=0.5)


def test_outlier_rows_decode(q4):
    # 3 of 32 rows of X scaled x8, as in the concurrent-decode workload
    M, N, K = 32, 96, 1024
    rng = np.random.default_rng(5)
    codes, scales, _ = rand_inputs(rng, M, N, K)
    X = workloads.gen_x(M, K, seed=77, outlier_rows=3)
    W = pack_on_gpu(q4, codes, scales)
    Y = torch.empty((M, N), dtype=torch.float32, device="cuda")
    q4.q4_0_gemm(W, dev(X), Y, M, N, K)
    Y_or, B_or = oracle.get().gemm(oracle.get().pack(codes, scales), X, M, N, K)
    check_gemm(Y.cpu().numpy(), Y_or, B_or, "outliers")


def test_special_structures(q4):
    """All-8 codes give exactly zero; one off-centre nibble gives (c-8)*d*x."""
    M, N, K = 2, 40, 512
    o = oracle.get()
    rng = np.random.default_rng(9)
    X = workloads.fp32_to_bf16_bits(rng.standard_normal(size=(M, K)).astype(np.float32) * 50)
    scales = np.full((N, K // 32), np.float16(3.5).view(np.uint16), np.uint16)
    codes = np.full((N, K), 8, np.uint8)
    for path in (0, q4.PATH_GENERIC):
        Y = torch.full((M, N), 1.0, dtype=torch.float32, device="cuda")
        q4.q4_0_force_path(path)
        q4.q4_0_gemm(pack_on_gpu(q4, codes, scales), dev(X), Y, M, N, K)
        q4.q4_0_force_path(0)
        assert torch.count_nonzero(Y).item() == 0
    codes[7, 300] = 13
    codes[39, 511] = 0
    Y = torch.empty((M, N), dtype=torch.float32, device="cuda")
    q4.q4_0_gemm(pack_on_gpu(q4, codes, scales), dev(X), Y, M, N, K)
    Y_or, B_or = o.gemm(o.pack(codes, scales), X, M, N, K)
    check_gemm(Y.cpu().numpy(), Y_or, B_or, "single nibble")


# --------------------------------------------------------------------------- empty inputs

def test_empty_problems(q4):
    Y = torch.full((3, 5), 7.0, device="cuda")
    q4.q4_0_gemm(None, None, Y, 0, 5, 64)
    q4.q4_0_gemm(None, None, Y, 3, 0, 64)
    assert torch.all(Y == 7.0)
    q4.q4_0_gemm(None, None, Y, 3, 5, 0)      # empty sum: zeros
    torch.cuda.synchronize()
    assert torch.all(Y == 0.0)


# --------------------------------------------------------------------------- grouped launch

def test_grouped_mixed_shapes(q4):
    o = oracle.get()
    rng = np.random.default_rng(21)
    shapes = [(1, 70, 512), (2, 33, 3072), (32, 40, 1024), (1, 5, 96), (48, 64, 256), (0, 5, 64), (3, 9, 0),
              (9, 300, 2048)]
    probs, refs, Ys = [], [], []
    for (M, N, K) in shapes:
        if M == 0 or K == 0:
            Y = torch.full((max(M, 1), N), 5.0, device="cuda")
            probs.append((None, None, Y, M, N, K))
            refs.append(None)
            Ys.append(Y)
            continue
        codes, scales, X = rand_inputs(rng, M, N, K)
        Y = torch.full((M, N), float("nan"), device="cuda")
        probs.append((pack_on_gpu(q4, codes, scales), dev(X), Y, M, N, K))
        refs.append(o.gemm(o.pack(codes, scales), X, M, N, K))
        Ys.append(Y)
    q4.q4_0_gemm_grouped(probs)
    for (M, N, K), Y, ref in zip(shapes, Ys, refs):
        if ref is None:
            assert torch.all(Y == (5.0 if M == 0 else 0.0))
        else:
            check_gemm(Y.cpu().numpy(), ref[0], ref[1], f"grouped {M}x{N}x{K}")


def test_non_default_stream(q4):
    M, N, K = 2, 64, 1024
    rng = np.random.default_rng(3)
    codes, scales, X = rand_inputs(rng, M, N, K)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        W = pack_on_gpu(q4, codes, scales)
        Y = torch.empty((M, N), device="cuda")
        q4.q4_0_gemm(W, dev(X), Y, M, N, K)
    s.synchronize()
    o = oracle.get()
    Y_or, B_or = o.gemm(o.pack(codes, scales), X, M, N, K)
    check_gemm(Y.cpu().numpy(), Y_or, B_or, "side stream")


# --------------------------------------------------------------------------- workload shapes

def test_gemv_workload_full(q4):
    b = build_workload(q4, workloads.workload("gemv"), full_oracle=True)
    q4.q4_0_gemm_grouped(b.problems())
    check_built(b, "gemv")


def test_layer_workload_full(q4):
    b = build_workload(q4, workloads.workload("layer"), full_oracle=True)
    q4.q4_0_gemm_grouped(b.problems())
    check_built(b, "layer")


@pytest.mark.parametrize("M,N,K", [(256, 128, 256), (300, 200, 512), (33, 1, 256), (512, 384, 2048)])
def test_tensor_core_path(q4, M, N, K):
    run_gemm(q4, M, N, K, x_sigma=0.5)


@pytest.mark.parametrize("name", ["adapter", "qkv_prefill"])
def test_prefill_workload_sampled(q4, name):
    b = build_workload(q4, workloads.workload(name), samples=2000)
    q4.q4_0_gemm_grouped(b.problems())
    check_built(b, name)


@pytest.mark.parametrize("M,N,K", [(1, 100, 1024), (2, 129, 3072), (8, 64, 512), (16, 33, 2048)])
def test_forced_warp_mma_decode(q4, M, N, K):
    run_gemm(q4, M, N, K, path=q4.PATH_DECODE_EXACT)


@pytest.mark.parametrize("M,N,K", [
    (1, 3072, 3072),   # 24 items: clusters of 4-8 cut them into pieces
    (2, 129, 3072),    # one 12-stage item in pieces
    (8, 1000, 1792),   # eight 7-stage items
    (5, 257, 768),     # ragged N, 3-stage items
    (3, 20000, 512),   # more items than SMs: plain mode
])
def test_forced_decode_256k_stages(q4, M, N, K):
    """The M <= 32 kernel (256-k stages) forced for M <= 8, where it runs one
    n tile with two stages per ring slot, in plain and cluster split modes."""
    run_gemm(q4, M, N, K, path=q4.PATH_DECODE)


def test_forced_decode_256k_stages_layer(q4):
    """A decoder layer (216 items) on the same kernel: split mode in pairs."""
    b = build_workload(q4, workloads.workload("layer"), full_oracle=True)
    q4.q4_0_force_path(q4.PATH_DECODE)
    try:
        q4.q4_0_gemm_grouped(b.problems())
    finally:
        q4.q4_0_force_path(0)
    check_built(b, "layer, 256-k stage kernel")


@pytest.mark.parametrize("name,layers", [("cfg_decode", [0, 13, 25]), ("concurrent", [0, 25]), ("flow_head", None)])
def test_decode_workloads_sampled(q4, name, layers):
    b = build_workload(q4, workloads.workload(name, layers=layers), samples=400)
    q4.q4_0_gemm_grouped(b.problems())
    check_built(b, name)


def test_split_mode_mixed_stage_counts(q4):
    """M <= 8 with between 148 and 1024 items runs in clusters of two CTAs:
    items longer than the mean load (K = 8192 here, 32 stages; and the odd
    7424, 29 stages, whose first half gets the extra stage) are halved
    between the pair, the rest (8-, 3- and 1-stage items) stay whole."""
    o = oracle.get()
    rng = np.random.default_rng(31)
    shapes = [(3, 12800, 2048), (3, 2900, 8192), (2, 300, 7424), (1, 3000, 256), (8, 1000, 768)]
    probs, refs, Ys = [], [], []
    for (M, N, K) in shapes:
        codes, scales, X = rand_inputs(rng, M, N, K)
        Y = torch.full((M, N), float("nan"), device="cuda")
        probs.append((pack_on_gpu(q4, codes, scales), dev(X), Y, M, N, K))
        refs.append(o.gemm(o.pack(codes, scales), X, M, N, K))
        Ys.append(Y)
    for rep in range(2):
        for Y in Ys:
            Y.fill_(float("nan"))
        q4.q4_0_gemm_grouped(probs)
        for (M, N, K), Y, (Y_or, B_or) in zip(shapes, Ys, refs):
            check_gemm(Y.cpu().numpy(), Y_or, B_or, f"split mode M={M} N={N} K={K} rep {rep}")
    no_device_error(q4)


@pytest.mark.parametrize("M,N,K", [
    (1, 100, 8192),    # one 32-stage item: eight pieces of 4 (cluster of 8)
    (2, 128, 1536),    # one 6-stage item: six pieces of 1 (cluster of 6; 8 would leave it whole)
    (3, 90, 1024),     # one 4-stage item: four pieces of 1 (cluster of 4)
    (8, 1000, 1792),   # eight 7-stage items in pieces of 2, 2, 2, 1 (clusters of 4)
])
def test_split_mode_few_items(q4, M, N, K):
    """M <= 8 with fewer items than SMs: each item is cut into pieces on the
    CTAs of one cluster (4, 6 or 8 of them), whose partial sums meet in rank
    0 of the cluster.  The second call reuses the schedule of the first."""
    rng = np.random.default_rng(M * 7 + N + K)
    codes, scales, X = rand_inputs(rng, M, N, K)
    W = pack_on_gpu(q4, codes, scales)
    o = oracle.get()
    Y_or, B_or = o.gemm(o.pack(codes, scales), X, M, N, K)
    Y = torch.empty((M, N), dtype=torch.float32, device="cuda")
    for rep in range(2):
        Y.fill_(float("nan"))
        q4.q4_0_gemm(W, dev(X), Y, M, N, K)
        check_gemm(Y.cpu().numpy(), Y_or, B_or, f"few items M={M} N={N} K={K} rep {rep}")
    no_device_error(q4)


def test_split_mode_few_items_grouped(q4):
    """A grouped launch of 14 items: the 32-, 8- and 7-stage items are cut
    into pieces (the 7-stage ones unevenly), the 1-stage items stay whole,
    and every problem's rows land in its own Y."""
    o = oracle.get()
    rng = np.random.default_rng(47)
    shapes = [(2, 1000, 1792), (5, 300, 256), (8, 129, 8192), (1, 1, 2048)]
    probs, refs, Ys = [], [], []
    for (M, N, K) in shapes:
        codes, scales, X = rand_inputs(rng, M, N, K)
        Y = torch.full((M, N), float("nan"), device="cuda")
        probs.append((pack_on_gpu(q4, codes, scales), dev(X), Y, M, N, K))
        refs.append(o.gemm(o.pack(codes, scales), X, M, N, K))
        Ys.append(Y)
    for rep in range(2):
        for Y in Ys:
            Y.fill_(float("nan"))
        q4.q4_0_gemm_grouped(probs)
        for (M, N, K), Y, (Y_or, B_or) in zip(shapes, Ys, refs):
            check_gemm(Y.cpu().numpy(), Y_or, B_or, f"few items grouped M={M} N={N} K={K} rep {rep}")
    no_device_error(q4)


def test_grouped_many_problems_mixed_m(q4):
    """70 problems, one of them at M = 16: the M <= 8 problems go to the
    M <= 8 kernel in one launch (split mode: fewer than 1024 items), the
    M = 16 problem to the M <= 32 kernel."""
    o = oracle.get()
    rng = np.random.default_rng(53)
    shapes = [(1 + i % 8, 8 + (7 * i) % 33, 256 * (2 + i % 3)) for i in range(69)] + [(16, 24, 256)]
    probs, refs, Ys = [], [], []
    for (M, N, K) in shapes:
        codes, scales, X = rand_inputs(rng, M, N, K)
        Y = torch.full((M, N), float("nan"), device="cuda")
        probs.append((pack_on_gpu(q4, codes, scales), dev(X), Y, M, N, K))
        refs.append(o.gemm(o.pack(codes, scales), X, M, N, K))
        Ys.append(Y)
    q4.q4_0_gemm_grouped(probs)
    for (M, N, K), Y, (Y_or, B_or) in zip(shapes, Ys, refs):
        check_gemm(Y.cpu().numpy(), Y_or, B_or, f"many problems M={M} N={N} K={K}")
    no_device_error(q4)


def test_grouped_many_problems_m_over_8(q4):
    """70 problems at 8 < M <= 32 in one grouped call: their X tensor maps fill
    the kernel parameters at 64 problems, so the call runs as two launches of
    the M <= 32 kernel (64 and 6 problems, sorted by K), each at the n-tile
    count of its largest M."""
    o = oracle.get()
    rng = np.random.default_rng(59)
    shapes = [(9 + (5 * i) % 24, 8 + (7 * i) % 41, 256 * (1 + i % 3)) for i in range(70)]
    probs, refs, Ys = [], [], []
    for (M, N, K) in shapes:
        codes, scales, X = rand_inputs(rng, M, N, K)
        Y = torch.full((M, N), float("nan"), device="cuda")
        probs.append((pack_on_gpu(q4, codes, scales), dev(X), Y, M, N, K))
        refs.append(o.gemm(o.pack(codes, scales), X, M, N, K))
        Ys.append(Y)
    q4.q4_0_gemm_grouped(probs)
    for (M, N, K), Y, (Y_or, B_or) in zip(shapes, Ys, refs):
        check_gemm(Y.cpu().numpy(), Y_or, B_or, f"many problems M={M} N={N} K={K}")
    no_device_error(q4)


def test_grouped_call_replays_from_cuda_graph(q4):
    """A grouped decode call captured in a CUDA graph (after one eager call,
    which does the per-device set-up) replays to the eager call's bits."""
    rng = np.random.default_rng(41)
    shapes = [(1, 5120, 3072), (1, 3072, 3072), (1, 16384, 3072), (1, 3072, 8192)]   # one decoder layer
    probs, Ys = [], []
    for (M, N, K) in shapes:
        codes, scales, X = rand_inputs(rng, M, N, K)
        Y = torch.full((M, N), float("nan"), device="cuda")
        probs.append((pack_on_gpu(q4, codes, scales), dev(X), Y, M, N, K))
        Ys.append(Y)
    arr = q4.make_problems(probs)
    q4.q4_0_gemm_grouped(arr, len(probs))
    torch.cuda.synchronize()
    eager = [Y.clone() for Y in Ys]
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        q4.q4_0_gemm_grouped(arr, len(probs))
    for rep in range(2):
        for Y in Ys:
            Y.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        for Y, E in zip(Ys, eager):
            assert torch.equal(Y, E)
    no_device_error(q4)


def test_plain_mode_many_items(q4):
    """More than 1024 items at M <= 8: one CTA per item, boustrophedon deal."""
    b = build_workload(q4, workloads.workload("cfg_decode", layers=[0, 1, 2, 3, 4]), samples=200)
    assert sum((N + 127) // 128 for (_, N, _) in b.shapes) > 1024
    q4.q4_0_gemm_grouped(b.problems())
    check_built(b, "cfg_decode 5 layers")
    no_device_error(q4)


@pytest.mark.parametrize("M,N,K", [(64, 128, 512), (300, 200, 1024), (4096, 256, 768)])
def test_workspace_path_matches(q4, M, N, K):
    """q4_0_gemm_ws (X converted to fp16 once, in the workspace) gives the
    oracle's answer within tolerance and q4_0_gemm's answer bit for bit."""
    rng = np.random.default_rng(M + N + K)
    codes, scales, X = rand_inputs(rng, M, N, K, 0.5)
    W = pack_on_gpu(q4, codes, scales)
    Xd = dev(X)
    ws_bytes = q4.q4_0_gemm_workspace_size(M, N, K)
    assert ws_bytes == ((M * K * 2 + 255) // 256) * 256
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    Y1 = torch.full((M, N), float("nan"), device="cuda")
    Y2 = torch.full((M, N), float("nan"), device="cuda")
    q4.q4_0_gemm_ws(W, Xd, Y1, M, N, K, ws)
    q4.q4_0_gemm(W, Xd, Y2, M, N, K)
    torch.cuda.synchronize()
    assert torch.equal(Y1, Y2)
    Y_or, B_or = oracle.get().gemm(oracle.get().pack(codes, scales), X, M, N, K)
    check_gemm(Y1.cpu().numpy(), Y_or, B_or, "workspace path")


def test_workspace_too_small_falls_back(q4):
    M, N, K = 64, 64, 512
    rng = np.random.default_rng(4)
    codes, scales, X = rand_inputs(rng, M, N, K, 0.5)
    W = pack_on_gpu(q4, codes, scales)
    ws = torch.empty(16, dtype=torch.uint8, device="cuda")
    Y = torch.empty((M, N), device="cuda")
    q4.q4_0_gemm_ws(W, dev(X), Y, M, N, K, ws)
    Y_or, B_or = oracle.get().gemm(oracle.get().pack(codes, scales), X, M, N, K)
    check_gemm(Y.cpu().numpy(), Y_or, B_or, "small workspace")
    assert q4.q4_0_gemm_workspace_size(8, 64, 512) == 0


def test_forced_tensor_path_small_m_small_workspace(q4):
    """The tensor-core path forced for M <= 32 with a workspace smaller than
    the fp16 copy of X (M*K*2 bytes): the library must not convert into it
    (that would write past its end); it converts X tile by tile instead, and
    the bytes just past the workspace stay untouched."""
    M, N, K = 24, 200, 1024
    rng = np.random.default_rng(5)
    codes, scales, X = rand_inputs(rng, M, N, K, 0.5)
    W = pack_on_gpu(q4, codes, scales)
    small = 256                                  # < M*K*2 = 48 KiB
    guard = torch.full((small + 4096,), 0x5A, dtype=torch.uint8, device="cuda")
    Y = torch.full((M, N), float("nan"), device="cuda")
    q4.q4_0_force_path(q4.PATH_TENSOR)
    try:
        q4.q4_0_gemm_ws(W, dev(X), Y, M, N, K, guard[:small])
    finally:
        q4.q4_0_force_path(0)
    torch.cuda.synchronize()
    assert bool((guard[small:] == 0x5A).all()), "bytes past the workspace were written"
    Y_or, B_or = oracle.get().gemm(oracle.get().pack(codes, scales), X, M, N, K)
    check_gemm(Y.cpu().numpy(), Y_or, B_or, "forced tensor path, M <= 32, small workspace")


@pytest.mark.parametrize("M,N,K", [(1, 100, 1024), (2, 129, 3072), (16, 33, 2048), (32, 70, 512)])
def test_forced_tmem_decode(q4, M, N, K):
    run_gemm(q4, M, N, K, path=q4.PATH_DECODE_TMEM)


@pytest.mark.parametrize("name", ["concurrent", "cfg_decode"])
def test_forced_tmem_decode_workload(q4, name):
    b = build_workload(q4, workloads.workload(name, layers=[0, 1]), samples=300)
    q4.q4_0_force_path(q4.PATH_DECODE_TMEM)
    try:
        q4.q4_0_gemm_grouped(b.problems())
    finally:
        q4.q4_0_force_path(0)
    check_built(b, f"{name} layers 0-1, tcgen05 decode")
    no_device_error(q4)


def test_decode_vocab_sized_gemv_sampled(q4):
    """M=1 against a 131072-row weight (an LM-head / embedding-table shape): 1024
    items, the edge of split mode, checked at sampled outputs including the
    last row."""
    M, N, K = 1, 131072, 3072
    rng = np.random.default_rng(12)
    o = oracle.get()
    codes = workloads.gen_codes(N, K, layer=77)
    scales = workloads.gen_scales(N, K, layer=77)
    X = workloads.gen_x(M, K, layer=77)
    W_host = o.pack(codes, scales)
    W = torch.from_numpy(W_host.reshape(-1)).cuda()
    del codes
    Y = torch.full((M, N), float("nan"), device="cuda")
    q4.q4_0_gemm(W, dev(X), Y, M, N, K)
    ns = np.concatenate([rng.integers(0, N, 300), [0, N - 1, 128 * 1023, 128 * 1023 + 127]])
    ms = np.zeros_like(ns)
    Y_or, B_or = o.gemm_sampled(W_host, X, M, N, K, ms, ns)
    check_gemm(Y.cpu().numpy()[ms, ns], Y_or, B_or, "vocab-sized gemv")
    no_device_error(q4)


@pytest.mark.parametrize("M,N,K", [(1, 200, 1024), (2, 300, 3072), (24, 129, 512), (64, 256, 512)])
def test_subnormal_scales(q4, M, N, K):
    """Scales in the fp16 subnormal range: every (q - 8) * d is then an exact
    fp16 subnormal, on the decode and the tensor-core paths alike."""
    rng = np.random.default_rng(M * 13 + N + K)
    codes = rng.integers(0, 16, size=(N, K), dtype=np.uint8)
    scales = rng.integers(1, 0x400, size=(N, K // 32)).astype(np.uint16)   # positive subnormals
    scales[::3] |= 0x8000                                                   # and negative ones
    X = workloads.fp32_to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32))
    W = pack_on_gpu(q4, codes, scales)
    Y = torch.full((M, N), float("nan"), device="cuda")
    q4.q4_0_gemm(W, dev(X), Y, M, N, K)
    o = oracle.get()
    Y_or, B_or = o.gemm(o.pack(codes, scales), X, M, N, K)
    check_gemm(Y.cpu().numpy(), Y_or, B_or, "subnormal scales")
    no_device_error(q4)
