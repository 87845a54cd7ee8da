"""The launch patterns the bench and a token loop use, against the float64
oracle: the workspace path (X converted to fp16 once, the bench's M > 32
path) at the full adapter and QKV sizes, decode launches back to back with
programmatic dependent launch where the second consumes the first's output,
and grouped calls running concurrently on two streams (the library's
per-thread and per-device host state under concurrent use)."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.gpu_helpers import build_workload, check_built, check_gemm, dev, no_device_error, pack_on_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q4():
    import bit_weight_only_matmul_b200 as q4
    q4.q4_0_force_path(q4.PATH_AUTO)
    yield q4
    q4.q4_0_force_path(q4.PATH_AUTO)


@pytest.fixture(autouse=True)
def _clean_error_word(q4):
    q4.q4_0_device_error(clear=True)
    yield
    no_device_error(q4)


def _weights(rng, N, K):
    codes = rng.integers(0, 16, size=(N, K), dtype=np.uint8)
    scales = (np.abs(rng.standard_normal((N, K // 32))) * 0.002 + 1e-4).astype(np.float16).view(np.uint16)
    return codes, scales


def _x(rng, M, K):
    return workloads.fp32_to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32))


@pytest.mark.parametrize("name", ["adapter", "qkv_prefill"])
def test_workspace_path_full_size_sampled(q4, name):
    """q4_0_gemm_ws with a full workspace, the path the bench times for
    M = 4096, at the configuration's full size: 2000 sampled outputs against
    the oracle, and bit-equal to the path that converts X tile by tile."""
    b = build_workload(q4, workloads.workload(name), samples=2000)
    (W, X, Y, M, N, K), = b.problems()
    ws = torch.empty(q4.q4_0_gemm_workspace_size(M, N, K), dtype=torch.uint8, device="cuda")
    q4.q4_0_gemm_ws(W, X, Y, M, N, K, ws)
    check_built(b, f"{name} through the workspace")
    Y2 = torch.full_like(Y, float("nan"))
    q4.q4_0_gemm(W, X, Y2, M, N, K)
    torch.cuda.synchronize()
    assert torch.equal(Y, Y2)


@pytest.mark.parametrize("M", [1, 2, 16])
def test_back_to_back_residual_chain(q4, M):
    """Two fused decode launches queued back to back on one stream: the
    second's residual R is the first's output Y1 (Y2 = X2 W2^T + Y1).  With
    programmatic dependent launch the second grid starts while the first
    drains and must still read the finished Y1."""
    rng = np.random.default_rng(40 + M)
    o = oracle.get()
    N, K = 3072, 3072
    (c1, s1), (c2, s2) = _weights(rng, N, K), _weights(rng, N, K)
    X1, X2 = _x(rng, M, K), _x(rng, M, K)
    R0 = rng.standard_normal((M, N)).astype(np.float32)
    W1, W2 = pack_on_gpu(q4, c1, s1), pack_on_gpu(q4, c2, s2)
    R0d = dev(R0)
    for rep in range(3):
        Y1 = torch.full((M, N), float("nan"), device="cuda")
        Y2 = torch.full((M, N), float("nan"), device="cuda")
        q4.q4_0_gemm_grouped_ex([(W1, dev(X1), Y1, M, N, K, R0d, q4.Q4_0_EPI_RESIDUAL)])
        q4.q4_0_gemm_grouped_ex([(W2, dev(X2), Y2, M, N, K, Y1, q4.Q4_0_EPI_RESIDUAL)])
        torch.cuda.synchronize()
        ya, ba = o.gemm(o.pack(c1, s1), X1, M, N, K)
        yb, bb = o.gemm(o.pack(c2, s2), X2, M, N, K)
        ref1 = ya + R0
        ref2 = yb + ref1
        t1 = 1e-3 * ba + 1e-6 + 2.0**-22 * np.abs(ref1)
        err1 = np.abs(Y1.cpu().numpy().astype(np.float64) - ref1)
        assert (err1 <= t1).all(), f"first launch: worst {float((err1 / t1).max())}"
        # the second inherits the first's error through R
        err2 = np.abs(Y2.cpu().numpy().astype(np.float64) - ref2)
        t2 = 1e-3 * bb + 1e-6 + t1 + 2.0**-22 * np.abs(ref2)
        assert (err2 <= t2).all(), f"chained launch: worst {float((err2 / t2).max())}"


def test_two_streams_concurrently(q4):
    """Two grouped calls with different shape sets on two streams, issued
    alternately so that their kernels can overlap on the device: a decode
    layer at M=2 and a set of M=1 / M=32 GEMMs; each result against the
    oracle."""
    rng = np.random.default_rng(11)
    o = oracle.get()
    sets = {
        "a": [(2, 5120, 3072), (2, 3072, 3072), (2, 3072, 8192)],
        "b": [(1, 1000, 1024), (32, 640, 2048), (7, 129, 768)],
    }
    built = {}
    for key, shapes in sets.items():
        items = []
        for (M, N, K) in shapes:
            codes, scales = _weights(rng, N, K)
            X = _x(rng, M, K)
            items.append((codes, scales, X, pack_on_gpu(q4, codes, scales), dev(X),
                          torch.full((M, N), float("nan"), device="cuda"), M, N, K))
        built[key] = items
    sa, sb = torch.cuda.Stream(), torch.cuda.Stream()
    torch.cuda.synchronize()
    for rep in range(4):
        for key, s in (("a", sa), ("b", sb)):
            with torch.cuda.stream(s):
                q4.q4_0_gemm_grouped([(W, X, Y, M, N, K) for (_, _, _, W, X, Y, M, N, K) in built[key]])
    sa.synchronize()
    sb.synchronize()
    for key, items in built.items():
        for codes, scales, X, W, Xd, Y, M, N, K in items:
            Y_or, B_or = o.gemm(o.pack(codes, scales), X, M, N, K)
            check_gemm(Y.cpu().numpy(), Y_or, B_or, f"stream {key} {M}x{N}x{K}")


@pytest.mark.parametrize("N,K", [(1, 256), (129, 3072), (3072, 8192), (1000, 5120)])
def test_stream_read_checksum(q4, N, K):
    """The streaming-ceiling instrument reads every byte of W once: its XOR of
    W's 32-bit words equals the same XOR on the host (rows past N count as
    zero)."""
    rng = np.random.default_rng(N + K)
    W = rng.integers(0, 256, size=q4.q4_0_bytes(N, K), dtype=np.uint8)
    cs = torch.zeros(1, dtype=torch.int32, device="cuda")
    q4.q4_0_stream_read(dev(W), N, K, cs)
    torch.cuda.synchronize()
    want = int(np.bitwise_xor.reduce(W.view(np.uint32)))
    assert int(cs.cpu().numpy().view(np.uint32)[0]) == want


@pytest.mark.parametrize("M,N,K", [(512, 18944, 256), (176, 300, 512), (177, 128, 1024), (4096, 256, 768),
                                   (300, 19000, 768), (4096, 2368, 5120), (1000, 5000, 256)])
def test_tensor_core_tiles_sampled(q4, M, N, K):
    """The tensor-core kernel on one and several activation tiles (ragged last
    tiles included, a grid of two tiles per SM, tile counts that leave a
    part-filled last wave: 298, 304 and 160 tiles): sampled outputs against
    the oracle, through both the in-kernel and the workspace conversion of X,
    which must agree bit for bit."""
    rng = np.random.default_rng(M + N + K)
    codes, scales = _weights(rng, N, K)
    X = _x(rng, M, K)
    W = pack_on_gpu(q4, codes, scales)
    Xd = dev(X)
    o = oracle.get()
    W_host = o.pack(codes, scales)
    ms = rng.integers(0, M, size=1500)
    ns = rng.integers(0, N, size=1500)
    ms[:4] = [0, M - 1, M - 1, min(M - 1, 175)]
    ns[:4] = [0, N - 1, 0, N - 1]
    Y_or, B_or = o.gemm_sampled(W_host, X, M, N, K, ms, ns)
    Y1 = torch.full((M, N), float("nan"), device="cuda")
    q4.q4_0_gemm(W, Xd, Y1, M, N, K)
    ws = torch.empty(q4.q4_0_gemm_workspace_size(M, N, K), dtype=torch.uint8, device="cuda")
    Y2 = torch.full((M, N), float("nan"), device="cuda")
    q4.q4_0_gemm_ws(W, Xd, Y2, M, N, K, ws)
    torch.cuda.synchronize()
    check_gemm(Y1.cpu().numpy()[ms, ns], Y_or, B_or, f"tensor core {M}x{N}x{K}")
    assert torch.equal(Y1, Y2)


def test_repeated_runs_bit_identical(q4):
    """Twenty runs of each path on the same inputs give the same bits: the
    tensor-core kernel with in-kernel and with workspace conversion of X (which
    must also agree with each other), and a grouped decode layer at M = 1 and
    M = 16 launched three times back to back per run.  A consumer that lets a
    copy engine refill a shared-memory slot before its own loads of the slot
    have completed shows up here as a few wrong rows in one tile of one run."""
    rng = np.random.default_rng(77)
    M, N, K = 4096, 3072, 5120
    codes, scales = _weights(rng, N, K)
    W, X = pack_on_gpu(q4, codes, scales), dev(_x(rng, M, K))
    ws = torch.empty(q4.q4_0_gemm_workspace_size(M, N, K), dtype=torch.uint8, device="cuda")
    ref = torch.full((M, N), float("nan"), device="cuda")
    q4.q4_0_gemm_ws(W, X, ref, M, N, K, ws)
    Y = torch.empty_like(ref)
    for rep in range(20):
        for use_ws in (False, True):
            Y.fill_(float("nan"))
            if use_ws:
                q4.q4_0_gemm_ws(W, X, Y, M, N, K, ws)
            else:
                q4.q4_0_gemm(W, X, Y, M, N, K)
            torch.cuda.synchronize()
            assert torch.equal(Y, ref), f"tensor core, run {rep}, workspace {use_ws}"
    shapes = [(5120, 3072), (3072, 3072), (16384, 3072), (3072, 8192)]
    for Md in (1, 16):
        probs = []
        for (Nd, Kd) in shapes:
            c, s = _weights(rng, Nd, Kd)
            probs.append((pack_on_gpu(q4, c, s), dev(_x(rng, Md, Kd)),
                          torch.full((Md, Nd), float("nan"), device="cuda"), Md, Nd, Kd))
        q4.q4_0_gemm_grouped(probs)
        torch.cuda.synchronize()
        refs = [p[2].clone() for p in probs]
        for rep in range(20):
            for p in probs:
                p[2].fill_(float("nan"))
            for _ in range(3):
                q4.q4_0_gemm_grouped(probs)
            torch.cuda.synchronize()
            for i, (p, r) in enumerate(zip(probs, refs)):
                assert torch.equal(p[2], r), f"decode M={Md} problem {i}, run {rep}"


@pytest.mark.parametrize("M,N,K", [(4096, 3072, 5120), (300, 19000, 768), (33, 200, 512), (8, 256, 1024)])
def test_prepared_path(q4, M, N, K):
    """q4_0_prepare_x then q4_0_gemm_prepared, the conversion on a second
    stream ordered by an event: for M > 32 bit-equal to q4_0_gemm_ws, for any
    M within the oracle's bound on sampled outputs (M <= 32 runs the
    tensor-core kernel too)."""
    rng = np.random.default_rng(M + 3 * N + K)
    codes, scales = _weights(rng, N, K)
    Xh = _x(rng, M, K)
    W, X = pack_on_gpu(q4, codes, scales), dev(Xh)
    xh = torch.empty(q4.q4_0_prepared_x_bytes(M, K), dtype=torch.uint8, device="cuda")
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        q4.q4_0_prepare_x(X, M, K, xh)
        done = torch.cuda.Event()
        done.record()
    torch.cuda.current_stream().wait_event(done)
    Y = torch.full((M, N), float("nan"), device="cuda")
    q4.q4_0_gemm_prepared(W, xh, Y, M, N, K)
    torch.cuda.synchronize()
    if M > 32:
        ws = torch.empty(q4.q4_0_gemm_workspace_size(M, N, K), dtype=torch.uint8, device="cuda")
        Y2 = torch.full((M, N), float("nan"), device="cuda")
        q4.q4_0_gemm_ws(W, X, Y2, M, N, K, ws)
        torch.cuda.synchronize()
        assert torch.equal(Y, Y2)
    o = oracle.get()
    ms = rng.integers(0, M, size=800)
    ns = rng.integers(0, N, size=800)
    ms[0], ns[0] = M - 1, N - 1
    Y_or, B_or = o.gemm_sampled(o.pack(codes, scales), Xh, M, N, K, ms, ns)
    check_gemm(Y.cpu().numpy()[ms, ns], Y_or, B_or, f"prepared {M}x{N}x{K}")


def test_prepared_pipeline_over_steps(q4):
    """The bench's pipeline for tensor-core steps: step k's X converted on a
    side stream into buffer k % 2 once the GEMM of step k - 2 (the buffer's
    last reader) is done, the GEMM of step k on the launching stream after
    its conversion; six steps over three operand sets, each output bit-equal
    to q4_0_gemm_ws on the same operands."""
    rng = np.random.default_rng(21)
    M, N, K = 600, 1536, 1024
    sets = []
    for _ in range(3):
        codes, scales = _weights(rng, N, K)
        sets.append((pack_on_gpu(q4, codes, scales), dev(_x(rng, M, K))))
    ws = torch.empty(q4.q4_0_gemm_workspace_size(M, N, K), dtype=torch.uint8, device="cuda")
    refs = []
    for W, X in sets:
        Y = torch.empty((M, N), device="cuda")
        q4.q4_0_gemm_ws(W, X, Y, M, N, K, ws)
        refs.append(Y)
    torch.cuda.synchronize()
    xh = [torch.empty(q4.q4_0_prepared_x_bytes(M, K), dtype=torch.uint8, device="cuda") for _ in range(2)]
    ys = [torch.full((M, N), float("nan"), device="cuda") for _ in range(6)]
    side, main = torch.cuda.Stream(), torch.cuda.current_stream()
    side.wait_stream(main)
    prep_done = [torch.cuda.Event(), torch.cuda.Event()]
    gemm_done = [torch.cuda.Event(), torch.cuda.Event()]
    for k in range(6):
        b = k % 2
        W, X = sets[k % 3]
        if k >= 2:
            side.wait_event(gemm_done[b])
        with torch.cuda.stream(side):
            q4.q4_0_prepare_x(X, M, K, xh[b])
            prep_done[b].record(side)
        main.wait_event(prep_done[b])
        q4.q4_0_gemm_prepared(W, xh[b], ys[k], M, N, K)
        gemm_done[b].record(main)
    torch.cuda.synchronize()
    for k in range(6):
        assert torch.equal(ys[k], refs[k % 3]), f"step {k}"


@pytest.mark.parametrize("M,N,K", [(1, 1, 256), (3, 2368, 512), (1, 2369, 512), (8, 4736, 768),
                                   (2, 4737, 768), (5, 300, 6144), (1, 3072, 8192),
                                   (1, 2000, 5120), (4, 3000, 2304), (6, 3000, 3072), (1, 3072, 4096)])
def test_one_problem_kernel_bounds(q4, M, N, K):
    """A lone problem at M <= 8 runs the one-problem kernel when its rows fit
    the SMs in CTAs of 16 rows (N <= 16 * 148), else of 32 (N <= 32 * 148),
    and its CTA fits in shared memory; one row more, or a K too long, takes
    the cluster path.  The CTA has 24 warps (M <= 4) or 32 (M > 4) where 16
    would leave a k-group two stages of at most 24 stage-row-tiles: here
    2000 x 5120 (16 rows a CTA, 20 stages) and 3000 x 2304 with 24, 300 x 6144
    and 3000 x 3072 with 32, 3072 x 4096 (32 stage-row-tiles) with 16.  Both
    sides of each bound against the oracle, with and without a residual (in
    place)."""
    rng = np.random.default_rng(M * 7 + N + K)
    codes, scales = _weights(rng, N, K)
    X = _x(rng, M, K)
    W, Xd = pack_on_gpu(q4, codes, scales), dev(X)
    o = oracle.get()
    ms = rng.integers(0, M, size=600)
    ns = rng.integers(0, N, size=600)
    ms[0], ns[0] = M - 1, N - 1
    Y_or, B_or = o.gemm_sampled(o.pack(codes, scales), X, M, N, K, ms, ns)
    Y = torch.full((M, N), float("nan"), device="cuda")
    q4.q4_0_gemm(W, Xd, Y, M, N, K)
    torch.cuda.synchronize()
    check_gemm(Y.cpu().numpy()[ms, ns], Y_or, B_or, f"lone {M}x{N}x{K}")
    R = rng.standard_normal((M, N)).astype(np.float32)
    Rd = dev(R)
    q4.q4_0_gemm_grouped_ex([(W, Xd, Rd, M, N, K, Rd, q4.Q4_0_EPI_RESIDUAL)])
    torch.cuda.synchronize()
    ref = Y_or + R[ms, ns]
    check_gemm(Rd.cpu().numpy()[ms, ns] - R[ms, ns], Y_or, B_or + 1e3 * 2.0**-22 * np.abs(ref),
               f"lone {M}x{N}x{K} + residual in place")
