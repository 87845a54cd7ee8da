"""Inputs outside the range the fp16 fast paths compute exactly.

The method takes X in bf16 (any finite value) and fp16 scales (up to 65504).
The fast kernels feed the tensor cores fp16: X overflows fp16 for
|x| > 65504, and (q - 8) * d for |d| > 8188.  Such inputs must set
Q4_DEVERR_FP16_RANGE on every fast path, the exact decode kernel
(q4_0_force_path(4)) must match the float64 oracle on them, and inputs at the
edges of the range (tiny values included) must pass without the flag and
within the method's tolerance.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.gpu_helpers import check_gemm, dev, pack_on_gpu

pytestmark = pytest.mark.gpu

# (M, what runs it by default): the M <= 8 decode kernel, the 8 < M <= 32
# decode kernel, the tensor-core kernel
SHAPES = [(1, 200, 1024), (2, 257, 3072), (16, 130, 2048), (64, 256, 512)]


@pytest.fixture(scope="module")
def q4():
    import bit_weight_only_matmul_b200 as q4
    q4.q4_0_force_path(q4.PATH_AUTO)
    yield q4
    q4.q4_0_force_path(q4.PATH_AUTO)


@pytest.fixture(autouse=True)
def _clean(q4):
    q4.q4_0_device_error(clear=True)
    yield
    q4.q4_0_force_path(q4.PATH_AUTO)
    q4.q4_0_device_error(clear=True)


def _codes_scales(rng, N, K):
    codes = rng.integers(0, 16, size=(N, K), dtype=np.uint8)
    scales = (np.abs(rng.standard_normal((N, K // 32))) * 0.002 + 1e-4).astype(np.float16).view(np.uint16)
    return codes, scales


def _run(q4, codes, scales, X, M, N, K, path=0):
    W = pack_on_gpu(q4, codes, scales)
    Y = torch.full((M, N), float("nan"), device="cuda")
    q4.q4_0_force_path(path)
    try:
        q4.q4_0_gemm(W, dev(X), Y, M, N, K)
    finally:
        q4.q4_0_force_path(q4.PATH_AUTO)
    torch.cuda.synchronize()
    flags = q4.q4_0_device_error(clear=True)
    return Y.cpu().numpy(), flags


def _wide_x(rng, M, K):
    """bf16 X spanning 1e-30 .. 1e30 in magnitude, both signs."""
    mag = 10.0 ** rng.uniform(-30, 30, size=(M, K))
    sign = np.where(rng.random((M, K)) < 0.5, -1.0, 1.0)
    return workloads.fp32_to_bf16_bits((sign * mag).astype(np.float32))


@pytest.mark.parametrize("M,N,K", SHAPES)
def test_wide_x_flagged_and_exact_path_matches(q4, M, N, K):
    rng = np.random.default_rng(M * 7 + N + K)
    codes, scales = _codes_scales(rng, N, K)
    X = _wide_x(rng, M, K)
    _, flags = _run(q4, codes, scales, X, M, N, K)
    assert flags & q4.Q4_DEVERR_FP16_RANGE, f"no range flag (flags {flags:#x})"
    o = oracle.get()
    Y_or, B_or = o.gemm(o.pack(codes, scales), X, M, N, K)
    if M <= 32:
        Y, flags = _run(q4, codes, scales, X, M, N, K, path=q4.PATH_DECODE_EXACT)
        assert flags == 0
        check_gemm(Y, Y_or, B_or, "exact decode path, wide X")


@pytest.mark.parametrize("M,N,K", SHAPES)
def test_large_scales_flagged_and_exact_path_matches(q4, M, N, K):
    """Scales up to 65504 with code 0 in their blocks: -8 d overflows fp16."""
    rng = np.random.default_rng(M * 11 + N + K)
    codes, scales = _codes_scales(rng, N, K)
    rows = rng.choice(N, size=3, replace=False)
    blocks = rng.integers(0, K // 32, size=3)
    big = np.array([65504.0, -20000.0, 9000.0], dtype=np.float16).view(np.uint16)
    for r, b, d in zip(rows, blocks, big):
        scales[r, b] = d
        codes[r, 32 * b:32 * b + 32] = 0
    X = workloads.fp32_to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32))
    _, flags = _run(q4, codes, scales, X, M, N, K)
    assert flags & q4.Q4_DEVERR_FP16_RANGE, f"no range flag (flags {flags:#x})"
    if M <= 32:
        o = oracle.get()
        Y_or, B_or = o.gemm(o.pack(codes, scales), X, M, N, K)
        Y, flags = _run(q4, codes, scales, X, M, N, K, path=q4.PATH_DECODE_EXACT)
        assert flags == 0
        check_gemm(Y, Y_or, B_or, "exact decode path, large scales")


@pytest.mark.parametrize("M,N,K", SHAPES)
def test_range_edges_pass_unflagged(q4, M, N, K):
    """X at the edges of the fp16 range (+-65280, the largest bf16 below
    65536; +-2^-17 and +-1e-7, below the fp16 normal range; zeros) and scales
    of +-8188: no flag, oracle tolerance."""
    rng = np.random.default_rng(M * 13 + N + K)
    codes, scales = _codes_scales(rng, N, K)
    scales[:, ::5] = np.array(8188.0, dtype=np.float16).view(np.uint16)
    scales[:, 1::7] = np.array(-8188.0, dtype=np.float16).view(np.uint16)
    vals = np.array([65280.0, -65280.0, 2.0**-17, -(2.0**-17), 1e-7, -1e-7, 0.0, 1.0, -3.5], dtype=np.float32)
    X = workloads.fp32_to_bf16_bits(rng.choice(vals, size=(M, K)))
    Y, flags = _run(q4, codes, scales, X, M, N, K)
    assert flags == 0, f"flags {flags:#x}"
    o = oracle.get()
    Y_or, B_or = o.gemm(o.pack(codes, scales), X, M, N, K)
    check_gemm(Y, Y_or, B_or, "range edges")
