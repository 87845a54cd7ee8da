"""Failure detection without a GPU fault: a bounded on-chip wait that nothing
completes gives up after its limit, reports Q4_DEVERR_WAIT_TIMEOUT through the
device error word, and leaves the context usable."""
import time

import numpy as np
import pytest
import torch

import oracle
from tests.gpu_helpers import check_gemm, dev, pack_on_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q4():
    import bit_weight_only_matmul_b200 as q4
    q4.q4_0_force_path(q4.PATH_AUTO)
    return q4


def test_bounded_wait_gives_up_and_reports(q4):
    q4.q4_0_device_error(clear=True)
    t0 = time.perf_counter()
    assert q4.lib.q4_0_selftest_wait_timeout(20000, None) == q4.Q4_OK      # 20 ms limit
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert q4.q4_0_device_error(clear=True) == q4.Q4_DEVERR_WAIT_TIMEOUT
    assert 0.015 <= elapsed < 5.0
    assert q4.q4_0_device_error(clear=True) == 0


def test_context_usable_after_a_timeout(q4):
    q4.lib.q4_0_selftest_wait_timeout(5000, None)
    torch.cuda.synchronize()
    assert q4.q4_0_device_error(clear=True) == q4.Q4_DEVERR_WAIT_TIMEOUT
    rng = np.random.default_rng(11)
    M, N, K = 2, 300, 1024
    codes = rng.integers(0, 16, size=(N, K), dtype=np.uint8)
    scales = (np.abs(rng.standard_normal((N, K // 32))) * 0.002 + 1e-4).astype(np.float16).view(np.uint16)
    import workloads
    X = workloads.fp32_to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32))
    Y = torch.full((M, N), float("nan"), device="cuda")
    q4.q4_0_gemm(pack_on_gpu(q4, codes, scales), dev(X), Y, M, N, K)
    o = oracle.get()
    Y_or, B_or = o.gemm(o.pack(codes, scales), X, M, N, K)
    check_gemm(Y.cpu().numpy(), Y_or, B_or, "after a timeout")
    assert q4.q4_0_device_error(clear=True) == 0
