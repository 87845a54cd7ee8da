"""q4_0_gemm_static_ws: the entry point that allocates nothing and takes its
workspace from the library's fixed device scratch array.

Called through the C ABI; each result is compared with q4_0_gemm on the same
inputs within the method's tolerance, |dY| <= 1e-3 * sum_k |x w| + 1e-6, with
sum_k |x w| taken in float64 from the library's own dequantized weights.  Two
calls in a row on different problems check that nothing of the first call
leaks into the second through the shared array.
"""
import numpy as np
import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q4():
    import bit_weight_only_matmul_b200 as q4
    q4.q4_0_force_path(q4.PATH_AUTO)
    return q4


def _inputs(q4, rng, M, N, K):
    codes = rng.integers(0, 16, size=(N, K), dtype=np.uint8)
    scales = (np.abs(rng.standard_normal(size=(N, K // 32))) * 0.002 + 1e-4).astype(np.float16).view(np.uint16)
    X = workloads.fp32_to_bf16_bits(rng.standard_normal(size=(M, K)).astype(np.float32))
    W = torch.empty(q4.q4_0_bytes(N, K), dtype=torch.uint8, device="cuda")
    q4.q4_0_pack(torch.from_numpy(codes).cuda(), torch.from_numpy(scales.view(np.int16)).cuda(), W, N, K)
    return W, torch.from_numpy(X.view(np.int16)).cuda()


def _abs_bound(q4, W, X, M, N, K):
    Wd = torch.empty((N, K), dtype=torch.float32, device="cuda")
    q4.q4_0_dequant(W, Wd, N, K)
    Xf = X.view(torch.bfloat16).to(torch.float64)
    return Xf.abs() @ Wd.to(torch.float64).abs().T


def _check_against_gemm(q4, rng, M, N, K):
    W, X = _inputs(q4, rng, M, N, K)
    Y_ref = torch.full((M, N), float("nan"), device="cuda")
    Y = torch.full((M, N), float("nan"), device="cuda")
    assert q4.lib.q4_0_gemm(W.data_ptr(), X.data_ptr(), Y_ref.data_ptr(), M, N, K, None) == q4.Q4_OK
    st = q4.lib.q4_0_gemm_static_ws(W.data_ptr(), X.data_ptr(), Y.data_ptr(), M, N, K,
                                    torch.cuda.current_stream().cuda_stream)
    assert st == q4.Q4_OK, q4.lib.q4_0_status_string(st)
    torch.cuda.synchronize()
    assert q4.q4_0_device_error() == 0
    bound = 1e-3 * _abs_bound(q4, W, X, M, N, K) + 1e-6
    err = (Y.to(torch.float64) - Y_ref.to(torch.float64)).abs()
    assert torch.isfinite(Y).all()
    assert bool((err <= bound).all()), f"max err/bound {float((err / bound).max())}"


def test_two_calls_in_a_row_match_gemm(q4):
    rng = np.random.default_rng(77)
    # tensor-core path (M > 32, ragged M and N), the scratch holding X in fp16
    _check_against_gemm(q4, rng, 300, 200, 1024)
    # a second, smaller problem right after it on the same array
    _check_against_gemm(q4, rng, 64, 136, 512)


def test_decode_sizes_need_no_scratch(q4):
    rng = np.random.default_rng(78)
    _check_against_gemm(q4, rng, 2, 129, 3072)


def test_too_large_is_rejected(q4):
    M, K, N = 4096, 16384, 64          # M*K*2 = 128 MiB > Q4_0_STATIC_WS_BYTES
    assert q4.q4_0_gemm_workspace_size(M, N, K) > q4.Q4_0_STATIC_WS_BYTES
    Y = torch.full((4, 4), float("nan"), device="cuda")
    A = 1 << 20                        # never dereferenced: the check comes first
    st = q4.lib.q4_0_gemm_static_ws(A, A, Y.data_ptr(), M, N, K, None)
    assert st == q4.Q4_ERR_TOO_LARGE
    assert b"Q4_0_STATIC_WS_BYTES" in q4.lib.q4_0_status_string(st)
    torch.cuda.synchronize()
    assert torch.isnan(Y).all()
