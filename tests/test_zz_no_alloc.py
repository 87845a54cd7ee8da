"""q4_0_gemm_static_ws: the entry point that allocates no device memory and
takes its workspace from the library's fixed device scratch array.

Called through the C ABI.  The header promises the result of q4_0_gemm bit for
bit, so every call is compared with q4_0_gemm on the same inputs with
torch.equal, and the first problem is also checked against the float64 oracle
within the method's tolerance (|dY| <= 1e-3 * sum_k |x w| + 1e-6).  Calls in a
row on different problems share the array: a later call with a larger M*K than
an earlier one would read stale fp16 rows of the earlier X if it read anything
it had not written first.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.gpu_helpers import check_gemm

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
    return codes, scales, X, W, torch.from_numpy(X.view(np.int16)).cuda()


def _check_against_gemm(q4, rng, M, N, K, with_oracle=False):
    codes, scales, Xh, W, X = _inputs(q4, rng, M, N, K)
    Y_ref = torch.full((M, N), float("nan"), device="cuda")
    Y = torch.full((M, N), float("nan"), device="cuda")
    assert q4.lib.q4_0_gemm(W.data_ptr(), X.data_ptr(), Y_ref.data_ptr(), M, N, K, None) == q4.Q4_OK
    st = q4.lib.q4_0_gemm_static_ws(W.data_ptr(), X.data_ptr(), Y.data_ptr(), M, N, K,
                                    torch.cuda.current_stream().cuda_stream)
    assert st == q4.Q4_OK, q4.lib.q4_0_status_string(st)
    torch.cuda.synchronize()
    assert q4.q4_0_device_error() == 0
    assert torch.isfinite(Y).all()
    assert torch.equal(Y, Y_ref), f"max |dY| {float((Y - Y_ref).abs().max())}"
    if with_oracle:
        Y_or, B_or = oracle.get().gemm(oracle.get().pack(codes, scales), Xh, M, N, K)
        check_gemm(Y.cpu().numpy(), Y_or, B_or, f"static workspace {M}x{N}x{K}")


def test_calls_in_a_row_match_gemm(q4):
    rng = np.random.default_rng(77)
    # tensor-core path (M > 32, ragged M and N), the scratch holding X in fp16
    _check_against_gemm(q4, rng, 300, 200, 1024, with_oracle=True)
    # a second, smaller problem right after it on the same array
    _check_against_gemm(q4, rng, 64, 136, 512)
    # a third, larger than the first: rows the first call left in the array
    # must not leak into it
    _check_against_gemm(q4, rng, 520, 72, 1536)


def test_decode_sizes_need_no_scratch(q4):
    rng = np.random.default_rng(78)
    _check_against_gemm(q4, rng, 2, 129, 3072, with_oracle=True)


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
