"""The debug build (Q4_DEBUG: index checks in the decode and tensor-core
kernels) on the GPU: small parity shapes through its C ABI match the float64
oracle, and no check fires (its device error word stays 0)."""
import ctypes
import importlib.util
import os

import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.gpu_helpers import check_gemm, dev

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def dlib():
    spec = importlib.util.spec_from_file_location("q4_0_b200_build", os.path.join(ROOT, "bit_weight_only_matmul_b200",
                                                                                  "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    lib = ctypes.CDLL(mod.build(debug=True))
    vp, i64 = ctypes.c_void_p, ctypes.c_int64
    lib.q4_0_pack.argtypes = [vp, vp, vp, i64, i64, vp]
    lib.q4_0_gemm.argtypes = [vp, vp, vp, i64, i64, i64, vp]
    lib.q4_0_device_error.argtypes = [ctypes.POINTER(ctypes.c_uint32), ctypes.c_int]
    return lib


def _flags(lib):
    f = ctypes.c_uint32(0)
    assert lib.q4_0_device_error(ctypes.byref(f), 1) == 0
    return f.value


# decode M <= 8 in split mode (few items) and plain mode (many items), the
# 8 < M <= 32 decode kernel, the tensor-core kernel (one and several tiles)
@pytest.mark.parametrize("M,N,K", [(1, 200, 1024), (2, 3072, 3072), (8, 129, 512), (2, 40000, 512),
                                   (16, 130, 1024), (64, 256, 512), (300, 200, 768)])
def test_debug_build_matches_oracle(dlib, M, N, K):
    rng = np.random.default_rng(M * 7 + N + K)
    codes = rng.integers(0, 16, size=(N, K), dtype=np.uint8)
    scales = (np.abs(rng.standard_normal((N, K // 32))) * 0.002 + 1e-4).astype(np.float16).view(np.uint16)
    X = workloads.fp32_to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32))
    _flags(dlib)
    W = torch.empty(N * (K // 32) * 18, dtype=torch.uint8, device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    cd, sd, Xd = dev(codes), dev(scales), dev(X)
    assert dlib.q4_0_pack(cd.data_ptr(), sd.data_ptr(), W.data_ptr(), N, K, s) == 0
    Y = torch.full((M, N), float("nan"), device="cuda")
    assert dlib.q4_0_gemm(W.data_ptr(), Xd.data_ptr(), Y.data_ptr(), M, N, K, s) == 0
    torch.cuda.synchronize()
    assert _flags(dlib) == 0
    o = oracle.get()
    Y_or, B_or = o.gemm(o.pack(codes, scales), X, M, N, K)
    check_gemm(Y.cpu().numpy(), Y_or, B_or, f"debug build {M}x{N}x{K}")
