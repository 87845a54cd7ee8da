"""Python binding of libq4_0_b200.so, the B200 (sm_100a) Q4_0 dequant-matmul
library (C ABI in include/q4_0.h).

Argument marshalling only: every function takes torch CUDA tensors (or raw
device addresses), passes their pointers, sizes and the current CUDA stream to
the C entry point of the same name, and raises ``Q4Error`` on a non-zero
status.  All arithmetic runs in the library's CUDA kernels; there is no CPU
path.  Importing this package fails loudly if the library has not been built
(``python bit_weight_only_matmul_b200/build.py``).
"""
from __future__ import annotations

import ctypes
import os
from typing import Iterable, Optional, Sequence

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libq4_0_b200.so")

Q4_OK = 0
Q4_ERR_INVALID_ARG = 1
Q4_ERR_MISALIGNED = 2
Q4_ERR_UNSUPPORTED_DEVICE = 3
Q4_ERR_CUDA = 4
Q4_ERR_TOO_LARGE = 5

Q4_DEVERR_WAIT_TIMEOUT = 1
Q4_DEVERR_BAD_INDEX = 2
Q4_DEVERR_FP16_RANGE = 4
Q4_DEVERR_DEBUG_CHECK = 8

Q4_0_MAX_GROUP = 256
Q4_0_STATIC_WS_BYTES = 64 << 20
Q4_0_EPI_NONE, Q4_0_EPI_RESIDUAL, Q4_0_EPI_SWIGLU = 0, 1, 2

PATH_AUTO, PATH_GENERIC, PATH_DECODE, PATH_TENSOR, PATH_DECODE_EXACT, PATH_DECODE_TMEM, PATH_DECODE_M8 = 0, 1, 2, 3, 4, 5, 6

# every symbol include/q4_0.h declares
EXPORTS = (
    "q4_0_status_string",
    "q4_0_last_cuda_error",
    "q4_0_bytes",
    "q4_0_pack",
    "q4_0_dequant",
    "q4_0_gemm",
    "q4_0_gemm_workspace_size",
    "q4_0_gemm_ws",
    "q4_0_gemm_static_ws",
    "q4_0_prepared_x_bytes",
    "q4_0_prepare_x",
    "q4_0_gemm_prepared",
    "q4_0_gemm_grouped",
    "q4_0_gemm_grouped_ex",
    "q4_0_interleave_gate_up",
    "q4_0_gather",
    "q4_0_quantize",
    "q4_0_selftest_wait_timeout",
    "q4_0_stream_read",
    "q4_0_device_error",
    "q4_0_force_path",
)


class Q4Error(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = _lib.q4_0_status_string(status).decode()
        if status == Q4_ERR_CUDA:
            msg += f" (cudaError {_lib.q4_0_last_cuda_error()})"
        super().__init__(f"{where}: {msg}")


class q4_0_problem(ctypes.Structure):
    _fields_ = [("W", ctypes.c_void_p), ("X", ctypes.c_void_p), ("Y", ctypes.c_void_p),
                ("M", ctypes.c_int64), ("N", ctypes.c_int64), ("K", ctypes.c_int64)]


class q4_0_problem_ex(ctypes.Structure):
    _fields_ = [("W", ctypes.c_void_p), ("X", ctypes.c_void_p), ("Y", ctypes.c_void_p),
                ("M", ctypes.c_int64), ("N", ctypes.c_int64), ("K", ctypes.c_int64),
                ("R", ctypes.c_void_p), ("epilogue", ctypes.c_int32)]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python bit_weight_only_matmul_b200/build.py`")
    lib = ctypes.CDLL(LIB_PATH)
    i64, vp, i32 = ctypes.c_int64, ctypes.c_void_p, ctypes.c_int
    sig = {
        "q4_0_status_string": (ctypes.c_char_p, [i32]),
        "q4_0_last_cuda_error": (i32, []),
        "q4_0_bytes": (i64, [i64, i64]),
        "q4_0_pack": (i32, [vp, vp, vp, i64, i64, vp]),
        "q4_0_dequant": (i32, [vp, vp, i64, i64, vp]),
        "q4_0_gemm": (i32, [vp, vp, vp, i64, i64, i64, vp]),
        "q4_0_gemm_workspace_size": (i64, [i64, i64, i64]),
        "q4_0_gemm_ws": (i32, [vp, vp, vp, i64, i64, i64, vp, i64, vp]),
        "q4_0_gemm_static_ws": (i32, [vp, vp, vp, i64, i64, i64, vp]),
        "q4_0_prepared_x_bytes": (i64, [i64, i64]),
        "q4_0_prepare_x": (i32, [vp, i64, i64, vp, i64, vp]),
        "q4_0_gemm_prepared": (i32, [vp, vp, vp, i64, i64, i64, vp]),
        "q4_0_gemm_grouped": (i32, [ctypes.POINTER(q4_0_problem), i32, vp]),
        "q4_0_gemm_grouped_ex": (i32, [ctypes.POINTER(q4_0_problem_ex), i32, vp]),
        "q4_0_interleave_gate_up": (i32, [vp, vp, vp, i64, i64, vp]),
        "q4_0_gather": (i32, [vp, vp, vp, i64, i64, i64, vp]),
        "q4_0_quantize": (i32, [vp, vp, i64, i64, vp]),
        "q4_0_device_error": (i32, [ctypes.POINTER(ctypes.c_uint32), i32]),
        "q4_0_selftest_wait_timeout": (i32, [ctypes.c_uint32, vp]),
        "q4_0_stream_read": (i32, [vp, i64, i64, vp, vp]),
        "q4_0_force_path": (i32, [i32]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype, f.argtypes = res, args
    return lib


_lib = _load()
lib = _lib


def _ptr(t) -> Optional[int]:
    """Device address of a tensor (or an int address, or None)."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status: int, where: str) -> None:
    if status != Q4_OK:
        raise Q4Error(status, where)


def q4_0_bytes(N: int, K: int) -> int:
    return int(_lib.q4_0_bytes(N, K))


def q4_0_pack(codes, scales, W, N: int, K: int, stream=None) -> None:
    """codes uint8 [N,K], scales fp16 bits (int16/uint16/float16 tensor) [N,K/32] -> W uint8 Q4_0."""
    _check(_lib.q4_0_pack(_ptr(codes), _ptr(scales), _ptr(W), N, K, _stream(stream)), "q4_0_pack")


def q4_0_dequant(W, out, N: int, K: int, stream=None) -> None:
    _check(_lib.q4_0_dequant(_ptr(W), _ptr(out), N, K, _stream(stream)), "q4_0_dequant")


def q4_0_gemm(W, X, Y, M: int, N: int, K: int, stream=None) -> None:
    """Y[M,N] = X[M,K] * dequant(W)^T; X bf16 (or int16 bit patterns), Y fp32."""
    _check(_lib.q4_0_gemm(_ptr(W), _ptr(X), _ptr(Y), M, N, K, _stream(stream)), "q4_0_gemm")


def q4_0_stream_read(W, N: int, K: int, checksum, stream=None) -> None:
    """Read the Q4_0 matrix W once with the decode kernels' weight stream and
    XOR its 32-bit words into `checksum` (a one-element int32/uint32 CUDA
    tensor the caller initialises): the read-only ceiling of that pattern."""
    _check(_lib.q4_0_stream_read(_ptr(W), N, K, _ptr(checksum), _stream(stream)), "q4_0_stream_read")


def q4_0_gemm_workspace_size(M: int, N: int, K: int) -> int:
    return int(_lib.q4_0_gemm_workspace_size(M, N, K))


def q4_0_gemm_ws(W, X, Y, M: int, N: int, K: int, workspace, workspace_bytes: Optional[int] = None,
                 stream=None) -> None:
    """q4_0_gemm with a device workspace (a CUDA tensor, its byte size taken
    from the tensor unless given)."""
    if workspace_bytes is None:
        workspace_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(_lib.q4_0_gemm_ws(_ptr(W), _ptr(X), _ptr(Y), M, N, K, _ptr(workspace), workspace_bytes,
                             _stream(stream)), "q4_0_gemm_ws")


def q4_0_gemm_static_ws(W, X, Y, M: int, N: int, K: int, stream=None) -> None:
    """q4_0_gemm_ws on the library's fixed device scratch array: the call
    allocates nothing (Q4Error Q4_ERR_TOO_LARGE when M*K*2 exceeds
    Q4_0_STATIC_WS_BYTES for M > 32)."""
    _check(_lib.q4_0_gemm_static_ws(_ptr(W), _ptr(X), _ptr(Y), M, N, K, _stream(stream)), "q4_0_gemm_static_ws")


def q4_0_prepared_x_bytes(M: int, K: int) -> int:
    return int(_lib.q4_0_prepared_x_bytes(M, K))


def q4_0_prepare_x(X, M: int, K: int, xh, xh_bytes: Optional[int] = None, stream=None) -> None:
    """X (bf16 [M, K]) into `xh` in the tensor-core kernel's fp16 layout (its
    byte size taken from the tensor unless given)."""
    if xh_bytes is None:
        xh_bytes = xh.numel() * xh.element_size()
    _check(_lib.q4_0_prepare_x(_ptr(X), M, K, _ptr(xh), xh_bytes, _stream(stream)), "q4_0_prepare_x")


def q4_0_gemm_prepared(W, xh, Y, M: int, N: int, K: int, stream=None) -> None:
    """The tensor-core GEMM on an X prepared by q4_0_prepare_x."""
    _check(_lib.q4_0_gemm_prepared(_ptr(W), _ptr(xh), _ptr(Y), M, N, K, _stream(stream)), "q4_0_gemm_prepared")


def make_problems(problems: Sequence) -> ctypes.Array:
    """Build a q4_0_problem array from (W, X, Y, M, N, K) tuples."""
    arr = (q4_0_problem * max(1, len(problems)))()
    for i, (W, X, Y, M, N, K) in enumerate(problems):
        arr[i] = q4_0_problem(_ptr(W), _ptr(X), _ptr(Y), M, N, K)
    return arr


def q4_0_gemm_grouped(problems, count: Optional[int] = None, stream=None) -> None:
    """`problems`: a ctypes q4_0_problem array (see make_problems) or a
    sequence of (W, X, Y, M, N, K) tuples."""
    if not isinstance(problems, ctypes.Array):
        count = len(problems)
        problems = make_problems(problems)
    elif count is None:
        count = len(problems)
    _check(_lib.q4_0_gemm_grouped(problems, count, _stream(stream)), "q4_0_gemm_grouped")


def make_problems_ex(problems: Sequence) -> ctypes.Array:
    """Build a q4_0_problem_ex array from (W, X, Y, M, N, K, R, epilogue) tuples."""
    arr = (q4_0_problem_ex * max(1, len(problems)))()
    for i, (W, X, Y, M, N, K, R, epi) in enumerate(problems):
        arr[i] = q4_0_problem_ex(_ptr(W), _ptr(X), _ptr(Y), M, N, K, _ptr(R), epi)
    return arr


def q4_0_gemm_grouped_ex(problems, count: Optional[int] = None, stream=None) -> None:
    """`problems`: a q4_0_problem_ex array or (W, X, Y, M, N, K, R, epilogue) tuples."""
    if not isinstance(problems, ctypes.Array):
        count = len(problems)
        problems = make_problems_ex(problems)
    elif count is None:
        count = len(problems)
    _check(_lib.q4_0_gemm_grouped_ex(problems, count, _stream(stream)), "q4_0_gemm_grouped_ex")


def q4_0_interleave_gate_up(W_gate, W_up, W_gu, F: int, K: int, stream=None) -> None:
    _check(_lib.q4_0_interleave_gate_up(_ptr(W_gate), _ptr(W_up), _ptr(W_gu), F, K, _stream(stream)),
           "q4_0_interleave_gate_up")


def q4_0_gather(W, ids, out, T: int, V: int, D: int, stream=None) -> None:
    """out[t] = dequant(W)[ids[t]] (float32 [T, D]); ids int32 on the device."""
    _check(_lib.q4_0_gather(_ptr(W), _ptr(ids), _ptr(out), T, V, D, _stream(stream)), "q4_0_gather")


def q4_0_quantize(X, W, N: int, K: int, stream=None) -> None:
    """float32 X [N, K] -> Q4_0 bytes W (GGUF Q4_0 rule, bit-exact)."""
    _check(_lib.q4_0_quantize(_ptr(X), _ptr(W), N, K, _stream(stream)), "q4_0_quantize")


def q4_0_device_error(clear: bool = True) -> int:
    v = ctypes.c_uint32(0)
    _check(_lib.q4_0_device_error(ctypes.byref(v), 1 if clear else 0), "q4_0_device_error")
    return int(v.value)


def q4_0_force_path(path: int) -> None:
    _check(_lib.q4_0_force_path(path), "q4_0_force_path")
