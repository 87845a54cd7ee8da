"""Float64 CPU oracle for the Q4_0 dequantize-and-matmul (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product library never imports it
and has no CPU fallback.

The arithmetic lives in ``q4_0_oracle.c`` (plain C, single-threaded, float64;
see its header for the definition and the passages it follows).  This module
compiles it with gcc into ``oracle/_build/`` and wraps it with ctypes for
numpy arrays.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "q4_0_oracle.c")
_BUILD = os.path.join(_HERE, "_build")

_i64 = ctypes.c_int64
_p = ctypes.c_void_p


def lib_path(mutant: int = 0) -> str:
    name = "liboracle.so" if mutant == 0 else f"liboracle_mutant{mutant}.so"
    return os.path.join(_BUILD, name)


def build(mutant: int = 0, force: bool = False) -> str:
    """Compile the oracle (or one planted-mistake variant) with gcc."""
    out = lib_path(mutant)
    if not force and os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(_SRC):
        return out
    os.makedirs(_BUILD, exist_ok=True)
    tmp = out + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math", "-ffp-contract=off",
           f"-DORACLE_MUTANT={mutant}", _SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


class Oracle:
    """ctypes view of one compiled oracle library."""

    def __init__(self, mutant: int = 0):
        self.mutant = mutant
        self._lib = ctypes.CDLL(build(mutant))
        L = self._lib
        L.oracle_half_to_double.restype = ctypes.c_double
        L.oracle_half_to_double.argtypes = [ctypes.c_uint16]
        L.oracle_bf16_to_double.restype = ctypes.c_double
        L.oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
        L.oracle_q4_0_row_bytes.restype = _i64
        L.oracle_q4_0_row_bytes.argtypes = [_i64]
        for name in ("oracle_q4_0_pack", "oracle_q4_0_unpack"):
            getattr(L, name).restype = None
            getattr(L, name).argtypes = [_p, _p, _p, _i64, _i64]
        for name in ("oracle_q4_0_dequant_f64", "oracle_q4_0_dequant_f32"):
            getattr(L, name).restype = None
            getattr(L, name).argtypes = [_p, _p, _i64, _i64]
        L.oracle_q4_0_gemm.restype = None
        L.oracle_q4_0_gemm.argtypes = [_p, _p, _p, _p, _i64, _i64, _i64]
        L.oracle_q4_0_gemm_sampled.restype = None
        L.oracle_q4_0_gemm_sampled.argtypes = [_p, _p, _i64, _i64, _i64, _p, _p, _i64, _p, _p]
        L.oracle_q4_0_gather_f32.restype = _i64
        L.oracle_q4_0_gather_f32.argtypes = [_p, _p, _p, _i64, _i64, _i64]
        L.oracle_float_to_half.restype = ctypes.c_uint16
        L.oracle_float_to_half.argtypes = [ctypes.c_float]
        L.oracle_q4_0_quantize.restype = None
        L.oracle_q4_0_quantize.argtypes = [_p, _p, _i64, _i64]
        L.oracle_swiglu.restype = None
        L.oracle_swiglu.argtypes = [_p, _p, _p, _i64]

    # -- scalar decoders -------------------------------------------------
    def half_to_double(self, h: int) -> float:
        return self._lib.oracle_half_to_double(int(h))

    def bf16_to_double(self, b: int) -> float:
        return self._lib.oracle_bf16_to_double(int(b))

    def row_bytes(self, K: int) -> int:
        return int(self._lib.oracle_q4_0_row_bytes(int(K)))

    # -- array entry points ---------------------------------------------
    @staticmethod
    def _c(a: np.ndarray, dtype) -> np.ndarray:
        a = np.ascontiguousarray(a)
        if a.dtype != dtype:
            raise TypeError(f"expected {np.dtype(dtype)}, got {a.dtype}")
        return a

    def pack(self, codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
        """codes uint8 [N,K], scales uint16 (fp16 bits) [N,K/32] -> W uint8 [N, K/32*18]."""
        codes = self._c(codes, np.uint8)
        scales = self._c(scales, np.uint16)
        N, K = codes.shape
        if K % 32 or scales.shape != (N, K // 32):
            raise ValueError("bad shapes")
        W = np.empty((N, K // 32 * 18), np.uint8)
        self._lib.oracle_q4_0_pack(codes.ctypes.data, scales.ctypes.data, W.ctypes.data, N, K)
        return W

    def unpack(self, W: np.ndarray, N: int, K: int):
        W = self._c(W, np.uint8)
        codes = np.empty((N, K), np.uint8)
        scales = np.empty((N, K // 32), np.uint16)
        self._lib.oracle_q4_0_unpack(W.ctypes.data, codes.ctypes.data, scales.ctypes.data, N, K)
        return codes, scales

    def dequant_f64(self, W: np.ndarray, N: int, K: int) -> np.ndarray:
        W = self._c(W, np.uint8)
        out = np.empty((N, K), np.float64)
        self._lib.oracle_q4_0_dequant_f64(W.ctypes.data, out.ctypes.data, N, K)
        return out

    def dequant_f32(self, W: np.ndarray, N: int, K: int) -> np.ndarray:
        W = self._c(W, np.uint8)
        out = np.empty((N, K), np.float32)
        self._lib.oracle_q4_0_dequant_f32(W.ctypes.data, out.ctypes.data, N, K)
        return out

    def gemm(self, W: np.ndarray, X: np.ndarray, M: int, N: int, K: int):
        """W uint8 Q4_0 [N, K/32*18], X uint16 (bf16 bits) [M,K] -> (Y, B) float64 [M,N]."""
        W = self._c(W, np.uint8)
        X = self._c(X, np.uint16)
        Y = np.empty((M, N), np.float64)
        B = np.empty((M, N), np.float64)
        self._lib.oracle_q4_0_gemm(W.ctypes.data, X.ctypes.data, Y.ctypes.data, B.ctypes.data, M, N, K)
        return Y, B

    def gemm_sampled(self, W: np.ndarray, X: np.ndarray, M: int, N: int, K: int,
                     ms: np.ndarray, ns: np.ndarray):
        """Only the outputs (ms[i], ns[i]) -> (Y, B) float64 [count]."""
        W = self._c(W, np.uint8)
        X = self._c(X, np.uint16)
        ms = self._c(ms.astype(np.int64), np.int64)
        ns = self._c(ns.astype(np.int64), np.int64)
        if ms.shape != ns.shape:
            raise ValueError("ms and ns differ in length")
        if len(ms) and (ms.min() < 0 or ms.max() >= M or ns.min() < 0 or ns.max() >= N):
            raise ValueError("sample index out of range")
        Y = np.empty(len(ms), np.float64)
        B = np.empty(len(ms), np.float64)
        self._lib.oracle_q4_0_gemm_sampled(W.ctypes.data, X.ctypes.data, M, N, K,
                                           ms.ctypes.data, ns.ctypes.data, len(ms),
                                           Y.ctypes.data, B.ctypes.data)
        return Y, B


    def gather_f32(self, W: np.ndarray, ids: np.ndarray, V: int, D: int):
        """Rows ids of W[V, D] (Q4_0) as float32 [T, D]; returns (out, count of ids outside [0, V))."""
        W = self._c(W, np.uint8)
        ids = self._c(ids, np.int32)
        out = np.empty((len(ids), D), np.float32)
        bad = self._lib.oracle_q4_0_gather_f32(W.ctypes.data, ids.ctypes.data, out.ctypes.data, len(ids), V, D)
        return out, int(bad)

    def float_to_half(self, f: float) -> int:
        return int(self._lib.oracle_float_to_half(float(f)))

    def quantize(self, X: np.ndarray) -> np.ndarray:
        """float32 [N, K] -> Q4_0 bytes [N, K/32*18] by the GGUF Q4_0 rule."""
        X = self._c(X, np.float32)
        N, K = X.shape
        if K % 32:
            raise ValueError("K must be a multiple of 32")
        W = np.empty((N, K // 32 * 18), np.uint8)
        self._lib.oracle_q4_0_quantize(X.ctypes.data, W.ctypes.data, N, K)
        return W


    def swiglu(self, g: np.ndarray, u: np.ndarray) -> np.ndarray:
        """silu(g) * u elementwise in float64 (same shapes)."""
        g = self._c(g, np.float64)
        u = self._c(u, np.float64)
        if g.shape != u.shape:
            raise ValueError("g and u differ in shape")
        out = np.empty(g.shape, np.float64)
        self._lib.oracle_swiglu(g.ctypes.data, u.ctypes.data, out.ctypes.data, g.size)
        return out


_default = None


def get() -> Oracle:
    """The (unmutated) oracle, built on first use."""
    global _default
    if _default is None:
        _default = Oracle(0)
    return _default
