"""Shared helpers of the GPU parity tests: upload seeded inputs, run the
library through its C ABI, and compare with the float64 oracle."""
from __future__ import annotations

import numpy as np
import torch

import oracle


def dev(a: np.ndarray) -> torch.Tensor:
    """numpy -> contiguous CUDA tensor with the same bytes (uint16 becomes int16)."""
    if a.dtype == np.uint16:
        a = a.view(np.int16)
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host_u16(t: torch.Tensor) -> np.ndarray:
    return t.cpu().numpy().view(np.uint16)


def pack_on_gpu(lib, codes: np.ndarray, scales: np.ndarray) -> torch.Tensor:
    N, K = codes.shape
    W = torch.empty(lib.q4_0_bytes(N, K), dtype=torch.uint8, device="cuda")
    lib.q4_0_pack(dev(codes), dev(scales), W, N, K)
    return W


def check_gemm(Y_gpu: np.ndarray, Y_or: np.ndarray, B_or: np.ndarray, what: str = "") -> float:
    """The tolerance of the method: |Y - Y_exact| <= 1e-3 * sum|x*w| + 1e-6
    per element.  Returns max(err / bound)."""
    Y_gpu = np.asarray(Y_gpu, np.float64)
    assert Y_gpu.shape == Y_or.shape, (Y_gpu.shape, Y_or.shape)
    bound = 1e-3 * B_or + 1e-6
    err = np.abs(Y_gpu - Y_or)
    bad = ~(err <= bound)
    if bad.any():
        i = np.argwhere(bad)[0]
        raise AssertionError(f"{what}: {bad.sum()} of {bad.size} outside tolerance; first at {tuple(i)}: "
                             f"gpu {Y_gpu[tuple(i)]!r} oracle {Y_or[tuple(i)]!r} bound {bound[tuple(i)]!r}")
    return float((err / bound).max()) if err.size else 0.0


def oracle_gemm(W_host: np.ndarray, X_host: np.ndarray, M: int, N: int, K: int):
    return oracle.get().gemm(W_host, X_host, M, N, K)


def no_device_error(lib) -> None:
    flags = lib.q4_0_device_error(clear=True)
    assert flags == 0, f"device error word = {flags:#x}"


class Built:
    """A workload resident on the GPU plus oracle values at sampled outputs."""

    def __init__(self):
        self.W, self.X, self.Y, self.shapes = [], [], [], []
        self.samples = []   # per linear: (ms, ns, Y_or, B_or)

    def problems(self):
        return [(W, X, Y, M, N, K) for W, X, Y, (M, N, K) in zip(self.W, self.X, self.Y, self.shapes)]


def build_workload(lib, wl, samples: int = 64, seed: int = 0, full_oracle: bool = False) -> Built:
    """Generate every linear of workload `wl` from its seeded streams, pack it
    on the GPU with q4_0_pack and, independently, with the oracle's pack, and
    take oracle values at `samples` random outputs per linear (all outputs if
    full_oracle)."""
    o = oracle.get()
    rng = np.random.default_rng(1000 + seed)
    out = Built()
    for lin in wl.linears:
        M, N, K = lin.M, lin.N, lin.K
        codes, scales, X = lin.codes(), lin.scales(), lin.x()
        W_host = o.pack(codes, scales)
        if full_oracle:
            Y_or, B_or = o.gemm(W_host, X, M, N, K)
            ms, ns = np.meshgrid(np.arange(M), np.arange(N), indexing="ij")
            out.samples.append((ms.reshape(-1), ns.reshape(-1), Y_or.reshape(-1), B_or.reshape(-1)))
        else:
            ms = rng.integers(0, M, size=samples)
            ns = rng.integers(0, N, size=samples)
            # always include the last row and column (tails)
            ms[0], ns[0] = M - 1, N - 1
            Y_or, B_or = o.gemm_sampled(W_host, X, M, N, K, ms, ns)
            out.samples.append((ms, ns, Y_or, B_or))
        out.W.append(pack_on_gpu(lib, codes, scales))
        out.X.append(dev(X))
        out.Y.append(torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda"))
        out.shapes.append((M, N, K))
        del codes, scales, W_host
    return out


def check_built(b: Built, what: str) -> float:
    worst = 0.0
    for i, (Y, (ms, ns, Y_or, B_or)) in enumerate(zip(b.Y, b.samples)):
        got = Y.cpu().numpy().astype(np.float64)[ms, ns]
        worst = max(worst, check_gemm(got, Y_or, B_or, f"{what} linear {i}"))
    return worst
