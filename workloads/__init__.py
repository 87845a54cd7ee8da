"""Seeded synthetic inputs and workload shapes for the Q4_0 dequant-matmul.

This module draws the *inputs* of the method -- 4-bit codes, fp16 scales and
bf16 activations -- and names the shapes of the workloads.  It holds none of
the method's arithmetic (no packing, no dequantization, no product): both the
float64 oracle and the CUDA library receive exactly these arrays.

Generator: numpy's Philox4x64-10 (Salmon et al., "Parallel random numbers: as
easy as 1, 2, 3", SC'11), a counter-based generator.  Every tensor has its own
stream, keyed by (seed, layer, tensor id, linear id), so any tensor of any
layer is reproducible on its own without generating the others.

Distributions (the workloads' recipe):
  * codes q: uniform integers in 0..15 (one uint8 per weight, low nibble);
  * scales d: fp16 round-to-nearest-even of |N(0,1)| * 0.002 + 1e-4
    (computed in float64, rounded once to fp16);
  * X: bf16 round-to-nearest-even of an fp32 N(0, sigma^2) draw, optionally
    times a per-row scale (uniform in [0.5, 2)) or with a fixed number of
    outlier rows multiplied by 8 (the scale is applied in fp32 before the
    single rounding to bf16).

Shapes follow the decoder of the Voxtral 4B speech models as the pages state
it (26 layers, width 3072, GQA 32Q/8KV; adapter 5120 -> 3072) --
voxtral-mini-realtime-rs (Shannon-Prime fork) README, "Architecture"; the
synthetic FFN width 8192 and K/V width 1024 are workload choices.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Optional

import numpy as np

SEED = 20261202

# tensor ids of the independent streams
T_CODES = 1
T_SCALES = 2
T_X = 3
T_ROWSCALE = 4
T_OUTLIER = 5


def _rng(seed: int, layer: int, tensor: int, linear: int) -> np.random.Generator:
    if not (0 <= seed < 2**63 and 0 <= layer < 2**20 and 0 <= tensor < 2**8 and 0 <= linear < 2**16):
        raise ValueError("stream id out of range")
    key = (int(seed) << 64) | (int(layer) << 24) | (int(tensor) << 16) | int(linear)
    return np.random.Generator(np.random.Philox(key=key))


def fp32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """bf16 round-to-nearest-even of float32 values, as uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    nan = (u & 0x7FFFFFFF) > 0x7F800000
    r = (u + np.uint32(0x7FFF) + ((u >> 16) & np.uint32(1))) >> 16
    r = r.astype(np.uint16)
    r[nan] = ((u[nan] >> 16) | 0x40).astype(np.uint16)
    return r


def bf16_bits_to_fp32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def gen_codes(N: int, K: int, seed: int = SEED, layer: int = 0, linear: int = 0) -> np.ndarray:
    """uint8 [N,K], uniform in 0..15."""
    return _rng(seed, layer, T_CODES, linear).integers(0, 16, size=(N, K), dtype=np.uint8)


def gen_scales(N: int, K: int, seed: int = SEED, layer: int = 0, linear: int = 0) -> np.ndarray:
    """uint16 fp16 bit patterns [N, K/32] of |N(0,1)|*0.002 + 1e-4."""
    if K % 32:
        raise ValueError("K must be a multiple of 32")
    z = _rng(seed, layer, T_SCALES, linear).standard_normal(size=(N, K // 32), dtype=np.float64)
    return (np.abs(z) * 0.002 + 1e-4).astype(np.float16).view(np.uint16)


def gen_x(M: int, K: int, seed: int = SEED, layer: int = 0, linear: int = 0,
          sigma: float = 1.0, row_scale: bool = False, outlier_rows: int = 0) -> np.ndarray:
    """uint16 bf16 bit patterns [M,K]."""
    x = _rng(seed, layer, T_X, linear).standard_normal(size=(M, K), dtype=np.float32)
    x *= np.float32(sigma)
    if row_scale:
        s = _rng(seed, layer, T_ROWSCALE, linear).uniform(0.5, 2.0, size=(M, 1)).astype(np.float32)
        x *= s
    if outlier_rows:
        rows = outlier_row_ids(M, outlier_rows, seed, layer, linear)
        x[rows] *= np.float32(8.0)
    return fp32_to_bf16_bits(x)


def outlier_row_ids(M: int, count: int, seed: int = SEED, layer: int = 0, linear: int = 0) -> np.ndarray:
    """The rows scaled x8: the first `count` of a seeded permutation of 0..M-1."""
    return np.sort(_rng(seed, layer, T_OUTLIER, linear).permutation(M)[:count])


# ---------------------------------------------------------------------------
# workload shapes
# ---------------------------------------------------------------------------

@dataclass
class Linear:
    """One Q4_0 linear: Y[M,N] = X[M,K] * dequant(W[N,K])^T."""
    name: str
    N: int
    K: int
    layer: int = 0
    linear: int = 0          # stream id of this linear within the layer
    M: int = 1
    sigma: float = 1.0
    row_scale: bool = False
    outlier_rows: int = 0

    @property
    def weight_bytes(self) -> int:
        return self.N * (self.K // 32) * 18

    @property
    def act_bytes(self) -> int:
        return self.M * self.K * 2 + self.M * self.N * 4

    @property
    def flops(self) -> int:
        return 2 * self.M * self.N * self.K

    def codes(self, seed: int = SEED) -> np.ndarray:
        return gen_codes(self.N, self.K, seed, self.layer, self.linear)

    def scales(self, seed: int = SEED) -> np.ndarray:
        return gen_scales(self.N, self.K, seed, self.layer, self.linear)

    def x(self, seed: int = SEED) -> np.ndarray:
        return gen_x(self.M, self.K, seed, self.layer, self.linear, self.sigma,
                     self.row_scale, self.outlier_rows)


D_MODEL = 3072
N_LAYERS = 26
FFN = 8192
Q_DIM, KV_DIM = 3072, 1024
ADAPTER_IN = 5120
FLOW_LAYERS = 3
FLOW_LAYER0 = 100   # stream ids of the flow head's layers, apart from the decoder's


def decoder_layer(layer: int, M: int, **xkw) -> List[Linear]:
    """The four Q4_0 GEMMs of one decoder layer: fused QKV (N = 3072 + 1024 +
    1024), O, fused gate/up (N = 2 x 8192) and down (K = 8192)."""
    return [
        Linear("qkv", Q_DIM + 2 * KV_DIM, D_MODEL, layer, 0, M, **xkw),
        Linear("o", D_MODEL, Q_DIM, layer, 1, M, **xkw),
        Linear("gate_up", 2 * FFN, D_MODEL, layer, 2, M, **xkw),
        Linear("down", D_MODEL, FFN, layer, 3, M, **xkw),
    ]


@dataclass
class Workload:
    name: str
    description: str
    linears: List[Linear] = field(default_factory=list)
    fused: bool = False   # gate/up -> SwiGLU (Y is half as wide), O and down + a residual read

    @property
    def weight_bytes(self) -> int:
        return sum(l.weight_bytes for l in self.linears)

    @property
    def hbm_bytes(self) -> int:
        """Algorithmic bytes: every weight byte once plus X and Y once (with
        the fused epilogues: the gate/up output is N/2 wide and the O and
        down outputs also read a residual of their own size)."""
        total = sum(l.weight_bytes + l.act_bytes for l in self.linears)
        if self.fused:
            for l in self.linears:
                if l.name == "gate_up":
                    total -= l.M * (l.N // 2) * 4
                elif l.name in ("o", "down"):
                    total += l.M * l.N * 4
        return total

    @property
    def flops(self) -> int:
        return sum(l.flops for l in self.linears)


def workload(name: str, layers: Optional[List[int]] = None) -> Workload:
    """The named workloads.  `layers` restricts the 26-layer sets to a subset
    (for fast tests); None means all."""
    if name == "gemv":
        return Workload(name, "single Q4_0 GEMV, M=1, K=N=3072",
                        [Linear("gemv", D_MODEL, D_MODEL, 0, 0, 1)])
    if name == "layer":
        return Workload(name, "one decoder-layer linear set at M=1 (QKV 5120, O 3072, gate/up 16384, down K=8192)",
                        decoder_layer(0, 1))
    if name == "cfg_decode":
        ls = range(N_LAYERS) if layers is None else layers
        return Workload(name, "batched-CFG decode step, M=2, 26 stacked layers, per-row X scale U(0.5,2)",
                        [l for i in ls for l in decoder_layer(i, 2, row_scale=True)])
    if name == "concurrent":
        ls = range(N_LAYERS) if layers is None else layers
        return Workload(name, "concurrent decode, M=32, 26 stacked layers, 3 of 32 X rows x8",
                        [l for i in ls for l in decoder_layer(i, 32, outlier_rows=3)])
    if name == "layer_fused":
        return Workload(name, "the layer set at M=1 with fused epilogues: O and down + residual, "
                              "gate/up -> SwiGLU (one grouped launch)", decoder_layer(0, 1), fused=True)
    if name == "flow_head":
        # the flow-matching head: 3 transformer layers run once per Euler step
        # on the batch-2 CFG rows (the pages give no width for it; reading:
        # the decoder's linear shapes, since it consumes the decoder's hidden
        # states); one step = one Euler step = the 3 layers' 12 GEMMs
        ls = range(FLOW_LAYERS) if layers is None else layers
        return Workload(name, "flow-head Euler step, M=2 (CFG), 3 layers of the decoder linear set",
                        [l for i in ls for l in decoder_layer(FLOW_LAYER0 + i, 2, row_scale=True)])
    if name == "adapter":
        return Workload(name, "adapter/prefill GEMM M=4096, K=5120, N=3072, X ~ N(0, 0.5^2)",
                        [Linear("adapter", D_MODEL, ADAPTER_IN, 0, 0, 4096, sigma=0.5)])
    if name == "qkv_prefill":
        return Workload(name, "fused-QKV prefill GEMM M=4096, K=3072, N=5120, X ~ N(0, 0.5^2)",
                        [Linear("qkv", Q_DIM + 2 * KV_DIM, D_MODEL, 0, 0, 4096, sigma=0.5)])
    raise KeyError(name)


WORKLOADS = ["gemv", "layer", "layer_fused", "cfg_decode", "concurrent", "flow_head", "adapter", "qkv_prefill"]

# ---------------------------------------------------------------------------
# the two utilities around the product (row gather, quantization)
# ---------------------------------------------------------------------------

T_IDS = 6
T_WEIGHTS = 7

EMBED_VOCAB, EMBED_DIM, EMBED_TOKENS = 131072, 3072, 4096
QUANT_N, QUANT_K = 16384, 3072


def gen_ids(T: int, V: int, seed: int = SEED, stream: int = 0) -> np.ndarray:
    """int32 [T] token ids, uniform in 0..V-1."""
    return _rng(seed, 0, T_IDS, stream).integers(0, V, size=T, dtype=np.int32)


def gen_weights(N: int, K: int, seed: int = SEED, stream: int = 0, sigma: float = 0.02) -> np.ndarray:
    """float32 [N, K] ~ N(0, sigma^2): unquantized weights to feed q4_0_quantize."""
    x = _rng(seed, 0, T_WEIGHTS, stream).standard_normal(size=(N, K), dtype=np.float32)
    x *= np.float32(sigma)
    return x


UTIL_WORKLOADS = {
    "embed": (f"Q4 embedding lookup: {EMBED_TOKENS} token ids uniform over a {EMBED_VOCAB} x {EMBED_DIM} "
              f"Q4_0 table ({EMBED_VOCAB * EMBED_DIM // 32 * 18 / 2**20:.1f} MiB), rows dequantized to fp32"),
    "quantize": f"quantize fp32 weights [{QUANT_N}, {QUANT_K}] ~ N(0, 0.02^2) to Q4_0",
}
