"""Pins that tie the float64 oracle to facts outside itself.

Each check takes an ``oracle.Oracle`` and raises AssertionError on a
mismatch.  ``test_oracle_pins.py`` runs them on the oracle; the mutant test
runs them on builds of the oracle with one planted mistake each and requires
that every mistake trips at least one pin.

What each pin is tied to:
  * fp16 / bf16 decoding: numpy's float16 and torch's bfloat16 types, on all
    65536 bit patterns;
  * block layout and dequantization: hand-built blocks in
    tests/golden/q4_0_blocks.txt (derived by hand from the Q4_0 convention);
  * packing: exhaustive round trip, every code at every position;
  * GEMM: closed forms (all codes 8 give exactly zero; a single off-centre
    nibble gives exactly (c-8)*d*x; constant codes with constant X give
    x*(c-8)*32*sum(d)), linearity in X, and brute force on tiny shapes via
    numpy's matmul on weights built straight from the unpacked codes;
  * fp32 -> fp16 rounding: numpy's float16 conversion (round to nearest
    even) on special values and random bit patterns;
  * quantization: hand-derived blocks in tests/golden/q4_0_quantize.txt, and
    properties of the rule computed independently with numpy (the extreme
    element maps to code 0, every other element is within half a step of
    its reconstruction, symmetry under negation and power-of-two scaling);
  * gather: equals the pinned dequantization row by row, zero rows for ids
    out of range;
  * swiglu: closed forms of silu (silu(0) = 0, silu(x) - silu(-x) = x,
    silu(1) = e/(1+e) from math.exp, silu(x) -> x and -> 0 at the ends) and
    the product with u;
  * sizes: 4.5 bits per weight, cross-checked with the pages' 1.5 GiB fp32
    embedding table that becomes 216 MB in Q4 (hakusoku.com story 5135,
    linear ops and embeddings; voxtral-mini-realtime-rs README, "WASM
    Constraints Solved", item 3).
"""
from __future__ import annotations

import math
import os
from fractions import Fraction

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "q4_0_blocks.txt")
QGOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "q4_0_quantize.txt")


def load_golden():
    cases, cur = [], None
    for raw in open(GOLDEN):
        line = raw.strip()
        if not line or line.startswith("#"):
            continue
        key, _, rest = line.partition(" ")
        if key == "case":
            cur = {"name": rest}
        elif key == "codes":
            cur["codes"] = np.array([int(c, 16) for c in rest], np.uint8)
        elif key == "d":
            cur["d"] = int(rest, 16)
        elif key == "d_value":
            cur["d_value"] = Fraction(rest)
        elif key == "bytes":
            cur["bytes"] = np.array([int(b, 16) for b in rest.split()], np.uint8)
        elif key == "w":
            cur["w"] = [Fraction(v) for v in rest.split()]
        elif key == "end":
            assert len(cur["codes"]) == 32 and len(cur["bytes"]) == 18 and len(cur["w"]) == 32
            cases.append(cur)
            cur = None
    return cases


def _bf16(values) -> np.ndarray:
    """bf16 bit patterns of values that are exactly representable in bf16."""
    f = np.asarray(values, np.float32)
    bits = (f.view(np.uint32) >> 16).astype(np.uint16)
    assert np.array_equal((bits.astype(np.uint32) << 16).view(np.float32), f), "not exact in bf16"
    return bits


def _fp16_bits(values) -> np.ndarray:
    f = np.asarray(values, np.float16)
    return f.view(np.uint16)


# ---------------------------------------------------------------------------

def pin_half_decoder(o):
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([o.half_to_double(int(b)) for b in bits])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


def pin_bf16_decoder(o):
    import torch
    bits = torch.arange(65536, dtype=torch.int32).to(torch.int16)
    ref = bits.view(torch.bfloat16).to(torch.float64).numpy()
    got = np.array([o.bf16_to_double(int(b) & 0xFFFF) for b in bits.tolist()])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


def pin_golden_blocks(o):
    for c in load_golden():
        codes = c["codes"].reshape(1, 32)
        scales = np.array([[c["d"]]], np.uint16)
        W = o.pack(codes, scales)
        assert np.array_equal(W.reshape(-1), c["bytes"]), c["name"]
        assert Fraction(o.half_to_double(c["d"])) == c["d_value"], c["name"]
        w = o.dequant_f64(c["bytes"].reshape(1, 18), 1, 32).reshape(-1)
        assert [Fraction(float(v)) for v in w] == c["w"], c["name"]
        w32 = o.dequant_f32(c["bytes"].reshape(1, 18), 1, 32).reshape(-1)
        assert [Fraction(float(v)) for v in w32] == c["w"], c["name"]
        uc, us = o.unpack(c["bytes"].reshape(1, 18), 1, 32)
        assert np.array_equal(uc.reshape(-1), c["codes"]) and int(us[0, 0]) == c["d"], c["name"]


def pin_pack_roundtrip_exhaustive(o):
    # row p*16+c: code c at position p, every other code 8
    N, K = 32 * 16, 32
    codes = np.full((N, K), 8, np.uint8)
    for p in range(32):
        for c in range(16):
            codes[p * 16 + c, p] = c
    rng = np.random.default_rng(7)
    scales = _fp16_bits(rng.uniform(0.5, 2.0, size=(N, 1)))
    W = o.pack(codes, scales)
    uc, us = o.unpack(W, N, K)
    assert np.array_equal(uc, codes) and np.array_equal(us, scales)
    w = o.dequant_f64(W, N, K)
    d = scales.view(np.float16).astype(np.float64)
    expect = np.zeros((N, K))
    for p in range(32):
        for c in range(16):
            expect[p * 16 + c, p] = (c - 8) * d[p * 16 + c, 0]
    assert np.array_equal(w, expect)


def pin_all_eight_is_zero(o):
    rng = np.random.default_rng(11)
    M, N, K = 3, 5, 96
    codes = np.full((N, K), 8, np.uint8)
    scales = _fp16_bits(rng.uniform(-50, 50, size=(N, K // 32)))
    X = _bf16(rng.integers(-100, 100, size=(M, K)))
    Y, B = o.gemm(o.pack(codes, scales), X, M, N, K)
    assert np.all(Y == 0.0) and np.all(B == 0.0)


def pin_single_nibble(o):
    rng = np.random.default_rng(12)
    M, N, K = 2, 3, 64
    for (n, k, c) in [(0, 0, 0), (1, 17, 15), (2, 63, 3), (1, 40, 9)]:
        codes = np.full((N, K), 8, np.uint8)
        codes[n, k] = c
        scales = _fp16_bits(rng.uniform(0.001, 3.0, size=(N, K // 32)))
        X = _bf16(rng.integers(-200, 200, size=(M, K)) / 8.0)
        Y, B = o.gemm(o.pack(codes, scales), X, M, N, K)
        d = float(scales.view(np.float16)[n, k // 32])
        x = (X.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        expect = np.zeros((M, N))
        expect[:, n] = (c - 8) * d * x[:, k]
        assert np.array_equal(Y, expect), (n, k, c)
        assert np.array_equal(B, np.abs(expect))


def pin_constant_closed_form(o):
    rng = np.random.default_rng(13)
    M, N, K = 2, 4, 32 * 7
    for c in (0, 3, 8, 15):
        for xi in (1.0, -0.375, 3.5):
            codes = np.full((N, K), c, np.uint8)
            scales = _fp16_bits(rng.uniform(1e-4, 0.01, size=(N, K // 32)))
            X = _bf16(np.full((M, K), xi))
            Y, _ = o.gemm(o.pack(codes, scales), X, M, N, K)
            for n in range(N):
                dsum = sum(Fraction(float(v)) for v in scales.view(np.float16)[n])
                exact = Fraction(xi) * (c - 8) * 32 * dsum
                for m in range(M):
                    assert abs(Fraction(Y[m, n]) - exact) <= abs(exact) * Fraction(1, 2**50), (c, xi, n)


def _numpy_reference(codes, scales, X):
    """Y from the unpacked codes via numpy's matmul (independent of the
    oracle's bit layout and of its fp16/bf16 decoders)."""
    import torch
    w = (codes.astype(np.float64) - 8.0) * np.repeat(scales.view(np.float16).astype(np.float64), 32, axis=1)
    x = torch.from_numpy(X.astype(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    return x @ w.T, np.abs(x) @ np.abs(w).T


def pin_brute_force_tiny(o):
    rng = np.random.default_rng(14)
    for M in (1, 2, 3):
        for N in (1, 5):
            for K in (32, 64, 96):
                codes = rng.integers(0, 16, size=(N, K), dtype=np.uint8)
                scales = _fp16_bits(np.abs(rng.standard_normal(size=(N, K // 32))) * 0.002 + 1e-4)
                X = _bf16(np.round(rng.standard_normal(size=(M, K)) * 64) / 64)
                Y, B = o.gemm(o.pack(codes, scales), X, M, N, K)
                Yr, Br = _numpy_reference(codes, scales, X)
                assert Y.shape == (M, N)
                assert np.all(np.abs(Y - Yr) <= 1e-12 * Br + 1e-300), (M, N, K)
                assert np.allclose(B, Br, rtol=1e-12, atol=0), (M, N, K)


def pin_one_hot_reads_weights(o):
    rng = np.random.default_rng(15)
    N, K = 6, 64
    codes = rng.integers(0, 16, size=(N, K), dtype=np.uint8)
    scales = _fp16_bits(rng.uniform(0.01, 1.0, size=(N, K // 32)))
    W = o.pack(codes, scales)
    d = np.repeat(scales.view(np.float16).astype(np.float64), 32, axis=1)
    X = _bf16(np.eye(K))
    Y, _ = o.gemm(W, X, K, N, K)   # row k of Y = column k of w
    assert np.array_equal(Y, ((codes.astype(np.float64) - 8) * d).T)


def pin_linearity(o):
    rng = np.random.default_rng(16)
    M, N, K = 3, 4, 128
    codes = rng.integers(0, 16, size=(N, K), dtype=np.uint8)
    scales = _fp16_bits(rng.uniform(0.001, 0.01, size=(N, K // 32)))
    W = o.pack(codes, scales)
    a = rng.integers(-60, 60, size=(M, K))
    b = rng.integers(-60, 60, size=(M, K))
    Ya, Ba = o.gemm(W, _bf16(a), M, N, K)
    Yb, Bb = o.gemm(W, _bf16(b), M, N, K)
    Yab, _ = o.gemm(W, _bf16(a + b), M, N, K)
    assert np.all(np.abs(Yab - (Ya + Yb)) <= 1e-12 * (Ba + Bb))


def pin_sampled_matches_full(o):
    rng = np.random.default_rng(17)
    M, N, K = 4, 7, 96
    codes = rng.integers(0, 16, size=(N, K), dtype=np.uint8)
    scales = _fp16_bits(rng.uniform(0.001, 0.01, size=(N, K // 32)))
    X = _bf16(rng.integers(-9, 9, size=(M, K)))
    W = o.pack(codes, scales)
    Y, B = o.gemm(W, X, M, N, K)
    ms = np.array([0, 3, 2, 1, 3]); ns = np.array([6, 0, 3, 5, 6])
    Ys, Bs = o.gemm_sampled(W, X, M, N, K, ms, ns)
    assert np.array_equal(Ys, Y[ms, ns]) and np.array_equal(Bs, B[ms, ns])


def pin_sizes(o):
    assert o.row_bytes(32) == 18
    assert o.row_bytes(3072) == 1728
    assert o.row_bytes(8192) == 4608
    # 1.5 GiB of fp32 embeddings (vocab 131072 x 3072) -> 216 MiB in Q4_0
    weights = int(1.5 * 2**30) // 4
    assert weights == 131072 * 3072
    assert 131072 * o.row_bytes(3072) == 216 * 2**20
    # 4.5 bits per weight
    assert o.row_bytes(3072) * 8 * 2 == 3072 * 9


def load_quantize_golden():
    cases, cur = [], None
    for raw in open(QGOLDEN):
        line = raw.strip()
        if not line or line.startswith("#"):
            continue
        key, _, rest = line.partition(" ")
        if key == "case":
            cur = {"name": rest}
        elif key == "x":
            vals = [Fraction(v) for v in rest.split()]
            x = np.array([float(v) for v in vals], np.float32)
            assert [Fraction(float(v)) for v in x] == vals, "fixture values must be exact in float32"
            cur["x"] = x
        elif key == "bytes":
            cur["bytes"] = np.array([int(b, 16) for b in rest.split()], np.uint8)
        elif key == "end":
            assert len(cur["x"]) == 32 and len(cur["bytes"]) == 18
            cases.append(cur)
            cur = None
    return cases


def pin_float_to_half(o):
    special = np.array([0.0, -0.0, 1.0, -1.0, 65504.0, 65519.99, 65520.0, 1e9, -1e9, np.inf, -np.inf,
                        2.0**-14, 2.0**-24, 2.0**-25, 2.0**-25 * 1.0000001, 2.0**-26, 3 * 2.0**-25,
                        2.0**-14 - 2.0**-25, 1.0 + 2.0**-11, 1.0 + 3 * 2.0**-11, 0.1, 1 / 3], np.float32)
    rng = np.random.default_rng(5)
    bits = rng.integers(0, 2**32, size=200000, dtype=np.uint64).astype(np.uint32)
    vals = np.concatenate([special, bits.view(np.float32)])
    with np.errstate(over="ignore"):
        ref = vals.astype(np.float16)
    for v, r in zip(vals, ref):
        h = o.float_to_half(float(v))
        if np.isnan(v):
            assert (h & 0x7c00) == 0x7c00 and (h & 0x3ff) != 0
        else:
            assert h == int(r.view(np.uint16)), (float(v), hex(h), hex(int(r.view(np.uint16))))


def pin_quantize_golden(o):
    for c in load_quantize_golden():
        W = o.quantize(c["x"].reshape(1, 32))
        assert np.array_equal(W.reshape(-1), c["bytes"]), (c["name"], W.reshape(-1).tobytes().hex(" "))


def _blocks(rng, n):
    """Blocks of 32 float32 values at scales over many binades, some with
    repeated extreme magnitudes."""
    x = rng.standard_normal((n, 32)).astype(np.float32)
    x *= np.exp2(rng.integers(-12, 12, size=(n, 1))).astype(np.float32)
    x[::7, 9] = -x[::7, 3]            # the same magnitude twice, opposite signs
    return x


def pin_quantize_rounding_bound(o):
    rng = np.random.default_rng(6)
    X = _blocks(rng, 400)
    W = o.quantize(X.reshape(-1, 64))   # 200 rows of two blocks
    codes, scales = o.unpack(W, 200, 64)
    codes = codes.reshape(-1, 32).astype(np.float64)
    scales = scales.reshape(-1)
    for x, q, dh in zip(X, codes, scales):
        i = int(np.argmax(np.abs(x)))          # first of the largest magnitudes
        d = np.float32(x[i]) / np.float32(-8.0)
        assert int(np.float16(d).view(np.uint16)) == int(dh)
        assert q[i] == 0
        err = np.abs((q - 8) * np.float64(d) - x.astype(np.float64))
        step = abs(float(d))
        # x/d lies in [-8, 8]; codes above 15 are clamped, so values with
        # x/d >= 7.5 (the far side from the extreme) may be off by one step
        clamped = x.astype(np.float64) / np.float64(d) >= 7.5 - 2.0**-18
        assert np.all(err[~clamped] <= 0.5 * step * (1 + 2.0**-20)), float(err[~clamped].max() / step)
        assert np.all(err[clamped] <= step * (1 + 2.0**-20))
        assert np.all(q[clamped] == 15)


def pin_quantize_sign_and_scale(o):
    rng = np.random.default_rng(7)
    X = _blocks(rng, 64).reshape(-1, 64)
    c0, s0 = o.unpack(o.quantize(X), 32, 64)
    c1, s1 = o.unpack(o.quantize(-X), 32, 64)
    assert np.array_equal(c0, c1) and np.array_equal(s0 ^ 0x8000, s1)
    for k in (-3, 5):
        c2, s2 = o.unpack(o.quantize(X * np.float32(2.0**k)), 32, 64)
        assert np.array_equal(c0, c2)
        d = s0.view(np.float16).astype(np.float64) * 2.0**k
        ok = np.abs(d) >= 2.0**-14           # scales that stay normal in fp16
        assert np.array_equal(s2.view(np.float16).astype(np.float64)[ok], d[ok])


def pin_gather_matches_dequant(o):
    rng = np.random.default_rng(8)
    V, D = 37, 96
    codes = rng.integers(0, 16, size=(V, D), dtype=np.uint8)
    scales = (rng.standard_normal((V, D // 32)) * 0.01).astype(np.float16).view(np.uint16)
    W = o.pack(codes, scales)
    full = o.dequant_f32(W, V, D)
    ids = np.concatenate([rng.permutation(V), rng.integers(0, V, 20), [0, V - 1, V - 1]]).astype(np.int32)
    out, bad = o.gather_f32(W, ids, V, D)
    assert bad == 0 and np.array_equal(out, full[ids])
    out, bad = o.gather_f32(W, np.array([-1, 3, V, 2**31 - 1], np.int32), V, D)
    assert bad == 3 and np.array_equal(out[1], full[3])
    assert not out[[0, 2, 3]].any()


def pin_swiglu_closed_forms(o):
    g = np.array([0.0, 1.0, -1.0, 2.5, -2.5, 40.0, -40.0, 1e-9])
    u = np.array([3.0, 1.0, 1.0, 1.0, 1.0, 1.0, 1.0, 1.0])
    out = o.swiglu(g, u)
    assert out[0] == 0.0
    assert abs(out[1] - math.e / (1 + math.e)) <= 1e-15
    assert abs(out[1] - out[2] - 1.0) <= 1e-15 and abs(out[3] - out[4] - 2.5) <= 1e-15
    assert abs(out[5] - 40.0) <= 1e-12 and abs(out[6]) <= 1e-15
    assert abs(out[7] - 0.5e-9) <= 1e-18          # silu(e) = e/2 + e^2/4 + ...
    gg = np.linspace(-8, 8, 33)
    assert np.allclose(o.swiglu(gg, np.full(33, -2.0)), -2.0 * o.swiglu(gg, np.ones(33)), rtol=0, atol=0)


ALL_PINS = [
    pin_half_decoder,
    pin_bf16_decoder,
    pin_golden_blocks,
    pin_pack_roundtrip_exhaustive,
    pin_all_eight_is_zero,
    pin_single_nibble,
    pin_constant_closed_form,
    pin_brute_force_tiny,
    pin_one_hot_reads_weights,
    pin_linearity,
    pin_sampled_matches_full,
    pin_sizes,
    pin_float_to_half,
    pin_quantize_golden,
    pin_quantize_rounding_bound,
    pin_quantize_sign_and_scale,
    pin_gather_matches_dequant,
    pin_swiglu_closed_forms,
]
