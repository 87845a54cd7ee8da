"""Fused epilogues (residual add, SwiGLU of a row-interleaved gate/up weight)
through q4_0_gemm_grouped_ex, against the float64 oracle: on the decode path
(M <= 32) and on the tensor-core kernel (M > 32, ragged activation tiles
included)."""
import numpy as np
import pytest
import torch

import oracle
from tests.gpu_helpers import dev, no_device_error, pack_on_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q4():
    import bit_weight_only_matmul_b200 as q4
    q4.q4_0_force_path(q4.PATH_AUTO)
    return q4


def _weights(rng, N, K):
    codes = rng.integers(0, 16, size=(N, K), dtype=np.uint8)
    scales = (np.abs(rng.standard_normal((N, K // 32))) * 0.002 + 1e-4).astype(np.float16).view(np.uint16)
    return codes, scales


def _x(rng, M, K):
    import workloads
    return workloads.fp32_to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32))


def _bound(B):
    return 1e-3 * B + 1e-6


def _check(got, ref, tol, what):
    err = np.abs(np.asarray(got, np.float64) - ref)
    bad = ~(err <= tol)
    assert not bad.any(), f"{what}: {bad.sum()} outside; worst {float((err / tol).max())}"


def test_interleave_bit_exact(q4):
    rng = np.random.default_rng(1)
    F, K = 192, 512
    o = oracle.get()
    Wg, Wu = o.pack(*_weights(rng, F, K)), o.pack(*_weights(rng, F, K))
    out = torch.empty(2 * F * (K // 32) * 18, dtype=torch.uint8, device="cuda")
    q4.q4_0_interleave_gate_up(dev(Wg.reshape(-1)), dev(Wu.reshape(-1)), out, F, K)
    want = np.concatenate([np.concatenate([Wg[64 * i:64 * i + 64], Wu[64 * i:64 * i + 64]]) for i in range(F // 64)])
    assert np.array_equal(out.cpu().numpy(), want.reshape(-1))


@pytest.mark.parametrize("M,N,K", [(1, 3072, 3072), (2, 200, 1024), (32, 300, 512), (7, 129, 768), (16, 257, 768),
                                   (33, 200, 512), (300, 129, 768), (600, 512, 1024)])
@pytest.mark.parametrize("inplace", [False, True])
def test_residual_epilogue(q4, M, N, K, inplace):
    rng = np.random.default_rng(M + N + K + inplace)
    o = oracle.get()
    codes, scales = _weights(rng, N, K)
    X = _x(rng, M, K)
    R = rng.standard_normal((M, N)).astype(np.float32)
    Rd = dev(R)
    Y = Rd if inplace else torch.full((M, N), float("nan"), device="cuda")
    q4.q4_0_gemm_grouped_ex([(pack_on_gpu(q4, codes, scales), dev(X), Y, M, N, K, Rd, q4.Q4_0_EPI_RESIDUAL)])
    Y_or, B_or = o.gemm(o.pack(codes, scales), X, M, N, K)
    ref = Y_or + R
    _check(Y.cpu().numpy(), ref, _bound(B_or) + 2.0**-22 * np.abs(ref), "residual")
    no_device_error(q4)


def _swiglu_case(q4, rng, M, F, K):
    o = oracle.get()
    (cg, sg), (cu, su) = _weights(rng, F, K), _weights(rng, F, K)
    X = _x(rng, M, K)
    Wgu = torch.empty(2 * F * (K // 32) * 18, dtype=torch.uint8, device="cuda")
    q4.q4_0_interleave_gate_up(pack_on_gpu(q4, cg, sg), pack_on_gpu(q4, cu, su), Wgu, F, K)
    Yg, Bg = o.gemm(o.pack(cg, sg), X, M, F, K)
    Yu, Bu = o.gemm(o.pack(cu, su), X, M, F, K)
    ref = o.swiglu(Yg, Yu)
    Tg, Tu = _bound(Bg), _bound(Bu)
    sil = np.abs(o.swiglu(Yg, np.ones_like(Yg)))
    # |d silu| <= 1.1 |dg|; plus fp32 rounding of the epilogue itself
    tol = 1.1 * Tg * (np.abs(Yu) + Tu) + (sil + 1.1 * Tg) * Tu + 1e-5 * np.abs(ref) + 1e-6
    return Wgu, X, ref, tol


@pytest.mark.parametrize("M,F,K", [(1, 64, 256), (2, 512, 1024), (32, 256, 512), (12, 192, 1024), (1, 8192, 3072),
                                   (33, 64, 256), (300, 320, 512), (513, 1024, 1024)])
def test_swiglu_epilogue(q4, M, F, K):
    rng = np.random.default_rng(M * 3 + F + K)
    Wgu, X, ref, tol = _swiglu_case(q4, rng, M, F, K)
    Y = torch.full((M, F), float("nan"), device="cuda")
    q4.q4_0_gemm_grouped_ex([(Wgu, dev(X), Y, M, 2 * F, K, None, q4.Q4_0_EPI_SWIGLU)])
    _check(Y.cpu().numpy(), ref, tol, "swiglu")
    no_device_error(q4)


@pytest.mark.parametrize("M,N,K", [(1, 3072, 3072), (5, 1000, 768)])
def test_epilogues_forced_256k_stage_kernel(q4, M, N, K):
    """Residual and SwiGLU on the M <= 32 kernel forced for M <= 8 (one n
    tile; cluster split mode for the few-item case)."""
    rng = np.random.default_rng(M + N + K + 5)
    o = oracle.get()
    codes, scales = _weights(rng, N, K)
    X = _x(rng, M, K)
    R = rng.standard_normal((M, N)).astype(np.float32)
    Y = torch.full((M, N), float("nan"), device="cuda")
    Wgu, Xs, ref_s, tol_s = _swiglu_case(q4, rng, M, N // 2 // 64 * 64, K)
    F = N // 2 // 64 * 64
    Ys = torch.full((M, F), float("nan"), device="cuda")
    q4.q4_0_force_path(q4.PATH_DECODE)
    try:
        q4.q4_0_gemm_grouped_ex([(pack_on_gpu(q4, codes, scales), dev(X), Y, M, N, K, dev(R), q4.Q4_0_EPI_RESIDUAL)])
        q4.q4_0_gemm_grouped_ex([(Wgu, dev(Xs), Ys, M, 2 * F, K, None, q4.Q4_0_EPI_SWIGLU)])
    finally:
        q4.q4_0_force_path(q4.PATH_AUTO)
    Y_or, B_or = o.gemm(o.pack(codes, scales), X, M, N, K)
    ref = Y_or + R
    _check(Y.cpu().numpy(), ref, _bound(B_or) + 2.0**-22 * np.abs(ref), "residual, 256-k stage kernel")
    _check(Ys.cpu().numpy(), ref_s, tol_s, "swiglu, 256-k stage kernel")
    no_device_error(q4)


def test_fused_decoder_layer_one_launch(q4):
    """A whole decoder layer's linears with their epilogues in one grouped
    launch at M=1: QKV plain, O + residual, gate/up -> SwiGLU, down +
    residual (216 items: split mode, the down items halved across a pair)."""
    rng = np.random.default_rng(5)
    o = oracle.get()
    M = 1
    cq, sq = _weights(rng, 5120, 3072)
    co, so = _weights(rng, 3072, 3072)
    cd, sd = _weights(rng, 3072, 8192)
    Xq, Xo, Xd = _x(rng, M, 3072), _x(rng, M, 3072), _x(rng, M, 8192)
    Ro = rng.standard_normal((M, 3072)).astype(np.float32)
    Rd = rng.standard_normal((M, 3072)).astype(np.float32)
    Wgu, Xg, ref_g, tol_g = _swiglu_case(q4, rng, M, 8192, 3072)
    Yq = torch.full((M, 5120), float("nan"), device="cuda")
    Yo = torch.full((M, 3072), float("nan"), device="cuda")
    Yg = torch.full((M, 8192), float("nan"), device="cuda")
    Yd = torch.full((M, 3072), float("nan"), device="cuda")
    Ro_d, Rd_d = dev(Ro), dev(Rd)
    probs = [(pack_on_gpu(q4, cq, sq), dev(Xq), Yq, M, 5120, 3072, None, q4.Q4_0_EPI_NONE),
             (pack_on_gpu(q4, co, so), dev(Xo), Yo, M, 3072, 3072, Ro_d, q4.Q4_0_EPI_RESIDUAL),
             (Wgu, dev(Xg), Yg, M, 16384, 3072, None, q4.Q4_0_EPI_SWIGLU),
             (pack_on_gpu(q4, cd, sd), dev(Xd), Yd, M, 3072, 8192, Rd_d, q4.Q4_0_EPI_RESIDUAL)]
    for rep in range(2):
        for Y in (Yq, Yo, Yg, Yd):
            Y.fill_(float("nan"))
        q4.q4_0_gemm_grouped_ex(probs)
        y, b = o.gemm(o.pack(cq, sq), Xq, M, 5120, 3072)
        _check(Yq.cpu().numpy(), y, _bound(b), "qkv")
        y, b = o.gemm(o.pack(co, so), Xo, M, 3072, 3072)
        _check(Yo.cpu().numpy(), y + Ro, _bound(b) + 2.0**-22 * np.abs(y + Ro), "o + residual")
        _check(Yg.cpu().numpy(), ref_g, tol_g, "gate/up swiglu")
        y, b = o.gemm(o.pack(cd, sd), Xd, M, 3072, 8192)
        _check(Yd.cpu().numpy(), y + Rd, _bound(b) + 2.0**-22 * np.abs(y + Rd), "down + residual")
    no_device_error(q4)


def test_mixed_paths_one_call(q4):
    """One grouped_ex call holding M <= 32 problems (one decode launch) and
    M > 32 problems (one tensor-core launch each), every epilogue kind."""
    rng = np.random.default_rng(9)
    o = oracle.get()
    cases = []
    for M, N, K, epi in [(2, 384, 512, q4.Q4_0_EPI_RESIDUAL), (100, 384, 512, q4.Q4_0_EPI_RESIDUAL),
                         (64, 256, 768, q4.Q4_0_EPI_NONE), (4, 256, 768, q4.Q4_0_EPI_NONE)]:
        codes, scales = _weights(rng, N, K)
        X = _x(rng, M, K)
        R = rng.standard_normal((M, N)).astype(np.float32)
        Y = torch.full((M, N), float("nan"), device="cuda")
        cases.append((codes, scales, X, R, Y, M, N, K, epi))
    Wgu, Xg, ref_g, tol_g = _swiglu_case(q4, rng, 70, 128, 512)
    Yg = torch.full((70, 128), float("nan"), device="cuda")
    probs = [(pack_on_gpu(q4, c, s), dev(X), Y, M, N, K, dev(R) if epi == q4.Q4_0_EPI_RESIDUAL else None, epi)
             for (c, s, X, R, Y, M, N, K, epi) in cases]
    probs.append((Wgu, dev(Xg), Yg, 70, 256, 512, None, q4.Q4_0_EPI_SWIGLU))
    q4.q4_0_gemm_grouped_ex(probs)
    for (c, s, X, R, Y, M, N, K, epi) in cases:
        y, b = o.gemm(o.pack(c, s), X, M, N, K)
        ref = y + R if epi == q4.Q4_0_EPI_RESIDUAL else y
        _check(Y.cpu().numpy(), ref, _bound(b) + 2.0**-22 * np.abs(ref), f"M={M} epilogue {epi}")
    _check(Yg.cpu().numpy(), ref_g, tol_g, "swiglu M=70")
    no_device_error(q4)
