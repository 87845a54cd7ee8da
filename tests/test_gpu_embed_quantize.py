"""Row gather (Q4 embedding lookup) and quantization on the GPU against the
oracle, bit for bit, through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
from tests.gpu_helpers import dev, no_device_error

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q4():
    import bit_weight_only_matmul_b200 as q4
    q4.q4_0_force_path(q4.PATH_AUTO)
    return q4


def _table(rng, V, D):
    codes = rng.integers(0, 16, size=(V, D), dtype=np.uint8)
    scales = (np.abs(rng.standard_normal((V, D // 32))) * 0.002 + 1e-4).astype(np.float16).view(np.uint16)
    return oracle.get().pack(codes, scales)


@pytest.mark.parametrize("V,D,T", [(1000, 3072, 257), (50, 96, 33), (7, 32, 5), (300, 4096, 1), (64, 160, 100)])
def test_gather_bit_exact(q4, V, D, T):
    rng = np.random.default_rng(V + D + T)
    W = _table(rng, V, D)
    ids = rng.integers(0, V, size=T).astype(np.int32)
    ids[:min(T, 3)] = [0, V - 1, 0][:min(T, 3)]
    out = torch.full((T, D), float("nan"), device="cuda")
    q4.q4_0_gather(dev(W.reshape(-1)), dev(ids), out, T, V, D)
    ref, bad = oracle.get().gather_f32(W, ids, V, D)
    assert bad == 0
    assert np.array_equal(out.cpu().numpy().view(np.uint32), ref.view(np.uint32))
    no_device_error(q4)


def test_gather_bad_ids_give_zero_rows_and_flag(q4):
    rng = np.random.default_rng(3)
    V, D = 40, 128
    W = _table(rng, V, D)
    ids = np.array([5, -1, V, 39, 2**31 - 1, 0], np.int32)
    out = torch.full((len(ids), D), float("nan"), device="cuda")
    q4.q4_0_device_error(clear=True)
    q4.q4_0_gather(dev(W.reshape(-1)), dev(ids), out, len(ids), V, D)
    ref, bad = oracle.get().gather_f32(W, ids, V, D)
    assert bad == 3
    assert np.array_equal(out.cpu().numpy().view(np.uint32), ref.view(np.uint32))
    assert q4.q4_0_device_error(clear=True) == q4.Q4_DEVERR_BAD_INDEX
    assert q4.q4_0_device_error(clear=True) == 0


def _weights(rng, N, K):
    x = rng.standard_normal((N, K)).astype(np.float32)
    x *= np.exp2(rng.integers(-20, 12, size=(N, K // 32, 1))).astype(np.float32).repeat(32, axis=2).reshape(N, K)
    x[::5, K - 24] = -x[::5, K - 31]                 # equal extreme magnitudes of opposite sign
    x[1, 0:32] = 0.0                                 # an all-zero block
    x[2, K - 32:K] = -0.0                            # all negative zeros
    x[3, 0:32] = 1e6 * np.sign(x[3, 0:32])           # d beyond the fp16 range (stored as inf)
    x[4, 0:32] *= np.float32(1e-5) / np.abs(x[4, 0:32]).max()   # d in the fp16 subnormal range
    return x


@pytest.mark.parametrize("N,K", [(64, 3072), (5, 32), (17, 256), (300, 1024)])
def test_quantize_bit_exact(q4, N, K):
    rng = np.random.default_rng(N * 7 + K)
    X = np.ascontiguousarray(_weights(rng, max(N, 5), K)[:N])
    W = torch.empty(q4.q4_0_bytes(N, K), dtype=torch.uint8, device="cuda")
    q4.q4_0_quantize(dev(np.ascontiguousarray(X)), W, N, K)
    ref = oracle.get().quantize(X)
    assert np.array_equal(W.cpu().numpy(), ref.reshape(-1))


def test_quantize_then_gather_round_trip(q4):
    """quantize -> gather reproduces each weight to within half a step
    (one step where the code is clamped at 15)."""
    rng = np.random.default_rng(9)
    V, D = 200, 512
    X = (rng.standard_normal((V, D)) * 0.02).astype(np.float32)
    W = torch.empty(q4.q4_0_bytes(V, D), dtype=torch.uint8, device="cuda")
    q4.q4_0_quantize(dev(X), W, V, D)
    ids = np.arange(V, dtype=np.int32)
    out = torch.empty((V, D), device="cuda")
    q4.q4_0_gather(W, dev(ids), out, V, V, D)
    codes, scales = oracle.get().unpack(W.cpu().numpy(), V, D)
    d = np.abs(scales.view(np.float16).astype(np.float64)).repeat(32, axis=1)
    err = np.abs(out.cpu().numpy().astype(np.float64) - X)
    assert np.all(err <= d * (1.0 + 1e-2) + 1e-12)
    no_device_error(q4)
