"""GPU quantisers (the export's dq4 and embedding_int8 steps, "ONNX export,
quantization and the browser runtime", section "Quantization
(train/quantize.py)", steps 2 and 3) against the oracle: the integer codes,
zero points and stored scales must be bit-identical (both sides take every
decision with the same fp64 operations)."""

import numpy as np
import pytest

import oracle
from gpu_util import dev, torch

pytestmark = pytest.mark.gpu


def w4():
    import int8_weight_quantized_w4_b200 as w
    return w


def _weights(K, N, seed):
    g = np.random.default_rng(seed)
    w = (g.standard_normal((K, N)) * 0.05).astype(np.float32)
    if N >= 8:
        w[:, 0] = 0.0                       # all-zero column: scale 1, zero point 0
        w[:, 1] = np.abs(w[:, 1])           # all positive: lo = 0
        w[:, 2] = -np.abs(w[:, 2])          # all negative: hi = 0
        w[K // 2, 3] = 40.0                 # an outlier
        w[:, 4] = np.round(w[:, 4] * 64) / 64  # values on a dyadic grid (ties possible)
    return w


@pytest.mark.parametrize("K,N,block,st", [
    (64, 96, 32, "fp32"),
    (768, 2304, 32, "fp32"),      # GPT-2 fused QKV
    (3072, 768, 64, "fp32"),
    (128, 100, 64, "fp16"),
    (96, 34, 32, "fp16"),         # N % 32 != 0
])
def test_w4_quantize_bit_exact(K, N, block, st):
    w = _weights(K, N, K + N)
    qw, sc, zp = w4().w4_quantize(dev(w), block=block, scale_type=st)
    torch().cuda.synchronize()
    rq, rs, rz = oracle.quantize_w4(w, block=block, scale_type=st)
    assert np.array_equal(qw.cpu().numpy(), rq)
    assert np.array_equal(zp.cpu().numpy(), rz)
    got_s = sc.cpu().numpy().reshape(-1)
    assert got_s.dtype == rs.dtype
    assert np.array_equal(got_s.view(np.uint32 if st == "fp32" else np.uint16),
                          rs.reshape(-1).view(np.uint32 if st == "fp32" else np.uint16))


def test_w4_quantize_padded_rows():
    T = torch()
    K, N, ld = 64, 40, 52
    w = _weights(K, N, 9)
    buf = T.full((K, ld), float("nan"), device="cuda")
    buf[:, :N] = dev(w)
    qw, sc, zp = w4().w4_quantize(buf[:, :N])
    T.cuda.synchronize()
    rq, rs, rz = oracle.quantize_w4(w)
    assert np.array_equal(qw.cpu().numpy(), rq) and np.array_equal(zp.cpu().numpy(), rz)
    assert np.array_equal(sc.cpu().numpy().reshape(-1), rs.reshape(-1))


def test_quantise_then_multiply():
    """GPU-quantised weights through the GEMV equal the oracle's matmul on the
    oracle-quantised weights (the same bits)."""
    K, N = 768, 768
    w = _weights(K, N, 5)
    x = np.random.default_rng(6).standard_normal((1, K)).astype(np.float32)
    qw, sc, zp = w4().w4_quantize(dev(w))
    y = w4().w4_matmul(dev(x), qw, sc, zp, K, N, path="gemv")
    torch().cuda.synchronize()
    rq, rs, rz = oracle.quantize_w4(w)
    y_ref, a = oracle.w4_matmul_ref(x, rq, rs, rz, K, N)
    assert oracle.max_violation(y.cpu().numpy(), y_ref, a) <= 0


@pytest.mark.parametrize("K,V", [(768, 50257), (16, 300)])
def test_i8_quantize_head_bit_exact(K, V):
    g = np.random.default_rng(K)
    w = (g.standard_normal((K, V)) * 0.1).astype(np.float32)
    w[:, 7] = 0.0
    w[3, 8] = -9.0
    t, s = w4().i8_quantize_head(dev(w))
    torch().cuda.synchronize()
    rt, rs = oracle.quantize_i8_head(w)
    assert np.array_equal(t.cpu().numpy(), rt)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), rs.view(np.uint32))
