"""GPU parity of the tensor-core (tcgen05, 3xTF32) path of w4_matmul against
the oracle: ragged tiles in M and N, several K-blocks, exact closed forms,
determinism, and the automatic choice for M above 16."""

import numpy as np
import pytest

import oracle
import pins
from gpu_util import check, dev, guarded, guards_intact, torch, upload_w4

from int8_weight_quantized_w4_b200 import synth

pytestmark = pytest.mark.gpu


def w4():
    import int8_weight_quantized_w4_b200 as w
    return w


def run_case(M, K, N, path="tc", seed=5, ldx=None, ldy=None):
    W = synth.w4_weight(K, N, M + 100, seed=seed)
    x = synth.activations(M, K, 17, seed=seed, ld=ldx)
    xd = dev(x)[:, :K] if ldx else dev(x)
    y, buf = guarded(M, N, ldy)
    Wd = upload_w4(W)
    w4().w4_matmul(xd, Wd["qw"], Wd["scales"], Wd["zp"], K, N, y=y, path=path)
    torch().cuda.synchronize()
    y_ref, a = oracle.w4_matmul_ref(x[:, :K], W["qw"], W["scales"], W["zp"], K, N)
    check(y, y_ref, a, f"tc M={M} K={K} N={N} path={path}")
    assert guards_intact(buf, M, N, ldy or N), "write outside y"
    return y


@pytest.mark.parametrize("M,K,N", [
    (17, 32, 32),       # one K-block, one ragged tile in both M and N
    (128, 64, 256),     # exactly one tile
    (129, 96, 288),     # one row and 32 columns past a tile
    (58, 768, 768),     # GPT-2 prefill, attention output projection
    (58, 768, 2304),    # GPT-2 prefill, fused QKV
    (300, 256, 544),    # three row tiles, three column tiles
    (64, 3072, 768),    # long K (96 blocks)
    (1, 64, 256),       # M = 1 forced onto the tensor cores
])
def test_tc_shapes(M, K, N):
    run_case(M, K, N)


def test_tc_padded_strides():
    run_case(70, 128, 320, ldx=132, ldy=333)


def test_auto_picks_tensor_cores_above_16_rows():
    # M = 40 goes to the tensor-core kernel on AUTO; same tolerance
    run_case(40, 256, 512, path="auto")


def _exact(q, zp, s, x):
    K, N = q.shape
    qw, sc, zpk = pins.make_w4(q, zp, s)
    y = w4().w4_matmul(dev(x), dev(qw), dev(sc), dev(zpk), K, N, path="tc")
    torch().cuda.synchronize()
    return y.cpu().numpy().astype(np.float64)


def test_tc_closed_forms_exact():
    # values with few significant bits: the tf32 high parts are exact, the low
    # parts zero, every partial sum exact
    M = 20
    y = _exact(np.full((32, 64), 9), np.full((1, 64), 8), np.full((1, 64), 0.5), np.ones((M, 32), np.float32))
    assert np.array_equal(y, np.full((M, 64), 16.0))
    q = np.concatenate([np.full((32, 64), 10), np.full((32, 64), 2)])
    y = _exact(q, np.full((2, 64), 7), np.array([[0.25] * 64, [2.0] * 64]), np.ones((M, 64), np.float32))
    assert np.array_equal(y, np.full((M, 64), 32 * 0.25 * 3 + 32 * 2.0 * -5))
    x = np.tile(((np.arange(64, dtype=np.float32) - 10) / 4)[None, :], (M, 1))
    y = _exact(np.zeros((64, 32)), np.full((2, 32), 15), np.full((2, 32), 0.125), x)
    assert np.array_equal(y, np.full((M, 32), -15 * 0.125 * float(x[0].sum())))
    g = np.random.default_rng(3)
    y = _exact(np.full((96, 64), 6), np.full((3, 64), 6), np.full((3, 64), 0.0173),
               g.standard_normal((M, 96)).astype(np.float32))
    assert np.all(y == 0)


def test_tc_one_hot_rows_within_tolerance():
    """x = e_k returns row k of W (to the 3xTF32 reading of w's low part)."""
    g = np.random.default_rng(4)
    K, N = 96, 256
    qi = g.integers(0, 16, (K, N))
    zi = g.integers(0, 16, (K // 32, N))
    s = g.uniform(0.005, 0.02, (K // 32, N)).astype(np.float32)
    qw, sc, zpk = pins.make_w4(qi, zi, s)
    Wf = oracle.dequantize_w4(qw, sc, zpk, K, N).astype(np.float64)
    ks = [0, 31, 32, 95, 50] * 4
    x = np.zeros((len(ks), K), np.float32)
    for r, k in enumerate(ks):
        x[r, k] = 1.0
    y = w4().w4_matmul(dev(x), dev(qw), dev(sc), dev(zpk), K, N, path="tc").cpu().numpy().astype(np.float64)
    for r, k in enumerate(ks):
        assert np.all(np.abs(y[r] - Wf[k]) <= 1e-5 * np.abs(Wf[k]) + 1e-6), k


def test_tc_deterministic():
    K, N, M = 768, 768, 58
    W = upload_w4(synth.w4_weight(K, N))
    x = dev(synth.activations(M, K))
    y1 = w4().w4_matmul(x, W["qw"], W["scales"], W["zp"], K, N, path="tc").clone()
    y2 = w4().w4_matmul(x, W["qw"], W["scales"], W["zp"], K, N, path="tc").clone()
    assert torch().equal(y1, y2)


def test_tc_refuses_unaligned_x():
    T = torch()
    K, N, M = 64, 64, 20
    W = upload_w4(synth.w4_weight(K, N))
    xb = dev(synth.activations(M, K + 1))
    with pytest.raises(RuntimeError):
        w4().w4_matmul(xb[:, 1:], W["qw"], W["scales"], W["zp"], K, N, path="tc")
    T.cuda.synchronize()
