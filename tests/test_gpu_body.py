"""GPU parity of w4_matmul (all of its kernels) against the oracle."""

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


def run_case(M, K, N, path, seed=1, ldx=None, ldy=None):
    W = synth.w4_weight(K, N, M, seed=seed)
    x = synth.activations(M, K, 7, seed=seed, ld=ldx)
    xd = dev(x)[:, :K] if ldx else dev(x)
    y, buf = guarded(M, N, ldy)
    Wd = upload_w4(W)
    w4().w4_matmul(xd, Wd["qw"], Wd["scales"], Wd["zp"], K, N, y=y, path=path)
    torch().cuda.synchronize()
    y_ref, a = oracle.w4_matmul_ref(x[:, :K], W["qw"], W["scales"], W["zp"], K, N)
    check(y, y_ref, a, f"M={M} K={K} N={N} path={path}")
    assert guards_intact(buf, M, N, ldy or N), "write outside y"
    return y


def test_config0_single_768x768_all_paths():
    for path in ("auto", "gemv", "generic"):
        run_case(1, 768, 768, path)


SHAPES = [(1, 32, 32), (1, 64, 288), (2, 96, 544), (3, 128, 96), (4, 256, 1024), (5, 160, 800), (8, 512, 256),
          (9, 64, 320), (16, 1024, 768), (1, 3072, 768), (2, 8192, 96), (6, 96, 2304), (1, 768, 3072),
          (12, 288, 160), (7, 2048, 64)]


@pytest.mark.parametrize("M,K,N", SHAPES)
@pytest.mark.parametrize("path", ["gemv", "generic"])
def test_shapes(M, K, N, path):
    run_case(M, K, N, path, seed=M * 1000 + N)


@pytest.mark.parametrize("M,K,N", [(1, 64, 34), (3, 96, 2), (7, 32, 30), (2, 64, 66), (17, 64, 50)])
def test_generic_only_shapes(M, K, N):
    run_case(M, K, N, "auto")
    with pytest.raises(w4().W4Error):
        run_case(M, K, N, "gemv")


@pytest.mark.parametrize("M,K,N,ldx,ldy,path", [
    (3, 96, 288, 100, 300, "gemv"),   # ldx % 4 == 0: TMA path
    (3, 96, 288, 97, 289, "auto"),    # ldx odd: generic path
    (2, 64, 64, 64, 65, "auto"),
])
def test_padded_strides(M, K, N, ldx, ldy, path):
    run_case(M, K, N, path, ldx=ldx, ldy=ldy)


def test_large_M_through_gemv_chunks():
    # the GEMV forced on M > 16: groups of 8 rows re-stream the weight
    run_case(37, 256, 512, "gemv")


def test_degenerate_sizes():
    T = torch()
    W = upload_w4(synth.w4_weight(64, 64))
    x = dev(synth.activations(2, 64))
    # M = 0: nothing written
    y, buf = guarded(0, 64)
    w4().w4_matmul(x[:0], W["qw"], W["scales"], W["zp"], 64, 64, y=y)
    # K = 0: y is the empty sum, zero
    y, buf = guarded(2, 64)
    e = T.empty(0, dtype=T.uint8, device="cuda")
    ef = T.empty(0, dtype=T.float32, device="cuda")
    w4().w4_matmul(T.empty((2, 0), device="cuda"), e, ef, e, 0, 64, y=y)
    T.cuda.synchronize()
    assert T.all(y == 0) and guards_intact(buf, 2, 64, 64)


def _exact_case(q, zp, s, x, path):
    K, N = q.shape
    qw, sc, zpk = pins.make_w4(q, zp, s)
    y = w4().w4_matmul(dev(x), dev(qw), dev(sc), dev(zpk), K, N, path=path)
    torch().cuda.synchronize()
    return y.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("path", ["gemv", "generic"])
def test_closed_forms_exact(path):
    # x = 1, q - zp = 1, s = 0.5, K = 32 -> 16 exactly
    y = _exact_case(np.full((32, 64), 9), np.full((1, 64), 8), np.full((1, 64), 0.5), np.ones((1, 32), np.float32), path)
    assert np.array_equal(y, np.full((1, 64), 16.0))
    # two blocks, scales 0.25 and 2, q - zp = 3 and -5
    q = np.concatenate([np.full((32, 64), 10), np.full((32, 64), 2)])
    y = _exact_case(q, np.full((2, 64), 7), np.array([[0.25] * 64, [2.0] * 64]), np.ones((2, 64), np.float32), path)
    assert np.array_equal(y, np.full((2, 64), 32 * 0.25 * 3 + 32 * 2.0 * -5))
    # q = 0, zp = 15 -> -15 * s * sum(x), dyadic x
    x = ((np.arange(64, dtype=np.float32) - 10) / 4)[None, :]
    y = _exact_case(np.zeros((64, 32)), np.full((2, 32), 15), np.full((2, 32), 0.125), x, path)
    assert np.array_equal(y, np.full((1, 32), -15 * 0.125 * float(x.sum())))
    # every q == zp -> exactly 0
    g = np.random.default_rng(3)
    y = _exact_case(np.full((96, 64), 6), np.full((3, 64), 6), np.full((3, 64), 0.0173),
                    g.standard_normal((3, 96)).astype(np.float32), path)
    assert np.all(y == 0)


def test_one_hot_rows_exact():
    """x = e_k returns row k of W: the fp32 dequantised weight, bit for bit."""
    g = np.random.default_rng(4)
    K, N = 96, 256
    qi = g.integers(0, 16, (K, N))
    zi = g.integers(0, 16, (K // 32, N))
    s = g.uniform(0.005, 0.02, (K // 32, N)).astype(np.float32)
    qw, sc, zpk = pins.make_w4(qi, zi, s)
    Wf = oracle.dequantize_w4(qw, sc, zpk, K, N)
    ks = [0, 31, 32, 95, 50]
    x = np.zeros((len(ks), K), np.float32)
    for r, k in enumerate(ks):
        x[r, k] = 1.0
    for path in ("gemv", "generic"):
        y = w4().w4_matmul(dev(x), dev(qw), dev(sc), dev(zpk), K, N, path=path)
        yh = y.cpu().numpy()
        for r, k in enumerate(ks):
            assert np.array_equal(yh[r], Wf[k]), (path, k)


def test_deterministic():
    K, N, M = 3072, 768, 1
    W = upload_w4(synth.w4_weight(K, N))
    x = dev(synth.activations(M, K))
    y1 = w4().w4_matmul(x, W["qw"], W["scales"], W["zp"], K, N).clone()
    y2 = w4().w4_matmul(x, W["qw"], W["scales"], W["zp"], K, N).clone()
    assert torch().equal(y1, y2)


def test_workspace_reused_across_shapes():
    """One workspace through calls whose grids and split tiles differ: the
    counters must be back at zero after every call."""
    T = torch()
    ws = T.zeros(1 << 22, dtype=T.uint8, device="cuda")
    for (M, K, N) in [(1, 768, 768), (1, 64, 288), (3, 3072, 768), (1, 8224, 64), (8, 96, 544), (1, 8192, 64)]:
        W = synth.w4_weight(K, N, 77)
        x = synth.activations(M, K, 77)
        Wd = upload_w4(W)
        y = w4().w4_matmul(dev(x), Wd["qw"], Wd["scales"], Wd["zp"], K, N, path="gemv", ws=ws)
        T.cuda.synchronize()
        y_ref, a = oracle.w4_matmul_ref(x, W["qw"], W["scales"], W["zp"], K, N)
        check(y, y_ref, a, f"reuse M={M} K={K} N={N}")
    assert int(ws[:4096].count_nonzero()) == 0


def test_workspace_too_small_is_refused():
    T = torch()
    K, N = 768, 768
    W = upload_w4(synth.w4_weight(K, N))
    x = dev(synth.activations(2, K))
    need = w4().w4_matmul_workspace_size(2, K, N)
    assert need > 0
    small = T.zeros(need // 2, dtype=T.uint8, device="cuda")
    with pytest.raises(w4().W4Error) as e:
        w4().w4_matmul(x, W["qw"], W["scales"], W["zp"], K, N, path="gemv", ws=small)
    assert e.value.status == 7


def test_bounded_wait_times_out_and_gpu_stays_usable():
    w = w4()
    w.device_error(clear=True)
    w.debug_wait_timeout(2_000_000)  # 2 ms limit on a barrier nothing completes
    torch().cuda.synchronize()
    st, info = w.device_error(clear=True)
    assert st == 6 and info[0] == 6 and info[1] == 9 and info[3] == 77
    assert w.device_error(clear=False)[0] == 0
    run_case(2, 256, 512, "gemv")  # the context is still healthy
    assert w.device_error(clear=False)[0] == 0


def test_m1_long_k():
    # 257 K-blocks: tall narrow tiles split over several CTAs
    run_case(1, 8224, 64, "gemv")
    run_case(1, 8224, 64, "auto")
