"""GPU: the decode matmuls (one row of x) on tile-layout weights with integer
tensor-core MMAs (w4i_matmul_grouped), against the oracle.

* x enters as 8 signed 7-bit digits against its largest magnitude and the
  codes as stored; the MMA sums digit x code exactly in int32 per block, the
  zero point enters exactly through the block sums of the digits, and each
  block is weighed and scaled in fp32. The outputs match the oracle within
  |y - y_ref| <= 1e-5 * sum|x*w| + 1e-6 for ragged column tiles, partial
  groups of blocks (K of 1 to 96 blocks), the GPT-2 decode stack in one
  grouped call and shared inputs; the dyadic closed forms, one-hot rows and
  awkward x values come out exactly; the fused epilogue, non-finite inputs,
  stream order across launches that start early, and the refusals hold."""

import numpy as np
import pytest

import oracle
import pins
from gpu_util import check, dev, torch, upload_w4

from int8_weight_quantized_w4_b200 import synth

pytestmark = pytest.mark.gpu


def w4():
    import int8_weight_quantized_w4_b200 as w
    return w


def _tiled(W):
    Wd = upload_w4(W)
    return w4().w4t_repack(Wd["qw"], Wd["scales"], Wd["zp"], W["K"], W["N"])


def _run(K, N, tag, epi=None, x=None):
    W = synth.w4_weight(K, N, tag)
    x = synth.activations(1, K, tag) if x is None else x
    wt = _tiled(W)
    T = torch()
    y = T.full((1, N), float("nan"), dtype=T.float32, device="cuda")
    kw = {k: (dev(v) if isinstance(v, np.ndarray) else v) for k, v in (epi or {}).items()}
    w4().w4i_matmul(dev(x), wt, K, N, y=y, **kw)
    T.cuda.synchronize()
    return W, x, y


SHAPES = [(32, 8), (64, 136), (96, 40), (160, 264), (224, 128), (768, 768), (768, 2304), (768, 3072), (3072, 768),
          (1536, 200), (3072, 9216)]


@pytest.mark.parametrize("K,N", SHAPES)
def test_gemv_matches_the_oracle(K, N):
    W, x, y = _run(K, N, K + 7 * N)
    y_ref, a = oracle.w4_matmul_ref(x, W["qw"], W["scales"], W["zp"], K, N)
    check(y, y_ref, a, f"w4i K={K} N={N}")


def test_gpt2_decode_stack_grouped_and_deterministic():
    """The 48 GPT-2 weights at M = 1, one grouped call, each with its own x:
    every output against the oracle, then bit-identical on a second run."""
    T = torch()
    host, items = [], []
    for i, (name, K, N) in enumerate(synth.gpt2_stack_shapes()):
        W = synth.w4_weight(K, N, i)
        x = synth.activations(1, K, i)
        items.append({"x": dev(x), "wr": _tiled(W), "y": T.full((1, N), float("nan"), device="cuda"), "K": K, "N": N})
        host.append((name, W, x))
    w4().w4i_matmul_grouped(items)
    T.cuda.synchronize()
    first = [it["y"].clone() for it in items]
    for (name, W, x), it in zip(host, items):
        y_ref, a = oracle.w4_matmul_ref(x, W["qw"], W["scales"], W["zp"], W["K"], W["N"])
        check(it["y"], y_ref, a, name)
    w4().w4i_matmul_grouped(items)
    T.cuda.synchronize()
    for a_, it in zip(first, items):
        assert T.equal(a_, it["y"]), "not run-to-run deterministic"


def test_shared_x_has_its_digits_once():
    T = torch()
    xs = dev(synth.activations(1, 768, 70))
    host, items = [], []
    for i in range(3):
        W = synth.w4_weight(768, 264, 70 + i)
        items.append({"x": xs, "wr": _tiled(W), "y": T.full((1, 264), float("nan"), device="cuda"), "K": 768,
                      "N": 264})
        host.append(W)
    W2 = synth.w4_weight(256, 136, 74)
    x2 = synth.activations(1, 256, 74)
    items.append({"x": dev(x2), "wr": _tiled(W2), "y": T.full((1, 136), float("nan"), device="cuda"), "K": 256,
                  "N": 136})
    descs = w4().make_rdescs(items)
    rnd = lambda v: -(-v // 256) * 256
    assert w4().w4i_workspace_size(descs) == rnd(8 * 768 + 768 // 2 + 16) + rnd(8 * 256 + 256 // 2 + 16)
    w4().w4i_matmul_grouped(descs=descs)
    T.cuda.synchronize()
    xh = xs.cpu().numpy()
    for W, it in zip(host, items[:3]):
        y_ref, a = oracle.w4_matmul_ref(xh, W["qw"], W["scales"], W["zp"], 768, 264)
        check(it["y"], y_ref, a, "shared x")
    y_ref, a = oracle.w4_matmul_ref(x2, W2["qw"], W2["scales"], W2["zp"], 256, 136)
    check(items[3]["y"], y_ref, a, "own x")


def _exact(q, zp, s, x):
    K, N = q.shape
    qw, sc, zpk = pins.make_w4(q, zp, s)
    wt = w4().w4t_repack(dev(qw), dev(sc), dev(zpk), K, N)
    y = w4().w4i_matmul(dev(x), wt, K, N)
    torch().cuda.synchronize()
    return y.cpu().numpy().astype(np.float64)


def test_closed_forms_exact():
    y = _exact(np.full((192, 64), 9), np.full((6, 64), 8), np.full((6, 64), 0.5), np.ones((1, 192), np.float32))
    assert np.array_equal(y, np.full((1, 64), 96.0))
    x = ((np.arange(192, dtype=np.float32) - 10) / 4)[None, :]
    y = _exact(np.zeros((192, 32)), np.full((6, 32), 15), np.full((6, 32), 0.125), x)
    assert np.array_equal(y, np.full((1, 32), -15 * 0.125 * x.astype(np.float64).sum()))
    q = np.concatenate([np.full((96, 64), 10), np.full((96, 64), 2)])
    s = np.array([[0.25] * 64] * 3 + [[2.0] * 64] * 3)
    y = _exact(q, np.full((6, 64), 7), s, np.ones((1, 192), np.float32))
    assert np.array_equal(y, np.full((1, 64), 96 * 0.25 * 3 + 96 * 2.0 * -5))
    g = np.random.default_rng(3)
    y = _exact(np.full((768, 64), 6), np.full((24, 64), 6), np.full((24, 64), 0.0173),
               g.standard_normal((1, 768)).astype(np.float32))
    assert np.all(y == 0)


def test_one_hot_x_gives_the_dequantised_row():
    g = np.random.default_rng(4)
    K, N = 192, 256
    qi = g.integers(0, 16, (K, N))
    zi = g.integers(0, 16, (K // 32, N))
    s = g.uniform(0.005, 0.02, (K // 32, N)).astype(np.float32)
    w = oracle.dequantize_w4(*pins.make_w4(qi, zi, s), K, N)
    for k in (0, 33, 100, K - 1):
        x = np.zeros((1, K), np.float32)
        x[0, k] = 1.0
        y = _exact(qi, zi, s, x)
        assert np.array_equal(y[0], w[k].astype(np.float64)), f"row {k}"


def test_awkward_x_values_come_back_exactly():
    """x values with all 24 significant bits over 2^28 of magnitudes: a
    one-hot weight column reads each back exactly."""
    K, N = 192, 8
    g = np.random.default_rng(9)
    for trial in range(6):
        mant = g.integers(2 ** 23, 2 ** 24, K).astype(np.float64)
        x = (mant * 2.0 ** g.integers(-20, 8, K) * np.where(g.random(K) < 0.5, -1, 1)).astype(np.float32)[None, :]
        k = int(g.integers(0, K))
        q = np.zeros((K, N), int)
        q[k, 3] = 1
        y = _exact(q, np.zeros((K // 32, N), int), np.ones((K // 32, N), np.float32), x)
        assert y[0, 3] == float(x[0, k]), (trial, k)
        assert np.all(np.delete(y[0], 3) == 0)


def test_wide_range_x_within_tolerance():
    K, N = 768, 264
    g = np.random.default_rng(12)
    x = (synth.activations(1, K, 12) * np.exp2(g.integers(-50, 50, K))).astype(np.float32)
    W, x, y = _run(K, N, 12, x=x)
    y_ref, a = oracle.w4_matmul_ref(x, W["qw"], W["scales"], W["zp"], K, N)
    check(y, y_ref, a, "wide x")


@pytest.mark.parametrize("act", ["none", "gelu_tanh", "gelu_erf"])
def test_fused_epilogue(act):
    K, N = 768, 3072
    b = synth.bias(N, 3)
    r = synth.activations(1, N, 77)
    W, x, y = _run(K, N, 5, epi={"bias": b, "residual": r, "act": act})
    y_ref, a = oracle.w4_matmul_ref(x, W["qw"], W["scales"], W["zp"], K, N)
    out, tol = oracle.epilogue_ref(y_ref, a, bias=b, residual=r, act=act)
    assert np.all(np.abs(y.cpu().numpy() - out) <= tol)


def test_zero_and_non_finite_x():
    K, N = 256, 136
    b = synth.bias(N, 8)
    W, x, y = _run(K, N, 8, epi={"bias": b}, x=np.zeros((1, K), np.float32))
    assert np.array_equal(y.cpu().numpy()[0], b)
    xn = synth.activations(1, K, 8).copy()
    xn[0, 77] = np.nan
    _, _, y = _run(K, N, 8, x=xn)
    assert np.all(np.isnan(y.cpu().numpy()))
    xi = synth.activations(1, K, 8).copy()
    xi[0, 5] = np.inf
    _, _, y = _run(K, N, 8, x=xi)
    assert np.all(np.isnan(y.cpu().numpy()))


def test_chained_launches_keep_stream_order():
    """Each launch's output is the next one's input, back to back on one
    stream (both launches of each call start early): each must read its
    finished input."""
    T = torch()
    K = 768
    Ws = [synth.w4_weight(K, K, 80 + i) for i in range(6)]
    wts = [_tiled(W) for W in Ws]
    x0 = dev(synth.activations(1, K, 80))
    ys = [T.full((1, K), float("nan"), dtype=T.float32, device="cuda") for _ in Ws]
    ws = [T.empty(w4().w4i_workspace_size(w4().make_rdescs([{"x": x0, "wr": wts[0], "y": ys[0], "K": K,
                                                                 "N": K}])) + 256, dtype=T.uint8, device="cuda")
          for _ in Ws]
    T.cuda.synchronize()
    cur = x0
    for i, wt in enumerate(wts):
        w4().w4i_matmul(cur, wt, K, K, y=ys[i], ws=ws[i])
        cur = ys[i]
    T.cuda.synchronize()
    xh = x0.cpu().numpy()
    for W, y in zip(Ws, ys):
        y_ref, a = oracle.w4_matmul_ref(xh, W["qw"], W["scales"], W["zp"], K, K)
        check(y, y_ref, a, "chained")
        xh = y.cpu().numpy()


def test_k_zero_writes_the_epilogue_of_zero():
    T = torch()
    N = 64
    b = synth.bias(N, 2)
    wt = T.zeros(16, dtype=T.uint8, device="cuda")
    y = T.full((1, N), float("nan"), device="cuda")
    w4().w4i_matmul(T.zeros((1, 0), device="cuda"), wt, 0, N, y=y, bias=dev(b))
    T.cuda.synchronize()
    assert np.array_equal(y.cpu().numpy()[0], b)


def test_refusals():
    T = torch()
    W = synth.w4_weight(256, 64, 1)
    wt = _tiled(W)
    x2 = T.zeros((2, 256), device="cuda")
    with pytest.raises(w4().W4Error):  # more than one row
        w4().w4i_matmul(x2, wt, 256, 64)
    Wb = synth.w4_weight(3104, 8, 1)
    with pytest.raises(w4().W4Error):  # K beyond 3072
        w4().w4i_matmul(T.zeros((1, 3104), device="cuda"), _tiled(Wb), 3104, 8)
    item = {"x": T.zeros((1, 256), device="cuda"), "wr": wt, "y": T.empty((1, 64), device="cuda"), "K": 256, "N": 64}
    descs = w4().make_rdescs([item])
    need = w4().w4i_workspace_size(descs)
    small = T.empty(need - 16, dtype=T.uint8, device="cuda")
    L = w4().lib()
    with pytest.raises(w4().W4Error):  # workspace too small
        w4()._check(L.w4i_matmul_grouped(descs, 1, w4()._ptr(small), small.numel(), None), "w4i")
    with pytest.raises(w4().W4Error):  # no workspace
        w4()._check(L.w4i_matmul_grouped(descs, 1, None, 0, None), "w4i")
