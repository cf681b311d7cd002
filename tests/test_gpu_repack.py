"""GPU: the streaming layout (w4_repack / w4_repack_restore) and the decode
GEMV that reads it (w4r_matmul, w4r_matmul_grouped), against the oracle.

* Repacking is a permutation of words: restoring gives the page-format
  buffers back bit for bit, and every nibble, scale and zero point sits where
  include/w4.h says, read through the oracle's own unpacking.
* The GEMV on repacked weights matches the oracle on the page-format weights
  within |y - y_ref| <= 1e-5 * sum|x*w| + 1e-6, equals the dyadic closed forms
  exactly, is deterministic, and keeps stream order when one launch's output
  is the next one's input (its launches start early, before the previous
  launch has finished)."""

import math

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


def _geom(K, N):
    nb = K // 32
    gs = 32 // math.gcd(nb, 32)
    return nb, gs, nb // math.gcd(nb, 32), -(-N // (8 * gs))


def _repacked(W):
    Wd = upload_w4(W)
    return Wd, w4().w4_repack(Wd["qw"], Wd["scales"], Wd["zp"], W["K"], W["N"])


SHAPES = [(32, 8), (64, 16), (96, 24), (768, 768), (768, 2304), (3072, 768), (1536, 200), (8192, 64), (256, 8),
          (32, 264), (4096, 48)]


@pytest.mark.parametrize("K,N", SHAPES)
def test_repack_then_restore_is_the_identity(K, N):
    W = synth.w4_weight(K, N, 11)
    _, wr = _repacked(W)
    assert wr.numel() == w4().w4_repacked_bytes(K, N)
    qw, sc, zp = w4().w4_repack_restore(wr, K, N)
    torch().cuda.synchronize()
    assert np.array_equal(qw.cpu().numpy(), W["qw"])
    assert np.array_equal(sc.cpu().numpy().reshape(-1).view(np.uint32), W["scales"].view(np.uint32))
    assert np.array_equal(zp.cpu().numpy(), W["zp"])


@pytest.mark.parametrize("K,N", [(768, 768), (3072, 768), (96, 40), (8192, 16)])
def test_repacked_words_sit_where_the_header_says(K, N):
    """Nibble, scale and zero point of sampled (k, n) read from the documented
    byte positions equal the oracle's unpacking of the page format."""
    W = synth.w4_weight(K, N, 12)
    _, wr = _repacked(W)
    buf = wr.cpu().numpy()
    q = oracle.unpack_nibbles(W["qw"], K * N).reshape(K, N)
    z = oracle.unpack_nibbles(W["zp"], (K // 32) * N).reshape(K // 32, N)
    s = W["scales"].reshape(K // 32, N)
    nb, gs, A, _ = _geom(K, N)
    g = np.random.default_rng(0)
    ks = np.concatenate([[0, K - 1], g.integers(0, K, 300)])
    ns = np.concatenate([[0, N - 1], g.integers(0, N, 300)])
    for k, n in zip(ks, ns):
        b, row = k // 32, k % 32
        strip_all = n // 8
        G, sidx = strip_all // gs, strip_all % gs
        phase, r = b % (32 // gs), b // (32 // gs)
        lane = phase * gs + sidx
        base = (G * A + r) * 5248
        c, j, i = row // 4, row % 4, n % 8
        word = int.from_bytes(buf[base + c * 512 + lane * 16 + j * 4:][:4].tobytes(), "little")
        assert (word >> (4 * i)) & 15 == q[k, n]
        sbytes = buf[base + 4096 + (i // 4) * 512 + lane * 16 + (i % 4) * 4:][:4].tobytes()
        assert np.frombuffer(sbytes, np.float32)[0].view(np.uint32) == s[b, n].view(np.uint32)
        zword = int.from_bytes(buf[base + 5120 + lane * 4:][:4].tobytes(), "little")
        assert (zword >> (4 * i)) & 15 == z[b, n]


def _run_r(K, N, tag, epi=None):
    W = synth.w4_weight(K, N, tag)
    x = synth.activations(1, K, tag)
    _, wr = _repacked(W)
    T = torch()
    y = T.full((1, N), float("nan"), dtype=T.float32, device="cuda")
    kw = {}
    if epi:
        kw = {k: (dev(v) if isinstance(v, np.ndarray) else v) for k, v in epi.items()}
    w4().w4r_matmul(dev(x), wr, K, N, y=y, **kw)
    T.cuda.synchronize()
    return W, x, y


@pytest.mark.parametrize("K,N", SHAPES)
def test_decode_gemv_matches_the_oracle(K, N):
    W, x, y = _run_r(K, N, K + N)
    y_ref, a = oracle.w4_matmul_ref(x, W["qw"], W["scales"], W["zp"], K, N)
    check(y, y_ref, a, f"w4r K={K} N={N}")


def test_gpt2_decode_stack_grouped_on_repacked_weights():
    T = torch()
    host, items = [], []
    for i, (name, K, N) in enumerate(synth.gpt2_stack_shapes()):
        W = synth.w4_weight(K, N, i)
        x = synth.activations(1, K, i)
        _, wr = _repacked(W)
        items.append({"x": dev(x), "wr": wr, "y": T.full((1, N), float("nan"), device="cuda"), "K": K, "N": N})
        host.append((name, W, x))
    w4().w4r_matmul_grouped(items)
    T.cuda.synchronize()
    first = [it["y"].clone() for it in items]
    for (name, W, x), it in zip(host, items):
        y_ref, a = oracle.w4_matmul_ref(x, W["qw"], W["scales"], W["zp"], W["K"], W["N"])
        check(it["y"], y_ref, a, name)
    w4().w4r_matmul_grouped(items)
    T.cuda.synchronize()
    for a_, it in zip(first, items):
        assert T.equal(a_, it["y"]), "not run-to-run deterministic"


def test_dense38_stack_in_one_launch_sampled():
    """The 128 weights of the 3.8B-shaped stack (K up to 8192) as one grouped
    call: one launch (every CTA's x fits its shared memory). The four layer
    weights are generated once and shared by the 32 layers' descriptors, each
    with its own x and y; 16 columns of every output are checked against the
    oracle on the same columns of the page-format buffers."""
    T = torch()
    shapes = synth.DENSE38_LAYER_SHAPES
    Ws = [synth.w4_weight(K, N, 300 + i) for i, (_, K, N) in enumerate(shapes)]
    wrs = [_repacked(W)[1] for W in Ws]
    items, host = [], []
    for layer in range(synth.DENSE38_LAYERS):
        for i, (_, K, N) in enumerate(shapes):
            x = synth.activations(1, K, 400 + 4 * layer + i)
            items.append({"x": dev(x), "wr": wrs[i], "y": T.full((1, N), float("nan"), device="cuda"), "K": K, "N": N})
            host.append((i, x))
    assert len(items) == 128
    w4().w4r_matmul_grouped(items)
    T.cuda.synchronize()
    g = np.random.default_rng(5)
    for (i, x), it in zip(host, items):
        W = Ws[i]
        K, N = W["K"], W["N"]
        y = it["y"].cpu().numpy()
        assert np.all(np.isfinite(y))
        for c0 in sorted(set([0, N - 8] + [int(v) * 8 for v in g.integers(0, N // 8, 2)])):
            qw = np.ascontiguousarray(W["qw"].reshape(K, N // 2)[:, c0 // 2:c0 // 2 + 4])
            sc = np.ascontiguousarray(W["scales"].reshape(K // 32, N)[:, c0:c0 + 8])
            zp = np.ascontiguousarray(W["zp"].reshape(K // 32, N // 2)[:, c0 // 2:c0 // 2 + 4])
            y_ref, a = oracle.w4_matmul_ref(x, qw, sc, zp, K, 8)
            check(y[:, c0:c0 + 8], y_ref, a, f"3.8B weight {i} K={K} N={N} columns {c0}..{c0 + 7}")


def _exact_r(q, zp, s, x):
    K, N = q.shape
    qw, sc, zpk = pins.make_w4(q, zp, s)
    wr = w4().w4_repack(dev(qw), dev(sc), dev(zpk), K, N)
    y = w4().w4r_matmul(dev(x), wr, K, N)
    torch().cuda.synchronize()
    return y.cpu().numpy().astype(np.float64)


def test_closed_forms_exact():
    y = _exact_r(np.full((32, 64), 9), np.full((1, 64), 8), np.full((1, 64), 0.5), np.ones((1, 32), np.float32))
    assert np.array_equal(y, np.full((1, 64), 16.0))
    q = np.concatenate([np.full((32, 64), 10), np.full((32, 64), 2)])
    y = _exact_r(q, np.full((2, 64), 7), np.array([[0.25] * 64, [2.0] * 64]), np.ones((1, 64), np.float32))
    assert np.array_equal(y, np.full((1, 64), 32 * 0.25 * 3 + 32 * 2.0 * -5))
    x = ((np.arange(64, dtype=np.float32) - 10) / 4)[None, :]
    y = _exact_r(np.zeros((64, 32)), np.full((2, 32), 15), np.full((2, 32), 0.125), x)
    assert np.array_equal(y, np.full((1, 32), -15 * 0.125 * float(x.sum())))
    g = np.random.default_rng(3)
    y = _exact_r(np.full((768, 64), 6), np.full((24, 64), 6), np.full((24, 64), 0.0173),
                 g.standard_normal((1, 768)).astype(np.float32))
    assert np.all(y == 0)


def test_one_hot_rows_give_the_dequantised_row():
    """x = e_k returns row k of W: the fp32 dequantised weight, bit for bit
    (the scale applied once to the exact (q - zp) is the same single
    rounding)."""
    g = np.random.default_rng(4)
    K, N = 96, 256
    qi = g.integers(0, 16, (K, N))
    zi = g.integers(0, 16, (K // 32, N))
    s = g.uniform(0.005, 0.02, (K // 32, N)).astype(np.float32)
    w = oracle.dequantize_w4(*pins.make_w4(qi, zi, s), K, N)
    for k in (0, 33, 95):
        x = np.zeros((1, K), np.float32)
        x[0, k] = 1.0
        y = _exact_r(qi, zi, s, x)
        assert np.array_equal(y[0], w[k].astype(np.float64))


@pytest.mark.parametrize("act", ["none", "gelu_tanh", "gelu_erf"])
def test_fused_epilogue(act):
    K, N = 768, 3072
    b = synth.bias(N, 3)
    r = synth.activations(1, N, 77)
    W, x, y = _run_r(K, N, 5, epi={"bias": b, "residual": r, "act": act})
    y_ref, a = oracle.w4_matmul_ref(x, W["qw"], W["scales"], W["zp"], K, N)
    out, tol = oracle.epilogue_ref(y_ref, a, bias=b, residual=r, act=act)
    assert np.all(np.abs(y.cpu().numpy() - out) <= tol)


def test_chained_launches_keep_stream_order():
    """Each launch reads the previous launch's output as its x: a launch that
    started early must still see the finished input (and the page-format
    GEMV between them must too)."""
    T = torch()
    K = N = 768
    Ws = [synth.w4_weight(K, N, 40 + i) for i in range(8)]
    wrs = [_repacked(W)[1] for W in Ws]
    Wd = upload_w4(Ws[3])
    x0 = dev(synth.activations(1, K, 40))
    ys = [T.full((1, N), float("nan"), dtype=T.float32, device="cuda") for _ in Ws]
    T.cuda.synchronize()
    cur = x0
    for i, wr in enumerate(wrs):
        if i == 3:  # a page-format launch in the middle of the chain
            w4().w4_matmul(cur, Wd["qw"], Wd["scales"], Wd["zp"], K, N, y=ys[i])
        else:
            w4().w4r_matmul(cur, wr, K, N, y=ys[i])
        cur = ys[i]
    T.cuda.synchronize()
    prev = x0.cpu().numpy()
    for i, W in enumerate(Ws):
        y_ref, a = oracle.w4_matmul_ref(prev, W["qw"], W["scales"], W["zp"], K, N)
        check(ys[i], y_ref, a, f"chain step {i}")
        prev = ys[i].cpu().numpy()
    assert np.all(np.isfinite(prev))


def test_refusals():
    T = torch()
    W = synth.w4_weight(64, 64, 1)
    _, wr = _repacked(W)
    x = dev(synth.activations(2, 64, 1))
    with pytest.raises(w4().W4Error):  # M = 2
        w4().w4r_matmul_grouped([{"x": x, "wr": wr, "y": T.empty((2, 64), device="cuda"), "K": 64, "N": 64}])
    with pytest.raises(w4().W4Error):  # x not 16-byte aligned
        xb = T.zeros(68, device="cuda")[1:65]
        w4().w4r_matmul(xb, wr, 64, 64)
    with pytest.raises(ValueError):
        w4().w4_repack(dev(W["qw"]), dev(W["scales"]), dev(W["zp"]), 64, 60)
