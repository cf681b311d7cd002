"""GPU: the tile layout (w4t_repack / w4t_repack_restore) and the tensor-core
tile GEMM that reads it (w4t_matmul_grouped), against the oracle.

* The tile layout reorders nibbles, scales and zero points only: restoring
  gives the page-format buffers back bit for bit, and every value sits where
  include/w4.h says, read through the oracle's own unpacking.
* The tile GEMM (tcgen05.mma on exact bf16 (q - zp) and an exact
  three-piece bf16 split of x, the scale applied per block in fp32) matches
  the oracle within |y - y_ref| <= 1e-5 * sum|x*w| + 1e-6 for every rows-per-
  tile class (M up to 16, 32, 64, beyond), ragged row and column tiles,
  strided x and y, the GPT-2 prefill stack and 3.8B layers at M = 2048
  (sampled); it gives the dyadic closed forms and one-hot rows exactly, is
  deterministic, and keeps stream order when launches start early."""

import numpy as np
import pytest

import oracle
import pins
from gpu_util import check, dev, guarded, guards_intact, torch, upload_w4

from int8_weight_quantized_w4_b200 import synth

pytestmark = pytest.mark.gpu

POS = [0, 16, 4, 20, 8, 24, 12, 28]


def w4():
    import int8_weight_quantized_w4_b200 as w
    return w


def _tiled(W):
    Wd = upload_w4(W)
    return Wd, w4().w4t_repack(Wd["qw"], Wd["scales"], Wd["zp"], W["K"], W["N"])


LAYOUT_SHAPES = [(32, 8), (64, 136), (192, 8), (768, 768), (768, 2304), (3072, 768), (8192, 64), (1536, 200),
                 (96, 40)]


@pytest.mark.parametrize("K,N", LAYOUT_SHAPES)
def test_tile_repack_then_restore_is_the_identity(K, N):
    W = synth.w4_weight(K, N, 21)
    _, wt = _tiled(W)
    assert wt.numel() == w4().w4t_repacked_bytes(K, N)
    qw, sc, zp = w4().w4t_repack_restore(wt, K, N)
    torch().cuda.synchronize()
    assert np.array_equal(qw.cpu().numpy(), W["qw"])
    assert np.array_equal(sc.cpu().numpy().reshape(-1).view(np.uint32), W["scales"].view(np.uint32))
    assert np.array_equal(zp.cpu().numpy(), W["zp"])


@pytest.mark.parametrize("K,N", [(768, 768), (3072, 200), (96, 40)])
def test_tile_words_sit_where_the_header_says(K, N):
    W = synth.w4_weight(K, N, 22)
    _, wt = _tiled(W)
    buf = wt.cpu().numpy()
    q = oracle.unpack_nibbles(W["qw"], K * N).reshape(K, N)
    z = oracle.unpack_nibbles(W["zp"], (K // 32) * N).reshape(K // 32, N)
    s = W["scales"].reshape(K // 32, N)
    nb = K // 32
    g = np.random.default_rng(1)
    for k, n in zip(np.concatenate([[0, K - 1], g.integers(0, K, 300)]), np.concatenate([[0, N - 1], g.integers(0, N, 300)])):
        T, c = n // 128, n % 128
        b, rr = k // 32, k % 32
        base = (T * nb + b) * 2624
        word = int.from_bytes(buf[base + c * 16 + (rr // 8) * 4:][:4].tobytes(), "little")
        assert (word >> POS[rr % 8]) & 15 == q[k, n]
        sb = buf[base + 2048 + 4 * c:][:4].tobytes()
        assert np.frombuffer(sb, np.uint32)[0] == s[b, n:n + 1].view(np.uint32)[0]
        zword = int.from_bytes(buf[base + 2560 + (c // 8) * 4:][:4].tobytes(), "little")
        assert (zword >> (4 * (c % 8))) & 15 == z[b, n]


def _run_t(M, K, N, tag, epi=None):
    W = synth.w4_weight(K, N, tag)
    x = synth.activations(M, K, tag)
    _, wt = _tiled(W)
    T = torch()
    y = T.full((M, N), float("nan"), dtype=T.float32, device="cuda")
    kw = {k: (dev(v) if isinstance(v, np.ndarray) else v) for k, v in (epi or {}).items()}
    w4().w4t_matmul(dev(x), wt, K, N, y=y, **kw)
    T.cuda.synchronize()
    return W, x, y


# M per rows-per-tile class (16, 32, 64, 128) with ragged row tiles; N with
# ragged column tiles; K from one block up
SHAPES = [(1, 32, 8), (7, 64, 136), (16, 768, 768), (17, 768, 2304), (32, 96, 128), (58, 768, 3072),
          (58, 3072, 768), (64, 256, 200), (65, 512, 384), (130, 768, 256), (300, 1024, 520), (128, 8192, 64)]


@pytest.mark.parametrize("M,K,N", SHAPES)
def test_tile_gemm_matches_the_oracle(M, K, N):
    W, x, y = _run_t(M, K, N, M + K + 3 * N)
    y_ref, a = oracle.w4_matmul_ref(x, W["qw"], W["scales"], W["zp"], K, N)
    check(y, y_ref, a, f"w4t M={M} K={K} N={N}")


def test_strided_x_and_y_leave_the_padding_alone():
    T = torch()
    M, K, N, ldx, ldy = 45, 512, 264, 520, 300
    W = synth.w4_weight(K, N, 41)
    xs = synth.activations(M, K, 41, ld=ldx)
    _, wt = _tiled(W)
    xd = dev(xs)[:, :K]
    y, buf = guarded(M, N, ldy)
    w4().w4t_matmul(xd, wt, K, N, y=y)
    T.cuda.synchronize()
    y_ref, a = oracle.w4_matmul_ref(np.ascontiguousarray(xs[:, :K]), W["qw"], W["scales"], W["zp"], K, N)
    check(y, y_ref, a, "strided")
    assert guards_intact(buf, M, N, ldy)


def test_gpt2_prefill_stack_grouped():
    """The 48 GPT-2 weights at M = 58 (a prompt), one grouped call, each with
    its own input: every output against the oracle, then bit-identical on a
    second run."""
    T = torch()
    host, items = [], []
    for i, (name, K, N) in enumerate(synth.gpt2_stack_shapes()):
        W = synth.w4_weight(K, N, i)
        x = synth.activations(58, K, i)
        _, wt = _tiled(W)
        items.append({"x": dev(x), "wr": wt, "y": T.full((58, N), float("nan"), device="cuda"), "K": K, "N": N})
        host.append((name, W, x))
    w4().w4t_matmul_grouped(items)
    T.cuda.synchronize()
    first = [it["y"].clone() for it in items]
    for (name, W, x), it in zip(host, items):
        y_ref, a = oracle.w4_matmul_ref(x, W["qw"], W["scales"], W["zp"], W["K"], W["N"])
        check(it["y"], y_ref, a, name)
    w4().w4t_matmul_grouped(items)
    T.cuda.synchronize()
    for a_, it in zip(first, items):
        assert T.equal(a_, it["y"]), "not run-to-run deterministic"


def test_dense38_layer_prefill_m2048_sampled():
    """One 3.8B layer (qkv, o_proj, gate_up, down) at M = 2048 in one grouped
    call; 4096 sampled outputs per weight against the oracle."""
    T = torch()
    M = 2048
    host, items = [], []
    for i, (name, K, N) in enumerate(synth.dense38_stack_shapes()[:4]):
        W = synth.w4_weight(K, N, 500 + i)
        x = synth.activations(M, K, 500 + i)
        _, wt = _tiled(W)
        items.append({"x": dev(x), "wr": wt, "y": T.full((M, N), float("nan"), device="cuda"), "K": K, "N": N})
        host.append((name, W, x))
    w4().w4t_matmul_grouped(items)
    T.cuda.synchronize()
    g = np.random.default_rng(2048)
    for (name, W, x), it in zip(host, items):
        rows = g.integers(0, M, 4096)
        cols = g.integers(0, W["N"], 4096)
        rows[:4] = [0, M - 1, 0, M - 1]
        cols[:4] = [0, W["N"] - 1, W["N"] - 1, 0]
        ys, a = oracle.w4_matmul_ref_entries(x, W["qw"], W["scales"], W["zp"], W["K"], W["N"], rows, cols)
        yg = it["y"].cpu().numpy()
        check(yg[rows, cols], ys, a, f"{name} M=2048")
        assert np.all(np.isfinite(yg)), f"{name}: output not fully written"


def test_mixed_row_classes_in_one_call_and_shared_x():
    """Matrices whose M fall in four rows-per-tile classes go to four GEMM
    launches after one split launch; three weights reading the same x share
    its pieces (the workspace holds them once)."""
    T = torch()
    host, items = [], []
    for i, M in enumerate([5, 20, 50, 100]):
        K, N = 256, 136
        W = synth.w4_weight(K, N, 60 + i)
        x = synth.activations(M, K, 60 + i)
        _, wt = _tiled(W)
        items.append({"x": dev(x), "wr": wt, "y": T.full((M, N), float("nan"), device="cuda"), "K": K, "N": N})
        host.append((W, x))
    xs = dev(synth.activations(40, 768, 70))
    for i in range(3):
        W = synth.w4_weight(768, 264, 70 + i)
        _, wt = _tiled(W)
        items.append({"x": xs, "wr": wt, "y": T.full((40, 264), float("nan"), device="cuda"), "K": 768, "N": 264})
        host.append((W, xs.cpu().numpy()))
    descs = w4().make_rdescs(items)
    want = sum((-(-M // c) * c) * K * 6 for M, K, c in [(5, 256, 16), (20, 256, 32), (50, 256, 64), (100, 256, 128)])
    want += 64 * 768 * 6  # the shared x once
    assert w4().w4t_workspace_size(descs) == want
    w4().w4t_matmul_grouped(descs=descs)
    T.cuda.synchronize()
    for (W, x), it in zip(host, items):
        y_ref, a = oracle.w4_matmul_ref(x, W["qw"], W["scales"], W["zp"], W["K"], W["N"])
        check(it["y"], y_ref, a, f"M={x.shape[0]} N={W['N']}")


def _exact_t(q, zp, s, x):
    K, N = q.shape
    qw, sc, zpk = pins.make_w4(q, zp, s)
    wt = w4().w4t_repack(dev(qw), dev(sc), dev(zpk), K, N)
    y = w4().w4t_matmul(dev(x), wt, K, N)
    torch().cuda.synchronize()
    return y.cpu().numpy().astype(np.float64)


def test_closed_forms_exact():
    M = 37
    y = _exact_t(np.full((192, 64), 9), np.full((6, 64), 8), np.full((6, 64), 0.5), np.ones((M, 192), np.float32))
    assert np.array_equal(y, np.full((M, 64), 96.0))
    x = np.stack([(np.arange(192, dtype=np.float32) - 10 - m) / 4 for m in range(M)])
    y = _exact_t(np.zeros((192, 32)), np.full((6, 32), 15), np.full((6, 32), 0.125), x)
    want = -15 * 0.125 * x.astype(np.float64).sum(axis=1)
    assert np.array_equal(y, np.repeat(want[:, None], 32, axis=1))
    q = np.concatenate([np.full((96, 64), 10), np.full((96, 64), 2)])
    s = np.array([[0.25] * 64] * 3 + [[2.0] * 64] * 3)
    y = _exact_t(q, np.full((6, 64), 7), s, np.ones((M, 192), np.float32))
    assert np.array_equal(y, np.full((M, 64), 96 * 0.25 * 3 + 96 * 2.0 * -5))
    g = np.random.default_rng(3)
    y = _exact_t(np.full((768, 64), 6), np.full((24, 64), 6), np.full((24, 64), 0.0173),
                 g.standard_normal((M, 768)).astype(np.float32))
    assert np.all(y == 0)


def test_one_hot_rows_give_the_dequantised_rows():
    g = np.random.default_rng(4)
    K, N, M = 192, 256, 70
    qi = g.integers(0, 16, (K, N))
    zi = g.integers(0, 16, (K // 32, N))
    s = g.uniform(0.005, 0.02, (K // 32, N)).astype(np.float32)
    w = oracle.dequantize_w4(*pins.make_w4(qi, zi, s), K, N)
    ks = g.integers(0, K, M)
    ks[:3] = [0, 33, K - 1]
    x = np.zeros((M, K), np.float32)
    x[np.arange(M), ks] = 1.0
    y = _exact_t(qi, zi, s, x)
    assert np.array_equal(y, w[ks].astype(np.float64))


def test_x_split_is_exact_for_awkward_values():
    """x values with all 24 significant bits, over many binades: the three
    bf16 pieces carry them exactly (a one-hot weight column reads x back)."""
    K, N, M = 192, 8, 24
    g = np.random.default_rng(9)
    mant = g.integers(2 ** 23, 2 ** 24, M).astype(np.float64)
    vals = (mant * 2.0 ** g.integers(-60, 40, M) * np.where(g.random(M) < 0.5, -1, 1)).astype(np.float32)
    q = np.zeros((K, N), int)
    q[37, 3] = 1
    x = np.zeros((M, K), np.float32)
    x[:, 37] = vals
    y = _exact_t(q, np.zeros((K // 32, N), int), np.ones((K // 32, N), np.float32), x)
    assert np.array_equal(y[:, 3], vals.astype(np.float64))
    assert np.all(np.delete(y, 3, axis=1) == 0)


@pytest.mark.parametrize("act", ["none", "gelu_tanh", "gelu_erf"])
def test_fused_epilogue(act):
    M, K, N = 58, 768, 3072
    b = synth.bias(N, 3)
    r = synth.activations(M, N, 77)
    W, x, y = _run_t(M, K, N, 5, epi={"bias": b, "residual": r, "act": act})
    y_ref, a = oracle.w4_matmul_ref(x, W["qw"], W["scales"], W["zp"], K, N)
    out, tol = oracle.epilogue_ref(y_ref, a, bias=b, residual=r, act=act)
    assert np.all(np.abs(y.cpu().numpy() - out) <= tol)


def test_chained_launches_keep_stream_order():
    """Each launch's output is the next one's input, back to back on one
    stream (every launch starts early): each must read finished input."""
    T = torch()
    M, K = 58, 768
    Ws = [synth.w4_weight(K, K, 80 + i) for i in range(6)]
    wts = [_tiled(W)[1] for W in Ws]
    x0 = dev(synth.activations(M, K, 80))
    ys = [T.full((M, K), float("nan"), dtype=T.float32, device="cuda") for _ in Ws]
    T.cuda.synchronize()
    cur = x0
    for i, wt in enumerate(wts):
        w4().w4t_matmul(cur, wt, K, K, y=ys[i])
        cur = ys[i]
    T.cuda.synchronize()
    prev = x0.cpu().numpy()
    for i, W in enumerate(Ws):
        y_ref, a = oracle.w4_matmul_ref(prev, W["qw"], W["scales"], W["zp"], K, K)
        check(ys[i], y_ref, a, f"chain step {i}")
        prev = ys[i].cpu().numpy()


def test_empty_and_zero_k():
    T = torch()
    W = synth.w4_weight(64, 64, 1)
    _, wt = _tiled(W)
    y0 = T.empty((0, 64), device="cuda")
    w4().w4t_matmul(T.empty((0, 64), device="cuda"), wt, 64, 64, y=y0)  # M = 0: nothing to do
    b = synth.bias(64, 9)
    y = T.full((5, 64), float("nan"), device="cuda")
    w4().w4t_matmul_grouped([{"x": T.empty((5, 0), device="cuda"), "wr": wt, "y": y, "K": 0, "N": 64,
                              "bias": dev(b)}])
    T.cuda.synchronize()
    assert np.array_equal(y.cpu().numpy(), np.repeat(b[None, :], 5, axis=0))


def test_refusals():
    T = torch()
    lib = w4().lib()
    W = synth.w4_weight(192, 64, 1)
    Wd, wt = _tiled(W)
    x = dev(synth.activations(20, 192, 1))
    y = T.empty((20, 64), device="cuda")
    descs = w4().make_rdescs([{"x": x, "wr": wt, "y": y, "K": 192, "N": 64}])
    need = w4().w4t_workspace_size(descs)
    assert need == 32 * 192 * 6
    ws = T.empty(need, dtype=T.uint8, device="cuda")
    st = T.cuda.current_stream().cuda_stream
    assert lib.w4t_matmul_grouped(descs, 1, ws.data_ptr(), need - 16, st) == 7  # workspace too small
    assert lib.w4t_matmul_grouped(descs, 1, None, 0, st) == 7  # no workspace
    assert lib.w4t_matmul_grouped(descs, 1, ws.data_ptr() + 4, need, st) == 7  # misaligned workspace
    descs[0].ldx = 100
    assert lib.w4t_matmul_grouped(descs, 1, ws.data_ptr(), need, st) == 2  # ldx < K
    descs[0].ldx = 192
    descs[0].K = 200
    assert lib.w4t_matmul_grouped(descs, 1, ws.data_ptr(), need, st) == 2  # K % 32
    with pytest.raises(ValueError):  # N % 8
        Wd = upload_w4(synth.w4_weight(64, 66, 2))
        w4().w4t_repack(Wd["qw"], Wd["scales"], Wd["zp"], 64, 66)
