"""GPU: the int8 head in the tensor cores' tile layout (i8t_head_repack /
i8t_head_repack_restore) and the tensor-core head that reads it
(i8t_head_logits, i8t_head_argmax, 1 to 8 rows), against the oracle.

* Repacking reorders and biases bytes only: restoring gives the page's table
  and scales back exactly, and every code and scale sits where include/w4.h
  says.
* The logits match the oracle within |l - l_ref| <= 1e-5 * sum|h*w| + 1e-6
  for every row count 1..8, ragged vocabularies, partial stages and strided
  rows. h enters as 8 signed 7-bit digits per row against the row's largest
  element and the sums are integers, so a one-hot table returns every h
  within 2^31 of its row's largest bit for bit, extreme codes give the exact
  sums, and a row with a NaN gives NaN logits.
* The greedy token is the argmax of exactly those logits (ties to the lowest
  id, -0 equal to +0); a head launched right after the body reads the body's
  finished output."""

import numpy as np
import pytest

import oracle
from gpu_util import check, dev, guarded, guards_intact, torch

from int8_weight_quantized_w4_b200 import synth

pytestmark = pytest.mark.gpu


def w4():
    import int8_weight_quantized_w4_b200 as w
    return w


def _head(K, V, tag, ldt=None):
    H = synth.i8_head(K, V, tag, ldt=ldt)
    tiles = w4().i8t_head_repack(dev(H["table"]), dev(H["scales"]), K, V, ldt=H["ldt"])
    return H, tiles


SHAPES = [(32, 5), (64, 1), (96, 300), (160, 129), (128, 128), (192, 129), (768, 50257), (1024, 300),
          (640, 1000)]


@pytest.mark.parametrize("K,V", SHAPES)
def test_repack_then_restore_is_the_identity(K, V):
    H, tiles = _head(K, V, 1)
    assert tiles.numel() == w4().i8t_head_repacked_bytes(K, V) == -(-V // 128) * (128 * K + 512)
    table, sc = w4().i8t_head_repack_restore(tiles, K, V)
    torch().cuda.synchronize()
    assert np.array_equal(table.cpu().numpy(), H["table"].reshape(K, H["ldt"])[:, :V])
    assert np.array_equal(sc.cpu().numpy().view(np.uint32), H["scales"].view(np.uint32))


def test_padded_row_stride_round_trip():
    K, V, ldt = 128, 200, 224
    H, tiles = _head(K, V, 2, ldt=ldt)
    table, _ = w4().i8t_head_repack_restore(tiles, K, V)
    torch().cuda.synchronize()
    assert np.array_equal(table.cpu().numpy(), H["table"].reshape(K, ldt)[:, :V])


@pytest.mark.parametrize("K,V", [(768, 50257), (192, 129)])
def test_tile_bytes_sit_where_the_header_says(K, V):
    H, tiles = _head(K, V, 3)
    buf = tiles.cpu().numpy()
    T = H["table"].reshape(K, H["ldt"])
    tb = 128 * K + 512
    g = np.random.default_rng(0)
    ks = np.concatenate([[0, K - 1], g.integers(0, K, 400)])
    vs = np.concatenate([[0, V - 1], g.integers(0, V, 400)])
    for k, v in zip(ks, vs):
        t, c = v // 128, v % 128
        u, hh, i = k // 32, (k % 32) // 16, k % 16
        byte = buf[t * tb + u * 4096 + (c // 8) * 256 + hh * 128 + (c % 8) * 16 + i]
        assert np.uint8(byte).view(np.int8) == T[k, v]
        sb = buf[t * tb + K * 128 + 4 * c:][:4].tobytes()
        assert np.frombuffer(sb, np.uint32)[0] == H["scales"][v:v + 1].view(np.uint32)[0]
    # padding tokens: code 0 and scale 0
    last = -(-V // 128) - 1
    for c in range(V - 128 * last, 128):
        assert buf[last * tb + (c // 8) * 256 + (c % 8) * 16] == 0
        assert np.frombuffer(buf[last * tb + K * 128 + 4 * c:][:4].tobytes(), np.uint32)[0] == 0


@pytest.mark.parametrize("K,V", SHAPES)
@pytest.mark.parametrize("M", [1, 3, 8])
def test_logits_match_the_oracle(K, V, M):
    H, tiles = _head(K, V, 4)
    h = synth.activations(M, K, 9, M)
    lg = w4().i8t_head_logits(dev(h), tiles, K, V)
    torch().cuda.synchronize()
    assert lg.shape == (M, V)
    ref, a = oracle.i8_head_ref(h, H["table"], H["scales"], K, V, H["ldt"])
    check(lg, ref, a, f"i8t M={M} K={K} V={V}")


@pytest.mark.parametrize("M", [2, 4, 5, 6, 7])
def test_every_row_count(M):
    K, V = 768, 50257
    H, tiles = _head(K, V, 5)
    h = synth.activations(M, K, 11, M)
    lg = w4().i8t_head_logits(dev(h), tiles, K, V)
    torch().cuda.synchronize()
    ref, a = oracle.i8_head_ref(h, H["table"], H["scales"], K, V)
    check(lg, ref, a, f"i8t M={M}")


def test_strided_rows_and_logits_leave_the_guards():
    K, V, M, ldh, ldl = 256, 1000, 5, 300, 1040
    H, tiles = _head(K, V, 6)
    hs = synth.activations(M, K, 12, ld=ldh)
    hbuf = dev(hs.reshape(-1))
    h = hbuf.view(M, ldh)[:, :K]
    y, buf = guarded(M, V, ld=ldl)
    w4().i8t_head_logits(h, tiles, K, V, logits=y)
    torch().cuda.synchronize()
    ref, a = oracle.i8_head_ref(hs.reshape(M, ldh)[:, :K], H["table"], H["scales"], K, V)
    check(y, ref, a, "i8t strided")
    assert guards_intact(buf, M, V, ldl)


def test_one_hot_table_returns_h_exactly():
    """T[k, v] = 1 for k = v mod K, scale 1: every logit is one h[m, k]; the
    digits hold every element within 2^31 of its row's largest exactly (rows
    here span at most 2^28), so the logits are h bit for bit."""
    K, V, M = 128, 1000, 8
    table = np.zeros((K, V), np.int8)
    table[np.arange(V) % K, np.arange(V)] = 1
    s = np.ones(V, np.float32)
    g = np.random.default_rng(21)
    sign = np.where(g.integers(0, 2, (M, K)) == 0, -1.0, 1.0)
    h = (sign * g.uniform(0.1, 4.0, (M, K)) * np.exp2(g.integers(-12, 13, (M, K)))).astype(np.float32)
    h[0] = (sign[0] * g.uniform(0.1, 4.0, K)).astype(np.float32)
    h[0, :4] = [1.0 + 2.0 ** -23, -(2.0 ** -20), 3.0e-3, 1000.0 + 2.0 ** -13]
    h[1, :] = 0.0
    h[1, 5] = -7.0  # one element; the rest exact zeros
    tiles = w4().i8t_head_repack(dev(table), dev(s), K, V)
    lg = w4().i8t_head_logits(dev(h), tiles, K, V)
    torch().cuda.synchronize()
    want = h[:, np.arange(V) % K]
    assert np.array_equal(lg.cpu().numpy().view(np.uint32), want.view(np.uint32))


def test_wide_rows_and_non_finite_rows():
    """A row spanning 2^120 of magnitudes stays within the tolerance (the
    elements below 2^-31 of the largest carry at most 2^-55 of it); an all-zero
    row gives zeros; a row holding a NaN gives NaN logits, the others not."""
    K, V, M = 256, 700, 4
    H = synth.i8_head(K, V, 14)
    g = np.random.default_rng(5)
    h = synth.activations(M, K, 14).copy()
    h[0] *= np.exp2(g.integers(-60, 60, K)).astype(np.float32)
    h[1] = 0.0
    h[3, 17] = np.nan
    tiles = w4().i8t_head_repack(dev(H["table"]), dev(H["scales"]), K, V)
    lg = w4().i8t_head_logits(dev(h), tiles, K, V).cpu().numpy()
    torch().cuda.synchronize()
    ref, a = oracle.i8_head_ref(h[:3], H["table"], H["scales"], K, V)
    check(lg[:3], ref, a, "wide rows")
    assert np.all(lg[1] == 0.0)
    assert np.all(np.isnan(lg[3]))


def test_extreme_codes_are_exact_and_deterministic():
    K, V, M = 1024, 300, 2
    table = np.where(np.arange(K * V).reshape(K, V) % 3 == 0, -128, 127).astype(np.int8)
    s = np.full(V, 0.25, np.float32)
    h = np.ones((M, K), np.float32)
    h[1] = -2.0
    tiles = w4().i8t_head_repack(dev(table), dev(s), K, V)
    a = w4().i8t_head_logits(dev(h), tiles, K, V)
    b = w4().i8t_head_logits(dev(h), tiles, K, V)
    torch().cuda.synchronize()
    assert torch().equal(a, b)
    col = table.astype(np.float64).sum(axis=0)
    want = np.stack([0.25 * col, -0.5 * col])
    assert np.array_equal(a.cpu().numpy().astype(np.float64), want)


def test_single_row_as_a_vector():
    K, V = 768, 4096
    H, tiles = _head(K, V, 7)
    h = synth.activations(1, K, 13)
    lg = w4().i8t_head_logits(dev(h.reshape(K)), tiles, K, V)
    torch().cuda.synchronize()
    ref, a = oracle.i8_head_ref(h, H["table"], H["scales"], K, V)
    check(lg, ref, a, "i8t vector row")


@pytest.mark.parametrize("M", [1, 8])
def test_argmax_is_the_argmax_of_the_logits(M):
    K, V = 768, 50257
    H, tiles = _head(K, V, 8)
    for tag in (1, 2):
        hn = synth.activations(M, K, tag, 30)
        h = dev(hn)
        lg = w4().i8t_head_logits(h, tiles, K, V).cpu().numpy()
        tok, best = w4().i8t_head_argmax(h, tiles, K, V)
        torch().cuda.synchronize()
        assert np.array_equal(tok.cpu().numpy(), np.argmax(lg, axis=1))
        assert np.array_equal(best.cpu().numpy(), lg.max(axis=1))
        rtok, _, _ = oracle.i8_head_argmax_ref(hn, H["table"], H["scales"], K, V)
        ref, a = oracle.i8_head_ref(hn, H["table"], H["scales"], K, V)
        tol = oracle.tolerance(a)
        for m in range(M):
            g_, r_ = int(tok[m].item()), int(rtok[m])
            assert g_ == r_ or ref[m, g_] >= ref[m, r_] - 2 * tol[m, r_]


def test_argmax_ties_and_signed_zero():
    K, V = 64, 1000
    table = np.full((K, V), -20, np.int8)
    table[:, 123] = 0
    table[:, 700] = 0
    s = np.full(V, 0.5, np.float32)
    s[123] = -0.5  # 0 * -0.5 = -0, equal to the +0 of token 700
    tiles = w4().i8t_head_repack(dev(table), dev(s), K, V)
    tok, best = w4().i8t_head_argmax(dev(np.ones((2, K), np.float32)), tiles, K, V)
    torch().cuda.synchronize()
    assert tok.cpu().tolist() == [123, 123] and best.cpu().tolist() == [0.0, 0.0]
    table[:, 123] = 100
    table[:, 700] = 100
    s[123] = 0.5
    tiles = w4().i8t_head_repack(dev(table), dev(s), K, V)
    tok, best = w4().i8t_head_argmax(dev(np.ones((1, K), np.float32)), tiles, K, V)
    torch().cuda.synchronize()
    assert int(tok.item()) == 123 and float(best.item()) == 0.5 * 100 * K


def test_head_after_body_reads_the_finished_output():
    """The body's output row is the head's input, launched back to back on
    one stream (both launches start early): the head must see it complete."""
    T = torch()
    K, V = 768, 50257
    W = synth.w4_weight(K, K, 62)
    Wd = {k: dev(W[k]) for k in ("qw", "scales", "zp")}
    wr = w4().w4_repack(Wd["qw"], Wd["scales"], Wd["zp"], K, K)
    H, tiles = _head(K, V, 9)
    x = dev(synth.activations(1, K, 62))
    y = T.full((1, K), float("nan"), dtype=T.float32, device="cuda")
    T.cuda.synchronize()
    for _ in range(3):
        w4().w4r_matmul(x, wr, K, K, y=y)
        lg = w4().i8t_head_logits(y, tiles, K, V)
    T.cuda.synchronize()
    ref, a = oracle.i8_head_ref(y.cpu().numpy(), H["table"], H["scales"], K, V)
    check(lg, ref, a, "tensor-core head after body")


def test_empty_calls_are_no_ops():
    T = torch()
    H, tiles = _head(64, 100, 10)
    out = T.full((0, 100), 1.0, device="cuda")
    w4().i8t_head_logits(T.zeros((0, 64), device="cuda"), tiles, 64, 100, logits=out)
    torch().cuda.synchronize()


def test_refusals():
    T = torch()
    H, tiles = _head(64, 100, 11)
    with pytest.raises(w4().W4Error):  # more than 8 rows
        w4().i8t_head_logits(T.zeros((9, 64), device="cuda"), tiles, 64, 100)
    h = T.zeros((2, 64), device="cuda")
    out = T.zeros((2, 100), device="cuda")
    L, P = w4().lib(), w4()._ptr
    with pytest.raises(w4().W4Error):  # h not 4-byte aligned
        w4()._check(L.i8t_head_logits(P(h) + 2, 64, P(tiles), 64, 100, 1, P(out), 100, None), "i8t_head_logits")
    with pytest.raises(w4().W4Error):  # tiles not 16-byte aligned
        w4()._check(L.i8t_head_logits(P(h), 64, P(tiles) + 8, 64, 100, 1, P(out), 100, None), "i8t_head_logits")
    with pytest.raises(w4().W4Error):  # ldh < K
        w4()._check(L.i8t_head_logits(P(h), 32, P(tiles), 64, 100, 2, P(out), 100, None), "i8t_head_logits")
    with pytest.raises(w4().W4Error):  # ldl < V
        w4()._check(L.i8t_head_logits(P(h), 64, P(tiles), 64, 100, 2, P(out), 50, None), "i8t_head_logits")
    with pytest.raises(w4().W4Error):  # K the layout does not take
        w4()._check(L.i8t_head_logits(P(h), 64, P(tiles), 80, 100, 1, P(out), 100, None), "i8t_head_logits")
    for K in (80, 1056, 0):  # K % 32 != 0, K > 1024, K = 0
        with pytest.raises(ValueError):
            w4().i8t_head_repack(dev(np.zeros((max(K, 1), 100), np.int8)), dev(np.ones(100, np.float32)), K, 100)
        assert w4().i8t_head_repacked_bytes(K, 100) == 0
