"""GPU: the int8 head in the streaming layout (i8_head_repack /
i8_head_repack_restore) and the M = 1 head GEMV that reads it
(i8r_head_logits, i8r_head_argmax), against the oracle.

* Repacking reorders and biases bytes only: restoring gives the page's table
  and scales back exactly, and every code and scale sits where include/w4.h
  says, read back through the oracle's own table.
* The logits match the oracle within |l - l_ref| <= 1e-5 * sum|h*w| + 1e-6;
  the greedy token is the argmax of exactly those logits (ties to the lowest
  id, -0 equal to +0); a head launched right after the body reads the body's
  finished output."""

import math

import numpy as np
import pytest

import oracle
from gpu_util import check, dev, torch

from int8_weight_quantized_w4_b200 import synth

pytestmark = pytest.mark.gpu


def w4():
    import int8_weight_quantized_w4_b200 as w
    return w


def _head(K, V, tag, ldt=None):
    H = synth.i8_head(K, V, tag, ldt=ldt)
    T = dev(H["table"])
    S = dev(H["scales"])
    tr = w4().i8_head_repack(T, S, K, V, ldt=H["ldt"])
    return H, tr


SHAPES = [(16, 1), (32, 7), (48, 100), (96, 8), (768, 50257), (256, 1000), (8192, 40), (64, 4096)]


@pytest.mark.parametrize("K,V", SHAPES)
def test_repack_then_restore_is_the_identity(K, V):
    H, tr = _head(K, V, 1)
    assert tr.numel() == w4().i8_head_repacked_bytes(K, V)
    table, sc = w4().i8_head_repack_restore(tr, K, V)
    torch().cuda.synchronize()
    assert np.array_equal(table.cpu().numpy(), H["table"].reshape(K, H["ldt"])[:, :V])
    assert np.array_equal(sc.cpu().numpy().view(np.uint32), H["scales"].view(np.uint32))


def test_padded_row_stride_round_trip():
    K, V, ldt = 48, 100, 112
    H, tr = _head(K, V, 2, ldt=ldt)
    table, sc = w4().i8_head_repack_restore(tr, K, V)
    torch().cuda.synchronize()
    assert np.array_equal(table.cpu().numpy(), H["table"].reshape(K, ldt)[:, :V])


@pytest.mark.parametrize("K,V", [(768, 50257), (48, 100)])
def test_repacked_bytes_sit_where_the_header_says(K, V):
    H, tr = _head(K, V, 3)
    buf = tr.cpu().numpy()
    T = H["table"].reshape(K, H["ldt"])
    nb = K // 16
    gs = 32 // math.gcd(nb, 32)
    A = gs * nb // 32
    gbytes = A * 4096 + 32 * gs
    g = np.random.default_rng(0)
    ks = np.concatenate([[0, K - 1], g.integers(0, K, 400)])
    vs = np.concatenate([[0, V - 1], g.integers(0, V, 400)])
    for k, v in zip(ks, vs):
        strip = v // 8
        G, s = strip // gs, strip % gs
        b = k // 16
        phase, r = b % (32 // gs), b // (32 // gs)
        lane = phase * gs + s
        c, e = (k % 16) // 2, k % 2
        hh, i = (v % 8) // 4, v % 4
        byte = buf[G * gbytes + r * 4096 + c * 512 + lane * 16 + (2 * e + hh) * 4 + i]
        assert np.int8(np.uint8(byte) ^ np.uint8(0x80)) == T[k, v]
        sb = buf[G * gbytes + A * 4096 + s * 32 + (v % 8) * 4:][:4].tobytes()
        assert np.frombuffer(sb, np.uint32)[0] == H["scales"][v:v + 1].view(np.uint32)[0]


@pytest.mark.parametrize("K,V", SHAPES)
def test_logits_match_the_oracle(K, V):
    H, tr = _head(K, V, 4)
    h = synth.activations(1, K, 9)
    lg = w4().i8r_head_logits(dev(h), tr, K, V)
    torch().cuda.synchronize()
    ref, a = oracle.i8_head_ref(h, H["table"], H["scales"], K, V, H["ldt"])
    check(lg, ref, a, f"i8r K={K} V={V}")


def test_logits_are_deterministic_and_extreme_codes_exact():
    K, V = 64, 300
    table = np.where(np.arange(K * V).reshape(K, V) % 2 == 0, -128, 127).astype(np.int8)
    s = np.full(V, 0.25, np.float32)
    h = np.ones((1, K), np.float32)
    tr = w4().i8_head_repack(dev(table), dev(s), K, V)
    a = w4().i8r_head_logits(dev(h), tr, K, V)
    b = w4().i8r_head_logits(dev(h), tr, K, V)
    torch().cuda.synchronize()
    assert torch().equal(a, b)
    want = 0.25 * table.astype(np.float64).sum(axis=0)
    assert np.array_equal(a.cpu().numpy()[0].astype(np.float64), want)


def test_argmax_is_the_argmax_of_the_logits():
    K, V = 768, 50257
    H, tr = _head(K, V, 5)
    for tag in (1, 2, 3):
        h = dev(synth.activations(1, K, tag))
        lg = w4().i8r_head_logits(h, tr, K, V).cpu().numpy()[0]
        tok, best = w4().i8r_head_argmax(h, tr, K, V)
        torch().cuda.synchronize()
        assert int(tok.item()) == int(np.argmax(lg)) and float(best.item()) == float(lg.max())
        rtok, _, gap = oracle.i8_head_argmax_ref(synth.activations(1, K, tag), H["table"], H["scales"], K, V)
        ref, a = oracle.i8_head_ref(synth.activations(1, K, tag), H["table"], H["scales"], K, V)
        g = int(tok.item())
        assert g == int(rtok[0]) or ref[0, g] >= ref[0, int(rtok[0])] - 2 * oracle.tolerance(a)[0, int(rtok[0])]


def test_argmax_ties_and_signed_zero():
    K, V = 32, 1000
    table = np.full((K, V), -20, np.int8)
    table[:, 123] = 0
    table[:, 700] = 0
    s = np.full(V, 0.5, np.float32)
    s[123] = -0.5  # 0 * -0.5 = -0, equal to the +0 of column 700
    tr = w4().i8_head_repack(dev(table), dev(s), K, V)
    tok, best = w4().i8r_head_argmax(dev(np.ones((1, K), np.float32)), tr, K, V)
    torch().cuda.synchronize()
    assert int(tok.item()) == 123 and float(best.item()) == 0.0
    table[:, 123] = 100
    table[:, 700] = 100
    s[123] = 0.5
    tr = w4().i8_head_repack(dev(table), dev(s), K, V)
    tok, best = w4().i8r_head_argmax(dev(np.ones((1, K), np.float32)), tr, K, V)
    torch().cuda.synchronize()
    assert int(tok.item()) == 123 and float(best.item()) == 0.5 * 100 * K


def test_head_after_body_reads_the_finished_output():
    """The body's output row is the head's input, launched back to back on
    one stream (both launches start early): the head must see it complete."""
    T = torch()
    K = 768
    W = synth.w4_weight(K, K, 61)
    Wd = {k: dev(W[k]) for k in ("qw", "scales", "zp")}
    wr = w4().w4_repack(Wd["qw"], Wd["scales"], Wd["zp"], K, K)
    H, tr = _head(K, 50257, 6)
    x = dev(synth.activations(1, K, 61))
    y = T.full((1, K), float("nan"), dtype=T.float32, device="cuda")
    T.cuda.synchronize()
    for _ in range(3):
        w4().w4r_matmul(x, wr, K, K, y=y)
        lg = w4().i8r_head_logits(y, tr, K, 50257)
    T.cuda.synchronize()
    ref, a = oracle.i8_head_ref(y.cpu().numpy(), H["table"], H["scales"], K, 50257)
    check(lg, ref, a, "head after body")


def test_refusals():
    T = torch()
    H, tr = _head(48, 100, 7)
    with pytest.raises(w4().W4Error):  # h not 16-byte aligned
        w4().i8r_head_logits(T.zeros(52, device="cuda")[1:49], tr, 48, 100)
    with pytest.raises(ValueError):
        w4().i8_head_repack(dev(H["table"]), dev(H["scales"]), 40, 100)
