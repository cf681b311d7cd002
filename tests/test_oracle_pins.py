"""The oracle pinned to facts outside itself (CPU only).

The pins live in ``pins.py`` as functions of the implementation under test.
Here they run against the oracle (all must pass) and against copies of it
with one planted mistake each (each copy must fail at least one pin), which
shows that the pins can see the mistakes they are meant to catch.
"""

import os
from fractions import Fraction
from types import SimpleNamespace

import numpy as np
import pytest

import oracle
import pins

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_oracle_passes_every_w4_pin():
    assert pins.run_w4_pins(oracle) == []


@pytest.mark.parametrize("chk", pins.ALL_W4_CHECKS, ids=lambda c: c.__name__)
def test_w4_pin(chk):
    assert chk(oracle) == []


# ---------------------------------------------------------------- mutants

def _impl(unpack=None, dequant=None, acc=np.float64, absum=True):
    unpack = unpack or oracle.unpack_nibbles
    dequant = dequant or (lambda qw, s, zp, K, N: _dequant_with(unpack, qw, s, zp, K, N))

    def matmul(x, qw, s, zp, K, N):
        w = np.asarray(dequant(qw, s, zp, K, N)).astype(acc)
        xx = np.asarray(x, np.float32).reshape(-1, K).astype(acc)
        y = (xx @ w).astype(np.float64)
        a = (np.abs(xx) @ np.abs(w)) if absum else np.abs(xx @ w)
        return y, a.astype(np.float64)

    return SimpleNamespace(unpack_nibbles=unpack, pack_nibbles=oracle.pack_nibbles,
                           dequantize_w4=dequant, w4_matmul_ref=matmul)


def _dequant_with(unpack, qw, s, zp, K, N, block=32, zp_sign=1, use_zp=True,
                  scale_rows=False, transpose=False, zp_block0=False, fp32_round=True,
                  drop_last_block=False):
    nb = K // 32
    q = unpack(qw, K * N).astype(np.int32)
    q = q.reshape(N, K).T if transpose else q.reshape(K, N)
    z = unpack(zp, nb * N).reshape(nb, N).astype(np.int32)
    sc = np.asarray(s, np.float32).reshape(nb, N)
    blk = np.minimum(np.arange(K) // block, nb - 1)
    if zp_block0:
        zb = np.zeros_like(blk)
    else:
        zb = blk
    sb = (np.arange(K) % nb) if scale_rows else blk
    d = (q - z[zb]) * zp_sign if use_zp else q
    if fp32_round:
        w = d.astype(np.float32) * sc[sb]
    else:
        w = d.astype(np.float64) * sc[sb].astype(np.float64)
    if drop_last_block:
        w = w.copy()
        w[K - 32:] = 0
    return w


def _high_first(packed, count):
    b = np.asarray(packed, np.uint8).reshape(-1)
    out = np.empty(2 * b.size, np.uint8)
    out[0::2] = b >> 4
    out[1::2] = b & 0x0F
    return out[:count]


MUTANTS = {
    "high_nibble_first": lambda: _impl(unpack=_high_first),
    "zero_point_ignored": lambda: _impl(dequant=lambda *a: _dequant_with(oracle.unpack_nibbles, *a, use_zp=False)),
    "sign_flipped": lambda: _impl(dequant=lambda *a: _dequant_with(oracle.unpack_nibbles, *a, zp_sign=-1)),
    "block_of_16": lambda: _impl(dequant=lambda *a: _dequant_with(oracle.unpack_nibbles, *a, block=16)),
    "scale_per_row": lambda: _impl(dequant=lambda *a: _dequant_with(oracle.unpack_nibbles, *a, scale_rows=True)),
    "weight_transposed": lambda: _impl(dequant=lambda *a: _dequant_with(oracle.unpack_nibbles, *a, transpose=True)),
    "zero_point_of_block0": lambda: _impl(dequant=lambda *a: _dequant_with(oracle.unpack_nibbles, *a, zp_block0=True)),
    "no_fp32_rounding": lambda: _impl(dequant=lambda *a: _dequant_with(oracle.unpack_nibbles, *a, fp32_round=False)),
    "last_block_dropped": lambda: _impl(dequant=lambda *a: _dequant_with(oracle.unpack_nibbles, *a, drop_last_block=True)),
    "fp32_accumulation": lambda: _impl(acc=np.float32),
    "abs_of_sum": lambda: _impl(absum=False),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name):
    failures = pins.run_w4_pins(MUTANTS[name]())
    assert failures, f"mutant {name} passed every pin"


# ---------------------------------------------------------------- golden

def _golden(path):
    meta, rows = {}, []
    for line in open(path):
        line = line.split("#", 1)[0].strip()
        if not line:
            continue
        parts = line.split()
        if parts[0] == "row":
            rows.append((parts[1], float(parts[2])))
        else:
            meta[parts[0]] = float(parts[1])
    return meta, rows


_ROWS = {
    "ones": lambda k: np.ones_like(k, dtype=np.float64),
    "mod7_minus3": lambda k: (k % 7) - 3.0,
    "alt_quarter": lambda k: 0.25 * (-1.0) ** k,
    "ramp_eighth": lambda k: k / 8.0,
}


def test_golden_halved_row_sums():
    meta, rows = _golden(os.path.join(GOLDEN, "halved_row_sums.txt"))
    K, N = int(meta["K"]), int(meta["N"])
    qw, sc, zp = pins.make_w4(np.full((K, N), int(meta["q"])), np.full((K // 32, N), int(meta["zp"])),
                              np.full((K // 32, N), meta["scale"]))
    k = np.arange(K)
    x = np.stack([_ROWS[name](k) for name, _ in rows]).astype(np.float32)
    y, _ = oracle.w4_matmul_ref(x, qw, sc, zp, K, N)
    want = np.array([[v] * N for _, v in rows])
    assert np.array_equal(y, want)


# ---------------------------------------------------------------- sampled oracle

def test_column_dequant_matches_full():
    g = np.random.default_rng(3)
    K, N = 96, 20
    qi, zi, s = pins._rand_w4(g, K, N)
    qw, sc, zp = pins.make_w4(qi, zi, s)
    full = oracle.dequantize_w4(qw, sc, zp, K, N)
    cols = np.array([0, 1, 2, 7, 19, 18, 1])
    assert np.array_equal(oracle.dequantize_w4_columns(qw, sc, zp, K, N, cols), full[:, cols])


def test_sampled_entries_match_full():
    g = np.random.default_rng(4)
    K, N, M = 128, 12, 5
    qi, zi, s = pins._rand_w4(g, K, N)
    qw, sc, zp = pins.make_w4(qi, zi, s)
    x = g.standard_normal((M, K)).astype(np.float32)
    y, a = oracle.w4_matmul_ref(x, qw, sc, zp, K, N)
    rows = np.array([0, 4, 2, 3, 0])
    cols = np.array([11, 0, 5, 5, 1])
    ys, as_ = oracle.w4_matmul_ref_entries(x, qw, sc, zp, K, N, rows, cols)
    assert np.allclose(ys, y[rows, cols], rtol=1e-14, atol=1e-14)
    assert np.allclose(as_, a[rows, cols], rtol=1e-14, atol=1e-14)


# ---------------------------------------------------------------- shape rules

@pytest.mark.parametrize("K,N", [(31, 4), (33, 4), (32, 3), (-32, 2)])
def test_bad_shapes_rejected(K, N):
    with pytest.raises(ValueError):
        oracle.check_w4_shape(K, N)


def test_empty_shapes():
    y, a = oracle.w4_matmul_ref(np.zeros((2, 0), np.float32), np.zeros(0, np.uint8),
                                np.zeros(0, np.float32), np.zeros(0, np.uint8), 0, 4)
    assert y.shape == (2, 4) and np.all(y == 0) and np.all(a == 0)
    y, _ = oracle.w4_matmul_ref(np.zeros((0, 32), np.float32), np.zeros(32, np.uint8),
                                np.ones(2, np.float32), np.zeros(1, np.uint8), 32, 2)
    assert y.shape == (0, 2)


# ---------------------------------------------------------------- quantiser

def _quant_err_ok(w):
    K, N = w.shape
    qw, s, zp = oracle.quantize_w4(w)
    q = oracle.unpack_nibbles(qw, K * N)
    z = oracle.unpack_nibbles(zp, (K // 32) * N)
    assert q.max() <= 15 and z.max() <= 15
    deq = oracle.dequantize_w4(qw, s, zp, K, N).astype(np.float64)
    sb = np.repeat(s.astype(np.float64), 32, axis=0)
    ulp = np.spacing(np.abs(w).astype(np.float32)).astype(np.float64)
    err = np.abs(deq - w.astype(np.float64))
    assert np.all(err <= sb / 2 * (1 + 1e-6) + ulp), float((err - sb / 2).max())
    return qw, s, zp


def test_quantizer_error_bound_random():
    g = np.random.default_rng(8)
    _quant_err_ok(g.standard_normal((128, 40)).astype(np.float32))


def test_quantizer_adversarial_blocks():
    g = np.random.default_rng(9)
    pos = np.abs(g.standard_normal((64, 8))).astype(np.float32) + 1.0  # all positive
    _quant_err_ok(pos)
    neg = -pos
    _quant_err_ok(neg)
    const = np.full((32, 4), 0.75, np.float32)  # all equal, nonzero
    _quant_err_ok(const)
    zero = np.zeros((32, 4), np.float32)  # all zero -> s = 1, zp = 0, exact zeros
    qw, s, zp = _quant_err_ok(zero)
    assert np.all(s == 1.0) and np.all(oracle.unpack_nibbles(zp, 4) == 0)
    assert np.all(oracle.dequantize_w4(qw, s, zp, 32, 4) == 0)


def test_quantizer_roundtrip_is_fixed_point():
    """Quantising an already-quantised weight recovers its codes' values."""
    g = np.random.default_rng(10)
    w = g.standard_normal((64, 16)).astype(np.float32)
    qw, s, zp = oracle.quantize_w4(w)
    deq = oracle.dequantize_w4(qw, s, zp, 64, 16)
    qw2, s2, zp2 = oracle.quantize_w4(deq)
    deq2 = oracle.dequantize_w4(qw2, s2, zp2, 64, 16)
    assert np.allclose(deq2, deq, rtol=0, atol=np.repeat(s, 32, axis=0) * 1e-5 + 1e-7)


# ---------------------------------------------------------------- head

def test_head_closed_forms():
    K, V = 16, 10
    t = np.ones(K * V, np.int8)
    s = np.full(V, 0.5, np.float32)
    h = (np.arange(K, dtype=np.float32) - 3)[None, :]
    y, a = oracle.i8_head_ref(h, t, s, K, V)
    assert np.array_equal(y, np.full((1, V), 0.5 * float(h.sum())))
    g = np.random.default_rng(1)
    t = g.integers(-128, 128, K * V).astype(np.int8)
    s = g.uniform(0.002, 0.01, V).astype(np.float32)
    for k in (0, 5, 15):
        h = np.zeros((1, K), np.float32)
        h[0, k] = 1.0
        y, _ = oracle.i8_head_ref(h, t, s, K, V)
        want = [np.float32(float(int(t[k * V + v]) * Fraction(float(s[v])))) for v in range(V)]
        assert np.array_equal(y[0], np.array(want, np.float64))


def test_head_brute_force_dyadic():
    g = np.random.default_rng(12)
    for M, K, V in ((1, 8, 5), (3, 12, 7)):
        t = g.integers(-128, 128, K * V).astype(np.int8)
        s = 2.0 ** -g.integers(1, 10, V).astype(np.float64)
        h = (g.integers(-20, 21, (M, K)) / 4.0).astype(np.float32)
        y, a = oracle.i8_head_ref(h, t, s.astype(np.float32), K, V)
        for m in range(M):
            for v in range(V):
                ex = sum(Fraction(float(h[m, k])) * int(t[k * V + v]) * Fraction(float(s[v])) for k in range(K))
                ax = sum(abs(Fraction(float(h[m, k])) * int(t[k * V + v]) * Fraction(float(s[v]))) for k in range(K))
                assert Fraction(float(y[m, v])) == ex
                assert Fraction(float(a[m, v])) == ax


def test_head_padded_rows_ignore_padding():
    g = np.random.default_rng(13)
    K, V, ldt = 9, 13, 21
    t = g.integers(-127, 128, (K, V)).astype(np.int8)
    padded = np.full((K, ldt), 127, np.int8)
    padded[:, :V] = t
    s = g.uniform(0.002, 0.01, V).astype(np.float32)
    h = g.standard_normal((2, K)).astype(np.float32)
    y1, _ = oracle.i8_head_ref(h, t.reshape(-1), s, K, V)
    y2, _ = oracle.i8_head_ref(h, padded.reshape(-1), s, K, V, ldt=ldt)
    assert np.array_equal(y1, y2)


def test_head_quantizer_bound():
    g = np.random.default_rng(14)
    w = g.standard_normal((24, 30)).astype(np.float32)
    q, s = oracle.quantize_i8_head(w)
    deq = q.astype(np.float64) * s.astype(np.float64)[None, :]
    assert np.all(np.abs(deq - w) <= s[None, :].astype(np.float64) / 2 * (1 + 1e-6) + 1e-7)
    assert q.min() >= -127 and q.max() <= 127


def test_last_position_rows():
    hs = np.arange(2 * 5 * 3, dtype=np.float32).reshape(2, 5, 3)
    r = oracle.last_position_rows(hs, 5, 3)
    assert np.array_equal(r, hs[:, 4, :])


# ---------------------------------------------------------------- tolerance

def test_tolerance_and_violation():
    y_ref = np.array([1.0, -2.0, 0.0])
    a = np.array([10.0, 100.0, 0.0])
    tol = oracle.tolerance(a)
    assert np.allclose(tol, [1e-4 + 1e-6, 1e-3 + 1e-6, 1e-6])
    assert oracle.max_violation(y_ref + 0.5 * tol, y_ref, a) < 0
    assert oracle.max_violation(y_ref + 2 * tol, y_ref, a) > 0
    assert oracle.max_violation(np.array([np.nan, 0, 0]), y_ref, a) == np.inf


def test_fp32_blocked_sum_meets_tolerance():
    """The tolerance admits an fp32 sum accumulated in 32-row blocks (the
    order a GPU reduction takes) on the config shapes; a sanity check of the
    tolerance, not of the oracle."""
    g = np.random.default_rng(15)
    K, N = 3072, 64
    qi, zi, s = pins._rand_w4(g, K, N)
    qw, sc, zp = pins.make_w4(qi, zi, s)
    x = g.standard_normal((1, K)).astype(np.float32)
    y, a = oracle.w4_matmul_ref(x, qw, sc, zp, K, N)
    w = oracle.dequantize_w4(qw, sc, zp, K, N)
    part = (x.reshape(K // 32, 32, 1) * w.reshape(K // 32, 32, N)).sum(axis=1, dtype=np.float32)
    y32 = part.sum(axis=0, dtype=np.float32)
    assert oracle.max_violation(y32[None, :], y, a) < 0


# ---------------------------------------------------------------- token lookup

def test_embed_literal():
    """Hand-computed: column t of the [K, V] table times scale t."""
    table = np.array([[1, -2, 3], [4, 5, -6]], np.int8)  # K = 2, V = 3
    s = np.array([0.5, 0.25, 2.0], np.float32)
    e = oracle.i8_embed_ref(table, s, [1, 2, 0], 2, 3)
    assert np.array_equal(e, np.array([[-0.5, 1.25], [6.0, -12.0], [0.5, 2.0]], np.float32))


def test_embed_is_the_head_column():
    """The head is tied: logit t of h equals h . embed(t) (both in fp64 from
    the same fp32 weights), for every t."""
    g = np.random.default_rng(11)
    K, V = 48, 70
    table = g.integers(-127, 128, (K, V)).astype(np.int8)
    s = g.uniform(0.002, 0.01, V).astype(np.float32)
    h = g.standard_normal((1, K)).astype(np.float32)
    y, _ = oracle.i8_head_ref(h, table, s, K, V)
    e = oracle.i8_embed_ref(table, s, np.arange(V), K, V).astype(np.float64)
    assert np.allclose(e @ h[0].astype(np.float64), y[0], rtol=0, atol=1e-12)


def test_embed_padded_rows_and_bounds():
    g = np.random.default_rng(12)
    K, V, ldt = 5, 9, 13
    t = g.integers(-128, 128, (K, V)).astype(np.int8)
    padded = np.full((K, ldt), 77, np.int8)
    padded[:, :V] = t
    s = g.uniform(0.01, 0.1, V).astype(np.float32)
    toks = [0, 8, 3, 3]
    assert np.array_equal(oracle.i8_embed_ref(padded.reshape(-1), s, toks, K, V, ldt=ldt),
                          oracle.i8_embed_ref(t, s, toks, K, V))
    with pytest.raises(ValueError):
        oracle.i8_embed_ref(t, s, [9], K, V)
    with pytest.raises(ValueError):
        oracle.i8_embed_ref(t, s, [-1], K, V)
    assert oracle.i8_embed_ref(t, s, [], K, V).shape == (0, K)


# ---------------------------------------------------------------- greedy decoding

def test_argmax_literal_and_ties():
    """Hand case: h = [1, 2]; columns give logits 0.5*(1+4)=2.5, 0.25*(-2+10)=2,
    2*(3-12)=-18, 1*(1+4)=5 (twice): the first of the two fives wins."""
    table = np.array([[1, -2, 3, 1, 1], [2, 5, -6, 2, 2]], np.int8)  # K = 2, V = 5
    s = np.array([0.5, 0.25, 2.0, 1.0, 1.0], np.float32)
    h = np.array([[1.0, 2.0]], np.float32)
    tok, best, gap = oracle.i8_head_argmax_ref(h, table, s, 2, 5)
    assert tok.tolist() == [3] and best.tolist() == [5.0] and gap.tolist() == [2.5]
