"""Checks that pin the oracle to facts outside itself.

Each check takes the implementation under test as an argument (an object with
``unpack_nibbles``, ``pack_nibbles``, ``dequantize_w4`` and ``w4_matmul_ref``)
and returns a list of failure messages. The real oracle must pass all of them;
``test_oracle_pins`` also runs them against oracle copies with one planted,
plausible mistake each and requires every mutant to fail at least one check.

The facts come from the quantisation section of the tokenling export page
("ONNX export, quantization and the browser runtime": dq4 stores 4-bit
asymmetric weights in blocks of 32 along K with an fp32 scale and a uint4
zero point per block, restored by DequantizeLinear) and from arithmetic:
exact rational results on dyadic inputs, closed forms, and invariants of a
linear map.
"""

from __future__ import annotations

from fractions import Fraction

import numpy as np

BLOCK = 32


def _pack_ref(q):
    """Pack two per byte, low nibble first, written as plain integer maths
    (byte = q[2i] + 16 * q[2i+1]) so the pins do not lean on the oracle's own
    packer."""
    q = [int(v) for v in np.asarray(q).reshape(-1)]
    if len(q) % 2:
        q.append(0)
    return np.array([q[2 * i] + 16 * q[2 * i + 1] for i in range(len(q) // 2)], dtype=np.uint8)


def make_w4(q_int, zp_int, scales):
    """Buffers for integer q [K, N], zp [K/32, N] and scales [K/32, N]."""
    q_int = np.asarray(q_int)
    zp_int = np.asarray(zp_int)
    return _pack_ref(q_int), np.asarray(scales, np.float32).reshape(-1), _pack_ref(zp_int)


def exact_matmul(x, q_int, zp_int, scales):
    """Exact rational y and sum|x*w| with w = fp32((q - zp) * s) (single RN)."""
    x = np.asarray(x, np.float32)
    K, N = np.asarray(q_int).shape
    M = x.shape[0]
    y = [[Fraction(0)] * N for _ in range(M)]
    a = [[Fraction(0)] * N for _ in range(M)]
    for n in range(N):
        col = []
        for k in range(K):
            b = k // BLOCK
            exact_w = (int(q_int[k][n]) - int(zp_int[b][n])) * Fraction(float(scales[b][n]))
            col.append(Fraction(float(np.float32(float(exact_w)))))
        for m in range(M):
            acc = Fraction(0)
            aa = Fraction(0)
            for k in range(K):
                t = Fraction(float(x[m, k])) * col[k]
                acc += t
                aa += abs(t)
            y[m][n] = acc
            a[m][n] = aa
    return y, a


# ---------------------------------------------------------------- packing

def check_nibble_literals(o):
    f = []
    if list(o.unpack_nibbles(np.array([0x21], np.uint8), 2)) != [1, 2]:
        f.append("byte 0x21 must unpack to (1, 2): low nibble first")
    if list(o.unpack_nibbles(np.array([0xF0], np.uint8), 2)) != [0, 15]:
        f.append("byte 0xF0 must unpack to (0, 15)")
    if list(o.pack_nibbles(np.array([1, 2]))) != [0x21]:
        f.append("(1, 2) must pack to 0x21")
    if list(o.pack_nibbles(np.array([7]))) != [0x07]:
        f.append("an odd count pads the high nibble with 0")
    return f


def check_pack_roundtrips(o):
    f = []
    allb = np.arange(256, dtype=np.uint8)
    if not np.array_equal(o.pack_nibbles(o.unpack_nibbles(allb, 512)), allb):
        f.append("pack(unpack(b)) != b for some byte")
    pairs = np.array([(lo, hi) for hi in range(16) for lo in range(16)], np.uint8).reshape(-1)
    if not np.array_equal(o.unpack_nibbles(o.pack_nibbles(pairs), 512), pairs):
        f.append("unpack(pack(q0, q1)) != (q0, q1) for some pair")
    if not np.array_equal(o.pack_nibbles(pairs), _pack_ref(pairs)):
        f.append("packing disagrees with byte = q0 + 16*q1")
    return f


# ---------------------------------------------------------------- dequantisation

def _all_pairs_weight(s):
    """K = 32, N = 256: column n carries (q, zp) = (n % 16, n // 16) in every row."""
    n = np.arange(256)
    q = np.tile(n % 16, (32, 1))
    zp = (n // 16)[None, :]
    sc = np.full((1, 256), s, np.float32)
    return q, zp, sc


def check_dequant_dyadic_all_pairs(o):
    f = []
    for e in (-1, 0, 1, 3, 7, 12):
        s = 2.0 ** (-e)
        q, zp, sc = _all_pairs_weight(s)
        qw, scales, zpk = make_w4(q, zp, sc)
        w = o.dequantize_w4(qw, scales, zpk, 32, 256)
        ints = w.astype(np.float64) * 2.0 ** e
        if not np.array_equal(ints, (q - zp).astype(np.float64)):
            f.append(f"w * 2^{e} != q - zp for dyadic scale 2^-{e}")
        zero = w[:, (np.arange(256) % 16) == (np.arange(256) // 16)]
        if np.any(zero != 0) or np.any(np.signbit(zero)):
            f.append("q == zp must dequantise to exactly +0")
    return f


def check_dequant_single_rounding(o):
    g = np.random.default_rng(11)
    q, zp, _ = _all_pairs_weight(1.0)
    sc = g.uniform(0.001, 0.05, size=(1, 256)).astype(np.float32)
    qw, scales, zpk = make_w4(q, zp, sc)
    w = o.dequantize_w4(qw, scales, zpk, 32, 256)
    want = np.array([np.float32(float((int(q[0, n]) - int(zp[0, n])) * Fraction(float(sc[0, n]))))
                     for n in range(256)], np.float32)
    if not np.array_equal(w[0], want) or not np.array_equal(w[31], want):
        return ["dequantised value is not (q - zp) * s rounded once to fp32"]
    return []


# ---------------------------------------------------------------- closed forms

def check_closed_forms(o):
    f = []
    # (i) K=32: x = 1, q - zp = 1, s = 0.5  ->  y = 16 in every column
    q = np.full((32, 4), 9)
    zp = np.full((1, 4), 8)
    qw, sc, zpk = make_w4(q, zp, np.full((1, 4), 0.5))
    y, a = o.w4_matmul_ref(np.ones((1, 32), np.float32), qw, sc, zpk, 32, 4)
    if not np.array_equal(y, np.full((1, 4), 16.0)) or not np.array_equal(a, np.full((1, 4), 16.0)):
        f.append("x=1, q-zp=1, s=0.5, K=32 must give y = 16")
    # (ii) K=64: two blocks with scales 0.25 and 2, q - zp = d1 and d2
    d1, d2 = 3, -5
    q = np.concatenate([np.full((32, 2), 7 + d1), np.full((32, 2), 7 + d2)])
    zp = np.full((2, 2), 7)
    sc = np.array([[0.25, 0.25], [2.0, 2.0]])
    qw, scv, zpk = make_w4(q, zp, sc)
    y, _ = o.w4_matmul_ref(np.ones((1, 64), np.float32), qw, scv, zpk, 64, 2)
    if not np.array_equal(y, np.full((1, 2), 32 * 0.25 * d1 + 32 * 2.0 * d2)):
        f.append("two-block closed form 32*0.25*d1 + 32*2*d2 violated")
    # (iii) one-hot x = e_k picks row k of W exactly
    g = np.random.default_rng(5)
    K, N = 64, 6
    qi = g.integers(0, 16, (K, N))
    zi = g.integers(0, 16, (K // 32, N))
    s = g.uniform(0.005, 0.02, (K // 32, N)).astype(np.float32)
    qw, scv, zpk = make_w4(qi, zi, s)
    w = o.dequantize_w4(qw, scv, zpk, K, N)
    for k in (0, 1, 31, 32, 63):
        x = np.zeros((1, K), np.float32)
        x[0, k] = 1.0
        y, _ = o.w4_matmul_ref(x, qw, scv, zpk, K, N)
        if not np.array_equal(y[0], w[k].astype(np.float64)):
            f.append(f"one-hot x at k={k} must return row {k} of W")
            break
        want = np.array([np.float32(float((int(qi[k, n]) - int(zi[k // 32, n])) * Fraction(float(s[k // 32, n]))))
                         for n in range(N)])
        if not np.array_equal(y[0], want.astype(np.float64)):
            f.append(f"one-hot x at k={k} disagrees with (q - zp) * s of row {k}")
            break
    # (iv) q = 0, zp = 15 -> y = -15 * s * sum(x)
    x = (np.arange(32, dtype=np.float32) - 10.0)[None, :] / 4.0
    qw, scv, zpk = make_w4(np.zeros((32, 2)), np.full((1, 2), 15), np.full((1, 2), 0.125))
    y, _ = o.w4_matmul_ref(x, qw, scv, zpk, 32, 2)
    if not np.array_equal(y, np.full((1, 2), -15 * 0.125 * float(x.sum()))):
        f.append("q=0, zp=15 must give -15 * s * sum(x)")
    # every q == zp -> exactly 0
    qw, scv, zpk = make_w4(np.full((64, 4), 6), np.full((2, 4), 6), np.full((2, 4), 0.0173))
    y, _ = o.w4_matmul_ref(g.standard_normal((3, 64)).astype(np.float32), qw, scv, zpk, 64, 4)
    if np.any(y != 0):
        f.append("a weight with every q == zp must give y exactly 0")
    return f


# ---------------------------------------------------------------- brute force

def check_brute_force_dyadic(o):
    """Tiny shapes, dyadic inputs: every fp64 step is exact, so y must equal
    the rational result bit for bit."""
    f = []
    g = np.random.default_rng(2024)
    for (M, K, N) in ((1, 32, 2), (2, 32, 8), (3, 64, 4), (2, 64, 6)):
        qi = g.integers(0, 16, (K, N))
        zi = g.integers(0, 16, (K // 32, N))
        s = 2.0 ** (-g.integers(1, 9, (K // 32, N)).astype(np.float64))
        x = (g.integers(-16, 17, (M, K)) / 8.0).astype(np.float32)
        qw, scv, zpk = make_w4(qi, zi, s)
        y, a = o.w4_matmul_ref(x, qw, scv, zpk, K, N)
        ye, ae = exact_matmul(x, qi, zi, s)
        if not np.array_equal(y, np.array([[float(v) for v in r] for r in ye])):
            f.append(f"dyadic brute force mismatch at M={M} K={K} N={N}")
        if not np.array_equal(a, np.array([[float(v) for v in r] for r in ae])):
            f.append(f"sum|x*w| mismatch at M={M} K={K} N={N}")
    return f


def check_brute_force_general(o):
    """Tiny shapes, general fp32 inputs: the fp64 result must lie within a few
    ulps (K * 2^-52 * sum|x*w|) of the exact rational result."""
    f = []
    g = np.random.default_rng(77)
    for (M, K, N) in ((2, 32, 4), (1, 64, 6), (3, 96, 2)):
        qi = g.integers(0, 16, (K, N))
        zi = g.integers(0, 16, (K // 32, N))
        s = g.uniform(0.005, 0.02, (K // 32, N)).astype(np.float32)
        x = g.standard_normal((M, K)).astype(np.float32)
        qw, scv, zpk = make_w4(qi, zi, s)
        y, _ = o.w4_matmul_ref(x, qw, scv, zpk, K, N)
        ye, ae = exact_matmul(x, qi, zi, s)
        for m in range(M):
            for n in range(N):
                err = abs(Fraction(float(y[m, n])) - ye[m][n])
                if err > Fraction(K) * Fraction(2) ** -52 * ae[m][n] + Fraction(2) ** -1000:
                    f.append(f"general brute force off by {float(err):.3g} at ({m},{n}) K={K}")
                    return f
    return f


# ---------------------------------------------------------------- invariants

def _rand_w4(g, K, N):
    qi = g.integers(0, 16, (K, N))
    zi = g.integers(0, 16, (K // 32, N))
    s = g.uniform(0.005, 0.02, (K // 32, N)).astype(np.float32)
    return qi, zi, s


def check_invariants(o):
    f = []
    g = np.random.default_rng(99)
    K, N, M = 96, 10, 3
    qi, zi, s = _rand_w4(g, K, N)
    qw, scv, zpk = make_w4(qi, zi, s)
    x1 = g.standard_normal((M, K)).astype(np.float32)
    x2 = g.standard_normal((M, K)).astype(np.float32)
    y1, a1 = o.w4_matmul_ref(x1, qw, scv, zpk, K, N)
    y2, a2 = o.w4_matmul_ref(x2, qw, scv, zpk, K, N)
    # linearity: x1 + x2 computed exactly in fp64 by passing the two halves
    y12, _ = o.w4_matmul_ref(np.concatenate([x1, x2]), qw, scv, zpk, K, N)
    if not np.allclose(y12, np.concatenate([y1, y2]), rtol=0, atol=1e-12):
        f.append("stacking rows must stack outputs")
    xs = (2.0 * x1).astype(np.float32)
    ys, _ = o.w4_matmul_ref(xs, qw, scv, zpk, K, N)
    if not np.allclose(ys, 2.0 * y1, rtol=1e-13, atol=1e-12):
        f.append("y(2x) != 2 y(x)")
    # column permutation of (q, zp, s) permutes y
    perm = g.permutation(N)
    qwp, scp, zpp = make_w4(qi[:, perm], zi[:, perm], s[:, perm])
    yp, _ = o.w4_matmul_ref(x1, qwp, scp, zpp, K, N)
    if not np.allclose(yp, y1[:, perm], rtol=1e-13, atol=1e-13):
        f.append("permuting columns of the weight must permute y")
    # K-block additivity: y over 96 rows = y over blocks {0} + y over blocks {1, 2}
    qa, sa, za = make_w4(qi[:32], zi[:1], s[:1])
    qb, sb, zb = make_w4(qi[32:], zi[1:], s[1:])
    ya, _ = o.w4_matmul_ref(np.ascontiguousarray(x1[:, :32]), qa, sa, za, 32, N)
    yb, _ = o.w4_matmul_ref(np.ascontiguousarray(x1[:, 32:]), qb, sb, zb, 64, N)
    if not np.allclose(ya + yb, y1, rtol=1e-13, atol=1e-13):
        f.append("K-block additivity violated")
    # row independence: changing row 1 of x leaves rows 0 and 2 unchanged
    x3 = x1.copy()
    x3[1] = g.standard_normal(K).astype(np.float32)
    y3, _ = o.w4_matmul_ref(x3, qw, scv, zpk, K, N)
    if not (np.array_equal(y3[0], y1[0]) and np.array_equal(y3[2], y1[2])):
        f.append("row m of y must depend on row m of x only")
    if np.any(a1 < np.abs(y1)):
        f.append("sum|x*w| must bound |y|")
    return f


ALL_W4_CHECKS = (
    check_nibble_literals,
    check_pack_roundtrips,
    check_dequant_dyadic_all_pairs,
    check_dequant_single_rounding,
    check_closed_forms,
    check_brute_force_dyadic,
    check_brute_force_general,
    check_invariants,
)


def run_w4_pins(o):
    out = []
    for chk in ALL_W4_CHECKS:
        try:
            out += [f"{chk.__name__}: {m}" for m in chk(o)]
        except Exception as e:  # a crash is a failure too
            out.append(f"{chk.__name__}: raised {type(e).__name__}: {e}")
    return out
