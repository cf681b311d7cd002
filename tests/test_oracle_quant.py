"""The oracle's quantisers (the export's dq4 and embedding_int8 steps, "ONNX
export, quantization and the browser runtime", section "Quantization
(train/quantize.py)", steps 2 and 3) pinned to facts outside themselves (CPU
only):

* weights that lie exactly on a quantisation grid (dyadic scale, integer
  codes spanning 0..15, or -127..127) come back as exactly that grid;
* rounding to the nearest code: every code that is not clamped reconstructs
  its weight within half a (stored) scale, and exact half steps go to the
  even code;
* an all-zero block or column takes scale 1, zero point 0, code 0.

Each check runs against the oracle and against copies with one planted
mistake; every copy must fail a check.
"""

from types import SimpleNamespace

import numpy as np
import pytest

import oracle


def _grid_block(rng, block, N, s, zp_lo=1, zp_hi=14):
    """w [block, N] = (q - zp) * s exactly, with codes 0 and 15 present in
    every column (in the block's second half) and zp in zp_lo..zp_hi."""
    zp = rng.integers(zp_lo, zp_hi + 1, size=N)
    q = rng.integers(0, 16, size=(block, N))
    q[block - 1, :] = 0
    q[block - 2, :] = 15
    return ((q - zp[None, :]) * s).astype(np.float32), q, zp


def check_grid_round_trip(impl):
    bad = []
    rng = np.random.default_rng(1)
    for block in (32, 64):
        for st in ("fp32", "fp16"):
            s = 2.0 ** -7
            blocks = [_grid_block(rng, block, 48, s) for _ in range(3)]
            w = np.concatenate([b[0] for b in blocks])
            qw, sc, zpk = impl.quantize_w4(w, block=block, scale_type=st)
            K, N = w.shape
            q = oracle.unpack_nibbles(qw, K * N).reshape(K, N)
            z = oracle.unpack_nibbles(zpk, (K // block) * N).reshape(K // block, N)
            if not np.array_equal(np.asarray(sc, np.float64), np.full((K // block, N), s)):
                bad.append(f"block {block} {st}: grid scale not recovered")
            if not np.array_equal(q, np.concatenate([b[1] for b in blocks])):
                bad.append(f"block {block} {st}: grid codes not recovered")
            if not np.array_equal(z, np.stack([b[2] for b in blocks])):
                bad.append(f"block {block} {st}: grid zero points not recovered")
            if st == "fp16" and np.asarray(sc).dtype != np.float16:
                bad.append("fp16 variant does not store fp16 scales")
    return bad


def check_nearest_code(impl):
    """Unclamped codes reconstruct within half the stored scale."""
    bad = []
    rng = np.random.default_rng(2)
    for block in (32, 64):
        for st in ("fp32", "fp16"):
            w = (rng.standard_normal((4 * block, 64)) * 0.05).astype(np.float32)
            w[:, 3] = np.abs(w[:, 3])  # an all-positive column: lo = 0
            qw, sc, zpk = impl.quantize_w4(w, block=block, scale_type=st)
            K, N = w.shape
            q = oracle.unpack_nibbles(qw, K * N).reshape(K, N).astype(np.int64)
            z = oracle.unpack_nibbles(zpk, (K // block) * N).reshape(K // block, N).astype(np.int64)
            s = np.asarray(sc, np.float64).reshape(K // block, N)
            blk = np.arange(K) // block
            rec = (q - z[blk]) * s[blk]
            err = np.abs(w.astype(np.float64) - rec)
            inner = (q > 0) & (q < 15)
            if np.any(err[inner] > 0.5 * s[blk][inner] * (1 + 1e-12)):
                bad.append(f"block {block} {st}: an unclamped code is not the nearest")
            if np.any(err > s[blk] * (1 + 1e-12)):
                bad.append(f"block {block} {st}: a code is more than one step off")
    return bad


def check_half_steps_go_even(impl):
    bad = []
    s = 2.0 ** -6
    block = 32
    zp = 7
    q = np.arange(32) % 16
    q[0], q[1] = 0, 15
    steps = (q - zp).astype(np.float64)
    w = np.zeros((block, 2), np.float32)
    w[:, 0] = steps * s
    w[:, 1] = steps * s
    # column 1: move interior weights to half steps (k + 0.5) * s, inside the range
    inner = (q > 0) & (q < 14)
    w[inner, 1] = ((steps[inner] + 0.5) * s).astype(np.float32)
    qw, sc, zpk = impl.quantize_w4(w, block=block)
    got = oracle.unpack_nibbles(qw, block * 2).reshape(block, 2)[:, 1].astype(np.int64)
    want = np.where(inner, np.rint(steps + 0.5) + zp, q)  # np.rint: half to even
    if not np.array_equal(got, want.astype(np.int64)):
        bad.append("half steps do not round to the even code")
    return bad


def check_zero_block_and_column(impl):
    bad = []
    w = np.zeros((64, 4), np.float32)
    w[32:, 2] = 0.5
    qw, sc, zpk = impl.quantize_w4(w, block=32)
    s = np.asarray(sc).reshape(2, 4)
    if not (s[0, 0] == 1.0 and s[1, 0] == 1.0 and s[0, 2] == 1.0):
        bad.append("an all-zero block does not take scale 1")
    if np.any(oracle.unpack_nibbles(zpk, 8).reshape(2, 4)[:, :2] != 0) or \
            np.any(oracle.unpack_nibbles(qw, 256).reshape(64, 4)[:, :2] != 0):
        bad.append("an all-zero block does not take zero point 0 and code 0")
    t, s8 = impl.quantize_i8_head(np.zeros((8, 3), np.float32))
    if not (np.all(t == 0) and np.all(s8 == 1.0)):
        bad.append("an all-zero head column does not take scale 1, code 0")
    return bad


def check_i8_grid_and_nearest(impl):
    bad = []
    rng = np.random.default_rng(3)
    s = 2.0 ** -8
    q = rng.integers(-127, 128, size=(40, 30))
    q[5, :] = np.where(np.arange(30) % 2 == 0, 127, -127)
    t, sc = impl.quantize_i8_head((q * s).astype(np.float32))
    if not (np.array_equal(t.astype(np.int64), q) and np.all(sc == np.float32(s))):
        bad.append("int8 grid not recovered")
    w = (rng.standard_normal((64, 50)) * 0.1).astype(np.float32)
    t, sc = impl.quantize_i8_head(w)
    err = np.abs(w.astype(np.float64) - t.astype(np.float64) * np.asarray(sc, np.float64)[None, :])
    if np.any(err > 0.5 * np.asarray(sc, np.float64)[None, :] * (1 + 1e-12)):
        bad.append("int8 code not the nearest")
    if not np.all(np.abs(t).max(axis=0) == 127):
        bad.append("a column's largest weight does not take code +-127")
    return bad


CHECKS = [check_grid_round_trip, check_nearest_code, check_half_steps_go_even, check_zero_block_and_column,
          check_i8_grid_and_nearest]


@pytest.mark.parametrize("chk", CHECKS, ids=lambda c: c.__name__)
def test_oracle_quantiser_pin(chk):
    assert chk(oracle) == []


# ---------------------------------------------------------------- mutants

def _q4(divisor=15.0, zp_sign=-1.0, add_zp=True, rnd=np.rint, round_scale=True, half_block=False):
    def quantize_w4(w, block=32, scale_type="fp32"):
        w = np.asarray(w, np.float32)
        K, N = w.shape
        nb = K // block
        wb = w.astype(np.float64).reshape(nb, block, N)
        rng_rows = wb[:, : block // 2, :] if half_block else wb
        lo = np.minimum(rng_rows.min(axis=1), 0.0)
        hi = np.maximum(rng_rows.max(axis=1), 0.0)
        s64 = (hi - lo) / divisor
        s = oracle.stored_scale(s64, scale_type)
        flat = s == 0
        s[flat] = 1.0
        sd = s.astype(np.float64) if round_scale else np.where(flat, 1.0, s64)
        zp = np.clip(rnd(zp_sign * lo / sd), 0, 15)
        zp[flat] = 0
        q = np.clip(rnd(wb / sd[:, None, :]) + (zp[:, None, :] if add_zp else 0), 0, 15)
        return oracle.pack_nibbles(q.reshape(K, N).astype(np.uint8)), s, oracle.pack_nibbles(zp.astype(np.uint8))
    return quantize_w4


def _i8(divisor=127.0, rnd=np.rint):
    def quantize_i8_head(w):
        w = np.asarray(w, np.float32)
        amax = np.abs(w.astype(np.float64)).max(axis=0)
        s = (amax / divisor).astype(np.float32)
        s[s == 0] = 1.0
        return np.clip(rnd(w.astype(np.float64) / s.astype(np.float64)), -127, 127).astype(np.int8), s
    return quantize_i8_head


def _half_away(x):
    return np.sign(x) * np.floor(np.abs(x) + 0.5)


MUTANTS = {
    "divide by 16": dict(quantize_w4=_q4(divisor=16.0)),
    "zero point sign": dict(quantize_w4=_q4(zp_sign=1.0)),
    "code without the zero point": dict(quantize_w4=_q4(add_zp=False)),
    "half away from zero": dict(quantize_w4=_q4(rnd=_half_away)),
    "codes from the unrounded scale": dict(quantize_w4=_q4(round_scale=False)),
    "range of half the block": dict(quantize_w4=_q4(half_block=True)),
    "int8 over 128": dict(quantize_i8_head=_i8(divisor=128.0)),
    "int8 truncation": dict(quantize_i8_head=_i8(rnd=np.trunc)),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_each_planted_mistake_fails_a_pin(name):
    impl = SimpleNamespace(quantize_w4=oracle.quantize_w4, quantize_i8_head=oracle.quantize_i8_head)
    for k, v in MUTANTS[name].items():
        setattr(impl, k, v)
    failures = [m for chk in CHECKS for m in chk(impl)]
    assert failures, f"no pin sees: {name}"
