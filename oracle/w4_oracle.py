"""Plain CPU oracle for the 4-bit blocked weight matmul and the int8 tied LM head.

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import, call or link
this module: only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` use it. It shares no code with the CUDA library; the two
meet only through the seeded input generators, which hold none of the method's
arithmetic.

What it follows
---------------
* "ONNX export, quantization and the browser runtime" (tokenling docs),
  section "Quantization (train/quantize.py)":
    - step 1 (``gemm_to_matmul``): every body weight is a plain [K, N]
      constant, K = in-features, N = out-features, so y = x @ W;
    - step 2 (``dq4``): each body weight is stored 4-bit asymmetric, in blocks
      of 32 along K, with an fp32 scale and a uint4 zero point per block (and
      column), as raw packed UINT4 tensors, restored to fp32 by one blocked
      DequantizeLinear:  w = (q - zp) * scale;
    - step 3 (``embedding_int8``): the tied embedding / LM head is int8 with
      one scale per token, in the head's [768, V] layout;
    - step 4 (``last_token_logits``): the head runs on the last position only.
  The same page's output list says "4-bit body, 8-bit embedding, fp32 compute".

Readings where the page is silent (each is listed in the design notes):
* nibble order: element i of a flat row-major tensor sits in byte i >> 1, in
  the low nibble when i is even (the ONNX UINT4 packing, low nibble first);
* zero points use the same packing over their [K/32, N] tensor;
* scales are fp32 [K/32, N] row-major;
* K must be a multiple of 32 and N even; anything else is rejected;
* dequantisation is exact in (q - zp) and then one fp32 multiply rounded to
  nearest-even, which is what DequantizeLinear computes in fp32;
* the head has no zero point (symmetric) and no bias.
* the optional fused epilogue restores the Add that step 1 splits off, then
  applies stock GPT-2's activation (the tanh form of GELU; the erf form is
  offered too) or its residual add: out = act(y + bias) + residual.

Accumulation is fp64. Every function also returns sum_k |x_k * w_kn| so that
callers can apply the tolerance |y - y_ref| <= 1e-5 * sum|x*w| + 1e-6.
"""

from __future__ import annotations

import math

import numpy as np

BLOCK = 32  # K-block length of the 4-bit format (dq4: "blocks of 32 along K")
QUANT_BLOCKS = (32, 64)  # the shipped block, and the group of 64 the page's MLX comparison uses
ABS_TOL = 1e-6
REL_TOL = 1e-5


# --------------------------------------------------------------------------
# nibble packing: "raw packed UINT4 tensors", two per byte, low nibble first
# --------------------------------------------------------------------------

def unpack_nibbles(packed, count: int) -> np.ndarray:
    """Return the first ``count`` uint4 values (as uint8 0..15) of a packed buffer.

    Element i is the low nibble of byte i >> 1 when i is even and the high
    nibble when i is odd.
    """
    b = np.ascontiguousarray(packed, dtype=np.uint8).reshape(-1)
    if count < 0 or count > 2 * b.size:
        raise ValueError(f"cannot unpack {count} nibbles from {b.size} bytes")
    out = np.empty(2 * b.size, dtype=np.uint8)
    out[0::2] = b & 0x0F
    out[1::2] = b >> 4
    return out[:count]


def pack_nibbles(q) -> np.ndarray:
    """Pack uint4 values (0..15) two per byte, low nibble first.

    An odd count leaves the high nibble of the last byte at zero.
    """
    v = np.ascontiguousarray(q).reshape(-1)
    if v.size and (v.min() < 0 or v.max() > 15):
        raise ValueError("uint4 values must lie in 0..15")
    v = v.astype(np.uint8)
    if v.size % 2:
        v = np.concatenate([v, np.zeros(1, np.uint8)])
    return (v[0::2] | (v[1::2] << 4)).astype(np.uint8)


# --------------------------------------------------------------------------
# 4-bit body weights
# --------------------------------------------------------------------------

def _rows(x, K: int) -> np.ndarray:
    """x as fp64 [M, K] rows (a 1-D x of length K is one row)."""
    a = np.asarray(x, dtype=np.float32)
    if a.ndim == 1:
        a = a.reshape(1, -1)
    if a.ndim != 2 or a.shape[1] != K:
        raise ValueError(f"x must be [M, {K}], got {a.shape}")
    return a.astype(np.float64)


def check_w4_shape(K: int, N: int, block: int = BLOCK) -> None:
    if K < 0 or N < 0:
        raise ValueError("negative shape")
    if block not in QUANT_BLOCKS:
        raise ValueError(f"block {block} is not one of {QUANT_BLOCKS}")
    if K % block:
        raise ValueError(f"K={K} is not a multiple of {block}")
    if N % 2:
        raise ValueError(f"N={N} is odd")


def dequantize_w4(qw, scales, zp, K: int, N: int, block: int = BLOCK) -> np.ndarray:
    """Blocked DequantizeLinear of one [K, N] weight: fp32 w = (q - zp) * s.

    ``qw`` holds K*N packed nibbles (flat [K, N] order), ``zp`` holds
    (K/block)*N packed nibbles (flat [K/block, N] order) and ``scales`` is
    [K/block, N], fp32 (or fp16, widened exactly). Row k uses block
    b = k // block; the shipped format has block = 32.
    """
    check_w4_shape(K, N, block)
    nb = K // block
    q = unpack_nibbles(qw, K * N).reshape(K, N).astype(np.int32)
    z = unpack_nibbles(zp, nb * N).reshape(nb, N).astype(np.int32)
    s = np.ascontiguousarray(scales).astype(np.float32).reshape(nb, N)
    blk = np.arange(K) // block
    diff = (q - z[blk, :]).astype(np.float32)  # small integers: exact in fp32
    return diff * s[blk, :]  # one fp32 multiply, round to nearest even


def dequantize_w4_columns(qw, scales, zp, K: int, N: int, cols) -> np.ndarray:
    """Columns ``cols`` of the dequantised [K, N] weight, without the rest.

    Column n of row k is nibble k*N + n; with N even that is byte
    k*(N/2) + n//2, low nibble when n is even.
    """
    check_w4_shape(K, N)
    cols = np.asarray(cols, dtype=np.int64).reshape(-1)
    nb = K // BLOCK
    rows_q = np.ascontiguousarray(qw, dtype=np.uint8).reshape(K, N // 2)
    rows_z = np.ascontiguousarray(zp, dtype=np.uint8).reshape(nb, N // 2)
    s = np.ascontiguousarray(scales, dtype=np.float32).reshape(nb, N)
    byte_q = rows_q[:, cols // 2]
    byte_z = rows_z[:, cols // 2]
    odd = (cols % 2).astype(bool)
    q = np.where(odd[None, :], byte_q >> 4, byte_q & 0x0F).astype(np.int32)
    z = np.where(odd[None, :], byte_z >> 4, byte_z & 0x0F).astype(np.int32)
    blk = np.arange(K) // BLOCK
    diff = (q - z[blk, :]).astype(np.float32)
    return diff * s[blk][:, cols]


def w4_matmul_ref(x, qw, scales, zp, K: int, N: int):
    """y = x @ W for the whole output, fp64 accumulation.

    Returns ``(y, a)`` with y = sum_k x_mk * w_kn and a = sum_k |x_mk * w_kn|,
    both fp64 [M, N]. The inputs are read as fp32 and widened exactly.
    """
    w = dequantize_w4(qw, scales, zp, K, N).astype(np.float64)
    x64 = _rows(x, K)
    return x64 @ w, np.abs(x64) @ np.abs(w)


def w4_matmul_ref_entries(x, qw, scales, zp, K: int, N: int, rows, cols):
    """Sampled outputs y[rows[i], cols[i]] (and a[...]) for shapes too large to
    dequantise whole. Only the named columns are dequantised."""
    rows = np.asarray(rows, dtype=np.int64).reshape(-1)
    cols = np.asarray(cols, dtype=np.int64).reshape(-1)
    ucols, inv = np.unique(cols, return_inverse=True)
    w = dequantize_w4_columns(qw, scales, zp, K, N, ucols).astype(np.float64)
    x64 = _rows(x, K)
    xr = x64[rows]  # [S, K]
    wc = w[:, inv].T  # [S, K]
    return np.einsum("sk,sk->s", xr, wc), np.einsum("sk,sk->s", np.abs(xr), np.abs(wc))


# --------------------------------------------------------------------------
# int8 tied head, last position only
# --------------------------------------------------------------------------

def dequantize_i8_head(table, scales, K: int, V: int, ldt: int | None = None) -> np.ndarray:
    """fp32 w[k, v] = q[k, v] * s[v] for the int8 [K, V] table (row stride ldt)."""
    ldt = V if ldt is None else ldt
    if ldt < V:
        raise ValueError("ldt < V")
    t = np.ascontiguousarray(table, dtype=np.int8).reshape(-1)
    if t.size < K * ldt - (ldt - V):
        raise ValueError("table too small")
    if K == 0 or V == 0:
        return np.zeros((K, V), np.float32)
    rows = np.lib.stride_tricks.as_strided(t, shape=(K, V), strides=(ldt, 1))
    s = np.ascontiguousarray(scales, dtype=np.float32).reshape(V)
    return rows.astype(np.float32) * s[None, :]  # exact int8 -> fp32, one RN multiply


def i8_head_ref(h, table, scales, K: int, V: int, ldt: int | None = None):
    """Logits of the last-position rows h [M, K]: fp64 (logits, sum|h*w|)."""
    w = dequantize_i8_head(table, scales, K, V, ldt).astype(np.float64)
    h64 = _rows(h, K)
    return h64 @ w, np.abs(h64) @ np.abs(w)


def i8_head_argmax_ref(h, table, scales, K: int, V: int, ldt: int | None = None):
    """Greedy decoding on the head: for each row of h, the token with the
    largest logit (the lowest id among equal ones), that logit, and the gap
    to the next-best distinct logit (fp64; inf when V == 1 or all equal)."""
    y, _ = i8_head_ref(h, table, scales, K, V, ldt)
    tok = np.argmax(y, axis=1)  # first maximum: the lowest id on ties
    best = y[np.arange(y.shape[0]), tok]
    gap = np.full(y.shape[0], np.inf)
    for m in range(y.shape[0]):
        rest = y[m][y[m] < best[m]]
        if rest.size:
            gap[m] = best[m] - rest.max()
    return tok.astype(np.int64), best, gap


def i8_embed_ref(table, scales, tokens, K: int, V: int, ldt: int | None = None) -> np.ndarray:
    """Token lookup from the tied int8 table ("ONNX export, quantization and
    the browser runtime", section "Quantization (train/quantize.py)", step 3:
    Gather(axis=1) + Transpose on the [K, V] table, dequantized): row i of the
    result is column tokens[i] of the table times that token's scale, fp32,
    one rounding per element. Shape [len(tokens), K]."""
    ldt = V if ldt is None else ldt
    if ldt < V:
        raise ValueError("ldt < V")
    tok = np.asarray(tokens, dtype=np.int64).reshape(-1)
    if tok.size and (tok.min() < 0 or tok.max() >= V):
        raise ValueError("token id out of range")
    t = np.ascontiguousarray(table, dtype=np.int8).reshape(-1)
    s = np.ascontiguousarray(scales, dtype=np.float32).reshape(V)
    out = np.empty((tok.size, K), np.float32)
    ks = np.arange(K, dtype=np.int64) * ldt
    for i, v in enumerate(tok):
        out[i] = t[ks + v].astype(np.float32) * s[v]  # exact int8 -> fp32, one RN multiply
    return out


def last_position_rows(hidden, T: int, K: int) -> np.ndarray:
    """Rows T-1 of M sequences of hidden states [M, T, K] (last_token_logits)."""
    hs = np.asarray(hidden, dtype=np.float32).reshape(-1, T, K)
    return np.ascontiguousarray(hs[:, T - 1, :])


# --------------------------------------------------------------------------
# fused epilogue: the Add that gemm_to_matmul splits off, and what follows it
# --------------------------------------------------------------------------
# The page's step 1 turns every GPT-2 Conv1D into MatMul + Add (bias). The
# model ("stock GPT-2 small") then applies GELU after the MLP's first weight
# and adds the residual stream after the attention and MLP output weights.
# Reading: GPT-2's activation is the tanh form of GELU ("gelu_new"); the erf
# form (the exact GELU) is offered beside it. Order: act(y + bias) + residual.

SQRT_2_OVER_PI = float(np.sqrt(2.0 / np.pi))
GELU_TANH_CUBIC = 0.044715
GELU_DERIV_MAX = 1.13  # max of d/dv GELU(v) over the reals (both forms): 1.1290 at v ~ 1.41


def gelu_tanh(v) -> np.ndarray:
    """0.5 v (1 + tanh(sqrt(2/pi) (v + 0.044715 v^3))), fp64."""
    v = np.asarray(v, dtype=np.float64)
    return 0.5 * v * (1.0 + np.tanh(SQRT_2_OVER_PI * (v + GELU_TANH_CUBIC * v ** 3)))


def gelu_erf(v) -> np.ndarray:
    """0.5 v (1 + erf(v / sqrt 2)) = v * Phi(v), fp64 (math.erf per element)."""
    v = np.asarray(v, dtype=np.float64)
    erf = np.vectorize(math.erf, otypes=[np.float64])
    return 0.5 * v * (1.0 + erf(v / math.sqrt(2.0)))


ACTIVATIONS = {"none": lambda v: np.asarray(v, dtype=np.float64), "gelu_tanh": gelu_tanh, "gelu_erf": gelu_erf}


def epilogue_ref(y, a, bias=None, residual=None, act: str = "none"):
    """out = act(y + bias) + residual in fp64 for y = x.W (fp64 [M, N]) with
    its sum|x*w| a; returns (out, tol), tol the per-output allowance for an
    fp32 kernel: the body's allowance carried through the activation's slope
    (at most GELU_DERIV_MAX), plus a few fp32 roundings of the bias add, the
    activation and the residual add (1e-6 relative to |pre| and |out|)."""
    y = np.asarray(y, dtype=np.float64)
    pre = y + (0.0 if bias is None else np.asarray(bias, dtype=np.float32).astype(np.float64)[None, :])
    out = ACTIVATIONS[act](pre)
    if residual is not None:
        out = out + np.asarray(residual, dtype=np.float32).astype(np.float64)
    slope = 1.0 if act == "none" else GELU_DERIV_MAX
    tol = slope * tolerance(a) + 1e-6 * (np.abs(pre) + np.abs(out))
    return out, tol


# --------------------------------------------------------------------------
# tolerance
# --------------------------------------------------------------------------

def tolerance(a) -> np.ndarray:
    """Allowed |y - y_ref| per output: 1e-5 * sum|x*w| + 1e-6."""
    return REL_TOL * np.asarray(a, dtype=np.float64) + ABS_TOL


def max_violation(y, y_ref, a) -> float:
    """max(|y - y_ref| - tol) over outputs; <= 0 means every output passes."""
    y = np.asarray(y, dtype=np.float64)
    d = np.abs(y - np.asarray(y_ref, dtype=np.float64)) - tolerance(a)
    if d.size == 0:
        return -np.inf
    if not np.all(np.isfinite(y)):
        return np.inf
    return float(d.max())


# --------------------------------------------------------------------------
# quantisers: the export's dq4 (step 2) and embedding_int8 (step 3), the
# reference of the GPU quantisers and of the oracle's own self-checks
# --------------------------------------------------------------------------

def stored_scale(s64, scale_type: str):
    """The stored form of a scale computed in fp64: fp32 (the shipped format)
    or fp16 (the page's "fp16 scales" variant), one round-to-nearest-even."""
    return np.asarray(s64, dtype=np.float64).astype(np.float16 if scale_type == "fp16" else np.float32)


def quantize_w4(w, block: int = BLOCK, scale_type: str = "fp32") -> tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Asymmetric min/max 4-bit quantiser, per (block of rows, column).

    The page says "asymmetric, blocks of 32 along K" and gives no formula; this
    is the plainest min/max reading, every step in fp64 (the differences of
    fp32 values are exact there, and each division rounds once):
      lo = min(min w, 0), hi = max(max w, 0) over the block (and column);
      s = (hi - lo) / 15, rounded once to the stored type (fp32 or fp16);
      a block whose stored s is 0 (all zeros, or a range below the type's
      smallest value) takes s = 1, zp = 0;
      zp = rint(-lo / s), q = rint(w / s) + zp, both clamped to 0..15, with
      s the stored value and rint rounding half to even.
    Returns packed qw, scales [K/block, N] of the stored type, packed zp.
    """
    if scale_type not in ("fp32", "fp16"):
        raise ValueError(f"scale_type {scale_type!r}")
    w = np.asarray(w, dtype=np.float32)
    K, N = w.shape
    check_w4_shape(K, N, block)
    nb = K // block
    wb = w.astype(np.float64).reshape(nb, block, N)
    lo = np.minimum(wb.min(axis=1), 0.0)
    hi = np.maximum(wb.max(axis=1), 0.0)
    s = stored_scale((hi - lo) / 15.0, scale_type)
    flat = s == 0
    s[flat] = 1.0
    s64 = s.astype(np.float64)
    zp = np.clip(np.rint(-lo / s64), 0, 15)
    zp[flat] = 0
    q = np.clip(np.rint(wb / s64[:, None, :]) + zp[:, None, :], 0, 15)
    q = q.reshape(K, N).astype(np.uint8)
    return pack_nibbles(q), s, pack_nibbles(zp.astype(np.uint8))


def quantize_i8_head(w) -> tuple[np.ndarray, np.ndarray]:
    """Symmetric int8 quantiser, one scale per column (token) of [K, V]
    (the page's embedding_int8: "int8 with one scale per token"), in fp64:
    s = max|w| / 127 rounded once to fp32, q = rint(w / s) clamped to
    -127..127; a column whose s is 0 (all zeros) takes s = 1."""
    w = np.asarray(w, dtype=np.float32)
    amax = np.abs(w.astype(np.float64)).max(axis=0)
    s = (amax / 127.0).astype(np.float32)
    s[s == 0] = 1.0
    q = np.clip(np.rint(w.astype(np.float64) / s.astype(np.float64)[None, :]), -127, 127)
    return q.astype(np.int8), s
