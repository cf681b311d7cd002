"""Seeded synthetic inputs for the W4 matmul and the int8 head.

This module holds shapes and value distributions only; it performs none of
the method's arithmetic (no packing, no dequantisation, no matmul). Both the
CUDA path's tests/bench and the CPU oracle's tests draw their inputs here.

Distributions (the workloads of the quantised-weight decode step):
* body weight [K, N]: every uint4 weight q and every zero point is uniform in
  0..15 and independent, so the packed byte buffers are uniform random bytes;
  fp32 scales are uniform in [0.005, 0.02], one per (32-row block, column);
* activations: fp32 N(0, 1);
* head table [K, V] (row stride ldt >= V): int8 uniform in -127..127, one fp32
  scale per token column uniform in [0.002, 0.01].

Every draw comes from numpy's PCG64 keyed by a SeedSequence over
(base seed, tag, *indices), so any single tensor can be regenerated alone.
"""

from __future__ import annotations

import numpy as np

BASE_SEED = 20261202
BLOCK = 32

# GPT-2 small: 12 layers; Conv1D weights as plain [in, out] matrices.
GPT2_LAYERS = 12
GPT2_HIDDEN = 768
GPT2_VOCAB = 50257
GPT2_LAYER_SHAPES = (  # (name, K, N)
    ("c_attn", 768, 2304),
    ("attn_c_proj", 768, 768),
    ("c_fc", 768, 3072),
    ("mlp_c_proj", 3072, 768),
)
GPT2_PROMPT = 58  # prefill rows

# 3.8B dense (hidden 3072, 32 layers)
DENSE38_LAYERS = 32
DENSE38_LAYER_SHAPES = (
    ("qkv", 3072, 9216),
    ("o_proj", 3072, 3072),
    ("gate_up", 3072, 16384),
    ("down", 8192, 3072),
)

_TAGS = {"w4": 1, "x": 2, "table": 3, "head_scales": 4, "h": 5, "misc": 6, "bias": 7}


def generator(tag: str, *idx: int, seed: int = BASE_SEED) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, _TAGS[tag], *map(int, idx)])))


def w4_weight(K: int, N: int, *idx: int, seed: int = BASE_SEED,
              scale_lo: float = 0.005, scale_hi: float = 0.02) -> dict:
    """Packed 4-bit weight buffers for a [K, N] matrix (K % 32 == 0, N even)."""
    g = generator("w4", K, N, *idx, seed=seed)
    nb = K // BLOCK
    qw = g.integers(0, 256, size=K * N // 2, dtype=np.uint8)
    zp = g.integers(0, 256, size=nb * N // 2, dtype=np.uint8)
    scales = g.uniform(scale_lo, scale_hi, size=nb * N).astype(np.float32)
    return {"qw": qw, "scales": scales, "zp": zp, "K": K, "N": N}


def activations(M: int, K: int, *idx: int, seed: int = BASE_SEED, ld: int | None = None) -> np.ndarray:
    """fp32 N(0,1) rows [M, K]; with ld > K the rows are padded (pad = NaN, never read)."""
    g = generator("x", M, K, *idx, seed=seed)
    x = g.standard_normal(size=(M, K)).astype(np.float32)
    if ld is None or ld == K:
        return x
    out = np.full((M, ld), np.nan, dtype=np.float32)
    out[:, :K] = x
    return out


def bias(N: int, *idx: int, seed: int = BASE_SEED, std: float = 0.5) -> np.ndarray:
    """fp32 N(0, std^2) vector [N] (a bias of the fused epilogue)."""
    g = generator("bias", N, *idx, seed=seed)
    return (std * g.standard_normal(size=N)).astype(np.float32)


def i8_head(K: int, V: int, *idx: int, seed: int = BASE_SEED, ldt: int | None = None) -> dict:
    """int8 [K, V] head table (row stride ldt) and its fp32 per-column scales."""
    ldt = V if ldt is None else ldt
    g = generator("table", K, V, ldt, *idx, seed=seed)
    table = g.integers(-127, 128, size=K * ldt, dtype=np.int16).astype(np.int8)
    gs = generator("head_scales", V, *idx, seed=seed)
    scales = gs.uniform(0.002, 0.01, size=V).astype(np.float32)
    return {"table": table, "scales": scales, "K": K, "V": V, "ldt": ldt}


def gpt2_stack_shapes() -> list[tuple[str, int, int]]:
    """The 48 body weights of GPT-2 small in layer order."""
    return [(f"h{l}.{name}", K, N) for l in range(GPT2_LAYERS) for name, K, N in GPT2_LAYER_SHAPES]


def dense38_stack_shapes() -> list[tuple[str, int, int]]:
    """The 128 body weights of the 3.8B-dense stack in layer order."""
    return [(f"l{l}.{name}", K, N) for l in range(DENSE38_LAYERS) for name, K, N in DENSE38_LAYER_SHAPES]


def w4_bytes(K: int, N: int) -> int:
    """Bytes of one packed weight: nibbles + fp32 scales + packed zero points."""
    nb = K // BLOCK
    return K * N // 2 + nb * N * 4 + nb * N // 2


def i8_head_bytes(K: int, V: int) -> int:
    return K * V + V * 4
