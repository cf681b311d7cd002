"""GPU parity of i8_head_logits (fast and plain kernels) against the oracle."""

import numpy as np
import pytest

import oracle
from gpu_util import check, dev, guarded, guards_intact, torch

from int8_weight_quantized_w4_b200 import synth

pytestmark = pytest.mark.gpu


def w4():
    import int8_weight_quantized_w4_b200 as w
    return w


def run_head(M, K, V, ldt=None, path="auto", seed=2, ldh=None):
    H = synth.i8_head(K, V, seed=seed, ldt=ldt)
    h = synth.activations(M, K, 3, seed=seed, ld=ldh)
    hd = dev(h)[:, :K]
    logits, buf = guarded(M, V)
    w4().i8_head_logits(hd, dev(H["table"]), dev(H["scales"]), K, V, ldt=H["ldt"], logits=logits, path=path)
    torch().cuda.synchronize()
    ref, a = oracle.i8_head_ref(h[:, :K], H["table"], H["scales"], K, V, H["ldt"])
    check(logits, ref, a, f"head M={M} K={K} V={V} ldt={H['ldt']} path={path}")
    assert guards_intact(buf, M, V, V)


@pytest.mark.parametrize("M", [1, 8])
@pytest.mark.parametrize("path", ["auto", "generic"])
def test_config2_gpt2_head(M, path):
    run_head(M, 768, 50257, path=path)


@pytest.mark.parametrize("M,K,V,ldt", [
    (1, 16, 20, 20), (1, 32, 500, 511), (2, 48, 1000, 1003), (3, 100, 777, 777), (5, 64, 2000, 2001),
    (4, 272, 300, 301), (1, 17, 33, 35), (2, 768, 4099, 4100), (6, 40, 1500, 1500), (8, 1, 64, 64),
    (11, 96, 999, 1001), (1, 2048, 31, 31),
])
@pytest.mark.parametrize("path", ["auto", "generic"])
def test_head_shapes(M, K, V, ldt, path):
    run_head(M, K, V, ldt, path, seed=K + V)


def test_head_closed_form_exact():
    K, V = 64, 3000
    table = np.ones(K * V, np.int8)
    s = np.full(V, 0.5, np.float32)
    h = ((np.arange(K, dtype=np.float32) - 20) / 8)[None, :]
    out = w4().i8_head_logits(dev(h), dev(table), dev(s), K, V)
    assert np.array_equal(out.cpu().numpy().astype(np.float64), np.full((1, V), 0.5 * float(h.sum())))


def test_head_extreme_codes():
    """-128 and 127 in every position, dyadic scales: exact."""
    K, V = 32, 257
    table = np.where(np.arange(K * V) % 2 == 0, -128, 127).astype(np.int8)
    s = np.full(V, 0.25, np.float32)
    h = np.ones((2, K), np.float32)
    out = w4().i8_head_logits(dev(h), dev(table), dev(s), K, V).cpu().numpy().astype(np.float64)
    ref, _ = oracle.i8_head_ref(h, table, s, K, V)
    assert np.array_equal(out, ref)


def test_last_position_rows_by_stride():
    """The head applied to row T-1 of [M, T, K] hidden states through a row stride."""
    T_, K, V, M = 5, 64, 700, 3
    hidden = synth.activations(M * T_, K, 9).reshape(M, T_, K)
    H = synth.i8_head(K, V, seed=11)
    hd = dev(hidden)
    last = hd[:, T_ - 1, :]  # stride T*K between rows
    out = w4().i8_head_logits(last, dev(H["table"]), dev(H["scales"]), K, V)
    torch().cuda.synchronize()
    ref, a = oracle.i8_head_ref(oracle.last_position_rows(hidden, T_, K), H["table"], H["scales"], K, V)
    check(out, ref, a, "last position")


def test_head_deterministic():
    K, V = 768, 50257
    H = synth.i8_head(K, V)
    h = dev(synth.activations(8, K))
    t, s = dev(H["table"]), dev(H["scales"])
    a = w4().i8_head_logits(h, t, s, K, V).clone()
    b = w4().i8_head_logits(h, t, s, K, V).clone()
    assert torch().equal(a, b)
