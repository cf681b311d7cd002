"""GPU parity of the decoder-stack workloads: the 48 GPT-2 weights in one
grouped launch (decode M=1 and prefill M=58 followed by the head on the last
row), and one layer of the 3.8B-dense stack at full size (sampled outputs),
as decode (M = 1, 8, 32) and as prefill (M = 2048)."""

import numpy as np
import pytest

import oracle
from gpu_util import check, dev, torch, upload_w4

from int8_weight_quantized_w4_b200 import synth

pytestmark = pytest.mark.gpu


def w4():
    import int8_weight_quantized_w4_b200 as w
    return w


def _stack(shapes, M, seed=synth.BASE_SEED):
    host, items = [], []
    T = torch()
    for i, (name, K, N) in enumerate(shapes):
        W = synth.w4_weight(K, N, i, seed=seed)
        x = synth.activations(M, K, i, seed=seed)
        Wd = upload_w4(W)
        y = T.empty((M, N), dtype=T.float32, device="cuda")
        items.append({"x": dev(x), "qw": Wd["qw"], "scales": Wd["scales"], "zp": Wd["zp"], "y": y, "K": K, "N": N})
        host.append((name, W, x))
    return host, items


def test_config1_gpt2_decode_stack_grouped():
    host, items = _stack(synth.gpt2_stack_shapes(), 1)
    w4().w4_matmul_grouped(items)
    torch().cuda.synchronize()
    for (name, W, x), it in zip(host, items):
        y_ref, a = oracle.w4_matmul_ref(x, W["qw"], W["scales"], W["zp"], W["K"], W["N"])
        check(it["y"], y_ref, a, name)


def test_config1_grouped_is_deterministic_and_matches_single_calls():
    host, items = _stack(synth.gpt2_stack_shapes()[:8], 1, seed=5)
    w4().w4_matmul_grouped(items)
    first = [it["y"].clone() for it in items]
    w4().w4_matmul_grouped(items)
    for a, it in zip(first, items):
        assert torch().equal(a, it["y"])
    for (name, W, x), it in zip(host, items):
        single = w4().w4_matmul(it["x"], it["qw"], it["scales"], it["zp"], it["K"], it["N"])
        y_ref, a = oracle.w4_matmul_ref(x, W["qw"], W["scales"], W["zp"], W["K"], W["N"])
        check(single, y_ref, a, name + " single")
        check(it["y"], y_ref, a, name + " grouped")


def test_config3_gpt2_prefill_then_head_on_last_row():
    M = synth.GPT2_PROMPT
    host, items = _stack(synth.gpt2_stack_shapes(), M)
    w4().w4_matmul_grouped(items)
    H = synth.i8_head(768, synth.GPT2_VOCAB)
    hidden = items[-1]["y"]  # layer 12 mlp c_proj output [58, 768]
    last = hidden[M - 1:M]   # the last position, by pointer offset
    logits = w4().i8_head_logits(last, dev(H["table"]), dev(H["scales"]), 768, synth.GPT2_VOCAB)
    torch().cuda.synchronize()
    refs = []
    for (name, W, x), it in zip(host, items):
        y_ref, a = oracle.w4_matmul_ref(x, W["qw"], W["scales"], W["zp"], W["K"], W["N"])
        check(it["y"], y_ref, a, name)
        refs.append((y_ref, a))
    # chained head: the oracle runs on its own last row; the allowed error adds
    # the body's per-output bound carried through |w| to the head's own bound.
    y_ref, a_body = refs[-1]
    h_ref = y_ref[M - 1].astype(np.float32)[None, :]
    wdq = oracle.dequantize_i8_head(H["table"], H["scales"], 768, synth.GPT2_VOCAB).astype(np.float64)
    l_ref, a_head = oracle.i8_head_ref(h_ref, H["table"], H["scales"], 768, synth.GPT2_VOCAB)
    carried = oracle.tolerance(a_body[M - 1])[None, :] @ np.abs(wdq)
    h_round = np.abs(y_ref[M - 1] - h_ref[0].astype(np.float64))[None, :] @ np.abs(wdq)
    err = np.abs(logits.cpu().numpy().astype(np.float64) - l_ref)
    allowed = oracle.tolerance(a_head) + carried + h_round
    assert np.all(err <= allowed), float((err - allowed).max())


def test_config3_head_on_seeded_last_row():
    """The head step of config 3 alone: seeded [58, 768] hidden rows, last row
    by pointer offset, against the oracle on the same input."""
    M, K, V = synth.GPT2_PROMPT, 768, synth.GPT2_VOCAB
    hidden = synth.activations(M, K, 123)
    H = synth.i8_head(K, V)
    logits = w4().i8_head_logits(dev(hidden)[M - 1:M], dev(H["table"]), dev(H["scales"]), K, V)
    torch().cuda.synchronize()
    ref, a = oracle.i8_head_ref(hidden[M - 1:M], H["table"], H["scales"], K, V)
    check(logits, ref, a, "config 3 head")


def _sample_idx(g, M, N, K, n=4096):
    rows = g.integers(0, M, n)
    cols = g.integers(0, N, n)
    rows[:4] = [0, M - 1, 0, M - 1]
    cols[:4] = [0, N - 1, N - 1, 0]
    return rows, cols


@pytest.mark.parametrize("M", [1, 8, 32, 2048])  # decode sizes, and the prefill size (tensor cores)
def test_config4_dense38_one_layer_full_size_sampled(M):
    shapes = synth.dense38_stack_shapes()[:4]
    host, items = _stack(shapes, M, seed=31)
    w4().w4_matmul_grouped(items)
    torch().cuda.synchronize()
    g = np.random.default_rng(M)
    for (name, W, x), it in zip(host, items):
        rows, cols = _sample_idx(g, M, W["N"], W["K"])
        ys, a = oracle.w4_matmul_ref_entries(x, W["qw"], W["scales"], W["zp"], W["K"], W["N"], rows, cols)
        yg = it["y"].cpu().numpy()[rows, cols]
        check(yg, ys, a, f"{name} M={M}")


def test_config4_single_calls_full_size_sampled():
    shapes = synth.dense38_stack_shapes()[:4]
    host, items = _stack(shapes, 1, seed=32)
    g = np.random.default_rng(0)
    for (name, W, x), it in zip(host, items):
        y = w4().w4_matmul(it["x"], it["qw"], it["scales"], it["zp"], it["K"], it["N"])
        rows, cols = _sample_idx(g, 1, W["N"], W["K"])
        ys, a = oracle.w4_matmul_ref_entries(x, W["qw"], W["scales"], W["zp"], W["K"], W["N"], rows, cols)
        check(y.cpu().numpy()[rows, cols], ys, a, name)
