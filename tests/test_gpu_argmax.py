"""GPU greedy decoding on the head (i8_head_argmax): the argmax of exactly
the logits i8_head_logits computes, ties to the lowest token id, and the
oracle's token wherever its top two logits are further apart than the
tolerance allows the GPU to move them."""

import numpy as np
import pytest

import oracle
from gpu_util import dev, torch

from int8_weight_quantized_w4_b200 import synth

pytestmark = pytest.mark.gpu


def w4():
    import int8_weight_quantized_w4_b200 as w
    return w


def run(M, K, V, ldt=None, seed=31):
    H = synth.i8_head(K, V, seed=seed, ldt=ldt)
    h = synth.activations(M, K, 5, seed=seed)
    hd, T, S = dev(h), dev(H["table"]), dev(H["scales"])
    tok, best = w4().i8_head_argmax(hd, T, S, K, V, ldt=H["ldt"])
    logits = w4().i8_head_logits(hd, T, S, K, V, ldt=H["ldt"])
    torch().cuda.synchronize()
    tok, best, lg = tok.cpu().numpy(), best.cpu().numpy(), logits.cpu().numpy()
    # the same logits the head writes: exact argmax (first maximum) and value
    assert np.array_equal(tok, np.argmax(lg, axis=1)), (M, K, V)
    assert np.array_equal(best, lg[np.arange(M), tok])
    # against the oracle where its decision is robust to fp32 rounding
    otok, obest, gap = oracle.i8_head_argmax_ref(h, H["table"], H["scales"], K, V, H["ldt"])
    _, a = oracle.i8_head_ref(h, H["table"], H["scales"], K, V, H["ldt"])
    tol = oracle.tolerance(a)
    for m in range(M):
        if gap[m] > 2 * tol[m].max():
            assert tok[m] == otok[m], (m, tok[m], otok[m])


@pytest.mark.parametrize("M", [1, 2])
def test_argmax_gpt2_head(M):
    run(M, 768, 50257)


@pytest.mark.parametrize("M,K,V,ldt", [(3, 768, 50257, None), (8, 256, 3001, 3005), (1, 20000, 300, None),
                                       (2, 64, 1, None)])
def test_argmax_other_paths(M, K, V, ldt):
    # M >= 3 and h too long for the fused kernel: logits through the workspace
    run(M, K, V, ldt)


def test_argmax_ties_go_to_the_lowest_token():
    K, V = 32, 1000
    g = np.random.default_rng(5)
    table = g.integers(-20, 20, (K, V)).astype(np.int8)
    table[:, 700] = 100
    table[:, 123] = 100
    s = np.full(V, 0.5, np.float32)
    h = np.ones((1, K), np.float32)
    tok, best = w4().i8_head_argmax(dev(h), dev(table), dev(s), K, V)
    torch().cuda.synchronize()
    assert int(tok.item()) == 123 and float(best.item()) == 0.5 * 100 * K


def test_argmax_signed_zero_tie_goes_to_the_lowest_token():
    """-0 and +0 are equal logits: the lower token id wins even when its
    logit is the negative zero (a zero column under a negative scale)."""
    K, V = 32, 1000
    table = np.full((K, V), -20, np.int8)
    table[:, 123] = 0
    table[:, 700] = 0
    s = np.full(V, 0.5, np.float32)
    s[123] = -0.5  # 0 * -0.5 = -0
    h = np.ones((1, K), np.float32)
    for M in (1, 3):  # the fused rows kernel and the workspace path
        hm = np.repeat(h, M, axis=0)
        tok, best = w4().i8_head_argmax(dev(hm), dev(table), dev(s), K, V)
        torch().cuda.synchronize()
        assert list(tok.cpu().numpy()) == [123] * M and np.all(best.cpu().numpy() == 0.0)


def test_argmax_leaves_the_counter_block_zero():
    """Calls share one workspace; its first 4 KB (the split-K counters of
    every kernel) must be zero after each of them."""
    w = w4()
    for case in [(3, 128, 2000), (1, 768, 4096), (8, 256, 3001), (1, 768, 4096)]:
        run(*case)  # logits through the workspace, then the fused path
        ws = w.workspace(int(w.lib().i8_head_argmax_workspace_size(*case)), "cuda")
        torch().cuda.synchronize()
        assert int(ws[:4096].count_nonzero()) == 0, case
