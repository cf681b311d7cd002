"""GPU: the decode step in one launch (w4r_decode_step): the body's matmuls on
repacked weights and the int8 head on its streaming layout, streamed by the
same persistent CTAs, against the oracle.

* Every output matches the oracle within |y - y_ref| <= 1e-5 * sum|x*w| +
  1e-6, and is bit-identical to the two separate calls (w4r_matmul_grouped,
  then i8r_head_logits): the same atoms sum in the same order.
* Ragged shapes (N not a multiple of a group's columns, V not a multiple of
  8), K = 0 descriptors, the fused epilogue, a head alone, and a step that one
  launch cannot hold (its head's K above 2048) all give the same results.
* The head's h may not be one of the body's outputs in the same step."""

import numpy as np
import pytest

import oracle
from gpu_util import check, dev, torch

from int8_weight_quantized_w4_b200 import synth

pytestmark = pytest.mark.gpu


def w4():
    import int8_weight_quantized_w4_b200 as w
    return w


def _body(shapes, tag0=0, epi=None):
    """Items (repacked weights, x, NaN-filled y) and the host copies."""
    T = torch()
    host, items = [], []
    for i, (K, N) in enumerate(shapes):
        if K > 0:
            W = synth.w4_weight(K, N, tag0 + i)
            x = synth.activations(1, K, tag0 + i)
            wr = w4().w4_repack(dev(W["qw"]), dev(W["scales"]), dev(W["zp"]), K, N)
        else:  # K = 0: y is the epilogue of 0, no weight is read
            W, x = {"K": 0, "N": N}, None
            wr = T.zeros(16, dtype=T.uint8, device="cuda")
        it = {"x": dev(x) if K > 0 else T.zeros((1, 4), device="cuda"), "wr": wr,
              "y": T.full((1, N), float("nan"), device="cuda"), "K": K, "N": N}
        if epi is not None and i in epi:
            for k, v in epi[i].items():
                it[k] = dev(v) if isinstance(v, np.ndarray) else v
        items.append(it)
        host.append((W, x))
    return host, items


def _head(K, V, tag):
    H = synth.i8_head(K, V, tag)
    tr = w4().i8_head_repack(dev(H["table"]), dev(H["scales"]), K, V, ldt=H["ldt"])
    return H, tr


def _step_and_separate(items, h, tr, K, V):
    """Logits and outputs of the fused step, then of the separate calls."""
    T = torch()
    lg = w4().w4r_decode_step(items, h, tr, K, V)
    T.cuda.synchronize()
    fused = [it["y"].clone() for it in items]
    for it in items:
        it["y"].fill_(float("nan"))
    if items:
        w4().w4r_matmul_grouped(items)
    lg2 = w4().i8r_head_logits(h, tr, K, V)
    T.cuda.synchronize()
    return lg, fused, lg2, [it["y"].clone() for it in items]


def _check_all(host, items, fused, H, h_host, lg, K, V, what):
    for i, ((W, x), y) in enumerate(zip(host, fused)):
        if W["K"] == 0:
            continue
        y_ref, a = oracle.w4_matmul_ref(x, W["qw"], W["scales"], W["zp"], W["K"], W["N"])
        check(y, y_ref, a, f"{what}: body {i} K={W['K']} N={W['N']}")
    ref, a = oracle.i8_head_ref(h_host, H["table"], H["scales"], K, V, H["ldt"])
    check(lg, ref, a, f"{what}: head K={K} V={V}")


def test_gpt2_decode_step_in_one_launch():
    T = torch()
    shapes = [(K, N) for _, K, N in synth.gpt2_stack_shapes()]
    host, items = _body(shapes)
    K, V = 768, 50257
    H, tr = _head(K, V, 1)
    h_host = synth.activations(1, K, 999)
    h = dev(h_host)
    lg, fused, lg2, sep = _step_and_separate(items, h, tr, K, V)
    _check_all(host, items, fused, H, h_host, lg, K, V, "GPT-2 step")
    assert T.equal(lg, lg2), "fused head differs from the separate head"
    for i, (a, b) in enumerate(zip(fused, sep)):
        assert T.equal(a, b), f"fused body output {i} differs from the separate call"
    again = w4().w4r_decode_step(items, h, tr, K, V)
    T.cuda.synchronize()
    assert T.equal(again, lg), "not run-to-run deterministic"


@pytest.mark.parametrize("K,V", [(64, 1000), (48, 7), (256, 20001), (2048, 300)])
def test_ragged_shapes_match_the_oracle_and_the_separate_calls(K, V):
    T = torch()
    shapes = [(64, 200), (96, 40), (32, 8), (1536, 264), (768, 2304)]
    host, items = _body(shapes, tag0=K)
    H, tr = _head(K, V, K + V)
    h_host = synth.activations(1, K, 7)
    h = dev(h_host)
    lg, fused, lg2, sep = _step_and_separate(items, h, tr, K, V)
    _check_all(host, items, fused, H, h_host, lg, K, V, f"step K={K} V={V}")
    assert T.equal(lg, lg2)
    for a, b in zip(fused, sep):
        assert T.equal(a, b)


def test_head_alone_and_zero_k_descriptor():
    T = torch()
    K, V = 128, 999
    H, tr = _head(K, V, 3)
    h_host = synth.activations(1, K, 3)
    h = dev(h_host)
    lg = w4().w4r_decode_step([], h, tr, K, V)
    T.cuda.synchronize()
    assert T.equal(lg, w4().i8r_head_logits(h, tr, K, V))
    b = synth.bias(64, 5)
    host, items = _body([(0, 64), (64, 64)], tag0=50, epi={0: {"bias": b, "act": "gelu_tanh"}})
    lg = w4().w4r_decode_step(items, h, tr, K, V)
    T.cuda.synchronize()
    want, tol = oracle.epilogue_ref(np.zeros((1, 64)), np.zeros((1, 64)), bias=b, act="gelu_tanh")
    assert np.all(np.abs(items[0]["y"].cpu().numpy() - want) <= tol)
    _check_all(host[1:], items[1:], [items[1]["y"]], H, h_host, lg, K, V, "K=0 step")


@pytest.mark.parametrize("act", ["none", "gelu_tanh", "gelu_erf"])
def test_fused_epilogue_in_the_step(act):
    N = 3072
    b = synth.bias(N, 3)
    r = synth.activations(1, N, 77)
    host, items = _body([(768, N), (3072, 768)], tag0=60, epi={0: {"bias": b, "residual": r, "act": act}})
    K, V = 768, 5000
    H, tr = _head(K, V, 8)
    h_host = synth.activations(1, K, 8)
    lg = w4().w4r_decode_step(items, dev(h_host), tr, K, V)
    torch().cuda.synchronize()
    W, x = host[0]
    y_ref, a = oracle.w4_matmul_ref(x, W["qw"], W["scales"], W["zp"], 768, N)
    out, tol = oracle.epilogue_ref(y_ref, a, bias=b, residual=r, act=act)
    assert np.all(np.abs(items[0]["y"].cpu().numpy() - out) <= tol)
    _check_all(host[1:], items[1:], [items[1]["y"]], H, h_host, lg, K, V, f"epilogue {act}")


def test_step_that_one_launch_cannot_hold():
    """A head with K above what the fused launch stages runs as the body's
    launches followed by the head's: same results."""
    T = torch()
    host, items = _body([(768, 768), (64, 128)], tag0=70)
    K, V = 4096, 777
    H, tr = _head(K, V, 9)
    h_host = synth.activations(1, K, 9)
    h = dev(h_host)
    lg, fused, lg2, sep = _step_and_separate(items, h, tr, K, V)
    _check_all(host, items, fused, H, h_host, lg, K, V, "two-launch step")
    assert T.equal(lg, lg2)


def test_chained_steps_keep_stream_order():
    """Each step's x is the previous step's output: a step that starts
    streaming early still reads the finished input."""
    T = torch()
    K = N = 768
    Ws = [synth.w4_weight(K, N, 80 + i) for i in range(4)]
    wrs = [w4().w4_repack(dev(W["qw"]), dev(W["scales"]), dev(W["zp"]), K, N) for W in Ws]
    H, tr = _head(K, 3000, 10)
    h_host = synth.activations(1, K, 10)
    h = dev(h_host)
    x0 = dev(synth.activations(1, K, 80))
    ys = [T.full((1, N), float("nan"), device="cuda") for _ in Ws]
    T.cuda.synchronize()
    cur = x0
    for wr, y in zip(wrs, ys):
        w4().w4r_decode_step([{"x": cur, "wr": wr, "y": y, "K": K, "N": N}], h, tr, K, 3000)
        cur = y
    T.cuda.synchronize()
    prev = x0.cpu().numpy()
    for i, W in enumerate(Ws):
        y_ref, a = oracle.w4_matmul_ref(prev, W["qw"], W["scales"], W["zp"], K, N)
        check(ys[i], y_ref, a, f"chained step {i}")
        prev = ys[i].cpu().numpy()


def test_refusals():
    T = torch()
    host, items = _body([(64, 64)], tag0=90)
    K, V = 64, 100
    H, tr = _head(K, V, 11)
    with pytest.raises(w4().W4Error):  # h is the body's output
        w4().w4r_decode_step(items, items[0]["y"], tr, K, V)
    with pytest.raises(w4().W4Error):  # h not 16-byte aligned
        hb = T.zeros(K + 4, device="cuda")[1:K + 1]
        w4().w4r_decode_step(items, hb, tr, K, V)
    with pytest.raises(w4().W4Error):  # K of the head not a multiple of 16
        w4().w4r_decode_step(items, T.zeros(72, device="cuda"), tr, 72, V)
    bad = dict(items[0])
    bad["x"] = dev(synth.activations(2, 64, 1))
    with pytest.raises(w4().W4Error):  # M = 2 in the body
        w4().w4r_decode_step([bad], dev(synth.activations(1, K, 1)), tr, K, V)


@pytest.mark.parametrize("K,V,tag", [(768, 50257, 1), (64, 1000, 2), (4096, 777, 3)])
def test_greedy_step_is_the_argmax_of_the_step_logits(K, V, tag):
    """The greedy step returns the token and logit of exactly the fused
    step's logits (ties to the lowest id), and the body outputs of the
    logits step; K = 4096 takes the two-launch form."""
    T = torch()
    shapes = [(K2, N) for _, K2, N in synth.gpt2_stack_shapes()][:6]
    host, items = _body(shapes, tag0=100 + tag)
    H, tr = _head(K, V, tag)
    h_host = synth.activations(1, K, 200 + tag)
    h = dev(h_host)
    lg = w4().w4r_decode_step(items, h, tr, K, V)
    T.cuda.synchronize()
    ys = [it["y"].clone() for it in items]
    for it in items:
        it["y"].fill_(float("nan"))
    tok, best = w4().w4r_decode_step_argmax(items, h, tr, K, V)
    T.cuda.synchronize()
    l = lg.cpu().numpy()[0]
    assert int(tok.item()) == int(np.argmax(l)) and float(best.item()) == float(l.max())
    for a, it in zip(ys, items):
        assert T.equal(a, it["y"])
    ref, a = oracle.i8_head_ref(h_host, H["table"], H["scales"], K, V, H["ldt"])
    rtok, _, _ = oracle.i8_head_argmax_ref(h_host, H["table"], H["scales"], K, V, H["ldt"])
    g = int(tok.item())
    assert g == int(rtok[0]) or ref[0, g] >= ref[0, int(rtok[0])] - 2 * oracle.tolerance(a)[0, int(rtok[0])]


def test_greedy_step_ties_and_signed_zero():
    K, V = 32, 1000
    table = np.full((K, V), -20, np.int8)
    table[:, 123] = 0
    table[:, 700] = 0
    s = np.full(V, 0.5, np.float32)
    s[123] = -0.5  # 0 * -0.5 = -0, equal to the +0 of column 700
    tr = w4().i8_head_repack(dev(table), dev(s), K, V)
    host, items = _body([(64, 64)], tag0=120)
    tok, best = w4().w4r_decode_step_argmax(items, dev(np.ones((1, K), np.float32)), tr, K, V)
    torch().cuda.synchronize()
    assert int(tok.item()) == 123 and float(best.item()) == 0.0
