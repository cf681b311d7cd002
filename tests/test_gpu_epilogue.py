"""GPU parity of the fused epilogue y = act(x.W + bias) + residual on every
kernel path, against the oracle (same seeded inputs):

* the bias Add that the export's gemm_to_matmul step splits off each GPT-2
  Conv1D ("ONNX export, quantization and the browser runtime", section
  "Quantization (train/quantize.py)", step 1);
* GELU (GPT-2's tanh form, and the erf form) and the residual add that follow
  it in the model.

Tolerance: the body's 1e-5 * sum|x*w| + 1e-6 carried through the activation's
slope (at most 1.13), plus 1e-6 of |pre| and |out| for the fp32 roundings of
the bias add, the activation and the residual add (oracle.epilogue_ref)."""

import numpy as np
import pytest

import oracle
from gpu_util import dev, guarded, guards_intact, torch, upload_w4

from int8_weight_quantized_w4_b200 import synth

pytestmark = pytest.mark.gpu


def w4():
    import int8_weight_quantized_w4_b200 as w
    return w


def _check(y, out_ref, tol, what):
    got = y.detach().cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(got)), what
    err = np.abs(got - out_ref) - tol
    assert err.max() <= 0, f"{what}: over by {err.max():.3e} (max |err| {np.abs(got - out_ref).max():.3e})"


def run(M, K, N, path, act, with_bias=True, with_res=True, seed=3, in_place=False):
    W = synth.w4_weight(K, N, M, seed=seed)
    x = synth.activations(M, K, seed=seed)
    b = synth.bias(N, seed=seed) if with_bias else None
    r = synth.activations(M, N, 77, seed=seed) if with_res else None
    y_mm, a = oracle.w4_matmul_ref(x, W["qw"], W["scales"], W["zp"], K, N)
    out_ref, tol = oracle.epilogue_ref(y_mm, a, bias=b, residual=r, act=act)
    Wd = upload_w4(W)
    T = torch()
    if in_place:
        y = dev(r)
        res = y
        buf = None
    else:
        y, buf = guarded(M, N)
        res = None if r is None else dev(r)
    w4().w4_matmul(dev(x), Wd["qw"], Wd["scales"], Wd["zp"], K, N, y=y, path=path,
                   bias=None if b is None else dev(b), residual=res, act=act)
    T.cuda.synchronize()
    _check(y, out_ref, tol, f"{path} M={M} K={K} N={N} act={act} bias={with_bias} res={with_res}")
    if buf is not None:
        assert guards_intact(buf, M, N, N), "write outside y"


@pytest.mark.parametrize("act", ["none", "gelu_tanh", "gelu_erf"])
@pytest.mark.parametrize("path,M,K,N", [
    ("gemv", 1, 768, 2304),     # GPT-2 fused QKV, decode
    ("gemv", 1, 3072, 768),     # GPT-2 MLP output: tiles split across CTAs
    ("gemv", 2, 768, 3072),
    ("gemv", 8, 256, 544),      # M = 5..8 kernel, narrow tail
    ("generic", 3, 96, 70),     # odd layout: N % 32 != 0
    ("tc", 58, 768, 768),       # GPT-2 prefill
    ("tc", 129, 96, 288),       # ragged tiles
])
def test_epilogue_paths(path, M, K, N, act):
    run(M, K, N, path, act)


@pytest.mark.parametrize("path,M", [("gemv", 1), ("tc", 40), ("generic", 2)])
def test_bias_only_and_residual_only(path, M):
    run(M, 256, 512, path, "none", with_bias=True, with_res=False)
    run(M, 256, 512, path, "none", with_bias=False, with_res=True)
    run(M, 256, 512, path, "gelu_tanh", with_bias=False, with_res=False)


@pytest.mark.parametrize("path,M", [("gemv", 1), ("gemv", 4), ("tc", 58), ("generic", 3)])
def test_in_place_residual(path, M):
    # y holds the residual stream and is updated in place: y = y + x.W + b
    run(M, 768, 768, path, "none", in_place=True)


def test_k_zero_goes_through_the_epilogue():
    T = torch()
    M, N = 3, 64
    b = synth.bias(N, 5)
    r = synth.activations(M, N, 5)
    out_ref, _ = oracle.epilogue_ref(np.zeros((M, N)), np.zeros((M, N)), bias=b, residual=r, act="gelu_erf")
    y = T.full((M, N), float("nan"), device="cuda")
    z = T.zeros(16, dtype=T.uint8, device="cuda")
    s = T.zeros(4, dtype=T.float32, device="cuda")
    w4().w4_matmul(T.zeros((M, 0), device="cuda"), z, s, z, 0, N, y=y, bias=dev(b), residual=dev(r), act="gelu_erf")
    T.cuda.synchronize()
    assert np.abs(y.cpu().numpy() - out_ref).max() <= 1e-6


@pytest.mark.parametrize("M", [1, 58])
def test_grouped_gpt2_layer_pattern(M):
    """Two GPT-2 layers in one grouped call, each weight with its own epilogue:
    qkv + bias, attention output + bias + residual, MLP in + bias + GELU(tanh),
    MLP out + bias + residual (M = 1: the GEMV, M = 58: the tensor cores)."""
    T = torch()
    pattern = [("qkv", 768, 2304, "none", False), ("proj", 768, 768, "none", True),
               ("fc", 768, 3072, "gelu_tanh", False), ("fc2", 3072, 768, "none", True)] * 2
    items, refs, keep = [], [], []
    for i, (_, K, N, act, with_res) in enumerate(pattern):
        W = synth.w4_weight(K, N, 900 + i)
        x = synth.activations(M, K, 900 + i)
        b = synth.bias(N, 900 + i)
        r = synth.activations(M, N, 950 + i) if with_res else None
        y_mm, a = oracle.w4_matmul_ref(x, W["qw"], W["scales"], W["zp"], K, N)
        refs.append(oracle.epilogue_ref(y_mm, a, bias=b, residual=r, act=act))
        Wd = upload_w4(W)
        y = T.full((M, N), float("nan"), device="cuda")
        it = {"x": dev(x), "y": y, "K": K, "N": N, "qw": Wd["qw"], "scales": Wd["scales"], "zp": Wd["zp"],
              "bias": dev(b), "act": act}
        if with_res:
            it["residual"] = dev(r)
        items.append(it)
        keep.append(it)
    w4().w4_matmul_grouped(items)
    T.cuda.synchronize()
    for i, (it, (out_ref, tol)) in enumerate(zip(items, refs)):
        _check(it["y"], out_ref, tol, f"grouped weight {i} ({pattern[i][0]}) M={M}")


def test_epilogue_leaves_workspace_counters_zero():
    """A split-tile GEMV with an epilogue still resets its counters."""
    T = torch()
    need = w4().w4_matmul_workspace_size(1, 3072, 768)
    ws = T.zeros(need, dtype=T.uint8, device="cuda")
    for _ in range(2):
        run_ws = ws
        W = synth.w4_weight(3072, 768, 1)
        Wd = upload_w4(W)
        x = dev(synth.activations(1, 3072, 1))
        w4().w4_matmul(x, Wd["qw"], Wd["scales"], Wd["zp"], 3072, 768, path="gemv", ws=run_ws,
                       bias=dev(synth.bias(768, 1)), act="gelu_tanh")
    T.cuda.synchronize()
    assert int(ws[:4096].count_nonzero()) == 0
