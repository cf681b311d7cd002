"""The allocation-free entry point, w4_matmul_noalloc, against w4_matmul (GPU).

w4_matmul_noalloc is for callers that cannot allocate device memory where
they multiply, for instance a plugin inside a framework that owns every
device allocation, or a process that forbids allocation once it has started.
They pass inputs and outputs only; the split-K scratch is an array held inside
the library. Two calls in a row (sharing that array) must each give what
w4_matmul gives, within the tests' tolerance 1e-5 * sum|x*w| + 1e-6, and a
shape needing more scratch than the array holds must be refused.

This file is collected last on purpose, so that a run stopping at the first
failure has already run every other test.
"""

import numpy as np
import pytest

import oracle

from int8_weight_quantized_w4_b200 import synth

pytestmark = pytest.mark.gpu


def _noalloc(lib, xd, Wd, y, K, N, stream):
    M = xd.shape[0]
    return lib.w4_matmul_noalloc(xd.data_ptr(), K, Wd["qw"].data_ptr(), Wd["scales"].data_ptr(),
                                 Wd["zp"].data_ptr(), y.data_ptr(), N, M, K, N, stream)


def test_noalloc_matches_w4_matmul_on_two_calls_in_a_row():
    import torch

    import int8_weight_quantized_w4_b200 as w4
    lib = w4.lib()
    stream = torch.cuda.current_stream().cuda_stream
    cases = [(1, 768, 3072, 901), (2, 3072, 768, 902)]
    host, dev, got = [], [], []
    for M, K, N, tag in cases:
        W = synth.w4_weight(K, N, tag)
        x = synth.activations(M, K, tag)
        Wd = {k: torch.from_numpy(W[k]).cuda() for k in ("qw", "scales", "zp")}
        host.append((W, x))
        dev.append((torch.from_numpy(x).cuda(), Wd))
    # two calls in a row, one after the other on the same stream and scratch
    for (M, K, N, _), (xd, Wd) in zip(cases, dev):
        y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
        st = _noalloc(lib, xd, Wd, y, K, N, stream)
        assert st == 0, lib.w4_last_error()
        got.append(y)
    for (M, K, N, _), (W, x), (xd, Wd), y in zip(cases, host, dev, got):
        y_ref = w4.w4_matmul(xd, Wd["qw"], Wd["scales"], Wd["zp"], K, N)
        torch.cuda.synchronize()
        _, a = oracle.w4_matmul_ref(x, W["qw"], W["scales"], W["zp"], K, N)
        diff = np.abs(y.cpu().numpy().astype(np.float64) - y_ref.cpu().numpy().astype(np.float64))
        assert np.all(np.isfinite(diff)), f"M={M} K={K} N={N}: output not fully written"
        assert np.all(diff <= oracle.tolerance(a)), f"M={M} K={K} N={N}: max diff {diff.max():.3e}"


def test_noalloc_refuses_shapes_beyond_its_scratch():
    import torch

    import int8_weight_quantized_w4_b200 as w4
    lib = w4.lib()
    M, K, N = 8, 3072, 768  # enough work to use every SM
    assert w4.w4_matmul_workspace_size(M, K, N) > 2 << 20
    W = synth.w4_weight(K, N, 903)
    Wd = {k: torch.from_numpy(W[k]).cuda() for k in ("qw", "scales", "zp")}
    xd = torch.from_numpy(synth.activations(M, K, 903)).cuda()
    y = torch.empty((M, N), dtype=torch.float32, device="cuda")
    st = _noalloc(lib, xd, Wd, y, K, N, torch.cuda.current_stream().cuda_stream)
    assert st == 7
    assert b"scratch" in lib.w4_last_error()
