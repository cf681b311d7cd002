"""The allocation-free entry point, w4_matmul_noalloc (GPU).

w4_matmul_noalloc is for callers that cannot allocate device memory where
they multiply, for instance a plugin inside a framework that owns every
device allocation, or a process that forbids allocation once it has started.
They pass inputs and outputs only; the split-K scratch is an array held inside
the library. Calls in a row (sharing that array) must each give what the
oracle gives within the tests' tolerance 1e-5 * sum|x*w| + 1e-6, and what
w4_matmul gives on the same inputs; a call that the tensor-core kernel takes
(M > 16) needs no scratch at all, and a shape needing more scratch than the
array holds must be refused.

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


def test_noalloc_matches_oracle_and_w4_matmul_on_calls_in_a_row():
    import torch

    import int8_weight_quantized_w4_b200 as w4
    lib = w4.lib()
    stream = torch.cuda.current_stream().cuda_stream
    # M = 1 and 2 go through the split-K GEMV (scratch), M = 17 through the
    # tensor cores (no scratch)
    cases = [(1, 768, 3072, 901), (2, 3072, 768, 902), (17, 768, 768, 904), (1, 768, 3072, 905)]
    host, dev, got = [], [], []
    for M, K, N, tag in cases:
        W = synth.w4_weight(K, N, tag)
        x = synth.activations(M, K, tag)
        Wd = {k: torch.from_numpy(W[k]).cuda() for k in ("qw", "scales", "zp")}
        host.append((W, x))
        dev.append((torch.from_numpy(x).cuda(), Wd))
    # the calls in a row, one after the other on the same stream and scratch
    for (M, K, N, _), (xd, Wd) in zip(cases, dev):
        y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
        st = _noalloc(lib, xd, Wd, y, K, N, stream)
        assert st == 0, lib.w4_last_error()
        got.append(y)
    torch.cuda.synchronize()
    for (M, K, N, _), (W, x), (xd, Wd), y in zip(cases, host, dev, got):
        y_or, a = oracle.w4_matmul_ref(x, W["qw"], W["scales"], W["zp"], K, N)
        yg = y.cpu().numpy().astype(np.float64)
        assert np.all(np.isfinite(yg)), f"M={M} K={K} N={N}: output not fully written"
        v = oracle.max_violation(yg, y_or, a)
        assert v <= 0, f"M={M} K={K} N={N}: oracle tolerance exceeded by {v:.3e}"
        y_ref = w4.w4_matmul(xd, Wd["qw"], Wd["scales"], Wd["zp"], K, N)
        torch.cuda.synchronize()
        diff = np.abs(yg - y_ref.cpu().numpy().astype(np.float64))
        assert np.all(diff <= oracle.tolerance(a)), f"M={M} K={K} N={N}: differs from w4_matmul by {diff.max():.3e}"


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
