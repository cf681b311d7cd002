"""The GEMV host side reuses the launch parameters of a repeated call (same
descriptor bytes, workspace and device). Calls that differ must not reuse
them, a repeated call must read its inputs afresh, and a too-small workspace
is still refused on a repeated call."""

import numpy as np
import pytest

import oracle
from gpu_util import check, dev, torch, upload_w4

from int8_weight_quantized_w4_b200 import synth

pytestmark = pytest.mark.gpu


def w4():
    import int8_weight_quantized_w4_b200 as w
    return w


SHAPES = [(768, 2304), (768, 768), (3072, 768)]


def _setup(tag):
    T = torch()
    host, items = [], []
    for i, (K, N) in enumerate(SHAPES):
        W = synth.w4_weight(K, N, 500 + i)
        x = synth.activations(1, K, tag, i)
        Wd = upload_w4(W)
        y = T.full((1, N), float("nan"), device="cuda")
        items.append({"x": dev(x), "y": y, "K": K, "N": N, "qw": Wd["qw"], "scales": Wd["scales"], "zp": Wd["zp"]})
        host.append((W, x))
    return host, items


def _check_all(host, items, what):
    torch().cuda.synchronize()
    for (W, x), it in zip(host, items):
        y_ref, a = oracle.w4_matmul_ref(x, W["qw"], W["scales"], W["zp"], it["K"], it["N"])
        check(it["y"], y_ref, a, what)


def test_repeated_and_interleaved_grouped_calls():
    T = torch()
    w = w4()
    host_a, items_a = _setup(1)
    host_b, items_b = _setup(2)
    da, db = w.make_descs(items_a), w.make_descs(items_b)
    need = max(w.w4_matmul_grouped_workspace_size(da), w.w4_matmul_grouped_workspace_size(db))
    ws = T.zeros(need, dtype=T.uint8, device="cuda")
    w.w4_matmul_grouped(descs=da, ws=ws)
    _check_all(host_a, items_a, "first call")
    w.w4_matmul_grouped(descs=db, ws=ws)
    _check_all(host_b, items_b, "a different call")
    # new input values at the same addresses: the repeated call reads them
    for i, ((W, x), it) in enumerate(zip(host_a, items_a)):
        x2 = synth.activations(1, it["K"], 3, i)
        it["x"].copy_(dev(x2))
        host_a[i] = (W, x2)
    for it in items_a:
        it["y"].fill_(float("nan"))
    w.w4_matmul_grouped(descs=da, ws=ws)
    _check_all(host_a, items_a, "repeated call, new inputs")
    assert int(ws[:4096].count_nonzero()) == 0


def test_repeated_call_still_checks_the_workspace():
    T = torch()
    w = w4()
    _, items = _setup(4)
    d = w.make_descs(items)
    need = w.w4_matmul_grouped_workspace_size(d)
    ws = T.zeros(need, dtype=T.uint8, device="cuda")
    w.w4_matmul_grouped(descs=d, ws=ws)
    T.cuda.synchronize()
    lib = w.lib()
    st = lib.w4_matmul_grouped(d, len(d), ws.data_ptr(), need - 16, int(T.cuda.current_stream().cuda_stream))
    assert st == 7  # W4_ERR_WORKSPACE
