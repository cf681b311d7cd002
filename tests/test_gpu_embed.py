"""GPU token lookup on the tied int8 table against the oracle: bit for bit
(one fp32 multiply per element on both sides)."""

import numpy as np
import pytest

import oracle
from gpu_util import dev, torch

from int8_weight_quantized_w4_b200 import synth

pytestmark = pytest.mark.gpu


def w4():
    import int8_weight_quantized_w4_b200 as w
    return w


def _tokens(ids):
    return torch().tensor(np.asarray(ids, np.int32), device="cuda")


def test_embed_gpt2_table_bit_exact():
    K, V = 768, 50257
    H = synth.i8_head(K, V, seed=21)
    g = np.random.default_rng(21)
    ids = np.concatenate([[0, V - 1, 1, V - 2], g.integers(0, V, 54), [7, 7]]).astype(np.int32)  # 60 tokens
    out = w4().i8_embed_lookup(dev(H["table"]), dev(H["scales"]), _tokens(ids), K, V, ldt=H["ldt"])
    torch().cuda.synchronize()
    ref = oracle.i8_embed_ref(H["table"], H["scales"], ids, K, V, H["ldt"])
    assert np.array_equal(out.cpu().numpy(), ref)


def test_embed_padded_table_and_output():
    K, V, ldt, ldo = 100, 777, 801, 130
    H = synth.i8_head(K, V, seed=22, ldt=ldt)
    ids = np.array([0, 776, 5, 400], np.int32)
    T = torch()
    out_buf = T.full((len(ids), ldo), 7.0, dtype=T.float32, device="cuda")
    w4().i8_embed_lookup(dev(H["table"]), dev(H["scales"]), _tokens(ids), K, V, ldt=ldt, out=out_buf[:, :K])
    T.cuda.synchronize()
    got = out_buf.cpu().numpy()
    assert np.array_equal(got[:, :K], oracle.i8_embed_ref(H["table"], H["scales"], ids, K, V, ldt))
    assert np.all(got[:, K:] == 7.0), "write past K"


def test_embed_out_of_range_token_zeroes_its_row_and_reports():
    w = w4()
    K, V = 64, 300
    H = synth.i8_head(K, V, seed=23)
    w.device_error(clear=True)
    ids = np.array([3, 300, -1, 299], np.int32)
    out = w.i8_embed_lookup(dev(H["table"]), dev(H["scales"]), _tokens(ids), K, V)
    torch().cuda.synchronize()
    got = out.cpu().numpy()
    st, info = w.device_error(clear=True)
    assert st == 8 and info[0] == 8  # W4_ERR_VALUE
    assert np.all(got[1] == 0) and np.all(got[2] == 0)
    ok = np.array([3, 299])
    assert np.array_equal(got[[0, 3]], oracle.i8_embed_ref(H["table"], H["scales"], ok, K, V))
    assert w.device_error(clear=False)[0] == 0
