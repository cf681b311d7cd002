"""The oracle's fused epilogue (bias Add, GELU, residual) pinned to facts
outside itself (CPU only).

The Add is the one the export page's gemm_to_matmul step splits off every
GPT-2 Conv1D ("ONNX export, quantization and the browser runtime", section
"Quantization (train/quantize.py)", step 1); GELU and the residual add are
what stock GPT-2 small applies after it. The facts used here are mathematical:
the erf form of GELU is v * Phi(v), Phi the standard normal CDF, whose values
at 0.5, 1 and 2 are textbook table entries; GELU(v) - GELU(-v) = v for both
forms (the tanh and erf terms are odd); the tanh form stays within 1e-3 of
the erf form and saturates to v and 0. Each check runs against the oracle and
against copies with one planted mistake, each of which must fail a check.
"""

from types import SimpleNamespace

import numpy as np
import pytest

import oracle

# standard normal CDF, from the table (Phi(-v) = 1 - Phi(v))
PHI = {0.5: 0.6914624612740131, 1.0: 0.8413447460685429, 2.0: 0.9772498680518208}


def check_erf_table(impl):
    bad = []
    for v, phi in PHI.items():
        for s in (1.0, -1.0):
            want = s * v * (phi if s > 0 else 1.0 - phi)
            got = float(impl.gelu_erf(np.array([s * v]))[0])
            if abs(got - want) > 1e-14:
                bad.append(f"gelu_erf({s * v}) = {got}, table gives {want}")
    if float(impl.gelu_erf(np.array([0.0]))[0]) != 0.0:
        bad.append("gelu_erf(0) != 0")
    return bad


def check_odd_part(impl):
    bad = []
    v = np.linspace(-7.0, 7.0, 1401)
    for name in ("gelu_tanh", "gelu_erf"):
        f = getattr(impl, name)
        d = f(v) - f(-v) - v
        if np.abs(d).max() > 1e-12:
            bad.append(f"{name}(v) - {name}(-v) != v (off by {np.abs(d).max():.3g})")
    return bad


def check_tanh_form_close_to_exact(impl):
    bad = []
    v = np.linspace(-8.0, 8.0, 16001)
    err = np.abs(impl.gelu_tanh(v) - impl.gelu_erf(v)).max()
    if err > 1e-3:
        bad.append(f"tanh form {err:.3g} away from the erf form")
    if float(impl.gelu_tanh(np.array([10.0]))[0]) != 10.0 or abs(float(impl.gelu_tanh(np.array([-10.0]))[0])) > 1e-12:
        bad.append("tanh form does not saturate to v and 0 at +-10")
    return bad


def _zero_weight_epilogue(impl, bias, residual, act):
    """y = x.W = 0 exactly (every q equals its zero point), then the epilogue."""
    M, N = 2, len(bias)
    y = np.zeros((M, N))
    a = np.zeros((M, N))
    out, _ = impl.epilogue_ref(y, a, bias=bias, residual=residual, act=act)
    return out


def check_epilogue_closed_forms(impl):
    bad = []
    b = np.array([1.0, 2.0, 0.5, -1.0], np.float32)
    r = np.array([[1.0, -2.0, 0.25, 3.0], [0.0, 0.5, -0.5, 1.0]], np.float32)
    phi = np.array([PHI[1.0], PHI[2.0], PHI[0.5], 1.0 - PHI[1.0]])
    want = b.astype(np.float64) * phi + r
    got = _zero_weight_epilogue(impl, b, r, "gelu_erf")
    if np.abs(got - want).max() > 1e-14:
        bad.append("act(bias) + residual on a zero product differs from the table")
    got = _zero_weight_epilogue(impl, b, None, "none")
    if not np.array_equal(got, np.tile(b.astype(np.float64), (2, 1))):
        bad.append("bias alone on a zero product is not the bias")
    got = _zero_weight_epilogue(impl, np.zeros(4, np.float32), r, "none")
    if not np.array_equal(got, r.astype(np.float64)):
        bad.append("residual alone on a zero product is not the residual")
    # the product itself goes through the activation: x.W = 1 with no bias
    out, _ = impl.epilogue_ref(np.ones((1, 1)), np.ones((1, 1)), act="gelu_erf")
    if abs(float(out[0, 0]) - PHI[1.0]) > 1e-14:
        bad.append("the product does not go through the activation")
    return bad


CHECKS = [check_erf_table, check_odd_part, check_tanh_form_close_to_exact, check_epilogue_closed_forms]


@pytest.mark.parametrize("chk", CHECKS, ids=lambda c: c.__name__)
def test_oracle_epilogue_pin(chk):
    assert chk(oracle) == []


def test_epilogue_tolerance_covers_the_slope():
    # the allowance grows with |pre| and |out| and with the activation's slope
    y = np.array([[3.0]])
    a = np.array([[10.0]])
    _, t0 = oracle.epilogue_ref(y, a, act="none")
    _, t1 = oracle.epilogue_ref(y, a, act="gelu_tanh")
    assert t1[0, 0] > t0[0, 0] > oracle.tolerance(a)[0, 0]


# ---------------------------------------------------------------- mutants

def _mutant(**over):
    base = dict(gelu_tanh=oracle.gelu_tanh, gelu_erf=oracle.gelu_erf)
    base.update({k: v for k, v in over.items() if k != "epilogue_ref"})
    ns = SimpleNamespace(**base)
    acts = {"none": lambda v: np.asarray(v, np.float64), "gelu_tanh": ns.gelu_tanh, "gelu_erf": ns.gelu_erf}

    def epi(y, a, bias=None, residual=None, act="none"):
        pre = np.asarray(y, np.float64) + (0.0 if bias is None else np.asarray(bias, np.float64)[None, :])
        out = acts[act](pre)
        if residual is not None:
            out = out + np.asarray(residual, np.float64)
        return out, oracle.tolerance(a)

    ns.epilogue_ref = over.get("epilogue_ref", epi)
    return ns


def _act_after_residual(y, a, bias=None, residual=None, act="none"):
    pre = np.asarray(y, np.float64) + (0.0 if bias is None else np.asarray(bias, np.float64)[None, :])
    if residual is not None:
        pre = pre + np.asarray(residual, np.float64)
    return oracle.ACTIVATIONS[act](pre), oracle.tolerance(a)


def _bias_dropped(y, a, bias=None, residual=None, act="none"):
    out = oracle.ACTIVATIONS[act](np.asarray(y, np.float64))
    if residual is not None:
        out = out + np.asarray(residual, np.float64)
    return out, oracle.tolerance(a)


MUTANTS = {
    "tanh form without the cubic term": _mutant(
        gelu_tanh=lambda v: 0.5 * np.asarray(v) * (1 + np.tanh(oracle.SQRT_2_OVER_PI * np.asarray(v)))),
    "tanh form with sqrt(1/pi)": _mutant(
        gelu_tanh=lambda v: 0.5 * np.asarray(v) * (1 + np.tanh(np.sqrt(1 / np.pi) * (np.asarray(v) + 0.044715 * np.asarray(v) ** 3)))),
    "erf form without the 1/sqrt(2)": _mutant(
        gelu_erf=lambda v: 0.5 * np.asarray(v) * (1 + np.vectorize(__import__("math").erf)(np.asarray(v, np.float64)))),
    "erf form as 1 - Phi": _mutant(gelu_erf=lambda v: np.asarray(v, np.float64) - oracle.gelu_erf(v)),
    "activation after the residual": _mutant(epilogue_ref=_act_after_residual),
    "bias dropped": _mutant(epilogue_ref=_bias_dropped),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_each_planted_mistake_fails_a_pin(name):
    impl = MUTANTS[name]
    failures = [m for chk in CHECKS for m in chk(impl)]
    assert failures, f"no pin sees: {name}"
