"""The softmax's polynomial 2^x (Cody-Waite reduction plus a minimax fit), on the CPU:
coefficients equal to the committed fit, error bound against exact 2^x, exact special
values, and the clamp."""
import importlib.util
import os

import numpy as np
import pytest

from tests.exp2_poly_ref import HEADER, exp2_poly_f32, header_constants

BOUND = 1.05e-4  # the fit's minimax relative error is 1.013e-4; fp32 evaluation adds < 2e-7


def _fit_module():
    path = os.path.join(os.path.dirname(HEADER), "exp2_poly_fit.py")
    spec = importlib.util.spec_from_file_location("exp2_poly_fit", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_coefficients_are_the_fit():
    pytest.importorskip("scipy")
    c, err = _fit_module().fit()
    k = header_constants()
    assert [k["c1"], k["c2"], k["c3"]] == [c[0], c[1], c[2]]
    assert err < 1.02e-4


def test_reduction_constants():
    k = header_constants()
    assert k["kRound"] == np.float32(1.5 * 2 ** 23)
    assert k["kLow"] == np.float32(-126.0)


def test_relative_error_bound():
    x = np.concatenate([np.linspace(-125.0, 8.0, 2_000_001, dtype=np.float64),
                        np.linspace(-1.0, 1.0, 200_001)]).astype(np.float32)
    y = exp2_poly_f32(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y / ref - 1.0)
    assert rel.max() <= BOUND, rel.max()


def test_exact_values():
    j = np.arange(-126, 9, dtype=np.float32)
    assert np.array_equal(exp2_poly_f32(j), np.exp2(j.astype(np.float64)).astype(np.float32))
    assert exp2_poly_f32(np.float32(0.0)) == np.float32(1.0)


def test_clamp_below():
    y = exp2_poly_f32(np.array([-126.0, -127.5, -1000.0, -np.inf], dtype=np.float32))
    assert np.all(y == np.float32(2.0 ** -126))


def test_planted_mistakes_fail():
    """A dropped term or a wrong sign in the restatement breaks the bound."""
    x = np.linspace(-4.0, 4.0, 10001, dtype=np.float32)
    ref = np.exp2(x.astype(np.float64))
    k = header_constants()
    f = x - np.rint(x)
    no_cubic = (1 + f * (k["c1"] + f * k["c2"])) * np.exp2(np.rint(x))
    assert np.abs(no_cubic / ref - 1).max() > 10 * BOUND
    wrong_sign = (1 + f * (k["c1"] - f * (k["c2"] + f * k["c3"]))) * np.exp2(np.rint(x))
    assert np.abs(wrong_sign / ref - 1).max() > 10 * BOUND
