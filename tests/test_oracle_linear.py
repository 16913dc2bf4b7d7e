"""Pins of the oracle's full linear-layer form: bias b and correction weight alpha.

Paper: "DyRA: Dynamic Residual Approximation for Efficient Matrix
Multiplication in DNNs", Sec. 2.4: the fused linear layer adds a bias and
weighs the correction, Y = Y_base + b + alpha L R (R is C here). Alg. 1 is
b = 0 and alpha = 1.

The pins check the oracle against closed forms: alpha = 0 is the weight-only
layer plus b; b shifts every row by b; the output is affine in alpha; and with
lam = 0 the correction is an orthogonal projection, so the fit error obeys
||E - alpha L C||^2 = ||E - L C||^2 + (1 - alpha)^2 ||L C||^2 (Pythagoras).
test_planted_linear_mistakes_are_caught swaps a mistaken copy of inference
into the oracle module and checks that some pin fails.
"""

import numpy as np
import pytest

from oracle import dyra_oracle as orc
from synth import LayerSpec, generate

B, T = 3, 9


def layer(lam=1e-3, seed=0):
    s = LayerSpec("lin", 20, 14, 3, 4, B, T, "f32", 0.6, "lognormal", seed=seed, lam=lam)
    w = generate(s)
    f = orc.offline_prepare_from_svd(w.left, w.sigma, w.right, s.r, s.k, lam)
    b = np.random.default_rng([seed, 7]).standard_normal(s.d_out)
    return w, f, b


def call(w, f, lam, **kw):
    return orc.inference(w.X, f.U, f.V, f.P, f.W_res, lam, B, T, **kw)


def check_defaults_are_algorithm_1():
    w, f, _ = layer()
    a = call(w, f, 1e-3)
    b = call(w, f, 1e-3, bias=None, alpha=1.0)
    np.testing.assert_array_equal(a, b)


def check_alpha_zero_is_weight_only_plus_bias():
    w, f, bias = layer()
    Y = call(w, f, 1e-3, bias=bias, alpha=0.0)
    np.testing.assert_allclose(Y, (w.X @ f.V) @ f.U.T + bias, rtol=0, atol=1e-12)


def check_bias_shifts_every_row():
    w, f, bias = layer(seed=1)
    for alpha in (1.0, 0.3):
        d = call(w, f, 1e-3, bias=bias, alpha=alpha) - call(w, f, 1e-3, alpha=alpha)
        np.testing.assert_allclose(d, np.broadcast_to(bias, d.shape), rtol=0, atol=1e-12)


def check_affine_in_alpha():
    w, f, bias = layer(seed=2)
    Y0 = call(w, f, 1e-3, bias=bias, alpha=0.0)
    Y1 = call(w, f, 1e-3, bias=bias, alpha=1.0)
    for alpha in (0.5, 2.0, -1.0):
        Ya = call(w, f, 1e-3, bias=bias, alpha=alpha)
        np.testing.assert_allclose(Ya, Y0 + alpha * (Y1 - Y0), rtol=0, atol=1e-11)


def check_pythagoras_at_lambda_zero():
    """lam = 0: L C projects E = X_b W_res^T onto col(L), so the error of the
    alpha-weighted correction splits into the fit error and (1 - alpha)^2 of
    the correction's energy. alpha in [0, 2] is never worse than weight-only."""
    w, f, bias = layer(lam=0.0, seed=3)
    Wd = f.U @ f.V.T + f.W_res
    Y1 = call(w, f, 0.0, alpha=1.0)
    Ywo = (w.X @ f.V) @ f.U.T
    for alpha in (0.0, 0.5, 1.5, 2.0):
        Ya = call(w, f, 0.0, bias=bias, alpha=alpha)
        for b in range(B):
            rows = slice(b * T, (b + 1) * T)
            Yd = w.X[rows] @ Wd.T + bias
            fit = np.sum((Yd - bias - Y1[rows]) ** 2)
            corr = np.sum((Y1[rows] - Ywo[rows]) ** 2)
            err = np.sum((Yd - Ya[rows]) ** 2)
            assert err == pytest.approx(fit + (1 - alpha) ** 2 * corr, rel=1e-9, abs=1e-12)
            assert err <= np.sum((Yd - bias - Ywo[rows]) ** 2) * (1 + 1e-12)


PINS = [check_defaults_are_algorithm_1, check_alpha_zero_is_weight_only_plus_bias,
        check_bias_shifts_every_row, check_affine_in_alpha, check_pythagoras_at_lambda_zero]


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_linear_pin(pin):
    pin()


_ORIG = orc.inference


def _alpha_on_static(X, U, V, P, W_res, lam, B_, T_, *, bias=None, alpha=1.0):
    Y = _ORIG(X, U, V, P, W_res, lam, B_, T_)
    return alpha * Y + (0 if bias is None else bias)


def _alpha_squared(X, U, V, P, W_res, lam, B_, T_, *, bias=None, alpha=1.0):
    Yw = (X @ V) @ U.T
    Y = _ORIG(X, U, V, P, W_res, lam, B_, T_)
    return Yw + alpha ** 2 * (Y - Yw) + (0 if bias is None else bias)


def _bias_subtracted(X, U, V, P, W_res, lam, B_, T_, *, bias=None, alpha=1.0):
    return _ORIG(X, U, V, P, W_res, lam, B_, T_, alpha=alpha) - (0 if bias is None else bias)


def _bias_on_first_row(X, U, V, P, W_res, lam, B_, T_, *, bias=None, alpha=1.0):
    Y = _ORIG(X, U, V, P, W_res, lam, B_, T_, alpha=alpha)
    if bias is not None:
        Y[0] += bias
    return Y


@pytest.mark.parametrize("mutant", [_alpha_on_static, _alpha_squared, _bias_subtracted,
                                    _bias_on_first_row], ids=lambda m: m.__name__)
def test_planted_linear_mistakes_are_caught(monkeypatch, mutant):
    monkeypatch.setattr(orc, "inference", mutant)
    failures = 0
    for pin in PINS:
        try:
            pin()
        except AssertionError:
            failures += 1
    assert failures > 0, "no pin catches the planted mistake %s" % mutant.__name__
