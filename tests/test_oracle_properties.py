"""Randomised pins of the oracle: the invariants of test_oracle.py over many
small shapes, drawn by hypothesis (bounded, seeded through hypothesis' own
database-free derandomised runs).

Paper: "DyRA: Dynamic Residual Approximation for Efficient Matrix
Multiplication in DNNs". Each property holds for every shape and ridge:
- k = 0 gives the weight-only layer (Eq. 2);
- the fit never loses to the weight-only layer, per instance (C = 0 is
  feasible in the ridge problem of Eq. 3-5);
- the fit is the ridge minimiser: the normal equations of Eq. 5 hold;
- a residual of rank k, fully covered, is reproduced exactly (lambda = 0);
- the instances are independent: permuting them permutes the outputs.
"""

import numpy as np
import pytest
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

from oracle import dyra_oracle as orc
from synth import LayerSpec, generate

SETTINGS = settings(max_examples=40, deadline=None, derandomize=True,
                    suppress_health_check=[HealthCheck.too_slow])


@st.composite
def layers(draw, exact_rank=False):
    d_in = draw(st.integers(4, 24))
    d_out = draw(st.integers(4, 24))
    m = min(d_in, d_out)
    r = draw(st.integers(1, m - 1))
    k = draw(st.integers(0, m - r))
    B = draw(st.integers(1, 4))
    T = draw(st.integers(max(1, k), max(12, k)))
    lam = draw(st.sampled_from([0.0, 1e-3, 0.3])) if not exact_rank else 0.0
    seed = draw(st.integers(0, 10_000))
    x_kind = draw(st.sampled_from(["normal", "lognormal", "outlier"]))
    s = LayerSpec("h", d_in, d_out, r, k, B, T, "f32", 0.8, x_kind, n_outlier=1,
                  outlier_scale=8.0, seed=seed, lam=lam)
    spectrum = None
    if exact_rank:
        spectrum = np.zeros(m)
        spectrum[: r + k] = np.linspace(2.0, 0.5, r + k)
    return s, generate(s, spectrum=spectrum)


def _run(s, w):
    f = orc.offline_prepare_from_svd(w.left, w.sigma, w.right, s.r, s.k, s.lam)
    Y = orc.inference(w.X, f.U, f.V, f.P, f.W_res, s.lam, s.B, s.T)
    return f, Y


@SETTINGS
@given(layers())
def test_never_worse_than_weight_only(layer):
    s, w = layer
    f, Y = _run(s, w)
    Yd = w.X @ w.weight().T
    Ywo = (w.X @ f.V) @ f.U.T
    for b in range(s.B):
        rows = slice(b * s.T, (b + 1) * s.T)
        assert np.linalg.norm(Yd[rows] - Y[rows]) <= \
            np.linalg.norm(Yd[rows] - Ywo[rows]) * (1 + 1e-10) + 1e-12


@SETTINGS
@given(layers())
def test_correction_solves_the_ridge_normal_equations(layer):
    """C = (L^T L + lam I)^-1 L^T E, i.e. (L^T L + lam I) C = L^T E with
    E = X_b W_res^T: checked through the output, since L C = Y - Y_wo."""
    s, w = layer
    if s.k == 0:
        return
    f, Y = _run(s, w)
    for b in range(s.B):
        rows = slice(b * s.T, (b + 1) * s.T)
        Xb = w.X[rows]
        L = Xb @ f.P
        E = Xb @ f.W_res.T
        LC = Y[rows] - (Xb @ f.V) @ f.U.T
        # recover C from L C where L has full column rank; otherwise check the
        # gradient of the ridge objective in the range of L
        grad = L.T @ (LC - E) + s.lam * np.linalg.lstsq(L, LC, rcond=None)[0]
        scale = np.linalg.norm(L) * (np.linalg.norm(E) + np.linalg.norm(LC)) + 1e-12
        if np.linalg.matrix_rank(L) == s.k:
            assert np.linalg.norm(grad) <= 1e-8 * scale


@SETTINGS
@given(layers(exact_rank=True))
def test_fully_covered_residual_is_exact(layer):
    s, w = layer
    if s.k == 0 or s.T < s.k:
        return
    f, Y = _run(s, w)
    Yd = w.X @ w.weight().T
    np.testing.assert_allclose(Y, Yd, rtol=0, atol=1e-8 * max(1.0, np.abs(Yd).max()))


@SETTINGS
@given(layers(), st.integers(0, 1000))
def test_instances_are_independent(layer, pseed):
    s, w = layer
    f, Y = _run(s, w)
    perm = np.random.default_rng(pseed).permutation(s.B)
    Xp = np.concatenate([w.X[b * s.T:(b + 1) * s.T] for b in perm])
    Yp = orc.inference(Xp, f.U, f.V, f.P, f.W_res, s.lam, s.B, s.T)
    want = np.concatenate([Y[b * s.T:(b + 1) * s.T] for b in perm])
    np.testing.assert_allclose(Yp, want, rtol=0, atol=1e-10 * max(1.0, np.abs(want).max()))


def test_weight_only_at_k0():
    s = LayerSpec("k0", 12, 10, 3, 0, 2, 5, "f32", 0.8, "lognormal", seed=1, lam=0.0)
    w = generate(s)
    f, Y = _run(s, w)
    np.testing.assert_allclose(Y, (w.X @ f.V) @ f.U.T, rtol=0, atol=1e-13)
