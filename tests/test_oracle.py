"""Pins of the fp64 oracle against what the DyRA paper and linear algebra fix.

Paper: "DyRA: Dynamic Residual Approximation for Efficient Matrix
Multiplication in DNNs". None of these tests re-types the oracle's formula:
each checks it against a closed form, an invariant, an optimality condition, a
library routine solving the defining problem another way, or a hand-derived
example. test_planted_mistakes_are_caught plants typical mistakes in the
oracle and checks that at least one pin fails for each.
"""

import json
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from oracle import dyra_oracle as orc
from synth import LayerSpec, generate, haar_orthonormal

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def small_layer(d_in=24, d_out=20, r=4, k=3, B=3, T=7, p=0.7, x_kind="lognormal", seed=0,
                spectrum=None):
    s = LayerSpec("small", d_in, d_out, r, k, B, T, "f32", p, x_kind, n_outlier=2,
                  outlier_scale=10.0, seed=seed)
    return generate(s, spectrum=spectrum)


def factors(w, r, k, lam):
    return orc.offline_prepare_from_svd(w.left, w.sigma, w.right, r, k, lam)


def run(w, r, k, lam, B, T, X=None):
    f = factors(w, r, k, lam)
    X = w.X if X is None else X
    return orc.inference(X, f.U, f.V, f.P, f.W_res, lam, B, T), f


# ---------------------------------------------------------------- pins ----

def check_k0_equals_weight_only(infer=orc.inference):
    """k = 0: only the first term of Eq. 2 remains, Y = (X V) U^T."""
    w = small_layer()
    f = factors(w, 4, 0, 0.0)
    Y = infer(w.X, f.U, f.V, f.P, f.W_res, 0.0, 3, 7)
    ref = w.X @ (w.right[:, :4] * w.sigma[:4]) @ w.left[:, :4].T
    np.testing.assert_allclose(Y, ref, rtol=0, atol=1e-12)


def check_full_residual_is_exact(infer=orc.inference):
    """rank(W_res) = k, T >= k, lambda = 0: L C is the projection of
    E = X W_res^T onto col(L), and E lies in col(L), so Y = X W^T."""
    d_in, d_out, r, k = 24, 20, 4, 3
    sig = np.zeros(20)
    sig[: r + k] = np.linspace(2.0, 0.5, r + k)
    w = small_layer(d_in, d_out, r, k, B=3, T=7, spectrum=sig)
    f = factors(w, r, k, 0.0)
    Y = infer(w.X, f.U, f.V, f.P, f.W_res, 0.0, 3, 7)
    Yd = w.X @ w.weight().T
    assert orc.rel_fro(Y, Yd) < 1e-11


def check_isotropic_prop1(infer=orc.inference):
    """Prop. 1 (Sec. 2.3, proof in App. C Eq. 16): if X_b^T X_b = I and
    lambda = 0, DyRA equals the static rank-(r+k) truncated SVD."""
    d_in, d_out, r, k, B = 12, 16, 3, 2, 2
    T = 15
    w = small_layer(d_in, d_out, r, k, B=B, T=T)
    rng = np.random.default_rng(5)
    X = np.concatenate([haar_orthonormal(rng, T, d_in) for _ in range(B)])
    f = factors(w, r, k, 0.0)
    Y = infer(X, f.U, f.V, f.P, f.W_res, 0.0, B, T)
    Wrk = (w.left[:, : r + k] * w.sigma[: r + k]) @ w.right[:, : r + k].T
    np.testing.assert_allclose(Y, X @ Wrk.T, rtol=0, atol=1e-12)


def check_augmented_lstsq(infer=orc.inference):
    """Eq. 5 with the footnote-2 ridge is the minimiser of
    ||E - L C||_F^2 + lambda ||C||_F^2 over C, E = X_b W_res^T. Solve that
    problem as the stacked least-squares system [L; sqrt(lambda) I] C = [E; 0]
    (numpy lstsq, no normal equations) and compare L C elementwise."""
    w = small_layer(B=3, T=7)
    for lam in (0.0, 1e-3, 0.37):
        f = factors(w, 4, 3, lam)
        Y = infer(w.X, f.U, f.V, f.P, f.W_res, lam, 3, 7)
        for b in range(3):
            Xb = w.X[b * 7:(b + 1) * 7]
            E = Xb @ f.W_res.T
            L = Xb @ f.P
            Aug = np.vstack([L, np.sqrt(lam) * np.eye(3)])
            rhs = np.vstack([E, np.zeros((3, E.shape[1]))])
            C = np.linalg.lstsq(Aug, rhs, rcond=None)[0]
            corr = Y[b * 7:(b + 1) * 7] - (Xb @ f.V) @ f.U.T
            np.testing.assert_allclose(corr, L @ C, rtol=0, atol=1e-11 * max(1, np.abs(E).max()))


def check_never_worse_than_weight_only(infer=orc.inference):
    """C = 0 is feasible in the ridge problem, so per instance
    ||E - L C||^2 + lambda ||C||^2 <= ||E||^2 and hence ||X W^T - Y|| <= ||X W^T - Y_wo||."""
    for seed, x_kind in ((0, "lognormal"), (1, "outlier"), (2, "normal")):
        w = small_layer(B=4, T=5, seed=seed, x_kind=x_kind)
        for lam in (0.0, 1e-3, 1.0, 100.0):
            f = factors(w, 4, 3, lam)
            Y = infer(w.X, f.U, f.V, f.P, f.W_res, lam, 4, 5)
            Yd = w.X @ w.weight().T
            Ywo = (w.X @ f.V) @ f.U.T
            for b in range(4):
                s = slice(b * 5, (b + 1) * 5)
                assert np.linalg.norm(Yd[s] - Y[s]) <= np.linalg.norm(Yd[s] - Ywo[s]) * (1 + 1e-12)


def check_eckart_young_bound(infer=orc.inference):
    """Sec. 2.2: the optimum of Eq. 3 is the truncated SVD of X W_res^T, so no
    rank-k correction beats sum_{i>k} sigma_i(E)^2."""
    w = small_layer(B=2, T=9)
    f = factors(w, 4, 3, 0.0)
    Y = infer(w.X, f.U, f.V, f.P, f.W_res, 0.0, 2, 9)
    for b in range(2):
        s = slice(b * 9, (b + 1) * 9)
        E = w.X[s] @ f.W_res.T
        sv = np.linalg.svd(E, compute_uv=False)
        got = np.linalg.norm(E - (Y[s] - (w.X[s] @ f.V) @ f.U.T))
        assert got >= np.sqrt(np.sum(sv[3:] ** 2)) * (1 - 1e-12)


def check_instances_independent(infer=orc.inference):
    """Sec. 2.4: the correction is fitted for each batch instance, so instance
    b's output depends on X_b only."""
    w = small_layer(B=3, T=6)
    f = factors(w, 4, 3, 1e-3)
    Y1 = infer(w.X, f.U, f.V, f.P, f.W_res, 1e-3, 3, 6)
    X2 = w.X.copy()
    X2[6:12] = 3.0 * X2[6:12][::-1] + 1.0
    Y2 = infer(X2, f.U, f.V, f.P, f.W_res, 1e-3, 3, 6)
    np.testing.assert_array_equal(Y1[:6], Y2[:6])
    np.testing.assert_array_equal(Y1[12:], Y2[12:])
    assert not np.allclose(Y1[6:12], Y2[6:12])


def check_single_row_closed_form(infer=orc.inference):
    """T = 1: with l = x P (1 x k), (l^T l + lambda I)^-1 l^T = l^T / (|l|^2 + lambda),
    so L C = |l|^2 / (|l|^2 + lambda) * x W_res^T."""
    w = small_layer(B=5, T=1)
    lam = 0.25
    f = factors(w, 4, 3, lam)
    Y = infer(w.X[:5], f.U, f.V, f.P, f.W_res, lam, 5, 1)
    for b in range(5):
        x = w.X[b:b + 1]
        l2 = float(np.sum((x @ f.P) ** 2))
        want = (x @ f.V) @ f.U.T + l2 / (l2 + lam) * (x @ f.W_res.T)
        np.testing.assert_allclose(Y[b:b + 1], want, rtol=0, atol=1e-12)


PINS = [check_k0_equals_weight_only, check_full_residual_is_exact, check_isotropic_prop1,
        check_augmented_lstsq, check_never_worse_than_weight_only, check_eckart_young_bound,
        check_instances_independent, check_single_row_closed_form]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_inference_pin(pin):
    pin()


# ------------------------------------------------- offline preparation ----

def test_projector_closed_form():
    """App. C Eq. 13 with the ridge: R0 has orthonormal rows, so
    P = W_res^T R0^T / (1 + lambda) = right_{r:r+k} sigma_{r:r+k} / (1 + lambda)."""
    w = small_layer()
    for lam in (0.0, 1e-3, 0.5):
        f = factors(w, 4, 3, lam)
        want = w.right[:, 4:7] * w.sigma[4:7] / (1.0 + lam)
        np.testing.assert_allclose(f.P, want, rtol=0, atol=1e-13)


def test_prop1_general_form():
    """Prop. 1 Eq. 8 (lambda = 0): Y = X V U^T + X A_res R1 with
    A_res = right_{r:r+k} sigma_{r:r+k} and R1 = (A^T X^T X A)^-1 A^T X^T X W_res^T."""
    w = small_layer(B=1, T=21)
    f = factors(w, 4, 3, 0.0)
    Y = orc.inference(w.X, f.U, f.V, f.P, f.W_res, 0.0, 1, 21)
    A = w.right[:, 4:7] * w.sigma[4:7]
    XtX = w.X.T @ w.X
    R1 = np.linalg.inv(A.T @ XtX @ A) @ A.T @ XtX @ f.W_res.T
    want = w.X @ (w.right[:, :4] * w.sigma[:4]) @ w.left[:, :4].T + w.X @ A @ R1
    np.testing.assert_allclose(Y, want, rtol=0, atol=1e-10)


def test_svd_route_matches_given_svd():
    """Alg. 1 offline via an SVD of the dense W gives the same layer as reading
    the generator's factors (singular-vector signs cancel in U V^T and in L C)."""
    w = small_layer()
    W = w.weight()
    lam = 1e-3
    a = orc.offline_prepare(W, 4, 3, lam)
    b = factors(w, 4, 3, lam)
    np.testing.assert_allclose(a.U @ a.V.T, b.U @ b.V.T, atol=1e-12)
    np.testing.assert_allclose(a.W_res, b.W_res, atol=1e-12)
    np.testing.assert_allclose(a.W_res, W - a.U @ a.V.T, atol=1e-13)
    Ya = orc.inference(w.X, a.U, a.V, a.P, a.W_res, lam, 3, 7)
    Yb = orc.inference(w.X, b.U, b.V, b.P, b.W_res, lam, 3, 7)
    np.testing.assert_allclose(Ya, Yb, atol=1e-10)


def test_r0_is_top_residual_direction():
    """App. D: R0 spans the top-k singular directions of W_res (output side)."""
    w = small_layer()
    a = orc.offline_prepare(w.weight(), 4, 3, 0.0)
    np.testing.assert_allclose(a.R0 @ a.R0.T, np.eye(3), atol=1e-12)
    proj = a.R0.T @ a.R0
    np.testing.assert_allclose(proj, w.left[:, 4:7] @ w.left[:, 4:7].T, atol=1e-10)


def test_hand_worked_example():
    """tests/golden/hand_example_diag321.json: Algorithm 1 worked by hand with
    exact fractions on W = diag(3,2,1)."""
    g = json.load(open(os.path.join(GOLDEN, "hand_example_diag321.json")))
    lam = float(Fraction(g["lam"]))
    W = np.array(g["W"], dtype=np.float64)
    X = np.array(g["X"], dtype=np.float64)
    want = np.array([[float(Fraction(v)) for v in row] for row in g["Y"]])
    for f in (orc.offline_prepare(W, g["r"], g["k"], lam),
              orc.offline_prepare_from_svd(np.eye(3), np.array([3.0, 2.0, 1.0]), np.eye(3),
                                           g["r"], g["k"], lam)):
        Y = orc.inference(X, f.U, f.V, f.P, f.W_res, lam, g["B"], g["T"])
        np.testing.assert_allclose(Y, want, rtol=0, atol=1e-14)
    f = orc.offline_prepare_from_svd(np.eye(3), np.array([3.0, 2.0, 1.0]), np.eye(3), 1, 1, lam)
    np.testing.assert_allclose(f.P, [[float(Fraction(v[0]))] for v in g["P"]], atol=1e-15)
    yd = np.array([[float(Fraction(v)) for v in row] for row in g["Y_dense"]])
    np.testing.assert_allclose(orc.dense(X, W), yd, atol=0)


def test_inference_rows_matches_full():
    """Row sampling evaluates the same per-instance fit as the whole-matrix path."""
    w = small_layer(B=4, T=6)
    f = factors(w, 4, 3, 1e-3)
    full = orc.inference(w.X, f.U, f.V, f.P, f.W_res, 1e-3, 4, 6)
    rows = np.array([23, 0, 5, 6, 17, 11])
    got = orc.inference_rows(w.X, f.U, f.V, f.P, f.W_res, 1e-3, 4, 6, rows)
    np.testing.assert_allclose(got, full[rows], rtol=0, atol=1e-13)


def test_error_report_orders():
    w = small_layer(B=2, T=12)
    f = factors(w, 4, 3, 1e-3)
    rep = orc.error_report(w.X, w.weight(), f, 1e-3, 2, 12)
    assert 0 < rep["err_dyra"] < rep["err_wo"] < 1


def test_round_to_bf16():
    """Round-to-nearest-even onto bf16 (8-bit mantissa): exact values stay,
    halfway cases go to the even neighbour, torch agrees on random data."""
    import torch
    vals = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 0.0, 1e-30, 3.0e38])
    got = orc.round_to(vals, "bf16")
    assert got[0] == 1.0 and got[1] == 1.0 and got[2] == 1.0 + 2 ** -6 and got[3] == -2.5
    x = np.random.default_rng(0).standard_normal(10000) * 10.0
    t = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(orc.round_to(x, "bf16"), t)


# ------------------------------------------------------ planted bugs ----

def _mutants():
    """Oracle variants with one plausible mistake each."""
    def drop_ridge(X, U, V, P, W_res, lam, B, T):
        return orc.inference(X, U, V, P, W_res, 0.0, B, T)

    def wrong_sign(X, U, V, P, W_res, lam, B, T):
        Y = orc.inference(X, U, V, P, W_res, lam, B, T)
        Ywo = (X @ V) @ U.T
        return Ywo - (Y - Ywo)

    def global_instance(X, U, V, P, W_res, lam, B, T):
        return orc.inference(X, U, V, P, W_res, lam, 1, B * T)

    def dropped_gram(X, U, V, P, W_res, lam, B, T):
        Y = np.empty((X.shape[0], U.shape[0]))
        for b in range(B):
            Xb = X[b * T:(b + 1) * T]
            L = Xb @ P
            Y[b * T:(b + 1) * T] = (Xb @ V) @ U.T + L @ ((L.T @ Xb) @ W_res.T)
        return Y

    def transposed_static(X, U, V, P, W_res, lam, B, T):
        Y = orc.inference(X, U, V, P, W_res, lam, B, T)
        return Y - (X @ V) @ U.T + (X @ V[:, ::-1]) @ U.T

    def half_correction(X, U, V, P, W_res, lam, B, T):
        Y = orc.inference(X, U, V, P, W_res, lam, B, T)
        Ywo = (X @ V) @ U.T
        return Ywo + 0.5 * (Y - Ywo)

    def lam_on_wrong_gram(X, U, V, P, W_res, lam, B, T):
        k = P.shape[1]
        Y = np.empty((X.shape[0], U.shape[0]))
        for b in range(B):
            Xb = X[b * T:(b + 1) * T]
            L = Xb @ P
            G = L.T @ L + (lam + 1.0) * np.eye(k)
            Y[b * T:(b + 1) * T] = (Xb @ V) @ U.T + L @ np.linalg.solve(G, (L.T @ Xb) @ W_res.T)
        return Y

    return [drop_ridge, wrong_sign, global_instance, dropped_gram, transposed_static,
            half_correction, lam_on_wrong_gram]


@pytest.mark.parametrize("mutant", _mutants(), ids=lambda m: m.__name__)
def test_planted_mistakes_are_caught(mutant):
    failures = 0
    for pin in PINS:
        try:
            pin(infer=mutant)
        except AssertionError:
            failures += 1
        except np.linalg.LinAlgError:
            failures += 1
    assert failures > 0, "no pin catches the planted mistake %s" % mutant.__name__
