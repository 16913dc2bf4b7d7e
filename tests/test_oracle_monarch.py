"""Pins of the oracle's Monarch static part (DyRA App. B) and of DyRA on top of it.

Paper: "DyRA: Dynamic Residual Approximation for Efficient Matrix
Multiplication in DNNs", Appendix B ("Monarch Matrix") and Sec. 2.3 (DyRA
corrects any structured static part).

The pins check the oracle against facts that do not depend on how it is
written:
- the entry formula a hand derivation gives for P L P^T R, element by element;
- exact recovery of a Monarch matrix;
- degenerate block counts (b1 = 1 or b2 = 1), where every matrix is Monarch;
- the block-wise Eckart-Young error, with the top singular value computed by
  power iteration rather than by an SVD;
- local optimality under perturbation of the factors;
- the DyRA invariants on the Monarch base: k = 0, a fully covered residual,
  and never worse than weight-only.
test_planted_monarch_mistakes_are_caught swaps mistaken copies into the
module and checks that some pin fails for each.
"""

import numpy as np
import pytest

from oracle import dyra_oracle as orc
from oracle import monarch as mon
from synth import LayerSpec, generate


def random_blocks(b1, b2, seed):
    rng = np.random.default_rng(seed)
    return ([rng.standard_normal((b1, b1)) for _ in range(b2)],
            [rng.standard_normal((b2, b2)) for _ in range(b1)])


def square_layer(N, k, B=2, T=9, seed=0, lam=1e-3):
    s = LayerSpec("mon", N, N, 1, k, B, T, "f32", 0.5, "lognormal", seed=seed, lam=lam)
    return s, generate(s)


def top_singular_value(S, iters=500):
    """Power iteration on S^T S (no SVD routine)."""
    v = np.ones(S.shape[1]) / np.sqrt(S.shape[1])
    for _ in range(iters):
        w = S.T @ (S @ v)
        v = w / np.linalg.norm(w)
    return np.linalg.norm(S @ v)


# ---------------------------------------------------------------- pins ----

def check_entry_formula():
    """Entry (m1*b2 + j2, j1*b2 + i2) of P L P^T R is L_j2[m1, j1] R_j1[j2, i2]."""
    for b1, b2 in ((3, 4), (2, 5), (4, 4)):
        Lb, Rb = random_blocks(b1, b2, seed=b1 * 10 + b2)
        W = mon.monarch_matrix(Lb, Rb)
        for m1 in range(b1):
            for j2 in range(b2):
                for j1 in range(b1):
                    for i2 in range(b2):
                        want = Lb[j2][m1, j1] * Rb[j1][j2, i2]
                        assert abs(W[m1 * b2 + j2, j1 * b2 + i2] - want) <= 1e-12


def check_shuffle_is_a_permutation():
    for b1, b2 in ((3, 4), (1, 5), (5, 1)):
        P = mon.shuffle(b1, b2)
        np.testing.assert_array_equal(P @ P.T, np.eye(b1 * b2))
        assert set(np.unique(P)) <= {0.0, 1.0}


def check_recovers_monarch_matrices():
    for b1, b2 in ((3, 4), (2, 5), (4, 4)):
        W = mon.monarch_matrix(*random_blocks(b1, b2, seed=7 + b1))
        Lb, Rb = mon.monarch_project(W, b1, b2)
        np.testing.assert_allclose(mon.monarch_matrix(Lb, Rb), W, rtol=0, atol=1e-11)


def check_degenerate_block_counts_are_exact():
    """b1 = 1: L is diagonal and R one N x N block; b2 = 1: L one block and R
    diagonal. Either way every N x N matrix is Monarch."""
    rng = np.random.default_rng(3)
    for b1, b2 in ((1, 6), (6, 1)):
        W = rng.standard_normal((6, 6))
        Lb, Rb = mon.monarch_project(W, b1, b2)
        np.testing.assert_allclose(mon.monarch_matrix(Lb, Rb), W, rtol=0, atol=1e-12)


def check_blockwise_eckart_young():
    """||W - W_hat||^2 = sum over the (j1, j2) blocks S of ||S||^2 - s1(S)^2."""
    b1, b2 = 3, 4
    W = np.random.default_rng(5).standard_normal((12, 12))
    Lb, Rb = mon.monarch_project(W, b1, b2)
    err = np.sum((W - mon.monarch_matrix(Lb, Rb)) ** 2)
    want = 0.0
    for j1 in range(b1):
        for j2 in range(b2):
            S = np.array([[W[m1 * b2 + j2, j1 * b2 + i2] for i2 in range(b2)] for m1 in range(b1)])
            want += np.sum(S ** 2) - top_singular_value(S) ** 2
    assert err == pytest.approx(want, rel=1e-9)


def check_locally_optimal():
    """No small perturbation of the projected factors lowers the error."""
    b1, b2 = 3, 4
    rng = np.random.default_rng(6)
    W = rng.standard_normal((12, 12))
    Lb, Rb = mon.monarch_project(W, b1, b2)
    best = np.sum((W - mon.monarch_matrix(Lb, Rb)) ** 2)
    for _ in range(50):
        Lp = [L + 1e-3 * rng.standard_normal(L.shape) for L in Lb]
        Rp = [R + 1e-3 * rng.standard_normal(R.shape) for R in Rb]
        assert np.sum((W - mon.monarch_matrix(Lp, Rp)) ** 2) >= best * (1 - 1e-12)


def check_dyra_k0_is_the_monarch_product():
    s, w = square_layer(12, 0)
    f = mon.offline_prepare_monarch(w.weight(), 3, 4, 0, s.lam)
    Y = mon.monarch_inference(w.X, f, s.lam, s.B, s.T)
    np.testing.assert_allclose(Y, w.X @ mon.monarch_matrix(f.Lb, f.Rb), rtol=0, atol=1e-12)


def check_dyra_full_residual_is_exact():
    """k = N and lam = 0 with T >= N: col(X P) = col(X_b) holds the residual
    output X_b W_res^T, so the correction restores X W^T."""
    s, w = square_layer(12, 12, T=20, lam=0.0, seed=1)
    f = mon.offline_prepare_monarch(w.weight(), 3, 4, 12, 0.0)
    Y = mon.monarch_inference(w.X, f, 0.0, s.B, s.T)
    Yd = w.X @ w.weight().T
    np.testing.assert_allclose(Y, Yd, rtol=0, atol=1e-9 * np.abs(Yd).max())


def check_dyra_never_worse_than_weight_only():
    s, w = square_layer(12, 3, seed=2)
    f = mon.offline_prepare_monarch(w.weight(), 3, 4, 3, s.lam)
    Y = mon.monarch_inference(w.X, f, s.lam, s.B, s.T)
    Yd = w.X @ w.weight().T
    Ywo = w.X @ f.What.T
    for b in range(s.B):
        rows = slice(b * s.T, (b + 1) * s.T)
        assert np.linalg.norm(Yd[rows] - Y[rows]) <= np.linalg.norm(Yd[rows] - Ywo[rows]) * (1 + 1e-12)
    # and the static part is the Monarch product of the weight's projection
    np.testing.assert_allclose(f.What, mon.monarch_matrix(*mon.monarch_project(w.weight().T, 3, 4)).T,
                               rtol=0, atol=1e-12)


# ------------------------------------------- rectangular blocks (reading) ----

RECT = ((3, 4, 2, 5), (2, 3, 4, 2), (1, 4, 3, 2))  # b1, b2, b1', b2'


def rect_blocks(b1, b2, b1o, b2o, seed):
    rng = np.random.default_rng(seed)
    return ([rng.standard_normal((b1, b1o)) for _ in range(b2)],
            [rng.standard_normal((b2, b2o)) for _ in range(b1o)])


def check_rect_entry_formula():
    """Entry (m1*b2 + j2, j1*b2' + i2) of P1 L P2^T R is L_j2[m1, j1] R_j1[j2, i2]
    for rectangular blocks, element by element (a c1 x c2 matrix)."""
    for b1, b2, b1o, b2o in RECT:
        Lb, Rb = rect_blocks(b1, b2, b1o, b2o, seed=b1 + 10 * b2 + 100 * b1o)
        W = mon.monarch_matrix(Lb, Rb)
        assert W.shape == (b1 * b2, b1o * b2o)
        for m1 in range(b1):
            for j2 in range(b2):
                for j1 in range(b1o):
                    for i2 in range(b2o):
                        want = Lb[j2][m1, j1] * Rb[j1][j2, i2]
                        assert abs(W[m1 * b2 + j2, j1 * b2o + i2] - want) <= 1e-12


def check_rect_recovery_and_blockwise_eckart_young():
    """A rectangular Monarch matrix is its own projection; for any matrix the
    projection error is the sum over the b1 x b2' blocks of ||S||^2 - s1(S)^2,
    with s1 by power iteration."""
    rng = np.random.default_rng(8)
    for b1, b2, b1o, b2o in RECT:
        M = mon.monarch_matrix(*rect_blocks(b1, b2, b1o, b2o, seed=3))
        np.testing.assert_allclose(mon.monarch_matrix(*mon.monarch_project(M, b1, b2, b1o, b2o)), M,
                                   rtol=0, atol=1e-10 * max(1.0, np.abs(M).max()))
        W = rng.standard_normal((b1 * b2, b1o * b2o))
        err = np.sum((W - mon.monarch_matrix(*mon.monarch_project(W, b1, b2, b1o, b2o))) ** 2)
        want = 0.0
        for j1 in range(b1o):
            for j2 in range(b2):
                S = np.array([[W[m1 * b2 + j2, j1 * b2o + i2] for i2 in range(b2o)]
                              for m1 in range(b1)])
                want += np.sum(S ** 2) - top_singular_value(S, iters=2000) ** 2
        assert err == pytest.approx(want, rel=1e-8, abs=1e-10)


def check_rect_dyra_invariants():
    """DyRA on a rectangular Monarch part (d_in = b1 b2, d_out = b1' b2'):
    k = 0 is the Monarch product, and no instance is worse than weight-only."""
    b1, b2, b1o, b2o = 3, 4, 2, 5
    s = LayerSpec("monr", b1 * b2, b1o * b2o, 1, 3, 2, 9, "f32", 0.5, "lognormal", seed=4)
    w = generate(s)
    f0 = mon.offline_prepare_monarch(w.weight(), b1, b2, 0, s.lam, b1o=b1o, b2o=b2o)
    Y0 = mon.monarch_inference(w.X, f0, s.lam, s.B, s.T)
    np.testing.assert_allclose(Y0, w.X @ mon.monarch_matrix(f0.Lb, f0.Rb), rtol=0, atol=1e-12)
    f = mon.offline_prepare_monarch(w.weight(), b1, b2, 3, s.lam, b1o=b1o, b2o=b2o)
    Y = mon.monarch_inference(w.X, f, s.lam, s.B, s.T)
    Yd = w.X @ w.weight().T
    Ywo = w.X @ f.What.T
    for b in range(s.B):
        rows = slice(b * s.T, (b + 1) * s.T)
        assert np.linalg.norm(Yd[rows] - Y[rows]) <= np.linalg.norm(Yd[rows] - Ywo[rows]) * (1 + 1e-12)


PINS = [check_entry_formula, check_shuffle_is_a_permutation, check_recovers_monarch_matrices,
        check_degenerate_block_counts_are_exact, check_blockwise_eckart_young, check_locally_optimal,
        check_dyra_k0_is_the_monarch_product, check_dyra_full_residual_is_exact,
        check_dyra_never_worse_than_weight_only, check_rect_entry_formula,
        check_rect_recovery_and_blockwise_eckart_young, check_rect_dyra_invariants]


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_monarch_pin(pin):
    pin()


def test_rejects_a_shape_that_does_not_match_the_blocks():
    with pytest.raises(ValueError):
        mon.monarch_project(np.zeros((12, 8)), 3, 4)
    with pytest.raises(ValueError):
        mon.monarch_project(np.zeros((12, 12)), 3, 4, 2, 5)


def test_rect_parameter_count():
    """b2 blocks of b1 x b1' and b1' blocks of b2 x b2'."""
    W = np.random.default_rng(0).standard_normal((12, 10))
    Lb, Rb = mon.monarch_project(W, 3, 4, 2, 5)
    assert len(Lb) == 4 and all(L.shape == (3, 2) for L in Lb)
    assert len(Rb) == 2 and all(R.shape == (4, 5) for R in Rb)


def test_parameter_count():
    """N (b1 + b2) parameters: b2 blocks of b1 x b1 and b1 blocks of b2 x b2."""
    Lb, Rb = mon.monarch_project(np.random.default_rng(0).standard_normal((12, 12)), 3, 4)
    assert len(Lb) == 4 and all(L.shape == (3, 3) for L in Lb)
    assert len(Rb) == 3 and all(R.shape == (4, 4) for R in Rb)
    assert sum(L.size for L in Lb) + sum(R.size for R in Rb) == 12 * (3 + 4)


# ------------------------------------------------------ planted bugs ----

_SHUFFLE, _PROJECT, _MATRIX = mon.shuffle, mon.monarch_project, mon.monarch_matrix


def _identity_shuffle(b1, b2):
    return np.eye(b1 * b2)


def _contiguous_rows(Wp, b1, b2, b1o=None, b2o=None):
    """Takes rows j2*b1 .. j2*b1 + b1 - 1 instead of the strided ones."""
    b1o = b1 if b1o is None else b1o
    b2o = b2 if b2o is None else b2o
    Lb = [np.zeros((b1, b1o)) for _ in range(b2)]
    Rb = [np.zeros((b2, b2o)) for _ in range(b1o)]
    for j1 in range(b1o):
        for j2 in range(b2):
            u, s, vt = np.linalg.svd(Wp[j2 * b1:(j2 + 1) * b1, j1 * b2o:(j1 + 1) * b2o])
            Lb[j2][:, j1] = np.sqrt(s[0]) * u[:, 0]
            Rb[j1][j2, :] = np.sqrt(s[0]) * vt[0]
    return Lb, Rb


def _sigma_twice(Wp, b1, b2, b1o=None, b2o=None):
    Lb, Rb = _PROJECT(Wp, b1, b2, b1o, b2o)
    return [L * 1.0 for L in Lb], [R * 2.0 for R in Rb]


def _swapped_factors(Lb, Rb):
    b2, b1 = len(Lb), len(Rb)
    P = _SHUFFLE(b1, b2)
    return P @ mon.block_diag(Rb) @ P.T @ mon.block_diag(Lb) if b1 == b2 else _MATRIX(Lb, Rb).T


MUTANTS = [("shuffle", _identity_shuffle), ("monarch_project", _contiguous_rows),
           ("monarch_project", _sigma_twice), ("monarch_matrix", _swapped_factors)]


@pytest.mark.parametrize("target,mutant", MUTANTS, ids=lambda m: getattr(m, "__name__", m))
def test_planted_monarch_mistakes_are_caught(monkeypatch, target, mutant):
    monkeypatch.setattr(mon, target, mutant)
    failures = 0
    for pin in PINS:
        try:
            pin()
        except (AssertionError, ValueError, np.linalg.LinAlgError):
            failures += 1
    assert failures > 0, "no pin catches the planted mistake %s" % mutant.__name__


# ------------------------------------------------ over random block counts ----

from hypothesis import given, settings  # noqa: E402
from hypothesis import strategies as st  # noqa: E402


@settings(max_examples=30, deadline=None, derandomize=True)
@given(st.integers(1, 5), st.integers(1, 5), st.integers(0, 10_000))
def test_projection_properties_over_block_counts(b1, b2, seed):
    """For any b1, b2: a Monarch matrix is its own projection, and the
    projection error is the block-wise Eckart-Young sum."""
    rng = np.random.default_rng(seed)
    N = b1 * b2
    Lb = [rng.standard_normal((b1, b1)) for _ in range(b2)]
    Rb = [rng.standard_normal((b2, b2)) for _ in range(b1)]
    M = mon.monarch_matrix(Lb, Rb)
    np.testing.assert_allclose(mon.monarch_matrix(*mon.monarch_project(M, b1, b2)), M, rtol=0,
                               atol=1e-10 * max(1.0, np.abs(M).max()))
    W = rng.standard_normal((N, N))
    err = np.sum((W - mon.monarch_matrix(*mon.monarch_project(W, b1, b2))) ** 2)
    want = 0.0
    for j1 in range(b1):
        for j2 in range(b2):
            S = np.array([[W[m1 * b2 + j2, j1 * b2 + i2] for i2 in range(b2)] for m1 in range(b1)])
            want += np.sum(S ** 2) - top_singular_value(S, iters=2000) ** 2
    assert err == pytest.approx(want, rel=1e-7, abs=1e-9)
