"""Pins of the oracle's multi-step ALS and of the Gaussian ALS start.

Paper: "DyRA: Dynamic Residual Approximation for Efficient Matrix
Multiplication in DNNs", Sec. 2.2 (Eq. 3-5 and footnote 2: the residual
output X W_res is fitted by alternating ridge least squares; Fig. 2 starts
from a Gaussian R^(0)) and Sec. 3.3, Fig. 9 right (t = 1, 1.5, 2 iterations).

As in test_oracle.py, no pin re-types the oracle's update formulas: each
checks them against an optimality condition, a monotonicity property of
alternating minimisation, the Eckart-Young optimum they converge to, a closed
form, exact rational arithmetic of the rank-1 case worked by hand, or a
least-squares solve of the augmented system by another routine.
test_planted_als_mistakes_are_caught swaps a mistaken copy into the oracle
module and checks that some pin fails.
"""

import numpy as np
import pytest
import torch

from oracle import dyra_oracle as orc
from rank_structured_matmul_b200 import prep
from synth import LayerSpec, gaussian_r0, generate, haar_orthonormal


def layer(d_in=16, d_out=12, r=3, k=3, B=2, T=10, seed=0, x_kind="lognormal"):
    s = LayerSpec("als", d_in, d_out, r, k, B, T, "f32", 0.6, x_kind, n_outlier=2,
                  outlier_scale=10.0, seed=seed)
    return s, generate(s)


def factors(w, s, lam, start="svd"):
    R0 = gaussian_r0(s.k, s.d_out, s.seed) if start == "gauss" else None
    return orc.offline_prepare_from_svd(w.left, w.sigma, w.right, s.r, s.k, lam, R0=R0)


def objective(E, L, R, lam):
    """The ridge objective both updates minimise (Eq. 3 plus footnote 2)."""
    return np.sum((E - L @ R) ** 2) + lam * (np.sum(L ** 2) + np.sum(R ** 2))


def gapped_instance(T=12, d_out=10, k=3, seed=5):
    """X_b (T x T, invertible) and W_res (d_out x T) whose residual output
    E = X_b W_res^T has the singular values 5, 4, 3 | 1, 0.6, 0.4, ... (a gap
    of 3 after the k-th), so alternating minimisation converges fast."""
    rng = np.random.default_rng(seed)
    Xb = rng.standard_normal((T, T)) + 3.0 * np.eye(T)
    s = np.concatenate([[5.0, 4.0, 3.0], np.geomspace(1.0, 0.05, d_out - 3)])
    E = haar_orthonormal(rng, T, d_out) @ np.diag(s) @ haar_orthonormal(rng, d_out, d_out).T
    W_res = np.linalg.solve(Xb, E).T
    return Xb, W_res, E, s


# ---------------------------------------------------------------- pins ----

def check_t1_is_algorithm_1():
    """t = 1 is Alg. 1: with P_L from the same start, the one-step layer."""
    for start in ("svd", "gauss"):
        for lam in (0.0, 1e-3):
            s, w = layer(seed=1)
            f = factors(w, s, lam, start)
            a = orc.als_inference(w.X, f.U, f.V, f.W_res, f.R0, lam, s.B, s.T, 1)
            b = orc.inference(w.X, f.U, f.V, f.P, f.W_res, lam, s.B, s.T)
            np.testing.assert_allclose(a, b, rtol=0, atol=1e-11 * np.abs(b).max())


def check_t0_is_weight_only():
    s, w = layer(seed=2)
    f = factors(w, s, 1e-3, "gauss")
    Y = orc.als_inference(w.X, f.U, f.V, f.W_res, f.R0, 1e-3, s.B, s.T, 0)
    np.testing.assert_allclose(Y, w.X @ f.V @ f.U.T, rtol=0, atol=1e-12)


def check_half_step_closed_form():
    """t = 0.5 ends on the first left update. With the singular-vector start
    (orthonormal rows, R0 R0^T = I) the fit is L R0 = E R0^T R0 / (1 + lam):
    the residual output projected on the start's row space, shrunk by the
    ridge."""
    s, w = layer(seed=3)
    for lam in (0.0, 0.25):
        f = factors(w, s, lam, "svd")
        np.testing.assert_allclose(f.R0 @ f.R0.T, np.eye(s.k), atol=1e-12)
        Y = orc.als_inference(w.X, f.U, f.V, f.W_res, f.R0, lam, s.B, s.T, 0.5)
        E = w.X @ f.W_res.T
        want = w.X @ f.V @ f.U.T + E @ f.R0.T @ f.R0 / (1.0 + lam)
        np.testing.assert_allclose(Y, want, rtol=0, atol=1e-11 * np.abs(want).max())


def check_half_steps_are_ridge_minimisers():
    """Each half-step zeroes the objective's gradient in the factor it
    updates and leaves the other factor as it was."""
    s, w = layer(seed=4)
    for lam in (0.0, 1e-3, 0.5):
        f = factors(w, s, lam, "gauss")
        Xb = w.X[: s.T]
        E = Xb @ f.W_res.T
        prev_L, prev_R = None, f.R0
        for h, (L, R) in enumerate(orc.als_half_steps(Xb, f.W_res, f.R0, lam, 7)):
            scale = np.linalg.norm(E) * (np.linalg.norm(L) + np.linalg.norm(R))
            if h % 2 == 0:
                grad = (L @ R - E) @ R.T + lam * L
                np.testing.assert_array_equal(R, prev_R)
            else:
                grad = L.T @ (L @ R - E) + lam * R
                np.testing.assert_array_equal(L, prev_L)
            assert np.linalg.norm(grad) <= 1e-11 * scale, (h, lam)
            prev_L, prev_R = L, R


def check_objective_never_increases():
    """Alternating exact minimisation cannot raise the ridge objective; with
    lam = 0 that objective is the fit error itself."""
    s, w = layer(seed=6, x_kind="outlier")
    for lam in (0.0, 1e-3, 0.5):
        f = factors(w, s, lam, "gauss")
        for b in range(s.B):
            Xb = w.X[b * s.T:(b + 1) * s.T]
            E = Xb @ f.W_res.T
            J = [objective(E, L, R, lam) for L, R in orc.als_half_steps(Xb, f.W_res, f.R0, lam, 12)]
            assert all(J[i + 1] <= J[i] * (1 + 1e-12) + 1e-300 for i in range(len(J) - 1)), (lam, J)


def check_converges_to_eckart_young():
    """lam = 0 from a Gaussian start: the fit reaches the optimal rank-k error
    (Eckart-Young, the bound cited in Sec. 2.2) and the product reaches the
    truncated SVD of E."""
    Xb, W_res, E, sv = gapped_instance()
    k = 3
    R0 = gaussian_r0(k, E.shape[1], seed=11)
    L, R = orc.als_half_steps(Xb, W_res, R0, 0.0, 60)[-1]
    best = np.sqrt(np.sum(sv[k:] ** 2))
    assert abs(np.linalg.norm(E - L @ R) - best) <= 1e-9 * best
    A, s, Bt = np.linalg.svd(E, full_matrices=False)
    Ek = (A[:, :k] * s[:k]) @ Bt[:k]
    np.testing.assert_allclose(L @ R, Ek, rtol=0, atol=1e-8 * np.abs(Ek).max())


def check_matches_augmented_lstsq():
    """Brute force: each update as a least-squares solve of the stacked
    system [factor; sqrt(lam) I] x = [E; 0] by numpy's SVD-based lstsq."""
    s, w = layer(d_in=9, d_out=7, r=2, k=2, B=1, T=6, seed=7)
    for lam in (0.0, 1e-3, 0.3):
        for start in ("svd", "gauss"):
            f = factors(w, s, lam, start)
            Xb = w.X
            E = Xb @ f.W_res.T
            k = s.k
            R = f.R0
            got = orc.als_half_steps(Xb, f.W_res, f.R0, lam, 4)
            for h in range(4):
                if h % 2 == 0:   # min_L ||E - L R||^2 + lam ||L||^2, as L^T rows
                    A = np.vstack([R.T, np.sqrt(lam) * np.eye(k)])
                    rhs = np.vstack([E.T, np.zeros((k, E.shape[0]))])
                    L = np.linalg.lstsq(A, rhs, rcond=None)[0].T
                else:            # min_R ||E - L R||^2 + lam ||R||^2
                    A = np.vstack([L, np.sqrt(lam) * np.eye(k)])
                    rhs = np.vstack([E, np.zeros((k, E.shape[1]))])
                    R = np.linalg.lstsq(A, rhs, rcond=None)[0]
                gl, gr = got[h]
                np.testing.assert_allclose(gl, L, rtol=0, atol=1e-9 * np.abs(L).max())
                np.testing.assert_allclose(gr, R, rtol=0, atol=1e-9 * np.abs(R).max())


def check_never_worse_than_weight_only():
    """Every ALS update is a ridge minimiser for which the zero factor is
    feasible, so ||E - L R|| <= ||E|| after any number of half-steps: no t is
    worse than the weight-only layer, per instance."""
    s, w = layer(seed=8, x_kind="outlier")
    lam = 1e-3
    for start in ("svd", "gauss"):
        f = factors(w, s, lam, start)
        Wd = f.U @ f.V.T + f.W_res
        for t in (0.5, 1, 1.5, 2, 3):
            Y = orc.als_inference(w.X, f.U, f.V, f.W_res, f.R0, lam, s.B, s.T, t)
            for b in range(s.B):
                rows = slice(b * s.T, (b + 1) * s.T)
                Yd = w.X[rows] @ Wd.T
                Ywo = w.X[rows] @ f.V @ f.U.T
                assert np.linalg.norm(Yd - Y[rows]) <= np.linalg.norm(Yd - Ywo) * (1 + 1e-12)


def check_iteration_count():
    """t counts (left, right) pairs: t = 2 equals running t = 1 and then one
    more pair from the R^(1) it produced; t = 1.5 stops after that pair's left
    update."""
    s, w = layer(seed=9)
    lam = 1e-3
    f = factors(w, s, lam, "gauss")
    Xb = w.X[: s.T]
    L1, R1 = orc.als_half_steps(Xb, f.W_res, f.R0, lam, 2)[-1]
    L2, R2 = orc.als_half_steps(Xb, f.W_res, R1, lam, 2)[-1]
    base = Xb @ f.V @ f.U.T
    for t, want in ((1, base + L1 @ R1), (1.5, base + L2 @ R1), (2, base + L2 @ R2)):
        Y = orc.als_inference(Xb, f.U, f.V, f.W_res, f.R0, lam, 1, s.T, t)
        np.testing.assert_allclose(Y, want, rtol=0, atol=1e-11 * np.abs(want).max())


def check_rank1_exact_rationals():
    """k = 1 by hand: each update is a scalar ridge regression,
    L_i = sum_j E_ij R_j / (sum_j R_j^2 + lam) and
    R_j = sum_i L_i E_ij / (sum_i L_i^2 + lam),
    run here in exact rational arithmetic on a 3 x 2 residual output."""
    from fractions import Fraction as F
    Wres = [[3, 1, 0], [0, 2, 1]]                    # d_out x d_in
    E = [[F(Wres[j][i]) for j in range(2)] for i in range(3)]   # X_b = I: E = W_res^T
    for lam in (F(0), F(1, 2)):
        R = [F(1), F(-2)]
        L = None
        want = []
        for h in range(5):
            if h % 2 == 0:
                den = sum(r * r for r in R) + lam
                L = [sum(E[i][j] * R[j] for j in range(2)) / den for i in range(3)]
            else:
                den = sum(l * l for l in L) + lam
                R = [sum(L[i] * E[i][j] for i in range(3)) / den for j in range(2)]
            want.append((list(L), list(R)))
        got = orc.als_half_steps(np.eye(3), np.array(Wres, dtype=np.float64),
                                 np.array([[1.0, -2.0]]), float(lam), 5)
        for (wl, wr), (gl, gr) in zip(want, got):
            np.testing.assert_allclose(gl[:, 0], [float(x) for x in wl], rtol=1e-13, atol=0)
            np.testing.assert_allclose(gr[0], [float(x) for x in wr], rtol=1e-13, atol=0)


def check_t15_closed_form():
    """t = 1.5 by hand from Alg. 1's quantities. With G = L^T L + lam I,
    Q = (L^T X_b) W_res^T and S = Q Q^T, the second L update simplifies to
    L(2) = X_b (Q W_res)^T (S + lam G^2)^-1 G, and the output adds L(2) R(1)
    = X_b (Q W_res)^T (S + lam G^2)^-1 Q."""
    s, w = layer(seed=12, x_kind="outlier")
    for lam in (0.0, 1e-3, 0.05):
        f = factors(w, s, lam, "gauss")
        Y = orc.als_inference(w.X, f.U, f.V, f.W_res, f.R0, lam, s.B, s.T, 1.5)
        for b in range(s.B):
            Xb = w.X[b * s.T:(b + 1) * s.T]
            L = Xb @ f.P
            G = L.T @ L + lam * np.eye(s.k)
            Q = (L.T @ Xb) @ f.W_res.T
            M = (Xb @ (Q @ f.W_res).T) @ np.linalg.inv(Q @ Q.T + lam * G @ G)
            want = Xb @ f.V @ f.U.T + M @ Q
            got = Y[b * s.T:(b + 1) * s.T]
            np.testing.assert_allclose(got, want, rtol=0, atol=1e-10 * np.abs(want).max())
            L2 = orc.als_half_steps(Xb, f.W_res, f.R0, lam, 3)[-1][0]
            np.testing.assert_allclose(L2, M @ G, rtol=0, atol=1e-10 * np.abs(L2).max())


PINS = [check_rank1_exact_rationals, check_t15_closed_form, check_t1_is_algorithm_1, check_t0_is_weight_only, check_half_step_closed_form,
        check_half_steps_are_ridge_minimisers, check_objective_never_increases,
        check_converges_to_eckart_young, check_matches_augmented_lstsq,
        check_never_worse_than_weight_only, check_iteration_count]


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_als_pin(pin):
    pin()


# ------------------------------------------------------ the Gaussian start ----

def test_gaussian_start_draw():
    """Seeded, of the asked shape, N(0, 1/d_out) entries (rows of squared norm
    about 1), and independent of the layer's own draws."""
    a = gaussian_r0(8, 4096, seed=0)
    assert a.shape == (8, 4096)
    np.testing.assert_array_equal(a, gaussian_r0(8, 4096, seed=0))
    assert not np.array_equal(a, gaussian_r0(8, 4096, seed=1))
    sd = 1.0 / np.sqrt(4096)
    assert abs(a.mean()) < 5 * sd / np.sqrt(a.size)
    assert abs(a.std() / sd - 1.0) < 0.02
    assert np.allclose(np.sum(a ** 2, axis=1), 1.0, atol=0.1)
    s, w1 = layer(seed=0)
    _, w2 = layer(seed=0)
    np.testing.assert_array_equal(w1.X, w2.X)


def test_prep_takes_a_given_start():
    """The library's host preparation and the oracle agree on P for a given
    start, from the SVD route and from the dense weight."""
    s, w = layer(seed=10)
    lam = 1e-3
    R0 = gaussian_r0(s.k, s.d_out, 10)
    a = prep.prepare_from_svd(w.left, w.sigma, w.right, s.r, s.k, lam, R0=R0)
    b = orc.offline_prepare_from_svd(w.left, w.sigma, w.right, s.r, s.k, lam, R0=R0)
    np.testing.assert_allclose(a.P.numpy(), b.P, atol=1e-12)
    c = prep.prepare_from_weight(torch.from_numpy(w.weight()), s.r, s.k, lam, R0=R0)
    # the static factors' signs may differ between SVD routes; the residual and P do not
    np.testing.assert_allclose(c.W_res.numpy(), b.W_res, atol=1e-12)
    np.testing.assert_allclose(c.P.numpy(), b.P, atol=1e-10)
    with pytest.raises(ValueError):
        prep.prepare_from_svd(w.left, w.sigma, w.right, s.r, s.k, lam, R0=R0[:, :-1])
    with pytest.raises(ValueError):
        orc.offline_prepare_from_svd(w.left, w.sigma, w.right, s.r, s.k, lam, R0=R0[:-1])


# ------------------------------------------------------ planted bugs ----

def _half_mutants():
    def no_ridge_left(Xb, W_res, R0, lam, steps):
        out, R, L = [], R0, None
        for h in range(steps):
            if h % 2 == 0:
                L = np.linalg.solve(R @ R.T, (Xb @ W_res.T @ R.T).T).T
            else:
                R = np.linalg.solve(L.T @ L + lam * np.eye(R0.shape[0]), L.T @ Xb @ W_res.T)
            out.append((L, R))
        return out

    def right_first(Xb, W_res, R0, lam, steps):
        L0 = Xb @ W_res.T @ R0.T
        out, L, R = [], L0, R0
        for h in range(steps):
            if h % 2 == 1:
                L = np.linalg.solve(R @ R.T + lam * np.eye(R0.shape[0]), (Xb @ W_res.T @ R.T).T).T
            else:
                R = np.linalg.solve(L.T @ L + lam * np.eye(R0.shape[0]), L.T @ Xb @ W_res.T)
            out.append((L, R))
        return out

    def stale_gram(Xb, W_res, R0, lam, steps):
        out, R, L = [], R0, None
        G0 = R0 @ R0.T + lam * np.eye(R0.shape[0])
        for h in range(steps):
            if h % 2 == 0:
                L = np.linalg.solve(G0, (Xb @ W_res.T @ R.T).T).T
            else:
                R = np.linalg.solve(L.T @ L + lam * np.eye(R0.shape[0]), L.T @ Xb @ W_res.T)
            out.append((L, R))
        return out

    def unsolved_left(Xb, W_res, R0, lam, steps):
        out, R, L = [], R0, None
        for h in range(steps):
            if h % 2 == 0:
                L = Xb @ W_res.T @ R.T
            else:
                R = np.linalg.solve(L.T @ L + lam * np.eye(R0.shape[0]), L.T @ Xb @ W_res.T)
            out.append((L, R))
        return out

    return [no_ridge_left, right_first, stale_gram, unsolved_left]


def _count_mutant(X, U, V, W_res, R0, lam, B, T, t):
    """Counts iterations as half-steps (t = 1 would run only L)."""
    Y = np.empty((X.shape[0], U.shape[0]))
    for b in range(B):
        Xb = X[b * T:(b + 1) * T]
        L, R = orc.als_half_steps(Xb, W_res, R0, lam, max(1, int(2 * t) - 1))[-1]
        Y[b * T:(b + 1) * T] = Xb @ V @ U.T + L @ R
    return Y


MUTANTS = [("als_half_steps", m) for m in _half_mutants()] + [("als_inference", _count_mutant)]


@pytest.mark.parametrize("target,mutant", MUTANTS, ids=lambda m: getattr(m, "__name__", m))
def test_planted_als_mistakes_are_caught(monkeypatch, target, mutant):
    monkeypatch.setattr(orc, target, mutant)
    failures = 0
    for pin in PINS:
        try:
            pin()
        except (AssertionError, np.linalg.LinAlgError, ValueError):
            failures += 1
    assert failures > 0, "no pin catches the planted mistake %s" % mutant.__name__


# ------------------------------------------- the printed t = 1.5 sequence ----

def test_printed_schedule_counts():
    """Sec. 3.3 prints t = 1.5 as L, R, L, R, L: five updates starting and
    ending with a left update. Integer t are the same under both schedules."""
    assert orc.als_updates(1.5, "printed") == 5
    assert orc.als_updates(1.5, "pairs") == 3
    for t in (0, 1, 2, 3):
        assert orc.als_updates(t, "printed") == orc.als_updates(t, "pairs") == 2 * t
    with pytest.raises(ValueError):
        orc.als_updates(1.25)
    with pytest.raises(ValueError):
        orc.als_updates(1.5, "other")


def test_printed_t15_is_two_pairs_then_a_left_update():
    """Under the printed schedule, t = 1.5 is t = 2 followed by one more left
    update: the right factor is t = 2's, and the left factor is the ridge
    minimiser against it (zero gradient), so the fit is never worse than t = 2's."""
    rng = np.random.default_rng(11)
    T, d_in, d_out, k, lam = 40, 12, 10, 3, 1e-3
    Xb = rng.standard_normal((T, d_in))
    W_res = rng.standard_normal((d_out, d_in))
    R0 = np.linalg.qr(rng.standard_normal((d_out, k)))[0].T
    E = Xb @ W_res.T
    pairs = orc.als_half_steps(Xb, W_res, R0, lam, 5)
    L5, R5 = pairs[-1]
    L4, R4 = pairs[3]
    np.testing.assert_array_equal(R5, R4)
    grad = (L5 @ R5 - E) @ R5.T + lam * L5
    assert np.abs(grad).max() < 1e-9 * max(1.0, np.abs(E).max())
    obj = lambda L, R: np.sum((E - L @ R) ** 2) + lam * (np.sum(L ** 2) + np.sum(R ** 2))
    assert obj(L5, R5) <= obj(L4, R4) + 1e-12
    U = rng.standard_normal((d_out, 2))
    V = rng.standard_normal((d_in, 2))
    Y = orc.als_inference(Xb, U, V, W_res, R0, lam, 1, T, 1.5, schedule="printed")
    np.testing.assert_allclose(Y, (Xb @ V) @ U.T + L5 @ R5, rtol=1e-12, atol=1e-12)
    Y2 = orc.als_inference(Xb, U, V, W_res, R0, lam, 1, T, 2.0, schedule="printed")
    np.testing.assert_allclose(Y2, orc.als_inference(Xb, U, V, W_res, R0, lam, 1, T, 2.0),
                               rtol=0, atol=0)
