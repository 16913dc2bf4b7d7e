"""Plain fp64 reference of the DyRA layer: a static part plus a one-step ALS correction.

TEST INFRASTRUCTURE ONLY: used by tests/, by the smoke check and by the
CPU-baseline leg of the benchmark. The CUDA library never calls into it and it
shares no code with the library.

Source: "DyRA: Dynamic Residual Approximation for Efficient Matrix
Multiplication in DNNs" (Chae, Chung, Lee, Kim), cited below as [DyRA].
  - Sec. 2.1, Eq. 1-2: W = W_hat + W_res, so X W = X W_hat + X W_res.
  - Sec. 2.2, Eq. 3-5: low-rank fit of the residual output by ALS, with the
    ridge term of footnote 2 added to both Gram matrices.
  - Sec. 2.3, Eq. 6-7: one ALS iteration; the left factor's projector P_L is
    precomputed offline.
  - Appendix A, Algorithm 1: the offline and inference procedures written out.
  - Appendix D: R^(0) is taken from the leading singular directions of W_res.
  - Sec. 2.4: one small SPD system per batch instance.
  - Sec. 3.3, Fig. 9 (right): more ALS iterations (als_inference), and
    Sec. 2.2: a Gaussian R^(0) (any R0 may be passed to the offline step).

Letters. The paper writes the product as X W with W of shape c1 x c2, static
rank k and correction rank r. This repository uses the PyTorch layout
Y = X W^T with W of shape d_out x d_in, static rank r and correction rank k:

    paper W            <->  W^T here
    paper U_k Sigma_k  <->  V here (d_in x r)    (the paper's left factor)
    paper V_k          <->  U here carries Sigma (d_out x r)
    paper P_L          <->  P (d_in x k)
    paper L^(1)        <->  L = X P (T x k per instance)
    paper R^(1)        <->  C (k x d_out per instance)

so the weight-only product X W_hat^T is (X V) U^T and DyRA adds L C.

Precision: everything here is float64; callers pass the dtype-rounded arrays
the GPU path consumes (see round_to), so a comparison measures kernel error and
not input quantisation.
"""

from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np


@dataclasses.dataclass
class Factors:
    """Output of the offline preparation, in this repository's letters.

    U     : d_out x r, static left factor with the singular values folded in
    V     : d_in x r, static right factor (orthonormal columns)
    P     : d_in x k, precomputed left projector of the correction
    W_res : d_out x d_in, residual weight W - U V^T
    R0    : k x d_out, fixed initial right factor of ALS
    """

    U: np.ndarray
    V: np.ndarray
    P: np.ndarray
    W_res: np.ndarray
    R0: np.ndarray


def _projector(W_res: np.ndarray, R0: np.ndarray, lam: float) -> np.ndarray:
    """[DyRA] Alg. 1 offline step 5 / Eq. 7, with the footnote-2 ridge term.

    Paper: P_L = (W_res R0^T)(R0 R0^T + lam I)^-1 with W_res of shape c1 x c2.
    Here W_res is d_out x d_in (transposed), so the paper's W_res R0^T is
    W_res^T R0^T, a d_in x k matrix.
    """
    k = R0.shape[0]
    gram = R0 @ R0.T + lam * np.eye(k)
    return np.linalg.solve(gram, (W_res.T @ R0.T).T).T


def _given_start(R0: np.ndarray, k: int, d_out: int) -> np.ndarray:
    R0 = np.array(R0, dtype=np.float64)
    if R0.shape != (k, d_out):
        raise ValueError("R0 must be k x d_out = %d x %d, got %s" % (k, d_out, R0.shape))
    return R0


def offline_prepare(W: np.ndarray, r: int, k: int, lam: float,
                    R0: Optional[np.ndarray] = None) -> Factors:
    """[DyRA] Alg. 1, procedure Offline Preparation, for the low-rank case.

    Step 2: the structured approximation is the rank-r truncated SVD
            (App. B, "Low-Rank Approximation"), with Sigma on the left factor.
    Step 3: W_res = W - W_hat.
    Step 4: R0 = top-k singular vectors of W_res on its output side (App. D;
            the paper's "right" singular vectors of its transposed W_res),
            unless a start R0 (k x d_out) is given, e.g. the Gaussian start
            of Sec. 2.2.
    Step 5: P from _projector.
    """
    W = np.asarray(W, dtype=np.float64)
    A, s, Bt = np.linalg.svd(W, full_matrices=False)
    U = A[:, :r] * s[:r]
    V = Bt[:r].T.copy()
    W_res = W - U @ V.T
    if R0 is not None:
        R0 = _given_start(R0, k, W.shape[0])
    elif k > 0:
        Ares, _, _ = np.linalg.svd(W_res, full_matrices=False)
        R0 = Ares[:, :k].T.copy()
    else:
        R0 = np.zeros((0, W.shape[0]))
    P = _projector(W_res, R0, lam) if k > 0 else np.zeros((W.shape[1], 0))
    return Factors(U, V, P, W_res, R0)


def offline_prepare_from_svd(left: np.ndarray, sigma: np.ndarray, right: np.ndarray,
                             r: int, k: int, lam: float,
                             R0: Optional[np.ndarray] = None) -> Factors:
    """Alg. 1 offline preparation when W = left . diag(sigma) . right^T is given.

    Same steps as offline_prepare, reading the SVD instead of computing it
    (synthetic weights are built from their singular factors). W_res is formed
    from the discarded singular triplets, which equals W - U V^T exactly in
    real arithmetic (Eq. 12 of App. C, in this repository's letters).
    """
    U = left[:, :r] * sigma[:r]
    V = right[:, :r].copy()
    W_res = (left[:, r:] * sigma[r:]) @ right[:, r:].T
    if R0 is not None:
        R0 = _given_start(R0, k, left.shape[0])
    else:
        R0 = left[:, r:r + k].T.copy()
    P = _projector(W_res, R0, lam) if k > 0 else np.zeros((right.shape[0], 0))
    return Factors(U, V, P, W_res, R0)


def weight_only(X: np.ndarray, U: np.ndarray, V: np.ndarray) -> np.ndarray:
    """[DyRA] Sec. 2.1: the conventional approximation keeps only X W_hat^T = (X V) U^T."""
    return (X @ V) @ U.T


def dense(X: np.ndarray, W: np.ndarray) -> np.ndarray:
    """[DyRA] Eq. 2: the exact product X W^T."""
    return X @ W.T


def inference(X: np.ndarray, U: np.ndarray, V: np.ndarray, P: np.ndarray,
              W_res: np.ndarray, lam: float, B: int, T: int, *,
              bias: Optional[np.ndarray] = None, alpha: float = 1.0) -> np.ndarray:
    """[DyRA] Alg. 1, procedure Inference, applied to each of B instances.

    The rows of X are B consecutive instances of T rows; the correction is
    fitted per instance (Sec. 2.4: one small SPD system per batch instance).
    For instance b with rows X_b, the procedure's steps in order:
      static part   Y_base = X_b W_hat^T              = (X_b V) U^T
      left factor   L      = X_b P                    (T x k)
      right factor  C      = (L^T L + lam I)^-1 (L^T X_b) W_res^T   (k x d_out)
      output        Y_b    = Y_base + L C
    Sec. 2.4 also writes the fused linear layer with a bias b (d_out) and a
    weight alpha on the correction, Y_b = Y_base + b + alpha L C; Alg. 1 is
    bias None and alpha 1 (the defaults).
    """
    X = np.asarray(X, dtype=np.float64)
    N = X.shape[0]
    if N != B * T:
        raise ValueError("X has %d rows, expected B*T = %d" % (N, B * T))
    k = P.shape[1]
    Y = np.empty((N, U.shape[0]))
    for b in range(B):
        Xb = X[b * T:(b + 1) * T]
        Yb = (Xb @ V) @ U.T
        if k > 0:
            L = Xb @ P
            G = L.T @ L + lam * np.eye(k)
            C = np.linalg.solve(G, (L.T @ Xb) @ W_res.T)
            Yb = Yb + alpha * (L @ C)
        if bias is not None:
            Yb = Yb + bias
        Y[b * T:(b + 1) * T] = Yb
    return Y


def inference_rows(X: np.ndarray, U: np.ndarray, V: np.ndarray, P: np.ndarray,
                   W_res: np.ndarray, lam: float, B: int, T: int, rows) -> np.ndarray:
    """Rows `rows` of inference(...), for layers too large to evaluate whole.

    Each instance that owns a requested row is fitted on all of its T rows
    exactly as in inference (its left and right factors); the static part and
    the output are then evaluated for the requested rows only.
    """
    X = np.asarray(X, dtype=np.float64)
    rows = np.asarray(rows, dtype=np.int64)
    k = P.shape[1]
    out = np.empty((rows.size, U.shape[0]))
    for b in np.unique(rows // T):
        Xb = X[b * T:(b + 1) * T]
        sel = np.nonzero(rows // T == b)[0]
        xr = X[rows[sel]]
        Yr = (xr @ V) @ U.T
        if k > 0:
            L = Xb @ P
            G = L.T @ L + lam * np.eye(k)
            C = np.linalg.solve(G, (L.T @ Xb) @ W_res.T)
            Yr = Yr + (xr @ P) @ C
        out[sel] = Yr
    return out


def als_half_steps(Xb: np.ndarray, W_res: np.ndarray, R0: np.ndarray, lam: float,
                   steps: int) -> list:
    """Alternating ridge least squares on one instance's residual output.

    [DyRA] Sec. 2.2: the residual product E = X_b W_res^T (T x d_out here) is
    fitted by a rank-k product L R, alternating the two exact minimisers of
    Eq. 4-5 with the ridge of footnote 2 on each Gram matrix:
      left update   L = (X_b W_res^T R^T)(R R^T + lam I)^-1
                      = argmin_L ||E - L R||^2 + lam ||L||^2
      right update  R = (L^T L + lam I)^-1 (L^T X_b) W_res^T
                      = argmin_R ||E - L R||^2 + lam ||R||^2
    starting from the fixed R = R0 with a left update. Alg. 1 is the first two
    half-steps (its P_L folds R0 into the left update). E is never formed: as
    in Alg. 1, X_b multiplies W_res^T R^T and L^T X_b multiplies W_res^T.
    Returns the pair (L, R) after each of `steps` half-steps.
    """
    Xb = np.asarray(Xb, dtype=np.float64)
    k = R0.shape[0]
    eye = np.eye(k)
    R = np.asarray(R0, dtype=np.float64)
    L = None
    pairs = []
    for h in range(steps):
        if h % 2 == 0:
            rhs = Xb @ (W_res.T @ R.T)                       # T x k
            L = np.linalg.solve(R @ R.T + lam * eye, rhs.T).T
        else:
            R = np.linalg.solve(L.T @ L + lam * eye, (L.T @ Xb) @ W_res.T)
        pairs.append((L, R))
    return pairs


def als_updates(t: float, schedule: str = "pairs") -> int:
    """How many ALS updates (half-steps) t iterations run.

    "pairs": an iteration is a left and a right update, as Alg. 1 runs for
    t = 1, and a half iteration ends on a left update; t = 1.5 runs L, R, L.
    "printed": Sec. 3.3 spells t = 1.5 as the five updates L, R, L, R, L. It
    gives no other half-integer sequence, so here a half-integer t runs
    ceil(t) pairs and then one more left update; integer t agree with "pairs".
    """
    steps = int(round(2 * t))
    if steps != 2 * t or steps < 0:
        raise ValueError("t must be a non-negative multiple of 0.5")
    if schedule == "pairs" or steps % 2 == 0:
        return steps
    if schedule == "printed":
        return steps + 2
    raise ValueError("unknown schedule %r" % schedule)


def als_inference(X: np.ndarray, U: np.ndarray, V: np.ndarray, W_res: np.ndarray,
                  R0: np.ndarray, lam: float, B: int, T: int, t: float,
                  schedule: str = "pairs") -> np.ndarray:
    """DyRA with t ALS iterations per instance ([DyRA] Sec. 3.3, Fig. 9 right).

    One iteration is a left and a right update (Alg. 1 is t = 1); a half
    iteration ends on a left update, so t = 1.5 runs L, R, L and t = 2 runs
    L, R, L, R. With schedule="printed", t = 1.5 runs the sequence the text
    prints, L, R, L, R, L (see als_updates). The output of instance b is
    (X_b V) U^T + L R with the last pair. t = 0 is the weight-only layer.
    """
    steps = als_updates(t, schedule)
    X = np.asarray(X, dtype=np.float64)
    if X.shape[0] != B * T:
        raise ValueError("X has %d rows, expected B*T = %d" % (X.shape[0], B * T))
    Y = np.empty((X.shape[0], U.shape[0]))
    for b in range(B):
        Xb = X[b * T:(b + 1) * T]
        Yb = (Xb @ V) @ U.T
        if steps > 0 and R0.shape[0] > 0:
            L, R = als_half_steps(Xb, W_res, R0, lam, steps)[-1]
            Yb = Yb + L @ R
        Y[b * T:(b + 1) * T] = Yb
    return Y


def rel_fro(A: np.ndarray, ref: np.ndarray) -> float:
    """Relative Frobenius error ||A - ref||_F / ||ref||_F ([DyRA] App. E.4)."""
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(np.asarray(A, np.float64) - ref) / (den if den > 0 else 1.0))


def error_report(X: np.ndarray, W: np.ndarray, f: Factors, lam: float, B: int, T: int,
                 Y: Optional[np.ndarray] = None) -> dict:
    """Normalised output errors of weight-only and DyRA against the dense product
    ([DyRA] App. E.4: ||X W - Y_approx||_F / ||X W||_F)."""
    Yd = dense(X, W)
    Ywo = weight_only(X, f.U, f.V)
    if Y is None:
        Y = inference(X, f.U, f.V, f.P, f.W_res, lam, B, T)
    return {"err_wo": rel_fro(Ywo, Yd), "err_dyra": rel_fro(Y, Yd)}


def round_to(a: np.ndarray, dtype: str) -> np.ndarray:
    """Round float64 values to the storage type ('f32' or 'bf16', round to
    nearest even) and return them as float64. bf16 is the upper half of the
    IEEE binary32 pattern; rounding adds 0x7FFF plus the kept LSB before the
    truncation. Inputs here are finite."""
    a32 = np.asarray(a, dtype=np.float32)
    if dtype == "f32":
        return a32.astype(np.float64)
    if dtype != "bf16":
        raise ValueError(dtype)
    bits = a32.view(np.uint32).astype(np.uint64)
    bits = (bits + 0x7FFF + ((bits >> 16) & 1)) >> 16 << 16
    return bits.astype(np.uint32).view(np.float32).astype(np.float64)
