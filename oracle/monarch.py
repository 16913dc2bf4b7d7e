"""Monarch static part for the DyRA layer, in float64: part of the oracle.

TEST INFRASTRUCTURE ONLY, like the rest of this package: the CUDA library
never calls into it and shares no code with it.

Source: "DyRA: Dynamic Residual Approximation for Efficient Matrix
Multiplication in DNNs", Appendix B, "Monarch Matrix" (cited as [DyRA]). DyRA
works with any structured static part (Sec. 2.3); Monarch is one of the three
the paper evaluates (Sec. 3.1). In the paper's layout (Y = X W, W of shape
N x N with N = b1 b2) the Monarch approximation is

    W_hat = P L P^T R,   L = diag(L_1, ..., L_b2), L_i of shape b1 x b1,
                         R = diag(R_1, ..., R_b1), R_j of shape b2 x b2,

with P a fixed permutation, and the factors come from a truncated SVD of each
block of the dense weight.

Readings (the pages leave these open):
  * P is the perfect shuffle: P^T moves the entry at position j1*b2 + j2 to
    position j2*b1 + j1 (a row-major b1 x b2 grid read column by column).
  * With that P, entry (m1*b2 + j2, j1*b2 + i2) of W_hat is
    L_j2[m1, j1] * R_j1[j2, i2]. For each pair (j1, j2) the b1 x b2 block of
    W_hat on rows m1*b2 + j2 and columns j1*b2 + i2 is therefore rank 1, and
    these blocks tile W_hat. The Frobenius-best Monarch approximation of W is
    the best rank-1 approximation (truncated SVD) of each such block of W,
    with the singular value split evenly between the two factors.
  * Only square weights are defined by the pages. Their experiments also put
    Monarch on rectangular MLP layers without saying how, so a rectangular
    weight of c1 = b1 b2 rows and c2 = b1' b2' columns is read the same way:
    L = diag(L_1, ..., L_b2) with L_j2 of shape b1 x b1', R = diag(R_1, ...,
    R_b1') with R_j1 of shape b2 x b2', W_hat = P1 L P2^T R with P1 the
    shuffle of the b1 x b2 grid and P2 that of the b1' x b2 grid. Entry
    (m1*b2 + j2, j1*b2' + i2) is then L_j2[m1, j1] * R_j1[j2, i2]: the same
    rank-1 blocks (now b1 x b2'), the same block-wise SVD projection, and the
    square form when b1' = b1 and b2' = b2.

This repository's letters are Y = X W^T with W of shape d_out x d_in, so the
static weight here is W_hat^T of the paper's W_hat, and the static output is
X W_hat (paper layout) = X What^T (these letters).
"""

from __future__ import annotations

import dataclasses
from typing import List, Optional

import numpy as np

from .dyra_oracle import _given_start, _projector, inference


def shuffle(b1: int, b2: int) -> np.ndarray:
    """The permutation matrix P of [DyRA] App. B (reading above), N x N,
    N = b1 b2."""
    N = b1 * b2
    Pt = np.zeros((N, N))
    for j1 in range(b1):
        for j2 in range(b2):
            Pt[j2 * b1 + j1, j1 * b2 + j2] = 1.0
    return Pt.T


def block_diag(blocks: List[np.ndarray]) -> np.ndarray:
    """diag(B_1, ..., B_n) of blocks of equal shape."""
    rows = sum(b.shape[0] for b in blocks)
    cols = sum(b.shape[1] for b in blocks)
    out = np.zeros((rows, cols))
    r = c = 0
    for b in blocks:
        out[r:r + b.shape[0], c:c + b.shape[1]] = b
        r += b.shape[0]
        c += b.shape[1]
    return out


def monarch_matrix(Lb: List[np.ndarray], Rb: List[np.ndarray]) -> np.ndarray:
    """W_hat = P1 L P2^T R in the paper's layout, as the product of App. B
    (P1 = P2 = P for square blocks; the rectangular reading above)."""
    b2, b1o = len(Lb), len(Rb)
    b1 = Lb[0].shape[0]
    P1 = shuffle(b1, b2)
    P2 = shuffle(b1o, b2)
    return P1 @ block_diag(Lb) @ P2.T @ block_diag(Rb)


def monarch_project(Wp: np.ndarray, b1: int, b2: int, b1o: Optional[int] = None,
                    b2o: Optional[int] = None):
    """Monarch factors of a c1 x c2 weight (paper layout), c1 = b1 b2 and
    c2 = b1o b2o (b1o = b1, b2o = b2 unless given: the square form).

    Each block of rows m1*b2 + j2 (m1 < b1) and columns j1*b2o + i2 (i2 < b2o)
    is replaced by its best rank-1 approximation s u v^T; its factors go to
    column j1 of L_j2 (sqrt(s) u) and row j2 of R_j1 (sqrt(s) v).
    Returns (Lb, Rb): b2 blocks of b1 x b1o and b1o blocks of b2 x b2o.
    """
    b1o = b1 if b1o is None else b1o
    b2o = b2 if b2o is None else b2o
    Wp = np.asarray(Wp, dtype=np.float64)
    if Wp.shape != (b1 * b2, b1o * b2o):
        raise ValueError("Monarch needs a %d x %d weight, got %s" % (b1 * b2, b1o * b2o, Wp.shape))
    Lb = [np.zeros((b1, b1o)) for _ in range(b2)]
    Rb = [np.zeros((b2, b2o)) for _ in range(b1o)]
    for j1 in range(b1o):
        for j2 in range(b2):
            block = Wp[j2::b2, j1 * b2o:(j1 + 1) * b2o]          # b1 x b2o
            u, s, vt = np.linalg.svd(block)
            Lb[j2][:, j1] = np.sqrt(s[0]) * u[:, 0]
            Rb[j1][j2, :] = np.sqrt(s[0]) * vt[0]
    return Lb, Rb


@dataclasses.dataclass
class MonarchFactors:
    """Offline preparation with a Monarch static part, in this repository's letters.

    Lb, Rb : the Monarch blocks of the paper-layout static weight What^T
    What   : d_out x d_in static weight (= W_hat of the paper, transposed)
    P      : d_in x k projector of the correction
    W_res  : d_out x d_in residual W - What
    R0     : k x d_out ALS start
    """

    Lb: List[np.ndarray]
    Rb: List[np.ndarray]
    What: np.ndarray
    P: np.ndarray
    W_res: np.ndarray
    R0: np.ndarray


def offline_prepare_monarch(W: np.ndarray, b1: int, b2: int, k: int, lam: float,
                            R0: Optional[np.ndarray] = None, b1o: Optional[int] = None,
                            b2o: Optional[int] = None) -> MonarchFactors:
    """[DyRA] Alg. 1, procedure Offline Preparation, with the Monarch structure.

    W is d_out x d_in with d_in = b1 b2 and d_out = b1o b2o (b1o = b1, b2o =
    b2 unless given).

    Step 2: What = the Monarch projection (App. B) of the paper-layout W^T.
    Step 3: W_res = W - What.
    Step 4: R0 = top-k output-side singular vectors of W_res (App. D), unless
            a start is given.
    Step 5: the projector P of Eq. 7 with the ridge.
    """
    W = np.asarray(W, dtype=np.float64)
    Lb, Rb = monarch_project(W.T, b1, b2, b1o, b2o)
    What = monarch_matrix(Lb, Rb).T
    W_res = W - What
    d_out, d_in = W.shape
    if R0 is not None:
        R0 = _given_start(R0, k, d_out)
    elif k > 0:
        R0 = np.linalg.svd(W_res)[0][:, :k].T.copy()
    else:
        R0 = np.zeros((0, d_out))
    P = _projector(W_res, R0, lam) if k > 0 else np.zeros((d_in, 0))
    return MonarchFactors(Lb, Rb, What, P, W_res, R0)


def monarch_inference(X: np.ndarray, f: MonarchFactors, lam: float, B: int, T: int) -> np.ndarray:
    """[DyRA] Alg. 1, procedure Inference, with the Monarch static part.

    The static product is X What^T. It is passed to the low-rank procedure as
    its factorisation (X V) U^T with V = I and U = What, so the correction
    steps are exactly those of `inference`.
    """
    d_in = f.What.shape[1]
    return inference(X, f.What, np.eye(d_in), f.P, f.W_res, lam, B, T)
