"""Offline preparation of a DyRA layer on the host (not on the hot path).

"DyRA: Dynamic Residual Approximation for Efficient Matrix Multiplication in
DNNs", Appendix A, Algorithm 1, procedure Offline Preparation, low-rank case
(App. B): truncated SVD W ~ U V^T with the singular values on U, the residual
W_res = W - U V^T, the fixed ALS start R0 = the top-k output-side singular
vectors of W_res (App. D) or a given k x d_out start (the Gaussian start of
Sec. 2.2), and the projector P = W_res^T R0^T (R0 R0^T +
lambda I)^-1 (Eq. 7 with the ridge of footnote 2). Computed in float64 with
torch on the CPU; the result is what dyra_load_factors takes.
"""

from __future__ import annotations

from typing import NamedTuple

import torch


class LayerFactors(NamedTuple):
    U: torch.Tensor      # d_out x r
    V: torch.Tensor      # d_in x r
    P: torch.Tensor      # d_in x k
    W_res: torch.Tensor  # d_out x d_in


def _p_from_r0(W_res: torch.Tensor, R0: torch.Tensor, lam: float) -> torch.Tensor:
    k = R0.shape[0]
    if R0.shape[1] != W_res.shape[0]:
        raise ValueError("R0 must be k x d_out, got %s for d_out = %d" % (tuple(R0.shape), W_res.shape[0]))
    gram = R0 @ R0.T + lam * torch.eye(k, dtype=torch.float64)
    return torch.linalg.solve(gram, R0 @ W_res).T.contiguous()


def _start(R0, k: int):
    R0 = torch.as_tensor(R0, dtype=torch.float64).cpu()
    if R0.dim() != 2 or R0.shape[0] != k:
        raise ValueError("R0 must have k = %d rows, got shape %s" % (k, tuple(R0.shape)))
    return R0


def prepare_from_weight(W, r: int, k: int, lam: float, R0=None) -> LayerFactors:
    """From a dense d_out x d_in weight (one SVD of W and, without a given
    start R0, one of W_res)."""
    W = torch.as_tensor(W, dtype=torch.float64).cpu()
    A, s, Bt = torch.linalg.svd(W, full_matrices=False)
    U = (A[:, :r] * s[:r]).contiguous()
    V = Bt[:r].T.contiguous()
    W_res = W - U @ V.T
    if k == 0:
        return LayerFactors(U, V, torch.zeros(W.shape[1], 0, dtype=torch.float64), W_res)
    if R0 is None:
        R0 = torch.linalg.svd(W_res, full_matrices=False)[0][:, :k].T
    return LayerFactors(U, V, _p_from_r0(W_res, _start(R0, k), lam), W_res)


def prepare_from_svd(left, sigma, right, r: int, k: int, lam: float, R0=None) -> LayerFactors:
    """From a weight given by its SVD W = left diag(sigma) right^T."""
    left = torch.as_tensor(left, dtype=torch.float64).cpu()
    sigma = torch.as_tensor(sigma, dtype=torch.float64).cpu()
    right = torch.as_tensor(right, dtype=torch.float64).cpu()
    U = (left[:, :r] * sigma[:r]).contiguous()
    V = right[:, :r].contiguous()
    W_res = (left[:, r:] * sigma[r:]) @ right[:, r:].T
    if k == 0:
        return LayerFactors(U, V, torch.zeros(right.shape[0], 0, dtype=torch.float64), W_res)
    R0 = left[:, r:r + k].T if R0 is None else _start(R0, k)
    return LayerFactors(U, V, _p_from_r0(W_res, R0, lam), W_res)


class MonarchLayerFactors(NamedTuple):
    Lblocks: torch.Tensor  # b2 x b1 x b1o: L_j2[m1][j1]
    Rblocks: torch.Tensor  # b1o x b2 x b2o: R_j1[j2][i2]
    P: torch.Tensor        # d_in x k
    W_res: torch.Tensor    # d_out x d_in


def prepare_monarch(W, b1: int, b2: int, k: int, lam: float, b1o=None, b2o=None,
                    R0=None) -> MonarchLayerFactors:
    """Offline preparation with a Monarch static part ("DyRA: Dynamic Residual
    Approximation for Efficient Matrix Multiplication in DNNs", App. B, and
    Alg. 1 Offline) for W of shape d_out x d_in, d_in = b1 b2, d_out = b1o b2o
    (b1o = b1, b2o = b2 unless given). In the paper's layout W^T, entry
    (m1 b2 + j2, j1 b2o + i2) of the Monarch matrix is L_j2[m1][j1] R_j1[j2][i2],
    so each block of rows m1 b2 + j2 (m1 < b1) and columns j1 b2o + i2 is rank
    one: its best rank-1 approximation sqrt(s) u . sqrt(s) v^T gives column j1
    of L_j2 and row j2 of R_j1. W_res = W - W_hat^T, R0 the top-k output-side
    singular vectors of W_res unless given, and the projector P of Eq. 7."""
    b1o = b1 if b1o is None else b1o
    b2o = b2 if b2o is None else b2o
    W = torch.as_tensor(W, dtype=torch.float64).cpu()
    if W.shape != (b1o * b2o, b1 * b2):
        raise ValueError("W must be %d x %d" % (b1o * b2o, b1 * b2))
    # blocks[j2][j1] = the b1 x b2o block of rows m1 b2 + j2, columns j1 b2o + i2
    blocks = W.T.reshape(b1, b2, b1o, b2o).permute(1, 2, 0, 3)
    u, s, vh = torch.linalg.svd(blocks)
    root = s[..., 0].sqrt()
    Lb = (u[..., :, 0] * root[..., None]).permute(0, 2, 1).contiguous()   # [j2][m1][j1]
    Rb = (vh[..., 0, :] * root[..., None]).permute(1, 0, 2).contiguous()  # [j1][j2][i2]
    What_p = torch.einsum("bmj,jbi->mbji", Lb, Rb).reshape(b1 * b2, b1o * b2o)
    W_res = W - What_p.T
    if k == 0:
        return MonarchLayerFactors(Lb, Rb, torch.zeros(W.shape[1], 0, dtype=torch.float64), W_res)
    if R0 is None:
        R0 = torch.linalg.svd(W_res, full_matrices=False)[0][:, :k].T
    return MonarchLayerFactors(Lb, Rb, _p_from_r0(W_res, _start(R0, k), lam), W_res)

