"""The library's host-side offline preparation agrees with the oracle's."""

import numpy as np
import torch

import oracle
from rank_structured_matmul_b200 import prep
from synth import LayerSpec, generate


def _layer():
    return generate(LayerSpec("p", 40, 32, 6, 4, 2, 9, "f32", 0.8, "lognormal", seed=3))


def test_prepare_from_svd_matches_oracle():
    w = _layer()
    for lam in (0.0, 1e-3):
        a = prep.prepare_from_svd(w.left, w.sigma, w.right, 6, 4, lam)
        b = oracle.offline_prepare_from_svd(w.left, w.sigma, w.right, 6, 4, lam)
        for x, y in zip(a, (b.U, b.V, b.P, b.W_res)):
            np.testing.assert_allclose(x.numpy(), y, atol=1e-13)


def test_prepare_from_weight_gives_same_layer():
    """Singular-vector signs may differ between the two SVD routes; the layer
    they define (U V^T, W_res, and the DyRA output) does not."""
    w = _layer()
    lam = 1e-3
    a = prep.prepare_from_weight(torch.from_numpy(w.weight()), 6, 4, lam)
    b = oracle.offline_prepare_from_svd(w.left, w.sigma, w.right, 6, 4, lam)
    np.testing.assert_allclose((a.U @ a.V.T).numpy(), b.U @ b.V.T, atol=1e-12)
    np.testing.assert_allclose(a.W_res.numpy(), b.W_res, atol=1e-12)
    ya = oracle.inference(w.X, a.U.numpy(), a.V.numpy(), a.P.numpy(), a.W_res.numpy(), lam, 2, 9)
    yb = oracle.inference(w.X, b.U, b.V, b.P, b.W_res, lam, 2, 9)
    np.testing.assert_allclose(ya, yb, atol=1e-10)


def test_k0_shapes():
    w = _layer()
    a = prep.prepare_from_svd(w.left, w.sigma, w.right, 6, 0, 0.0)
    assert a.P.shape == (40, 0)
