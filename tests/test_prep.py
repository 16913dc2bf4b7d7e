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


def test_monarch_preparation_matches_the_oracle():
    """The host Monarch preparation (torch) and the oracle's (NumPy), written
    independently, give the same static matrix and residual, square and
    rectangular (signs of the block factors may differ; their products may not)."""
    import numpy as np
    from oracle import monarch as mon
    rng = np.random.default_rng(3)
    for b1, b2, b1o, b2o in ((4, 3, 4, 3), (4, 3, 2, 5)):
        W = rng.standard_normal((b1o * b2o, b1 * b2))
        f = prep.prepare_monarch(W, b1, b2, 2, 1e-3, b1o, b2o)
        fo = mon.offline_prepare_monarch(W, b1, b2, 2, 1e-3, b1o=b1o, b2o=b2o)
        np.testing.assert_allclose(f.W_res.numpy(), fo.W_res, rtol=0, atol=1e-12)
        What = mon.monarch_matrix(list(f.Lblocks.numpy()), list(f.Rblocks.numpy())).T
        np.testing.assert_allclose(What, fo.What, rtol=0, atol=1e-12)
        Pn = f.P.numpy()
        np.testing.assert_allclose(np.abs(Pn), np.abs(fo.P), rtol=0, atol=1e-10)
