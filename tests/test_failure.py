"""Failure handling on the device without a GPU fault.

Every pipeline wait inside the tensor-core kernels is bounded. A diagnostic
setter shortens the limit of the Gram stage's waits so that one of them runs
out: the kernel must raise DYRA_STATUS_WAIT_TIMEOUT, let the copies and MMAs
it already issued finish, free its tensor memory and return, so that the
context stays usable. The next forward on the same plan, with the default
limit restored, must then give exactly the output of a forward before the
failure. Nothing here traps, asserts on the device or reads out of bounds.
"""

import numpy as np
import pytest
import torch

import oracle
from rank_structured_matmul_b200 import dyra
from synth import LayerSpec, generate

pytestmark = pytest.mark.gpu

GRAM_STAGE = 1


def _layer(s: LayerSpec):
    w = generate(s)
    f = oracle.offline_prepare_from_svd(w.left, w.sigma, w.right, s.r, s.k, s.lam)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(oracle.round_to(a, "bf16"))).to(
        "cuda", torch.bfloat16)
    layer = dyra.DyraLinear(s.d_in, s.d_out, s.r, s.k, "bf16")
    layer.load(dev(f.U), dev(f.V), dev(f.P), dev(f.W_res), s.lam)
    return layer, dev(w.X)


@pytest.mark.parametrize("B,T", [(3, 201), (1, 2048)])
def test_gram_wait_that_runs_out_is_reported_and_the_context_stays_usable(B, T):
    """(3, 201): one CTA per Gram tile; (1, 2048): the instance's rows are
    split over a cluster of CTAs that sum their partials through distributed
    shared memory, which every CTA reaches even after giving up."""
    s = LayerSpec("timeout", 256, 512, 64, 32, B, T, "bf16", 0.7, "lognormal", seed=5)
    layer, X = _layer(s)
    try:
        if B == 1:
            splits, _ = dyra.dyra_debug_gram_split(layer.plan, B, T)
            assert splits > 1
        before = layer.forward(X, B=B, T=T)
        assert layer.status() == 0
        dyra.dyra_debug_set_wait_limit(layer.plan, GRAM_STAGE, 1)  # 1 ns: the first wait runs out
        layer.forward(X, B=B, T=T)
        status = layer.status()
        assert status & dyra.DYRA_STATUS_WAIT_TIMEOUT, status
        dyra.dyra_debug_set_wait_limit(layer.plan, GRAM_STAGE, 0)
        after = layer.forward(X, B=B, T=T)
        assert layer.status() == 0
        assert torch.equal(after, before)
    finally:
        layer.close()


def test_wait_limit_only_for_the_gram_stage():
    s = LayerSpec("timeout", 256, 512, 64, 32, 2, 64, "bf16", 0.7, "lognormal", seed=5)
    layer, _ = _layer(s)
    try:
        for stage in (0, 2, 3, 4):
            with pytest.raises(dyra.DyraError) as e:
                dyra.dyra_debug_set_wait_limit(layer.plan, stage, 1)
            assert e.value.code == dyra.DYRA_ERR_UNSUPPORTED
    finally:
        layer.close()
