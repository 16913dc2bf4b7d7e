"""The allocation-free forward, dyra_forward_batched_noalloc.

It exists for callers that may not allocate device memory once serving has
started (a memory manager owns the device, or an allocation's implicit
synchronisation is not acceptable): the intermediates live in one fixed array
inside the library instead of the plan's workspace. These tests call it
through the C ABI and compare it with dyra_forward_batched, which uses the
plan's workspace, on two calls in a row with different inputs (the shared
array keeps the first call's contents, which must not leak into the second).
Both entry points run the same deterministic kernels on the same inputs, so
their outputs must agree bit for bit.
This file is collected last on purpose.
"""

import dataclasses
import os

import numpy as np
import pytest
import torch

import oracle
from rank_structured_matmul_b200 import dyra
from synth import LayerSpec, generate

pytestmark = pytest.mark.gpu


def _layer(s: LayerSpec):
    # draw 2*N rows: the first N feed the first call, the rest the second
    w = generate(dataclasses.replace(s, n_draw=2 * s.N).with_rows(1, 2 * s.N))
    f = oracle.offline_prepare_from_svd(w.left, w.sigma, w.right, s.r, s.k, s.lam)
    td = torch.bfloat16 if s.dtype == "bf16" else torch.float32
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(oracle.round_to(a, s.dtype))).to(
        "cuda", td)
    plan = dyra.dyra_plan_create(s.d_in, s.d_out, s.r, s.k,
                                 dyra.DYRA_BF16 if s.dtype == "bf16" else dyra.DYRA_F32)
    P = dev(f.P) if s.k > 0 else None
    Wr = dev(f.W_res) if s.k > 0 else None
    dyra.dyra_load_factors(plan, dev(f.U), dev(f.V), P, Wr, s.lam)
    X = dev(w.X)
    return plan, X[: s.N].contiguous(), X[s.N:].contiguous(), td


def _compare(s: LayerSpec):
    plan, Xa, Xb, td = _layer(s)
    try:
        for X in (Xa, Xb):  # two calls in a row, different inputs
            want = torch.empty(s.N, s.d_out, device="cuda", dtype=td)
            got = torch.full((s.N, s.d_out), float("nan"), device="cuda", dtype=td)
            dyra.dyra_forward_batched(plan, X, want, s.B, s.T)
            dyra.dyra_forward_batched_noalloc(plan, X, got, s.B, s.T)
            torch.cuda.synchronize()
            assert dyra.dyra_last_status(plan) == 0
            assert bool(torch.isfinite(got.float()).all())
            assert torch.equal(got, want)
    finally:
        dyra.dyra_plan_destroy(plan)


def test_noalloc_matches_workspace_forward_bf16():
    _compare(LayerSpec("noalloc_bf16", 256, 512, 64, 32, 3, 201, "bf16", 0.7, "lognormal",
                       seed=7))


def test_noalloc_matches_workspace_forward_split_k_projection():
    """Few rows and a long K: the projection splits K across a cluster of
    CTAs; the allocation-free forward agrees with the workspace forward."""
    _compare(LayerSpec("noalloc_sk", 2048, 512, 256, 32, 1, 64, "bf16", 0.7, "lognormal",
                       seed=7))


def test_noalloc_matches_workspace_forward_weight_only():
    """k = 0: only the static part's intermediate lives in the array."""
    _compare(LayerSpec("noalloc_k0", 256, 512, 64, 0, 2, 130, "bf16", 0.7, "lognormal", seed=7))


def test_noalloc_matches_workspace_forward_large_k():
    """k = 72 (above 64): no per-instance factor records in the array."""
    _compare(LayerSpec("noalloc_k72", 256, 512, 64, 72, 2, 150, "bf16", 0.7, "lognormal",
                       seed=7))


def test_noalloc_matches_workspace_forward_bf16_cuda_cores(monkeypatch):
    """A bf16 plan on the CUDA-core kernels (chosen when the plan is created)."""
    monkeypatch.setenv("DYRA_KERNELS", "simt")
    _compare(LayerSpec("noalloc_simt", 256, 512, 64, 32, 2, 100, "bf16", 0.7, "lognormal",
                       seed=7))


def test_noalloc_matches_workspace_forward_fp32():
    _compare(LayerSpec("noalloc_f32", 256, 256, 32, 8, 2, 64, "f32", 1.0, "outlier",
                       n_outlier=4, outlier_scale=20.0, seed=7))


def test_noalloc_first_call_allocates_nothing(monkeypatch):
    """On a fresh plan (no workspace yet) the allocation-free forward is the
    first forward, with every device allocation of the library made to fail:
    it still succeeds, and the plan's device footprint does not change. The
    workspace forward afterwards gives the same output bit for bit."""
    s = LayerSpec("noalloc_fresh", 256, 512, 64, 32, 3, 201, "bf16", 0.7, "lognormal", seed=8)
    plan, Xa, Xb, td = _layer(s)
    try:
        before = dyra.dyra_plan_device_bytes(plan)
        got = [torch.full((s.N, s.d_out), float("nan"), device="cuda", dtype=td)
               for _ in range(2)]
        monkeypatch.setenv("DYRA_TEST_FAIL_ALLOC", "1")
        for X, G in zip((Xa, Xb), got):
            dyra.dyra_forward_batched_noalloc(plan, X, G, s.B, s.T)
        torch.cuda.synchronize()
        # the workspace forward, by contrast, needs an allocation here
        with pytest.raises(dyra.DyraError) as e:
            dyra.dyra_forward_batched(plan, Xa, torch.empty_like(got[0]), s.B, s.T)
        assert e.value.code == dyra.DYRA_ERR_ALLOC
        monkeypatch.delenv("DYRA_TEST_FAIL_ALLOC")
        assert dyra.dyra_plan_device_bytes(plan) == before
        assert dyra.dyra_last_status(plan) == 0
        for X, G in zip((Xa, Xb), got):
            want = torch.empty_like(G)
            dyra.dyra_forward_batched(plan, X, want, s.B, s.T)
            torch.cuda.synchronize()
            assert torch.equal(G, want)
    finally:
        os.environ.pop("DYRA_TEST_FAIL_ALLOC", None)
        dyra.dyra_plan_destroy(plan)


def test_noalloc_rejects_sizes_beyond_the_array():
    """A request whose intermediates exceed the fixed array is refused before
    anything is enqueued, and the output is left untouched."""
    s = LayerSpec("noalloc_big", 1024, 4096, 256, 32, 64, 201, "bf16", 0.7, "lognormal", seed=7)
    plan = dyra.dyra_plan_create(s.d_in, s.d_out, s.r, s.k, dyra.DYRA_BF16)
    try:
        z = lambda *shape: torch.zeros(*shape, device="cuda", dtype=torch.bfloat16)
        dyra.dyra_load_factors(plan, z(4096, 256), z(1024, 256), z(1024, 32), z(4096, 1024), 1e-3)
        X = z(s.N, s.d_in)
        Y = torch.full((s.N, s.d_out), 7.0, device="cuda", dtype=torch.bfloat16)
        with pytest.raises(dyra.DyraError) as e:
            dyra.dyra_forward_batched_noalloc(plan, X, Y, s.B, s.T)
        assert e.value.code == dyra.DYRA_ERR_INVALID_ARG
        torch.cuda.synchronize()
        assert bool(torch.all(Y == 7.0))
    finally:
        dyra.dyra_plan_destroy(plan)
