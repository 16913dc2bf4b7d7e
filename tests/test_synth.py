"""The seeded workload generator: shapes, determinism and statistics."""

import numpy as np

from synth import CONFIGS, LLAMA_SWEEP, generate, spec


def test_config_table():
    assert spec("tiny_f32").N == 64 and spec("tiny_f32").dtype == "f32"
    v = spec("vit_fc1")
    assert (v.d_in, v.d_out, v.r, v.k, v.B, v.T) == (1024, 4096, 256, 32, 32, 201)
    for nm, (di, do) in {"qkv": (1024, 3072), "proj": (1024, 1024), "fc1": (1024, 4096),
                         "fc2": (4096, 1024)}.items():
        s = spec("vit_block_" + nm)
        assert (s.d_in, s.d_out, s.r, s.k, s.B, s.T) == (di, do, min(di, do) // 4, 32, 64, 201)
    w = spec("whisper_fc1")
    assert (w.d_in, w.d_out, w.r, w.k, w.N) == (1280, 5120, 320, 64, 12000)
    for n in LLAMA_SWEEP:
        s = spec("llama_up_%d" % n)
        assert (s.d_in, s.d_out, s.r, s.k, s.N, s.n_outlier) == (4096, 14336, 1024, 64, n, 41)
    assert all(c.lam == 1e-3 for c in CONFIGS.values())


def test_tiny_is_deterministic_and_well_formed():
    a = generate(spec("tiny_f32"))
    b = generate(spec("tiny_f32"))
    np.testing.assert_array_equal(a.X, b.X)
    np.testing.assert_allclose(a.left.T @ a.left, np.eye(256), atol=1e-12)
    np.testing.assert_allclose(a.right.T @ a.right, np.eye(256), atol=1e-12)
    np.testing.assert_allclose(a.sigma, 1.0 / np.arange(1, 257))
    sv = np.linalg.svd(a.weight(), compute_uv=False)
    np.testing.assert_allclose(sv, a.sigma, atol=1e-12)
    # 4 channels scaled x20 over N(0,1) rows
    colstd = a.X.std(axis=0)
    assert np.sum(colstd > 8) == 4


def test_prefix_draw():
    s = spec("tiny_f32")
    full = generate(s.with_rows(1, 64))
    part = generate(s.with_rows(2, 16))
    np.testing.assert_array_equal(part.X, full.X[:32])
