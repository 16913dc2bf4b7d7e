"""GPU parity: the CUDA DyRA forward (through the C ABI) against the fp64 oracle.

Both sides receive the same seeded inputs, rounded once to the plan's storage
type. Tolerances are the layer's bar: relative Frobenius error <= 1e-5 for
fp32 plans and <= 1e-2 for bf16 plans (fp32 accumulation). Full-size layers
whose oracle output is too large are compared on sampled rows (the oracle
still fits each sampled instance on all of its rows), always including the
first and last row of every instance and the rows around tile boundaries.
"""

import os

import numpy as np
import pytest
import torch

import oracle
from rank_structured_matmul_b200 import dyra
from synth import CONFIGS, LayerSpec, gaussian_r0, generate

pytestmark = pytest.mark.gpu

TOL = {"bf16": 1e-2, "f32": 1e-5}
ROW_TOL = 5e-2  # any single row: ||dy|| / rms row norm
_CACHE = {}


def prepared(s: LayerSpec):
    """Workload + oracle factors, rounded to the storage type (cached per layer)."""
    key = (s.d_in, s.d_out, s.r, s.k, s.p, s.x_kind, s.n_outlier, s.outlier_scale, s.seed,
           s.lam, s.dtype, s.n_draw if s.n_draw else s.N)
    if key not in _CACHE:
        n_draw = s.n_draw if s.n_draw else s.N
        w = generate(s.with_rows(1, n_draw))  # the whole draw; prefixes are sliced below
        f = oracle.offline_prepare_from_svd(w.left, w.sigma, w.right, s.r, s.k, s.lam)
        r = {n: oracle.round_to(a, s.dtype) for n, a in
             (("X", w.X), ("U", f.U), ("V", f.V), ("P", f.P), ("W_res", f.W_res))}
        _CACHE.clear()
        _CACHE[key] = r
    r = _CACHE[key]
    return dict(r, X=r["X"][: s.N])


def to_dev(a, dtype):
    td = torch.bfloat16 if dtype == "bf16" else torch.float32
    return torch.from_numpy(np.ascontiguousarray(a)).to("cuda", td)


def make_layer(s: LayerSpec, f, kernels="umma"):
    os.environ["DYRA_KERNELS"] = kernels
    try:
        layer = dyra.DyraLinear(s.d_in, s.d_out, s.r, s.k, s.dtype)
    finally:
        os.environ.pop("DYRA_KERNELS", None)
    layer.load(to_dev(f["U"], s.dtype), to_dev(f["V"], s.dtype),
               to_dev(f["P"], s.dtype) if s.k else None,
               to_dev(f["W_res"], s.dtype) if s.k else None, s.lam)
    return layer


def sample_rows(s: LayerSpec, n=384, seed=0):
    rng = np.random.default_rng(seed)
    rows = set(rng.choice(s.N, size=min(n, s.N), replace=False).tolist())
    for b in range(s.B):
        rows |= {b * s.T, b * s.T + s.T - 1}
    for m in range(128, s.N, 128 * 7):
        rows |= {m - 1, m}
    return np.array(sorted(r for r in rows if r < s.N))


def check(s: LayerSpec, Y: torch.Tensor, f, full=None):
    Yg = Y.double().cpu().numpy()
    if full is None:
        full = s.N * s.d_out <= 60_000_000
    if full:
        rows = np.arange(s.N)
        Yo = oracle.inference(f["X"], f["U"], f["V"], f["P"], f["W_res"], s.lam, s.B, s.T)
    else:
        rows = sample_rows(s)
        Yo = oracle.inference_rows(f["X"], f["U"], f["V"], f["P"], f["W_res"], s.lam, s.B, s.T,
                                   rows)
    Yg = Yg[rows]
    err = oracle.rel_fro(Yg, Yo)
    rms = np.sqrt(np.mean(np.sum(Yo ** 2, axis=1))) + 1e-300
    worst_row = float(np.max(np.linalg.norm(Yg - Yo, axis=1)) / rms)
    assert np.all(np.isfinite(Yg))
    assert err <= TOL[s.dtype], "%s: rel Frobenius %.3e > %.0e" % (s.name, err, TOL[s.dtype])
    assert worst_row <= ROW_TOL * (1 if s.dtype == "bf16" else 1e-3), \
        "%s: worst row %.3e" % (s.name, worst_row)
    return err


def run_spec(s: LayerSpec, kernels="umma"):
    f = prepared(s)
    layer = make_layer(s, f, kernels)
    X = to_dev(f["X"], s.dtype)
    Y = layer.forward(X, B=s.B, T=s.T)
    assert layer.status() == 0
    err = check(s, Y, f)
    layer.close()
    return err


# ------------------------------------------------------- the workloads ----

@pytest.mark.parametrize("name", sorted(CONFIGS))
def test_config_parity(name):
    """Every configuration at full size, in the launch configuration the
    benchmark times (one dyra_forward_batched of B x T rows)."""
    run_spec(CONFIGS[name])


# ------------------------------------------------------------ edge cases ----

EDGE = [
    # name, d_in, d_out, r, k, B, T, lam
    ("ragged_tiles", 256, 512, 64, 32, 3, 201, 1e-3),      # N = 603, instances straddle tiles
    ("many_small_instances", 256, 256, 64, 16, 40, 5, 1e-3),  # 26 instances per 128-row tile
    ("one_row_instances", 128, 192, 32, 8, 300, 1, 1e-3),   # T = 1, k > T
    ("single_row", 256, 512, 64, 32, 1, 1, 1e-3),           # N = 1
    ("odd_sizes", 200, 328, 40, 8, 5, 37, 1e-3),            # d_in, d_out, r off the 64 grid
    ("k72_two_chunks", 256, 512, 64, 72, 2, 300, 1e-3),     # k > 64
    ("k128_max", 512, 384, 128, 128, 2, 260, 1e-3),         # largest supported k
    ("row_splits", 256, 256, 64, 32, 1, 3000, 1e-3),        # Gram reduced over row splits
    ("lambda_zero", 256, 512, 64, 32, 2, 150, 0.0),         # plain ALS normal equations
    ("k_below_rows_lam", 256, 512, 64, 64, 4, 20, 1e-3),    # T < k, ridge keeps G SPD
    ("tall_out", 64, 2048, 16, 16, 2, 100, 1e-3),
    ("wide_in", 2048, 64, 16, 16, 2, 100, 1e-3),
]


@pytest.mark.parametrize("case", EDGE, ids=[c[0] for c in EDGE])
def test_edge_shapes(case):
    name, d_in, d_out, r, k, B, T, lam = case
    run_spec(LayerSpec(name, d_in, d_out, r, k, B, T, "bf16", 0.7, "lognormal", seed=1, lam=lam))


def test_fp32_batched():
    run_spec(LayerSpec("f32_batched", 96, 80, 12, 8, 3, 50, "f32", 0.9, "outlier", n_outlier=3,
                       outlier_scale=20.0, seed=2))


def test_simt_variant_bf16():
    """DYRA_KERNELS=simt runs the bf16 plan on the CUDA-core kernels (a
    debugging variant); it meets the same bar."""
    run_spec(LayerSpec("simt", 256, 512, 64, 32, 3, 201, "bf16", 0.7, "lognormal", seed=1),
             kernels="simt")


GAUSS = [
    # name, d_in, d_out, r, k, B, T, dtype, x_kind (outliers: 8 channels x 20)
    ("gauss_start_ragged", 256, 512, 64, 32, 3, 201, "bf16", "lognormal"),
    ("gauss_start_outliers", 1024, 2048, 128, 64, 1, 128, "bf16", "outlier"),
    ("gauss_start_f32", 96, 80, 12, 8, 3, 50, "f32", "outlier"),
]


@pytest.mark.parametrize("case", GAUSS, ids=[c[0] for c in GAUSS])
def test_gaussian_start(case):
    """A Gaussian ALS start R0 (DyRA Sec. 2.2) changes only the offline
    projector P; the forward is the same one-step layer, checked here against
    the oracle's t = 1 alternating least squares from that start."""
    name, d_in, d_out, r, k, B, T, dtype, x_kind = case
    s = LayerSpec(name, d_in, d_out, r, k, B, T, dtype, 0.7, x_kind, n_outlier=8,
                  outlier_scale=20.0, seed=6)
    w = generate(s)
    R0 = gaussian_r0(k, d_out, s.seed)
    fo = oracle.offline_prepare_from_svd(w.left, w.sigma, w.right, r, k, s.lam, R0=R0)
    f = {n: oracle.round_to(a, dtype) for n, a in
         (("X", w.X), ("U", fo.U), ("V", fo.V), ("P", fo.P), ("W_res", fo.W_res))}
    layer = make_layer(s, f)
    Y = layer.forward(to_dev(f["X"], dtype), B=B, T=T)
    assert layer.status() == 0
    check(s, Y, f, full=True)
    layer.close()
    # the oracle's one-step ALS from R0 is the layer the projector defines: it
    # differs from the reference above only by P's rounding to the storage type
    Ya = oracle.als_inference(f["X"], f["U"], f["V"], f["W_res"], fo.R0, s.lam, B, T, 1)
    Yo = oracle.inference(f["X"], f["U"], f["V"], f["P"], f["W_res"], s.lam, B, T)
    assert oracle.rel_fro(Ya, Yo) < TOL[dtype] / 10


LINEAR = [
    # name, d_in, d_out, r, k, B, T, dtype, alpha, pairs
    ("linear_pairs", 256, 512, 64, 32, 3, 201, "bf16", 0.5, True),
    ("linear_alpha1", 256, 512, 64, 32, 3, 201, "bf16", 1.0, True),
    ("linear_alpha0", 256, 512, 64, 32, 3, 201, "bf16", 0.0, True),
    ("linear_single_cta", 256, 512, 64, 32, 3, 201, "bf16", 0.5, False),
    ("linear_odd_d_out", 200, 328, 40, 8, 5, 37, "bf16", 1.5, True),   # last box past d_out
    ("linear_k72", 256, 512, 64, 72, 2, 300, "bf16", 0.5, True),        # the general solve
    ("linear_weight_only", 256, 512, 64, 0, 3, 201, "bf16", 1.0, True),
    ("linear_f32", 96, 80, 12, 8, 3, 50, "f32", 0.5, True),
    ("linear_vit_fc1", 1024, 4096, 256, 32, 32, 201, "bf16", 0.7, True),  # the ViT-L fc1 shape
    ("linear_compensated", 512, 1024, 64, 64, 1, 300, "bf16", 0.7, True),  # one instance: hi/lo parts
]


@pytest.mark.parametrize("case", LINEAR, ids=[c[0] for c in LINEAR])
def test_bias_and_alpha(case):
    """The full linear layer (DyRA Sec. 2.4): Y = static + b + alpha * correction,
    against the oracle with the same bias (rounded to the storage type) and alpha."""
    name, d_in, d_out, r, k, B, T, dtype, alpha, pairs = case
    s = LayerSpec(name, d_in, d_out, r, k, B, T, dtype, 0.7, "lognormal", seed=3)
    f = prepared(s)
    bias = oracle.round_to(np.random.default_rng(5).standard_normal(d_out) * 0.3, dtype)
    if not pairs:
        os.environ["DYRA_PAIR"] = "0"
    try:
        layer = make_layer(s, f)
    finally:
        os.environ.pop("DYRA_PAIR", None)
    X = to_dev(f["X"], dtype)
    Y0 = layer.forward(X, B=B, T=T).double().cpu().numpy()  # captures a graph first
    layer.set_linear(to_dev(bias, dtype), alpha)
    Y = layer.forward(X, B=B, T=T)
    assert layer.status() == 0
    Yg = Y.double().cpu().numpy()
    Yo = oracle.inference(f["X"], f["U"], f["V"], f["P"], f["W_res"], s.lam, B, T, bias=bias,
                          alpha=alpha)
    err = oracle.rel_fro(Yg, Yo)
    assert err <= TOL[dtype], "%s: rel Frobenius %.3e" % (name, err)
    # the weight-only entry adds the bias too
    Yw = layer.forward_weight_only(X).double().cpu().numpy()
    Ywo = (f["X"] @ f["V"]) @ f["U"].T + bias
    assert oracle.rel_fro(Yw, Ywo) <= TOL[dtype]
    # removing the bias and restoring alpha gives the plain layer back
    layer.set_linear(None, 1.0)
    Y1 = layer.forward(X, B=B, T=T).double().cpu().numpy()
    np.testing.assert_array_equal(Y1, Y0)
    layer.close()


NEWTON_SCHULZ = [
    # name, d_in, d_out, r, k, B, T
    ("ns_instances", 256, 512, 64, 32, 3, 201),       # straddling tiles, k = 32
    ("ns_k64_one", 512, 1024, 64, 64, 1, 700),        # one instance: compensated correction
    ("ns_k40", 200, 328, 40, 40, 2, 150),             # k not a multiple of 16
    ("ns_vit_fc1", 1024, 4096, 256, 32, 32, 201),     # the ViT-L fc1 shape
]


@pytest.mark.parametrize("case", NEWTON_SCHULZ, ids=[c[0] for c in NEWTON_SCHULZ])
def test_newton_schulz_solver(case):
    """The Newton-Schulz solver of the small ridge systems (DyRA Sec. 2.4)
    meets the oracle's exact solve, and agrees with the LDL^T solver's layer."""
    name, d_in, d_out, r, k, B, T = case
    s = LayerSpec(name, d_in, d_out, r, k, B, T, "bf16", 0.7, "lognormal", seed=6)
    f = prepared(s)
    layer = make_layer(s, f)
    X = to_dev(f["X"], "bf16")
    Y_ldl = layer.forward(X, B=B, T=T).clone()
    dyra.dyra_set_solver(layer.plan, dyra.DYRA_SOLVER_NEWTON_SCHULZ, 40)
    Y = layer.forward(X, B=B, T=T)
    assert layer.status() == 0
    check(s, Y, f)
    d = oracle.rel_fro(Y.double().cpu().numpy(), Y_ldl.double().cpu().numpy())
    assert d <= 1e-2, "%s: Newton-Schulz vs LDL %.3e" % (name, d)
    dyra.dyra_set_solver(layer.plan, dyra.DYRA_SOLVER_LDL, 40)
    assert torch.equal(layer.forward(X, B=B, T=T), Y_ldl)
    layer.close()


def test_newton_schulz_solver_limits():
    s, f = _small(k=72)
    layer = make_layer(s, f)
    with pytest.raises(dyra.DyraError) as e:
        dyra.dyra_set_solver(layer.plan, dyra.DYRA_SOLVER_NEWTON_SCHULZ, 40)
    assert e.value.code == dyra.DYRA_ERR_UNSUPPORTED
    for bad in ((2, 40), (1, 0), (1, 201)):
        with pytest.raises(dyra.DyraError) as e:
            dyra.dyra_set_solver(layer.plan, *bad)
        assert e.value.code == dyra.DYRA_ERR_INVALID_ARG
    layer.close()


ALS = [
    # name, d_in, d_out, r, k, B, T, dtype, t, kernels
    ("als_f32_t1.5", 96, 80, 12, 8, 3, 50, "f32", 1.5, "simt"),
    ("als_f32_t2", 96, 80, 12, 8, 3, 50, "f32", 2.0, "simt"),
    ("als_f32_t3_k40", 128, 96, 16, 40, 2, 60, "f32", 3.0, "simt"),
    ("als_bf16_simt_t2", 256, 512, 64, 32, 3, 201, "bf16", 2.0, "simt"),
    # the tensor-core chain: instances straddling 128-row tiles, a ragged tail
    ("als_bf16_t1.5", 256, 512, 64, 32, 3, 201, "bf16", 1.5, "umma"),
    ("als_bf16_t2", 256, 512, 64, 32, 3, 201, "bf16", 2.0, "umma"),
    ("als_bf16_t3", 256, 512, 64, 32, 3, 201, "bf16", 3.0, "umma"),
    ("als_bf16_t2.5_k40", 200, 328, 40, 40, 2, 150, "bf16", 2.5, "umma"),  # k, d_in, d_out odd
    ("als_bf16_t1.5_k64_one", 512, 1024, 64, 64, 1, 700, "bf16", 1.5, "umma"),  # row splits
    ("als_bf16_t2_k72", 256, 512, 64, 72, 2, 300, "bf16", 2.0, "umma"),  # the general solve
    ("als_vit_fc1_t1.5", 1024, 4096, 256, 32, 32, 201, "bf16", 1.5, "umma"),  # the ViT-L fc1 shape
]


@pytest.mark.parametrize("case", ALS, ids=[c[0] for c in ALS])
def test_als_iterations(case):
    """t alternating least-squares iterations (DyRA Sec. 2.2, Sec. 3.3) on the
    CUDA-core or the tensor-core kernels, against the oracle's ALS from the
    same start; t = 1 again afterwards gives the one-step layer."""
    name, d_in, d_out, r, k, B, T, dtype, t, kernels = case
    s = LayerSpec(name, d_in, d_out, r, k, B, T, dtype, 0.7, "outlier", n_outlier=4,
                  outlier_scale=10.0, seed=2)
    w = generate(s)
    fo = oracle.offline_prepare_from_svd(w.left, w.sigma, w.right, r, k, s.lam)
    f = {n: oracle.round_to(a, dtype) for n, a in
         (("X", w.X), ("U", fo.U), ("V", fo.V), ("P", fo.P), ("W_res", fo.W_res))}
    layer = make_layer(s, f, kernels=kernels)
    X = to_dev(f["X"], dtype)
    layer.set_als_iterations(t)
    Y = layer.forward(X, B=B, T=T)
    assert layer.status() == 0
    Yo = oracle.als_inference(f["X"], f["U"], f["V"], f["W_res"], fo.R0, s.lam, B, T, t)
    err = oracle.rel_fro(Y.double().cpu().numpy(), Yo)
    assert err <= TOL[dtype], "%s: rel Frobenius %.3e" % (name, err)
    layer.set_als_iterations(1)
    check(s, layer.forward(X, B=B, T=T), f, full=True)
    layer.close()


def test_als_iterations_on_the_tensor_cores_keep_the_one_step_path():
    """Switching a tensor-core plan to t = 2 and back gives the one-step output
    bit for bit, and the allocation-free entry refuses t > 1."""
    s, f = _small()
    layer = make_layer(s, f)
    X = to_dev(f["X"], "bf16")
    Y1 = layer.forward(X, B=s.B, T=s.T).clone()
    layer.set_als_iterations(2)
    Y2 = layer.forward(X, B=s.B, T=s.T).clone()
    assert layer.status() == 0 and not torch.equal(Y1, Y2)
    Yn = torch.empty_like(Y2)
    with pytest.raises(dyra.DyraError) as e:
        dyra.dyra_forward_batched_noalloc(layer.plan, X, Yn, s.B, s.T)
    assert e.value.code == dyra.DYRA_ERR_UNSUPPORTED
    layer.set_als_iterations(1)
    assert torch.equal(layer.forward(X, B=s.B, T=s.T), Y1)
    layer.close()


def test_als_printed_t15_schedule_on_the_tensor_cores():
    """The update sequence the text prints for t = 1.5 (L, R, L, R, L: five
    updates) runs as half_steps = 5 and matches the oracle's printed schedule."""
    s = LayerSpec("als_printed", 256, 512, 64, 32, 3, 201, "bf16", 0.7, "outlier", n_outlier=4,
                  outlier_scale=10.0, seed=2)
    w = generate(s)
    fo = oracle.offline_prepare_from_svd(w.left, w.sigma, w.right, s.r, s.k, s.lam)
    f = {n: oracle.round_to(a, "bf16") for n, a in
         (("X", w.X), ("U", fo.U), ("V", fo.V), ("P", fo.P), ("W_res", fo.W_res))}
    layer = make_layer(s, f)
    X = to_dev(f["X"], "bf16")
    dyra.dyra_set_als_steps(layer.plan, oracle.als_updates(1.5, "printed"))
    Y = layer.forward(X, B=s.B, T=s.T)
    assert layer.status() == 0
    Yo = oracle.als_inference(f["X"], f["U"], f["V"], f["W_res"], fo.R0, s.lam, s.B, s.T, 1.5,
                              schedule="printed")
    assert oracle.rel_fro(Y.double().cpu().numpy(), Yo) <= TOL["bf16"]
    layer.close()


@pytest.mark.parametrize("B,T", [(32, 201), (3, 201), (1, 600)])
def test_host_forward_matches_device_forward(B, T):
    """dyra_forward_batched_host (host buffers, copies overlapped by chunks of
    instances) meets the oracle like the device-buffer forward. The chunks are
    forwards of fewer instances, whose Gram reduction may split rows
    differently, so the two agree to rounding, not bit for bit."""
    s = LayerSpec("host", 256, 512, 64, 32, B, T, "bf16", 0.7, "lognormal", seed=4)
    f = prepared(s)
    layer = make_layer(s, f)
    Xd = to_dev(f["X"], "bf16")
    Yd = layer.forward(Xd, B=B, T=T).cpu()
    Xh = Xd.cpu().pin_memory()
    Yh = layer.forward_host(Xh, B=B, T=T)
    torch.cuda.current_stream().synchronize()
    assert layer.status() == 0
    check(s, Yh, f, full=True)
    assert oracle.rel_fro(Yh.double().numpy(), Yd.double().numpy()) <= TOL["bf16"] / 2
    layer.close()


HILO = [
    # name, d_in, d_out, r, k, B, T, outlier channels (x20)
    ("hilo_single", 1024, 2048, 128, 64, 1, 128, 8),
    ("hilo_batched", 256, 512, 64, 32, 3, 201, 8),
    ("hilo_needed", 512, 1024, 64, 64, 1, 128, 6),   # modelled 1.1e-2 without it, 6.8e-3 with
]


def _run_hilo(s, f, mode):
    os.environ["DYRA_HILO"] = mode
    try:
        layer = make_layer(s, f)
    finally:
        os.environ.pop("DYRA_HILO", None)
    Y = layer.forward(to_dev(f["X"], s.dtype), B=s.B, T=s.T)
    assert layer.status() == 0
    layer.close()
    Yo = oracle.inference(f["X"], f["U"], f["V"], f["P"], f["W_res"], s.lam, s.B, s.T)
    return oracle.rel_fro(Y.double().cpu().numpy(), Yo)


@pytest.mark.parametrize("case", HILO, ids=[c[0] for c in HILO])
def test_compensated_correction(case):
    """L~ and Q^T with their bf16 rounding errors (hi.hi + hi.lo + lo.hi in
    the output stage) cut the error the grouping L~ . Q amplifies on
    ill-conditioned instances (outlier channels)."""
    name, d_in, d_out, r, k, B, T, nout = case
    s = LayerSpec(name, d_in, d_out, r, k, B, T, "bf16", 0.6, "outlier", n_outlier=nout,
                  outlier_scale=20.0, seed=5)
    f = prepared(s)
    err_on = _run_hilo(s, f, "1")
    assert err_on <= TOL["bf16"], "%s: %.3e" % (name, err_on)
    if name != "hilo_needed":
        err_off = _run_hilo(s, f, "0")
        assert err_on < 0.8 * err_off, (err_on, err_off)


MONARCH = [
    # name, b1, b2, b1', b2', k, B, T, dtype, kernels
    ("monarch_f32", 8, 12, 8, 12, 8, 3, 50, "f32", "simt"),
    ("monarch_f32_k0", 6, 6, 6, 6, 0, 2, 40, "f32", "simt"),
    ("monarch_f32_rect", 6, 8, 4, 10, 8, 2, 45, "f32", "simt"),
    ("monarch_bf16_simt", 16, 16, 16, 16, 32, 3, 201, "bf16", "simt"),
    # the tensor cores: instances straddling tiles, blocks narrower than a tile
    ("monarch_bf16", 16, 16, 16, 16, 32, 3, 201, "bf16", "umma"),
    ("monarch_bf16_k0", 16, 16, 16, 16, 0, 2, 150, "bf16", "umma"),
    ("monarch_bf16_rect", 16, 16, 8, 64, 32, 3, 201, "bf16", "umma"),
    ("monarch_bf16_narrow", 32, 32, 64, 16, 32, 2, 130, "bf16", "umma"),
    ("monarch_bf16_k64_one", 16, 32, 32, 16, 64, 1, 700, "bf16", "umma"),
    ("monarch_vit_block_proj", 32, 32, 32, 32, 32, 64, 201, "bf16", "umma"),
]


def _monarch_layer(case, seed=8):
    from oracle import monarch as mon
    name, b1, b2, b1o, b2o, k, B, T, dtype, kernels = case
    d_in, d_out = b1 * b2, b1o * b2o
    s = LayerSpec(name, d_in, d_out, 1, k, B, T, dtype, 0.7, "lognormal", seed=seed)
    w = generate(s)
    fo = mon.offline_prepare_monarch(w.weight(), b1, b2, k, s.lam, b1o=b1o, b2o=b2o)
    rd = lambda a: oracle.round_to(a, dtype)
    Lb = rd(np.stack(fo.Lb))
    Rb = rd(np.stack(fo.Rb))
    P, W_res, X = rd(fo.P), rd(fo.W_res), rd(w.X)
    os.environ["DYRA_KERNELS"] = kernels
    try:
        layer = dyra.DyraMonarchLinear(d_in, b1, b2, k, dtype, b1o=b1o, b2o=b2o)
    finally:
        os.environ.pop("DYRA_KERNELS", None)
    layer.load(to_dev(Lb, dtype), to_dev(Rb, dtype), to_dev(P, dtype) if k else None,
               to_dev(W_res, dtype) if k else None, s.lam)
    fr = mon.MonarchFactors(list(Lb), list(Rb), mon.monarch_matrix(list(Lb), list(Rb)).T, P, W_res,
                            fo.R0)
    return s, layer, X, fr


@pytest.mark.parametrize("case", MONARCH, ids=[c[0] for c in MONARCH])
def test_monarch_static_part(case):
    """A Monarch static part (DyRA App. B; square, or rectangular blocks as read
    for rectangular layers) under the same correction, on the tensor cores
    (bf16) or the CUDA cores, against the oracle's Monarch layer."""
    from oracle import monarch as mon
    s, layer, X, fr = _monarch_layer(case)
    dtype = s.dtype
    Y = layer.forward(to_dev(X, dtype), B=s.B, T=s.T)
    assert layer.status() == 0
    Yo = mon.monarch_inference(X, fr, s.lam, s.B, s.T)
    err = oracle.rel_fro(Y.double().cpu().numpy(), Yo)
    assert err <= TOL[dtype], "%s: rel Frobenius %.3e" % (s.name, err)
    layer.close()


def test_monarch_bias_alpha_and_newton_schulz():
    """The full linear layer (bias, alpha) and the Newton-Schulz solver on a
    tensor-core Monarch plan, against the oracle."""
    from oracle import monarch as mon
    case = ("monarch_linear", 16, 16, 8, 64, 32, 3, 201, "bf16", "umma")
    s, layer, X, fr = _monarch_layer(case, seed=9)
    bias = oracle.round_to(np.random.default_rng(2).standard_normal(s.d_out) * 0.3, "bf16")
    layer.set_linear(to_dev(bias, "bf16"), 0.6)
    dyra.dyra_set_solver(layer.plan, dyra.DYRA_SOLVER_NEWTON_SCHULZ, 40)
    Y = layer.forward(to_dev(X, "bf16"), B=s.B, T=s.T)
    assert layer.status() == 0
    Ys = X @ fr.What.T
    Yc = mon.monarch_inference(X, fr, s.lam, s.B, s.T) - Ys
    Yo = Ys + bias + 0.6 * Yc
    assert oracle.rel_fro(Y.double().cpu().numpy(), Yo) <= TOL["bf16"]
    with pytest.raises(dyra.DyraError) as e:
        layer.set_als_iterations(2)
    assert e.value.code == dyra.DYRA_ERR_UNSUPPORTED
    layer.close()


# ----------------------------------------------------------- properties ----

def _small(k=32, lam=1e-3, B=3, T=201, dtype="bf16"):
    s = LayerSpec("p", 256, 512, 64, k, B, T, dtype, 0.7, "lognormal", seed=4, lam=lam)
    return s, prepared(s)


def test_weight_only_k0_plan_matches_oracle_and_weight_only_entry():
    s0, f0 = _small(k=0)
    layer0 = make_layer(s0, f0)
    X = to_dev(f0["X"], "bf16")
    Y0 = layer0.forward(X, B=s0.B, T=s0.T)
    Ywo = oracle.weight_only(f0["X"], f0["U"], f0["V"])
    assert oracle.rel_fro(Y0.double().cpu().numpy(), Ywo) <= 1e-2
    s, f = _small(k=32)
    layer = make_layer(s, f)
    Y1 = layer.forward_weight_only(X)
    assert torch.equal(Y0, Y1)
    layer.close()
    layer0.close()


def test_forward_is_batched_with_one_instance_and_deterministic():
    s, f = _small(B=1, T=603)
    layer = make_layer(s, f)
    X = to_dev(f["X"], "bf16")
    Y1 = torch.empty(603, 512, device="cuda", dtype=torch.bfloat16)
    Y2 = torch.empty_like(Y1)
    Y3 = torch.empty_like(Y1)
    dyra.dyra_forward(layer.plan, X, Y1, 603)
    dyra.dyra_forward_batched(layer.plan, X, Y2, 1, 603)
    dyra.dyra_forward(layer.plan, X, Y3, 603)
    torch.cuda.synchronize()
    assert torch.equal(Y1, Y2) and torch.equal(Y1, Y3)
    layer.close()


def test_side_stream():
    s, f = _small()
    layer = make_layer(s, f)
    X = to_dev(f["X"], "bf16")
    Y1 = layer.forward(X, B=s.B, T=s.T)
    st = torch.cuda.Stream()
    with torch.cuda.stream(st):
        Y2 = layer.forward(X, B=s.B, T=s.T, stream=st)
    st.synchronize()
    assert torch.equal(Y1, Y2)
    layer.close()


def test_graph_replay_matches_direct_launches():
    """The per-plan CUDA-graph cache replays exactly the launches a direct
    forward makes (DYRA_GRAPHS=0 disables the cache)."""
    s, f = _small()
    X = to_dev(f["X"], "bf16")
    os.environ["DYRA_GRAPHS"] = "0"
    try:
        direct = make_layer(s, f)
    finally:
        os.environ.pop("DYRA_GRAPHS")
    cached = make_layer(s, f)
    Yd = direct.forward(X, B=s.B, T=s.T)
    Yc = [cached.forward(X, B=s.B, T=s.T) for _ in range(3)]  # new Y each call: new graphs
    Y = torch.empty_like(Yd)
    for _ in range(3):
        cached.forward(X, B=s.B, T=s.T, Y=Y)  # same arguments: replays one graph
    torch.cuda.synchronize()
    assert all(torch.equal(Yd, y) for y in Yc + [Y])
    direct.close()
    cached.close()


def test_pair_output_stage_matches_single_cta():
    """The output stage on CTA pairs (default) and on single CTAs
    (DYRA_PAIR=0) agree and both meet the oracle bar."""
    s, f = _small(B=3, T=201)
    X = to_dev(f["X"], "bf16")
    os.environ["DYRA_PAIR"] = "0"
    try:
        single = make_layer(s, f)
    finally:
        os.environ.pop("DYRA_PAIR")
    pair = make_layer(s, f)
    Y1 = single.forward(X, B=s.B, T=s.T)
    Y2 = pair.forward(X, B=s.B, T=s.T)
    assert pair.status() == 0
    assert oracle.rel_fro(Y2.double().cpu().numpy(), Y1.double().cpu().numpy()) <= 1e-3
    check(s, Y2, f)
    single.close()
    pair.close()


def _layer_with_factor(s, f, placement):
    """placement: 'shared' (the first solve block of each instance factors G_b
    and publishes it) or 'self' (every solve block factors it)."""
    os.environ["DYRA_FACTOR"] = placement
    try:
        return make_layer(s, f)
    finally:
        os.environ.pop("DYRA_FACTOR", None)


@pytest.mark.parametrize("placement", ["self"])
@pytest.mark.parametrize("k,B,T", [(32, 3, 201), (64, 2, 150), (24, 1, 3000), (64, 1, 3000),
                                   (32, 40, 64)])
def test_factor_placements_agree(placement, k, B, T):
    """G_b factored once per instance by the first solve block or by every
    solve block gives the same layer, also on a second call (the per-instance
    flags start from zero again)."""
    s, f = _small(k=k, B=B, T=T)
    X = to_dev(f["X"], "bf16")
    other = _layer_with_factor(s, f, placement)
    shared = _layer_with_factor(s, f, "shared")
    Ys1 = shared.forward(X, B=s.B, T=s.T)
    Ys2 = shared.forward(X, B=s.B, T=s.T)
    Yo1 = other.forward(X, B=s.B, T=s.T)
    Yo2 = other.forward(X, B=s.B, T=s.T)
    assert other.status() == 0 and shared.status() == 0
    assert torch.equal(Ys1, Ys2) and torch.equal(Yo1, Yo2)
    assert oracle.rel_fro(Yo1.double().cpu().numpy(), Ys1.double().cpu().numpy()) <= 1e-3
    check(s, Ys1, f)
    other.close()
    shared.close()


@pytest.mark.parametrize("d_in,B,T", [(1024, 1, 64), (2048, 2, 40), (4096, 1, 1)])
def test_projection_split_k(d_in, B, T):
    """Few row tiles and a long K: the projection splits K across the CTAs of
    a cluster, which sum their fp32 partials over distributed shared memory
    in split order. Repeated calls agree bit for bit, and the weight-only
    layer (another tiling of the same stage) stays right."""
    s = LayerSpec("sk", d_in, 512, 256, 32, B, T, "bf16", 0.7, "lognormal", seed=5, lam=1e-3)
    f = prepared(s)
    layer = make_layer(s, f)
    X = to_dev(f["X"], "bf16")
    Y1 = layer.forward(X, B=s.B, T=s.T)
    Y2 = layer.forward(X, B=s.B, T=s.T)
    Ywo = layer.forward_weight_only(X)
    Y3 = layer.forward(X, B=s.B, T=s.T)
    assert layer.status() == 0
    assert torch.equal(Y1, Y2) and torch.equal(Y1, Y3)
    check(s, Y1, f)
    wo = oracle.weight_only(f["X"], f["U"], f["V"])
    assert oracle.rel_fro(Ywo.double().cpu().numpy(), wo) <= 1e-2
    layer.close()


def test_forward_inside_caller_graph_capture():
    """A forward issued while the caller captures its stream is recorded into
    the caller's graph (the workspace is reserved beforehand)."""
    s, f = _small()
    layer = make_layer(s, f)
    X = to_dev(f["X"], "bf16")
    want = layer.forward(X, B=s.B, T=s.T)
    Y = torch.zeros_like(want)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        layer.forward(X, B=s.B, T=s.T, Y=Y)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(Y, want)
    del g
    layer.close()


def test_rank_deficient_is_an_error():
    s, f = _small(k=32, lam=0.0, B=2, T=20)
    layer = make_layer(s, f)
    X = to_dev(f["X"], "bf16")
    with pytest.raises(dyra.DyraError) as e:
        layer.forward(X, B=2, T=20)
    assert e.value.code == dyra.DYRA_ERR_RANK_DEFICIENT
    layer.close()


@pytest.mark.parametrize("placement", ["shared", "self"])
def test_zero_input_without_ridge_flags_pivot(placement):
    """X_b = 0 and lambda = 0 make L^T L = 0: the factorisation (wherever it
    runs) flags the pivot and drops that instance's correction, leaving the
    weight-only output (0)."""
    s, f = _small(k=32, lam=0.0, B=2, T=64)
    layer = _layer_with_factor(s, f, placement)
    X = torch.zeros(128, 256, device="cuda", dtype=torch.bfloat16)
    Y = layer.forward(X, B=2, T=64)
    st = layer.status()
    assert st & dyra.DYRA_STATUS_NONPOSITIVE_PIVOT
    assert torch.count_nonzero(Y).item() == 0
    assert layer.status() == 0  # cleared by the read
    layer.close()


def test_not_loaded_and_misaligned():
    plan = dyra.dyra_plan_create(256, 512, 64, 32, dyra.DYRA_BF16)
    X = torch.zeros(64, 256, device="cuda", dtype=torch.bfloat16)
    Y = torch.zeros(64, 512, device="cuda", dtype=torch.bfloat16)
    with pytest.raises(dyra.DyraError) as e:
        dyra.dyra_forward(plan, X, Y, 64)
    assert e.value.code == dyra.DYRA_ERR_NOT_LOADED
    s, f = _small()
    U, V, P, W = (to_dev(f[n], "bf16") for n in ("U", "V", "P", "W_res"))
    dyra.dyra_load_factors(plan, U, V, P, W, 1e-3)
    with pytest.raises(dyra.DyraError) as e:
        dyra.dyra_forward(plan, X.data_ptr() + 2, Y, 63)
    assert e.value.code == dyra.DYRA_ERR_ALIGNMENT
    with pytest.raises(dyra.DyraError) as e:
        dyra.dyra_load_factors(plan, U, V, P, W, -1.0)
    assert e.value.code == dyra.DYRA_ERR_INVALID_ARG
    dyra.dyra_forward(plan, X, Y, 0)  # empty input is a no-op
    dyra.dyra_plan_destroy(plan)


def test_allocation_failure_is_reported():
    os.environ["DYRA_TEST_FAIL_ALLOC"] = "1"
    try:
        with pytest.raises(dyra.DyraError) as e:
            dyra.dyra_plan_create(256, 512, 64, 32, dyra.DYRA_BF16)
        assert e.value.code == dyra.DYRA_ERR_ALLOC
    finally:
        os.environ.pop("DYRA_TEST_FAIL_ALLOC")
