"""Seeded synthetic layers and activations with the shapes of the DyRA workloads.

Source: "DyRA: Dynamic Residual Approximation for Efficient Matrix Multiplication
in DNNs" (Chae, Chung, Lee, Kim). The paper evaluates ViT-L (Sec. 3.1, App. D),
Wav2Vec2/Whisper-class speech encoders (Table 1, App. D) and LLaMA-7B / LLaDA-8B
linear layers (Sec. 3.1, App. E.1). None of those weights or datasets is
available here, so each workload below is a seeded stand-in with the layer's
shape, a power-law singular spectrum and activation statistics of the stated
kind (per-channel log-normal scales, or a few large outlier channels).

Conventions (PyTorch layout, used everywhere in this repository):
  X  : N x d_in activations, N = B*T rows, B independent instances of T rows
  W  : d_out x d_in weight, Y = X . W^T
  W  = left . diag(sigma) . right^T with left (d_out x m), right (d_in x m)
       orthonormal and m = min(d_in, d_out).

Draw order for one layer (fixed, so any consumer reproduces the same arrays):
  1. left basis  (Haar: QR of a d_out x m Gaussian, signs fixed by diag(R))
  2. right basis (Haar: QR of a d_in x m Gaussian, signs fixed by diag(R))
  3. X noise     (N_draw x d_in standard normal)
  4. channel scales (log-normal: s_j = exp(z_j), z_j ~ N(0,1)) or outlier
     channels (chosen without replacement, multiplied by a constant)
All draws come from numpy.random.default_rng(seed).
"""

from __future__ import annotations

import dataclasses
from typing import Dict, Optional, Tuple

import numpy as np


@dataclasses.dataclass(frozen=True)
class LayerSpec:
    """One DyRA layer workload.

    name      : identifier used by tests and the benchmark
    d_in      : input features
    d_out     : output features
    r         : static rank of the low-rank weight factorisation
    k         : rank of the input-dependent residual correction
    B, T      : instances and rows per instance (N = B*T rows in total)
    dtype     : storage type of the GPU path, 'f32' or 'bf16'
    p         : spectrum exponent, sigma_i = i^(-p), i = 1..min(d_in, d_out)
    x_kind    : 'lognormal' or 'outlier'
    n_outlier : outlier channel count (x_kind == 'outlier')
    outlier_scale : multiplier of the outlier channels
    seed      : numpy default_rng seed
    lam       : ridge constant of the Gram matrices
    n_draw    : rows drawn for X (>= B*T); the workload uses the first B*T rows
    """

    name: str
    d_in: int
    d_out: int
    r: int
    k: int
    B: int
    T: int
    dtype: str
    p: float
    x_kind: str
    n_outlier: int = 0
    outlier_scale: float = 1.0
    seed: int = 0
    lam: float = 1e-3
    n_draw: Optional[int] = None

    @property
    def N(self) -> int:
        return self.B * self.T

    @property
    def m(self) -> int:
        return min(self.d_in, self.d_out)

    def with_rows(self, B: int, T: int) -> "LayerSpec":
        """Same layer and draw, a different instance split (prefix of the draw)."""
        n_draw = self.n_draw if self.n_draw is not None else self.N
        if B * T > n_draw:
            raise ValueError("more rows than the draw holds")
        return dataclasses.replace(self, B=B, T=T, n_draw=n_draw)


# Llama-shaped up-projection: N swept over these token counts, X is the
# N-row prefix of one 8192-row draw.
LLAMA_SWEEP: Tuple[int, ...] = (1, 16, 128, 1024, 8192)


def _configs() -> Dict[str, LayerSpec]:
    c = {}
    # Tiny fp32 single linear: X 64x256 (N(0,1) rows, 4 outlier channels x20),
    # W 256x256 with sigma_i = 1/i, r=32, k=8, seed 0.
    c["tiny_f32"] = LayerSpec("tiny_f32", 256, 256, 32, 8, 1, 64, "f32", 1.0,
                              "outlier", n_outlier=4, outlier_scale=20.0, seed=0)
    # ViT-L/16 MLP fc1, 32 images x 201 tokens.
    c["vit_fc1"] = LayerSpec("vit_fc1", 1024, 4096, 256, 32, 32, 201, "bf16", 0.7,
                             "lognormal", seed=0)
    # ViT-L/16 block linears, batch 64 x 201 tokens, r = min(d_in, d_out)/4,
    # seed = layer index within the block.
    for i, (nm, di, do) in enumerate((("qkv", 1024, 3072), ("proj", 1024, 1024),
                                      ("fc1", 1024, 4096), ("fc2", 4096, 1024))):
        c["vit_block_" + nm] = LayerSpec("vit_block_" + nm, di, do, min(di, do) // 4, 32,
                                         64, 201, "bf16", 0.7, "lognormal", seed=i)
    # Whisper-large-shaped encoder fc1, 8 clips x 1500 frames.
    c["whisper_fc1"] = LayerSpec("whisper_fc1", 1280, 5120, 320, 64, 8, 1500, "bf16", 0.6,
                                 "lognormal", seed=0)
    # Llama-shaped MLP up-projection; one instance of N tokens, 1% outlier
    # channels (round(0.01*4096) = 41) scaled x50.
    for n in LLAMA_SWEEP:
        c["llama_up_%d" % n] = LayerSpec("llama_up_%d" % n, 4096, 14336, 1024, 64, 1, n,
                                         "bf16", 0.5, "outlier", n_outlier=41,
                                         outlier_scale=50.0, seed=0, n_draw=max(LLAMA_SWEEP))
    return c


CONFIGS: Dict[str, LayerSpec] = _configs()


def spec(name: str) -> LayerSpec:
    return CONFIGS[name]


@dataclasses.dataclass
class Workload:
    spec: LayerSpec
    X: np.ndarray       # N x d_in float64
    left: np.ndarray    # d_out x m float64, orthonormal columns
    sigma: np.ndarray   # m float64, decreasing
    right: np.ndarray   # d_in x m float64, orthonormal columns

    def weight(self) -> np.ndarray:
        """The dense weight W = left . diag(sigma) . right^T (d_out x d_in)."""
        return (self.left * self.sigma) @ self.right.T


def haar_orthonormal(rng: np.random.Generator, d: int, m: int) -> np.ndarray:
    """d x m matrix with orthonormal columns, Haar-distributed.

    QR of a Gaussian matrix with the column signs fixed so that diag(R) > 0
    (Mezzadri's recipe for the Haar measure).
    """
    g = rng.standard_normal((d, m))
    q, r = np.linalg.qr(g)
    return q * np.sign(np.diag(r))


def make_activations(rng: np.random.Generator, n_rows: int, d_in: int, x_kind: str,
                     n_outlier: int = 0, outlier_scale: float = 1.0) -> np.ndarray:
    """X noise then channel scaling, in that draw order."""
    X = rng.standard_normal((n_rows, d_in))
    if x_kind == "lognormal":
        X *= np.exp(rng.standard_normal(d_in))
    elif x_kind == "outlier":
        idx = rng.choice(d_in, size=n_outlier, replace=False)
        X[:, idx] *= outlier_scale
    elif x_kind == "normal":
        pass
    else:
        raise ValueError("unknown x_kind %r" % x_kind)
    return X


def generate(s: LayerSpec, spectrum: Optional[np.ndarray] = None) -> Workload:
    """Draw one workload. `spectrum` overrides sigma (used by invariant tests)."""
    rng = np.random.default_rng(s.seed)
    m = s.m
    left = haar_orthonormal(rng, s.d_out, m)
    right = haar_orthonormal(rng, s.d_in, m)
    n_draw = s.n_draw if s.n_draw is not None else s.N
    X = make_activations(rng, n_draw, s.d_in, s.x_kind, s.n_outlier, s.outlier_scale)[: s.N]
    if spectrum is None:
        sigma = np.arange(1, m + 1, dtype=np.float64) ** (-s.p)
    else:
        sigma = np.asarray(spectrum, dtype=np.float64)
        if sigma.shape != (m,):
            raise ValueError("spectrum must have min(d_in, d_out) entries")
    return Workload(s, np.ascontiguousarray(X), left, sigma, right)


def gaussian_r0(k: int, d_out: int, seed: int) -> np.ndarray:
    """A Gaussian start R0 (k x d_out) for the alternating least squares.

    The DyRA paper initialises R^(0) from a Gaussian distribution in its ALS
    convergence study (Sec. 2.2, Fig. 2; App. E.3) without giving the variance.
    Entries here are i.i.d. N(0, 1/d_out), so each row has squared norm about
    1, like the orthonormal rows of the singular-vector start, and the ridge
    term weighs the same against either. The draws come from their own stream,
    numpy.random.default_rng([seed, 1]), so the layer draws above are unchanged.
    """
    rng = np.random.default_rng([seed, 1])
    return rng.standard_normal((k, d_out)) / np.sqrt(d_out)
