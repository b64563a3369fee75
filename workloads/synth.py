"""Seeded synthetic inputs shaped like the pages' workloads.

The pages calibrate on 2048 WikiText tokens of SmolLM-135M, Qwen2.5-0.5B and
TinyLlama-1.1B ("Warum Geometrie Gewichte nicht komprimiert", Methodik and
Teil 1).  Neither the models nor the text are available, so these generators
stand in for them:

* cone activations x = 3·u + z, u a seeded unit vector, z ~ N(0, diag(σ²)) with
  σ_k = k^-0.7 (k = 1..n): a narrow cone with mean pairwise cosine ≈ 0.75, as
  Teil 1 of that page measures;
* weights ~ N(0, 0.02²);
* a stress input of Student-t (3 degrees of freedom) noise with 1 % of the
  channels scaled by 20.

Every draw uses its own torch CPU generator seeded with
42 + 1000·layer + tensor_id, so the CUDA path and the oracle see identical bits.
"""
from __future__ import annotations

import torch

BASE_SEED = 42


def seed_for(layer: int, tensor_id: int) -> int:
    return BASE_SEED + 1000 * int(layer) + int(tensor_id)


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def cone_activations(T: int, n: int, seed: int, radius: float = 3.0,
                     decay: float = 0.7) -> torch.Tensor:
    """T × n float32 activations x = radius·u + z (see module docstring)."""
    g = _gen(seed)
    u = torch.randn(n, generator=g, dtype=torch.float64)
    u = u / torch.linalg.vector_norm(u)
    sigma = torch.arange(1, n + 1, dtype=torch.float64).pow(-decay)
    z = torch.randn(T, n, generator=g, dtype=torch.float64) * sigma
    return (radius * u + z).to(torch.float32)


def gaussian_weights(rows: int, cols: int, seed: int,
                     std: float = 0.02) -> torch.Tensor:
    """rows × cols float32 weights ~ N(0, std²)."""
    g = _gen(seed)
    return torch.randn(rows, cols, generator=g, dtype=torch.float32) * std


def student_t_activations(T: int, n: int, seed: int, df: int = 3,
                          outlier_frac: float = 0.01,
                          outlier_scale: float = 20.0) -> torch.Tensor:
    """T × n float32 Student-t(df) noise; round(frac·n) channels × scale.

    t = z / sqrt(χ²_df/df) with χ²_df a sum of df squared standard normals.
    The outlier channels are a seeded choice of distinct columns.
    """
    g = _gen(seed)
    z = torch.randn(T, n, generator=g, dtype=torch.float32)
    chi2 = torch.zeros(T, n, dtype=torch.float32)
    for _ in range(df):
        chi2 += torch.randn(T, n, generator=g, dtype=torch.float32).square()
    x = z / torch.sqrt(chi2 / df)
    k = int(round(outlier_frac * n))
    if k > 0:
        cols = torch.randperm(n, generator=g)[:k]
        x[:, cols] *= outlier_scale
    return x


def swiglu_input(X: torch.Tensor, W_gate: torch.Tensor,
                 W_up: torch.Tensor) -> torch.Tensor:
    """down_proj input SiLU(X·W_gateᵀ)·(X·W_upᵀ), float32 then rounded to bf16.

    X, W_gate and W_up are taken as the bf16 values the layer holds.
    """
    Xf = X.to(torch.bfloat16).to(torch.float32)
    G = Xf @ W_gate.to(torch.bfloat16).to(torch.float32).T
    Up = Xf @ W_up.to(torch.bfloat16).to(torch.float32).T
    return (torch.nn.functional.silu(G) * Up).to(torch.bfloat16)


def normal_matrix(rows: int, cols: int, seed: int) -> torch.Tensor:
    """rows × cols float32 standard normal entries (e.g. a randomized SVD's
    test matrix, drawn by the caller)."""
    g = _gen(seed)
    return torch.randn(rows, cols, generator=g, dtype=torch.float32)


def spectral_weights(rows: int, cols: int, seed: int, decay: float = 0.8,
                     std: float = 0.02) -> torch.Tensor:
    """rows × cols float32 weights with singular values k^−decay (random
    orthonormal bases), scaled to an entry std of about ``std``."""
    g = _gen(seed)
    k = min(rows, cols)
    a = torch.randn(rows, k, generator=g, dtype=torch.float64)
    b = torch.randn(cols, k, generator=g, dtype=torch.float64)
    qa, _ = torch.linalg.qr(a)
    qb, _ = torch.linalg.qr(b)
    sig = torch.arange(1, k + 1, dtype=torch.float64).pow(-decay)
    w = (qa * sig) @ qb.T
    w = w * (std / w.std())
    return w.to(torch.float32)


def student_t_weights(rows: int, cols: int, seed: int, df: int = 3,
                      std: float = 0.02) -> torch.Tensor:
    """rows × cols float32 weights std·t with t ~ Student-t(df) (z over
    sqrt(χ²_df/df)): a heavy-tailed layer, the case outlier-keeping schemes
    are made for."""
    g = _gen(seed)
    z = torch.randn(rows, cols, generator=g, dtype=torch.float32)
    chi2 = torch.zeros(rows, cols, dtype=torch.float32)
    for _ in range(df):
        chi2 += torch.randn(rows, cols, generator=g, dtype=torch.float32).square()
    return z / torch.sqrt(chi2 / df) * std
