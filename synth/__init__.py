"""Seeded synthetic inputs shared by the CPU oracle, the tests and ``bench.py``.

This module only draws random numbers and shapes them; it holds none of the
codec's arithmetic (no rotation, no codebook, no quantization, no attention).
Both the oracle and the CUDA path receive the same arrays from here, so a
parity test compares the two implementations on identical inputs.

Workload recipes (the pages print no data; these stand in for the protein and
LLM activations, and for the GloVe search set, that the pages evaluate on):

* ``heavy_tailed``: i.i.d. N(0, 1) entries; per (layer, kv-head) a seeded set
  of 4 channels is scaled by 20 for every token.  Channel outliers that persist
  across tokens are the failure mode TurboESM's problem statement describes
  (values 10-100x the median; TurboESM, "Résumé technique" §1).
* ``lognormal_channels``: per (layer, head, channel) scale ~ LogNormal(0, 0.5);
  each channel independently becomes an outlier (x15) with probability 0.02.
* ``anisotropic``: x = U (lambda^1/2 * g), lambda_i = i^-0.8 (i = 1..d),
  U a seeded Haar-random orthogonal basis, g ~ N(0, I).

Random numbers that the method itself draws (the Hadamard sign diagonal, the
Gaussian QJL projection, the Gaussian matrix whose QR gives a dense rotation)
are also produced here and passed to both sides as inputs.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "rotation_randomness",
    "heavy_tailed",
    "lognormal_channels",
    "anisotropic",
    "haar_basis",
    "outlier_channels",
    "CONFIGS",
]


# Configuration presets: the five workloads, by what they are.
CONFIGS = {
    "tiny_d128_t1024": dict(
        heads=1, head_dim=128, tokens=1024, code_bits=2, dtype="f32",
        law="heavy_tailed", rope_base=10000.0, seed=1001),
    "esm2_650m_encoder": dict(
        layers=33, batch=8, heads=20, head_dim=64, tokens=1024, code_bits=2,
        dtype="bf16", law="lognormal_channels", rope_base=10000.0, seed=1002),
    "llama31_8b_gqa_decode": dict(
        layers=32, batch=16, q_heads=32, kv_heads=8, head_dim=128,
        tokens=32768, code_bits=(2, 3), dtype="bf16", law="heavy_tailed",
        rope_base=10000.0, seed=1003),
    "llama31_70b_long_slice": dict(
        layers=1, batch=1, q_heads=64, kv_heads=8, head_dim=128,
        tokens=1 << 20, code_bits=2, dtype="bf16", law="heavy_tailed",
        rope_base=10000.0, seed=1004),
    "vector_search_d1536": dict(
        n_db=1_000_000, dim=1536, n_queries=1000, code_bits=(1, 3), top_k=10,
        law="anisotropic", seed=1005),
}


def _rng(seed) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence(seed))


def rotation_randomness(d: int, seed: int, dense: bool = False, m: int | None = None):
    """Random draws a rotation handle is built from.

    Returns a dict with
      ``signs``: int8 [d] of +-1 (the sign diagonal of a randomized Hadamard),
      ``gauss_s``: float32 [m, d] i.i.d. N(0, 1) (the QJL projection before
        the codec rounds it to bf16-representable values),
      ``gauss_pi``: float64 [d, d] i.i.d. N(0, 1) when ``dense`` (its QR factor
        is the dense rotation), else None.
    """
    m = d if m is None else m
    g = _rng([*np.atleast_1d(seed).tolist(), 0x5107])
    signs = np.where(g.random(d) < 0.5, -1, 1).astype(np.int8)
    gauss_s = g.standard_normal((m, d), dtype=np.float32)
    gauss_pi = g.standard_normal((d, d)) if dense else None
    return {"signs": signs, "gauss_s": gauss_s, "gauss_pi": gauss_pi}


def outlier_channels(seed, n_groups: int, d: int, count: int = 4) -> np.ndarray:
    """int64 [n_groups, count]: distinct channel ids per (layer, kv-head) group."""
    g = _rng([*np.atleast_1d(seed).tolist(), 0x0C4A])
    return np.stack([g.choice(d, size=count, replace=False) for _ in range(n_groups)])


def heavy_tailed(shape, seed, n_outliers: int = 4, outlier_scale: float = 20.0,
                 dtype=np.float32) -> np.ndarray:
    """N(0,1) array of ``shape`` = [..., H, T, d] with per-[..., H] outlier channels.

    Every leading index combination except the token axis forms one
    (layer, head) group whose ``n_outliers`` channels are scaled by
    ``outlier_scale`` for all tokens.
    """
    shape = tuple(shape)
    *lead, T, d = shape
    n_groups = int(np.prod(lead)) if lead else 1
    g = _rng([*np.atleast_1d(seed).tolist(), 0xD47A])
    x = g.standard_normal((n_groups, T, d), dtype=np.float32)
    ch = outlier_channels(seed, n_groups, d, n_outliers)
    for i in range(n_groups):
        x[i][:, ch[i]] *= outlier_scale
    return x.reshape(shape).astype(dtype, copy=False)


def lognormal_channels(shape, seed, sigma: float = 0.5, p_outlier: float = 0.02,
                       outlier_scale: float = 15.0, dtype=np.float32) -> np.ndarray:
    """N(0,1) array [..., H, T, d] with per-(group, channel) LogNormal(0, sigma)
    scales; each channel is additionally an outlier (x outlier_scale) with
    probability ``p_outlier``."""
    shape = tuple(shape)
    *lead, T, d = shape
    n_groups = int(np.prod(lead)) if lead else 1
    g = _rng([*np.atleast_1d(seed).tolist(), 0x109A])
    scale = np.exp(sigma * g.standard_normal((n_groups, 1, d)))
    scale = scale * np.where(g.random((n_groups, 1, d)) < p_outlier, outlier_scale, 1.0)
    x = g.standard_normal((n_groups, T, d), dtype=np.float32) * scale.astype(np.float32)
    return x.reshape(shape).astype(dtype, copy=False)


def haar_basis(d: int, seed) -> np.ndarray:
    """Seeded Haar-random orthogonal matrix [d, d] (float64), from scipy."""
    from scipy.stats import ortho_group
    return ortho_group.rvs(dim=d, random_state=_rng([*np.atleast_1d(seed).tolist(), 0xBA5E]))


def anisotropic(n: int, d: int, seed, basis: np.ndarray | None = None,
                decay: float = 0.8, dtype=np.float32) -> np.ndarray:
    """n draws of U (lambda^1/2 * g) with lambda_i = i^-decay; returns [n, d]."""
    U = haar_basis(d, seed) if basis is None else basis
    lam_sqrt = np.arange(1, d + 1, dtype=np.float64) ** (-decay / 2.0)
    g = _rng([*np.atleast_1d(seed).tolist(), 0xA150, n])
    out = np.empty((n, d), dtype=dtype)
    step = 65536
    for s in range(0, n, step):
        e = min(n, s + step)
        z = g.standard_normal((e - s, d)) * lam_sqrt
        out[s:e] = (z @ U.T).astype(dtype)
    return out


# --------------------------------------------------------------------------
# Device-side generators for workloads too large for the host (torch only).
# --------------------------------------------------------------------------

def heavy_tailed_torch(shape, seed, device, n_outliers: int = 4,
                       outlier_scale: float = 20.0, dtype=None):
    """Device version of :func:`heavy_tailed` (different random stream).

    Same law, drawn with a seeded ``torch.Generator`` on ``device``; outlier
    channel ids come from :func:`outlier_channels` with the same seed.
    """
    import torch
    dtype = torch.bfloat16 if dtype is None else dtype
    *lead, T, d = tuple(shape)
    n_groups = int(np.prod(lead)) if lead else 1
    gen = torch.Generator(device=device)
    gen.manual_seed(int(np.random.SeedSequence([*np.atleast_1d(seed).tolist(), 0x7011]).generate_state(1)[0]))
    x = torch.empty((n_groups, T, d), dtype=dtype, device=device)
    scale = torch.ones((n_groups, 1, d), dtype=torch.float32, device=device)
    ch = torch.as_tensor(outlier_channels(seed, n_groups, d, n_outliers), device=device)
    scale.scatter_(2, ch.view(n_groups, 1, -1), outlier_scale)
    chunk = max(1, (1 << 28) // max(1, T * d))
    for s in range(0, n_groups, chunk):
        e = min(n_groups, s + chunk)
        y = torch.randn((e - s, T, d), generator=gen, device=device, dtype=torch.float32)
        x[s:e] = (y * scale[s:e]).to(dtype)
    return x.view(*lead, T, d) if lead else x.view(T, d)


def lognormal_channels_torch(shape, seed, device, sigma: float = 0.5, p_outlier: float = 0.02,
                             outlier_scale: float = 15.0, dtype=None):
    """Device version of :func:`lognormal_channels` (different random stream):
    per-(group, channel) LogNormal(0, sigma) scales, x outlier_scale with
    probability ``p_outlier``, drawn on the host; the N(0, 1) rows are drawn
    on ``device`` with a seeded ``torch.Generator``."""
    import torch
    dtype = torch.bfloat16 if dtype is None else dtype
    *lead, T, d = tuple(shape)
    n_groups = int(np.prod(lead)) if lead else 1
    g = _rng([*np.atleast_1d(seed).tolist(), 0x109B])
    scale = np.exp(sigma * g.standard_normal((n_groups, 1, d)))
    scale = scale * np.where(g.random((n_groups, 1, d)) < p_outlier, outlier_scale, 1.0)
    scale = torch.as_tensor(scale.astype(np.float32), device=device)
    gen = torch.Generator(device=device)
    gen.manual_seed(int(np.random.SeedSequence([*np.atleast_1d(seed).tolist(), 0x7012]).generate_state(1)[0]))
    x = torch.empty((n_groups, T, d), dtype=dtype, device=device)
    chunk = max(1, (1 << 28) // max(1, T * d))
    for s in range(0, n_groups, chunk):
        e = min(n_groups, s + chunk)
        y = torch.randn((e - s, T, d), generator=gen, device=device, dtype=torch.float32)
        x[s:e] = (y * scale[s:e]).to(dtype)
    return x.view(*lead, T, d) if lead else x.view(T, d)
