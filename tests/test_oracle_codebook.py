"""Pins for the oracle's Lloyd-Max codebook (CPU only).

Each check is independent of the oracle's own route (regularized incomplete
beta + closed-form first moment + Lloyd iteration)."""
import math

import numpy as np
import pytest
from scipy import integrate, stats
from scipy.special import gammaln

from conftest import read_golden
from oracle import codebook as cb


@pytest.mark.parametrize("d", [3, 8, 64, 128, 1536])
def test_one_bit_level_closed_form(d):
    # 1-bit Lloyd-Max on a symmetric law: level = E|T| =
    # Gamma(d/2) / (sqrt(pi) Gamma((d+1)/2)).
    levels, thr = cb.lloyd_max(d, 1)
    expect = math.exp(gammaln(d / 2) - 0.5 * math.log(math.pi) - gammaln((d + 1) / 2))
    assert levels[1] == pytest.approx(expect, rel=1e-13)
    assert levels[0] == -levels[1]
    assert thr[0] == 0.0


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_d3_is_uniform_quantizer(bits):
    # On S^2 a coordinate is uniform on [-1, 1] (Archimedes); Lloyd-Max of a
    # uniform law is the uniform quantizer with levels (2j+1)/2^b - 1.
    levels, _ = cb.lloyd_max(3, bits)
    n = 1 << bits
    expect = (2 * np.arange(n) + 1) / n - 1
    np.testing.assert_allclose(levels, expect, atol=1e-12)


def test_large_d_tends_to_gaussian_table():
    rows = read_golden("gaussian_lloyd_max.txt")
    d = 200_000
    for row in rows:
        bits, mse = int(row[0]), float(row[1])
        pos_levels = np.array([float(v) for v in row[2:]])
        levels, _ = cb.lloyd_max(d, bits)
        got = math.sqrt(d) * levels[len(levels) // 2:]
        np.testing.assert_allclose(got, pos_levels, rtol=2e-3, atol=6e-4)
        assert d * cb.codebook_mse(d, levels) == pytest.approx(mse, rel=4e-3)


@pytest.mark.parametrize("d,bits", [(64, 2), (128, 2), (128, 3), (1536, 1), (1536, 3), (16, 3)])
def test_optimality_conditions_by_quadrature(d, bits):
    levels, thr = cb.lloyd_max(d, bits)
    edges = np.concatenate(([-1.0], thr, [1.0]))
    f = lambda t: float(cb.coord_pdf(t, d))
    width = 1.0 / math.sqrt(d)
    for j, c in enumerate(levels):
        a, b = edges[j], edges[j + 1]
        pts = [p for p in (c - 8 * width, c, c + 8 * width) if a < p < b]
        mass = integrate.quad(f, a, b, points=pts or None, limit=400, epsabs=0, epsrel=1e-13)[0]
        mom = integrate.quad(lambda t: t * f(t), a, b, points=pts or None, limit=400,
                             epsabs=0, epsrel=1e-13)[0]
        assert mom / mass == pytest.approx(c, rel=1e-9, abs=1e-13)
        if a >= 0:
            assert cb.coord_mass(a, b, d) == pytest.approx(mass, rel=1e-9)
    # nearest-neighbour condition
    np.testing.assert_allclose(thr, 0.5 * (levels[:-1] + levels[1:]), rtol=0, atol=0)
    assert np.all(np.diff(levels) > 0)


def test_density_matches_sphere_samples():
    d = 16
    g = np.random.default_rng(7).standard_normal((200_000, d))
    t = g[:, 0] / np.linalg.norm(g, axis=1)

    def cdf(x):
        x = np.asarray(x, dtype=np.float64)
        out = np.empty_like(x)
        for i, v in enumerate(x.ravel()):
            out.ravel()[i] = 0.5 + (1 if v >= 0 else -1) * cb.coord_mass(0.0, min(abs(v), 1.0), d)
        return out

    sub = t[:20_000]
    ks = stats.kstest(sub, cdf)
    assert ks.pvalue > 1e-3
    assert integrate.quad(lambda s: float(cb.coord_pdf(s, d)), -1, 1)[0] == pytest.approx(1.0, rel=1e-12)


@pytest.mark.parametrize("d", [64, 128, 1536])
def test_mse_falls_with_bits(d):
    mses = [cb.codebook_mse(d, cb.lloyd_max(d, b)[0]) for b in (1, 2, 3, 4)]
    assert all(a > b for a, b in zip(mses, mses[1:]))
    assert 0 < mses[-1] < mses[0] < 1.0 / d


def test_mse_monte_carlo():
    d, bits = 128, 2
    levels, thr = cb.lloyd_max(d, bits)
    g = np.random.default_rng(11).standard_normal((20_000, d))
    u = g / np.linalg.norm(g, axis=1, keepdims=True)
    q = levels[np.searchsorted(thr, u, side="right")]
    emp = np.mean(np.sum((u - q) ** 2, axis=1))
    assert emp == pytest.approx(d * cb.codebook_mse(d, levels), rel=0.01)


@pytest.mark.parametrize("bits", [1, 2, 3])
def test_walsh_form_reproduces_levels(bits):
    levels, _ = cb.lloyd_max(128, bits)
    a = cb.walsh_coefficients(levels)
    n = 1 << bits
    for idx in range(n):
        v = 0.0
        for S in range(n):
            prod = 1.0
            for k in range(bits):
                if S >> k & 1:
                    prod *= 2 * ((idx >> k) & 1) - 1
            v += a[S] * prod
        assert v == pytest.approx(levels[idx], abs=1e-15)
    # odd-symmetric codebook: only odd-size subsets carry weight
    for S in range(n):
        if bin(S).count("1") % 2 == 0:
            assert abs(a[S]) < 1e-15
