"""Lloyd-Max scalar codebook for one coordinate of a randomly rotated unit vector.

TEST INFRASTRUCTURE ONLY (see the package header).

The pages fix the quantizer as "a standard high-quality quantizer applied to
each part of the vector after a random rotation" ([TurboQuant] "Principe",
Étape 1) whose "boundaries and reconstruction values are optimised with the
Lloyd-Max algorithm" ([TurboQuant] comments; [TurboESM] §2.C).  After a
uniformly random rotation a unit vector is uniform on S^{d-1}, and one of its
coordinates T has the exact density

    f_d(t) = C_d (1 - t^2)^((d-3)/2),  t in [-1, 1],
    C_d = Gamma(d/2) / (sqrt(pi) Gamma((d-1)/2)).

This module computes the Lloyd-Max quantizer of that law (reading: the exact
law, not its N(0, 1/d) approximation).  It is the fixed point of

    t_j = (c_j + c_{j+1}) / 2                (nearest-neighbour condition)
    c_j = E[T | t_{j-1} <= T < t_j]          (centroid condition)

iterated in float64 until no level moves by more than 1e-15.  f_d is
log-concave for d >= 3, so the fixed point is unique.

Pins (tests/test_oracle_codebook.py): the 1-bit level against its closed form
Gamma(d/2)/(sqrt(pi) Gamma((d+1)/2)); d = 3 (uniform law, Archimedes) against
the uniform quantizer; large d against the textbook Gaussian Lloyd-Max table;
both optimality conditions against direct numerical quadrature of f_d;
the density against Monte-Carlo samples of the sphere; MSE decreasing in bits.
"""
from __future__ import annotations

import math

import numpy as np
from scipy.special import betainc, gammaln


def _log_cd(d: int) -> float:
    return gammaln(d / 2.0) - 0.5 * math.log(math.pi) - gammaln((d - 1) / 2.0)


def coord_pdf(t, d: int):
    """Density f_d(t) of one coordinate of a uniform point on S^{d-1}."""
    t = np.asarray(t, dtype=np.float64)
    with np.errstate(divide="ignore", invalid="ignore"):
        val = np.exp(_log_cd(d) + 0.5 * (d - 3) * np.log1p(-t * t))
    return np.where(np.abs(t) < 1.0, val, 0.0)


def coord_mass(a: float, b: float, d: int) -> float:
    """P(a <= T < b) for 0 <= a <= b <= 1.

    For t >= 0, P(0 <= T < t) = I_{t^2}(1/2, (d-1)/2) / 2, with I the
    regularized incomplete beta function (T^2 ~ Beta(1/2, (d-1)/2)).  In the
    upper tail the complementary form I_{1-t^2}((d-1)/2, 1/2) avoids
    cancellation.
    """
    assert 0.0 <= a <= b <= 1.0
    k = (d - 1) / 2.0
    lo_a = betainc(0.5, k, a * a)
    if lo_a <= 0.5:
        return 0.5 * (betainc(0.5, k, b * b) - lo_a)
    return 0.5 * (betainc(k, 0.5, 1.0 - a * a) - betainc(k, 0.5, 1.0 - b * b))


def coord_first_moment(a: float, b: float, d: int) -> float:
    """Integral of t f_d(t) over [a, b], 0 <= a <= b <= 1 (closed form).

    d/dt (1-t^2)^((d-1)/2) = -(d-1) t (1-t^2)^((d-3)/2), hence
    int_a^b t f_d = C_d [(1-a^2)^((d-1)/2) - (1-b^2)^((d-1)/2)] / (d-1).
    """
    k = (d - 1) / 2.0
    lc = _log_cd(d) - math.log(d - 1)
    pa = math.exp(lc + k * math.log1p(-a * a)) if a < 1.0 else 0.0
    pb = math.exp(lc + k * math.log1p(-b * b)) if b < 1.0 else 0.0
    return pa - pb


def _centroid(a: float, b: float, d: int) -> float:
    return coord_first_moment(a, b, d) / coord_mass(a, b, d)


def lloyd_max(d: int, bits: int, tol: float = 1e-15, max_iter: int = 200000):
    """Lloyd-Max levels and thresholds for f_d with 2**bits levels.

    Returns ``(levels, thresholds)`` as float64 arrays, levels ascending
    (code 0 = most negative level), thresholds[j] = (levels[j] + levels[j+1])/2.
    The law is symmetric, so the positive half is solved on [0, 1] with the
    middle threshold fixed at 0.
    """
    if d < 3:
        raise ValueError("d >= 3 required")
    if not 1 <= bits <= 8:
        raise ValueError("1 <= bits <= 8")
    L = 1 << (bits - 1)
    spread = min(1.0, 3.0 / math.sqrt(d))
    c = np.array([(j + 0.5) / L * spread for j in range(L)])
    best, stalled = math.inf, 0
    for _ in range(max_iter):
        tau = np.concatenate(([0.0], 0.5 * (c[:-1] + c[1:]), [1.0]))
        c_new = np.array([_centroid(tau[j], tau[j + 1], d) for j in range(L)])
        moved = float(np.max(np.abs(c_new - c))) / float(np.max(np.abs(c_new)))
        c = c_new
        if moved <= tol * 10:
            break
        # At very large d the incomplete-beta evaluations carry ~1e-12
        # relative noise; stop once the iteration sits on that floor.
        stalled = stalled + 1 if moved >= best else 0
        best = min(best, moved)
        if best < 1e-10 and stalled > 200:
            break
    else:  # pragma: no cover
        raise RuntimeError("Lloyd-Max did not converge")
    levels = np.concatenate((-c[::-1], c))
    thresholds = 0.5 * (levels[:-1] + levels[1:])
    return levels, thresholds


def codebook_mse(d: int, levels: np.ndarray) -> float:
    """E[(T - Q(T))^2] per coordinate for a symmetric codebook of centroids.

    With every level the centroid of its cell, E[(T - Q(T))^2] =
    E[T^2] - sum_j c_j^2 P(cell_j), and E[T^2] = 1/d exactly.
    """
    L = len(levels) // 2
    c = levels[L:]
    tau = np.concatenate(([0.0], 0.5 * (c[:-1] + c[1:]), [1.0]))
    energy = sum(c[j] ** 2 * coord_mass(tau[j], tau[j + 1], d) for j in range(L))
    return 1.0 / d - 2.0 * energy


def walsh_coefficients(levels: np.ndarray) -> np.ndarray:
    """Coefficients a_S with level(idx) = sum_S a_S prod_{k in S} s_k(idx).

    s_k(idx) = 2 * bit_k(idx) - 1 is the +-1 value of bit k of the code.
    Returned as an array indexed by the subset bitmask S (length 2**bits); it
    is the Walsh-Hadamard transform of the level table over the bit cube.
    Used by the tests to check that a codebook written in this form gives the
    same levels; not needed by the oracle's own arithmetic.
    """
    n = len(levels)
    bits = n.bit_length() - 1
    a = np.zeros(n)
    for S in range(n):
        tot = 0.0
        for idx in range(n):
            prod = 1.0
            for k in range(bits):
                if S >> k & 1:
                    prod *= 2 * ((idx >> k) & 1) - 1
            tot += levels[idx] * prod
        a[S] = tot / n
    return a
