"""Pins of the oracle's counter-based generator (oracle/philox.py).

The generator is pinned to the published known-answer vectors of
Philox4x32-10 (tests/golden/philox4x32_10_kat.txt), which a wrong multiplier,
a swapped output word, a missing key bump or an off-by-one round count all
fail.  The derived draws are pinned by their laws: 52-bit uniforms strictly
inside (0, 1) with the moments of U(0, 1), Box-Muller normals with the
moments of N(0, 1) and a Kolmogorov-Smirnov test, and +-1 signs with balanced
frequencies."""
import numpy as np
import pytest
from scipy import stats

from conftest import read_golden
from oracle import philox


def _kat():
    for row in read_golden("philox4x32_10_kat.txt"):
        rounds = int(row[0])
        vals = [int(v, 16) for v in row[1:]]
        yield rounds, vals[0:4], vals[4:6], vals[6:10]


def test_scalar_round_function_matches_published_vectors():
    for rounds, ctr, key, out in _kat():
        assert list(philox.philox4x32_scalar(ctr, key, rounds)) == out


def test_vectorised_generator_matches_published_vectors():
    for rounds, ctr, key, out in _kat():
        got = philox.philox4x32(*[np.array([c], dtype=np.uint64) for c in ctr], key[0], key[1], rounds)
        assert [int(g[0]) for g in got] == out


def test_vectorised_equals_scalar_on_many_counters():
    rng = np.random.default_rng(5)
    ctr = rng.integers(0, 2**32, size=(200, 4), dtype=np.uint64)
    key = (0x01234567, 0x89ABCDEF)
    got = philox.philox4x32(ctr[:, 0], ctr[:, 1], ctr[:, 2], ctr[:, 3], *key)
    for i in range(200):
        assert tuple(int(g[i]) for g in got) == philox.philox4x32_scalar(ctr[i], key)


def test_uniforms_inside_unit_interval_with_uniform_moments():
    w = philox._blocks(12345, 7, 200000)
    u = philox.uniform52(w[0], w[1])
    assert u.min() > 0.0 and u.max() < 1.0
    assert abs(u.mean() - 0.5) < 5 * np.sqrt(1 / 12 / u.size)
    assert abs(u.var() - 1 / 12) < 0.002
    # the extreme grid points map strictly inside (0, 1)
    assert philox.uniform52(np.uint64(0), np.uint64(0)) == 0.5 / 2**52
    assert philox.uniform52(np.uint64(2**32 - 1), np.uint64(2**32 - 1)) == 1.0 - 0.5 / 2**52
    assert 1.0 - 0.5 / 2**52 < 1.0


def test_gaussians_have_the_standard_normal_law():
    z = philox.gaussians(2024, philox.STREAM_S, 400001)
    assert z.shape == (400001,)
    assert abs(z.mean()) < 5 / np.sqrt(z.size)
    assert abs(z.var() - 1.0) < 0.01
    assert abs(stats.skew(z)) < 0.02 and abs(stats.kurtosis(z)) < 0.04
    assert stats.kstest(z, "norm").pvalue > 1e-4
    # a prefix of a stream does not depend on how many draws follow it
    np.testing.assert_array_equal(philox.gaussians(2024, philox.STREAM_S, 1001), z[:1001])


def test_signs_are_balanced_and_streams_and_seeds_differ():
    s = philox.sign_diagonal(99, 100000)
    assert set(np.unique(s)) == {-1, 1}
    assert abs(s.mean()) < 5 / np.sqrt(s.size)
    a = philox.rotation_draws(128, 1, dense=True)
    b = philox.rotation_draws(128, 2, dense=True)
    assert not np.array_equal(a["signs"], b["signs"])
    assert not np.allclose(a["gauss_s"], b["gauss_s"])
    # S and the dense Gaussian come from different streams of one seed
    assert not np.allclose(a["gauss_s"].ravel()[:1000], a["gauss_pi"].ravel()[:1000])
    assert a["gauss_s"].dtype == np.float32 and a["gauss_pi"].dtype == np.float64


@pytest.mark.parametrize("seed", [0, 2**63 + 12345])
def test_seed_splits_into_the_two_key_words(seed):
    k0, k1 = philox._key(seed)
    assert k0 + (k1 << 32) == seed
