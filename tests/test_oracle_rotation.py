"""Pins for the oracle's rotations, RoPE and bf16 rounding (CPU only)."""
import numpy as np
import pytest
import scipy.linalg
import torch

import synth
from oracle import rotation as ro


@pytest.mark.parametrize("d", [2, 4, 8, 16, 32, 64, 128])
def test_sylvester_matches_scipy(d):
    np.testing.assert_array_equal(ro.sylvester_hadamard(d), scipy.linalg.hadamard(d))


def test_small_hadamard_closed_forms():
    np.testing.assert_array_equal(ro.sylvester_hadamard(2), [[1, 1], [1, -1]])
    np.testing.assert_array_equal(ro.sylvester_hadamard(4),
                                  [[1, 1, 1, 1], [1, -1, 1, -1], [1, 1, -1, -1], [1, -1, -1, 1]])


@pytest.mark.parametrize("d", [64, 128])
def test_randomized_hadamard_is_orthogonal(d):
    r = synth.rotation_randomness(d, 3)
    pi = ro.hadamard_rotation(r["signs"])
    np.testing.assert_allclose(pi.T @ pi, np.eye(d), atol=1e-13)
    x = np.random.default_rng(0).standard_normal((10, d))
    np.testing.assert_allclose(np.linalg.norm(x @ pi.T, axis=1), np.linalg.norm(x, axis=1), rtol=1e-13)


@pytest.mark.parametrize("d", [48, 96, 1536])
def test_dense_rotation_qr_convention(d):
    r = synth.rotation_randomness(d, 5, dense=True)
    g = r["gauss_pi"]
    pi = ro.dense_rotation(g)
    np.testing.assert_allclose(pi.T @ pi, np.eye(d), atol=1e-12)
    rr = pi.T @ g                                   # R = Q^T G
    assert np.all(np.diag(rr) > 0)
    np.testing.assert_allclose(np.tril(rr, -1), 0, atol=1e-9 * np.abs(rr).max())


def test_rope_complex_form_and_properties():
    d, base = 128, 10000.0
    rng = np.random.default_rng(1)
    x = rng.standard_normal((5, d))
    pos = np.array([0, 1, 17, 4096, 1 << 20])
    out = ro.apply_rope(x, pos, base)
    # complex form: (x_i + i x_{i+d/2}) * exp(i pos theta_i)
    theta = base ** (-np.arange(d // 2) * 2.0 / d)
    z = (x[:, : d // 2] + 1j * x[:, d // 2:]) * np.exp(1j * pos[:, None] * theta[None, :])
    np.testing.assert_allclose(out, np.concatenate((z.real, z.imag), axis=1), atol=1e-12)
    np.testing.assert_allclose(out[0], x[0], atol=0)                 # R_0 = I
    np.testing.assert_allclose(np.linalg.norm(out, axis=1), np.linalg.norm(x, axis=1), rtol=1e-13)
    q, k = rng.standard_normal(d), rng.standard_normal(d)
    for i, j, c in [(5, 3, 100), (1000, 10, 7), (0, 50, 123456)]:
        a = ro.apply_rope(q, i, base) @ ro.apply_rope(k, j, base)
        b = ro.apply_rope(q, i + c, base) @ ro.apply_rope(k, j + c, base)
        assert a == pytest.approx(b, rel=1e-9, abs=1e-9)


@pytest.mark.parametrize("kind,d", [("hadamard", 128), ("dense", 96)])
def test_rope_first_rotation_invariance(kind, d):
    # (Pi R_i q)^T (Pi R_j k) = (R_i q)^T (R_j k) since Pi^T Pi = I
    r = synth.rotation_randomness(d, 9, dense=(kind == "dense"))
    pi = ro.hadamard_rotation(r["signs"]) if kind == "hadamard" else ro.dense_rotation(r["gauss_pi"])
    rng = np.random.default_rng(2)
    q, k = rng.standard_normal(d), rng.standard_normal(d)
    rq, rk = ro.apply_rope(q, 77, 10000.0), ro.apply_rope(k, 3, 10000.0)
    assert (pi @ rq) @ (pi @ rk) == pytest.approx(rq @ rk, rel=1e-12)


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(3)
    x = np.concatenate([rng.standard_normal(100_000).astype(np.float32),
                        np.array([0.0, -0.0, 1.0, 1.00390625, 1.005859375, 3.0e38, 1e-40], np.float32)])
    ref = torch.from_numpy(x).to(torch.bfloat16).float().numpy()
    np.testing.assert_array_equal(ro.round_to_bf16(x), ref)


def test_build_rotation_fields():
    r = synth.rotation_randomness(128, 4)
    rot = ro.build_rotation(128, 2, r, "hadamard", rope_base=10000.0)
    assert rot.pi.shape == (128, 128) and rot.s.shape == (128, 128)
    assert len(rot.levels) == 4 and len(rot.thresholds) == 3
    np.testing.assert_array_equal(rot.s, ro.round_to_bf16(r["gauss_s"]))
