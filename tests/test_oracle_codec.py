"""Pins for the oracle's encode / pack / dequantize and the QJL estimator (CPU only)."""
import math

import numpy as np
import pytest

import synth
from oracle import codebook as cb
from oracle import codec, rotation as ro


def _rot(d=128, bits=2, seed=1, rope=0.0, kind="hadamard"):
    return ro.build_rotation(d, bits, synth.rotation_randomness(d, seed, dense=(kind == "dense")),
                             kind, rope_base=rope)


@pytest.mark.parametrize("bits", [1, 2, 3])
def test_pack_roundtrip(bits):
    rng = np.random.default_rng(bits)
    codes = rng.integers(0, 1 << bits, size=(50, 128))
    packed = codec.pack_planes(codes, bits)
    assert packed.shape == (50, bits * 16)
    np.testing.assert_array_equal(codec.unpack_planes(packed, bits, 128), codes)
    z = rng.random((50, 128)) < 0.5
    np.testing.assert_array_equal(codec.unpack_bits(codec.pack_bits(z), 128), z)


def test_pack_known_bytes():
    # codes i mod 4 over 16 coordinates: plane 0 = 0,1,0,1,... -> 0xAA;
    # plane 1 = 0,0,1,1,... -> 0xCC (bit i%8 of byte i//8, LSB first)
    codes = (np.arange(16) % 4)[None, :]
    np.testing.assert_array_equal(codec.pack_planes(codes, 2)[0], [0xAA, 0xAA, 0xCC, 0xCC])
    z = (np.arange(16) % 2 == 0)[None, :]
    np.testing.assert_array_equal(codec.pack_bits(z)[0], [0x55, 0x55])
    codes3 = np.full((1, 8), 5)                      # 0b101
    np.testing.assert_array_equal(codec.pack_planes(codes3, 3)[0], [0xFF, 0x00, 0xFF])


@pytest.mark.parametrize("bits", [1, 2, 3])
def test_zero_vector(bits):
    rot = _rot(bits=bits)
    e = codec.encode(rot, np.zeros((1, 128)))
    assert e["norm"][0] == 0 and e["rnorm"][0] == 0
    assert np.all(e["codes"] == (1 << (bits - 1)))    # y = 0 sits on the middle threshold
    assert np.all(e["signs"])                          # sign(0) = +1


def test_codes_are_nearest_level():
    rot = _rot(bits=3)
    x = synth.heavy_tailed((64, 128), 5)
    e = codec.encode(rot, x)
    dist = np.abs(e["y"][:, :, None] - rot.levels[None, None, :])
    np.testing.assert_array_equal(np.argmin(dist, axis=2), e["codes"])


def test_residual_is_rotated_error():
    rot = _rot(bits=2)
    x = synth.heavy_tailed((32, 128), 6)
    e = codec.encode(rot, x)
    x_mse = (e["norm"][:, None] * rot.levels[e["codes"]]) @ rot.pi     # Pi^T ||x|| c[idx]
    np.testing.assert_allclose(e["rnorm"], np.linalg.norm(x - x_mse, axis=1), rtol=1e-10)


def test_mse_matches_codebook_distortion():
    d, bits = 128, 2
    rot = _rot(d, bits)
    x = np.random.default_rng(12).standard_normal((4000, d))          # isotropic inputs
    e = codec.encode(rot, x)
    rel = np.mean((e["rnorm"] / e["norm"]) ** 2)
    assert rel == pytest.approx(d * cb.codebook_mse(d, rot.levels), rel=0.03)


def test_qjl_sign_identity():
    # E[sign(<s, r>) s] = sqrt(2/pi) r / ||r|| for s ~ N(0, I)
    rng = np.random.default_rng(21)
    r = rng.standard_normal(32)
    s = rng.standard_normal((400_000, 32))
    est = np.mean(np.sign(s @ r)[:, None] * s, axis=0)
    np.testing.assert_allclose(est, math.sqrt(2 / math.pi) * r / np.linalg.norm(r), atol=6e-3)


def test_qjl_estimator_unbiased_and_variance():
    # Over many Gaussian S: mean of ||r|| sqrt(pi/2)/m <S q, sign(S r)> -> <q, r>,
    # variance [(pi/2)||q||^2||r||^2 - <q,r>^2] / m.
    d = m = 64
    rng = np.random.default_rng(22)
    q, r = rng.standard_normal(d), rng.standard_normal(d)
    n = 20000
    vals = np.empty(n)
    for i in range(n):
        S = rng.standard_normal((m, d))
        vals[i] = np.linalg.norm(r) * codec.QJL_CONST / m * (S @ q) @ np.where(S @ r >= 0, 1.0, -1.0)
    ip = q @ r
    var = ((math.pi / 2) * (q @ q) * (r @ r) - ip ** 2) / m
    assert abs(vals.mean() - ip) < 4 * math.sqrt(var / n)
    assert vals.var() == pytest.approx(var, rel=0.05)


@pytest.mark.parametrize("kind,d,bits", [("hadamard", 128, 2), ("hadamard", 64, 3), ("dense", 96, 1)])
def test_score_routes_agree(kind, d, bits):
    # estimator on the codes == <q, dequantized x> (rotation-invariance route)
    rot = _rot(d, bits, 3, kind=kind)
    x = synth.heavy_tailed((40, d), 8)
    e = codec.encode(rot, x)
    q = np.random.default_rng(9).standard_normal((3, d))
    s1 = codec.score_from_codes(rot, q, e["codes"], e["signs"], e["norm"], e["rnorm"])
    xt = codec.dequantize(rot, e["codes"], e["signs"], e["norm"], e["rnorm"])
    np.testing.assert_allclose(s1, q @ xt.T, rtol=1e-10, atol=1e-10)


def test_quality_improves_with_bits():
    d = 128
    x = synth.heavy_tailed((500, d), 13)
    q = synth.heavy_tailed((20, d), 14)
    exact = q.astype(np.float64) @ x.T.astype(np.float64)
    errs = []
    for bits in (1, 2, 3, 4):
        rot = _rot(d, bits, 4)
        e = codec.encode(rot, x)
        est = codec.score_from_codes(rot, q, e["codes"], e["signs"], e["norm"], e["rnorm"])
        errs.append(np.sqrt(np.mean((est - exact) ** 2)))
    assert all(a > b for a, b in zip(errs, errs[1:]))


def test_flags_mark_boundary_coordinates():
    rot = _rot(bits=2)
    x = synth.heavy_tailed((200, 128), 15)
    e = codec.encode(rot, x)
    gap = np.min(np.abs(e["y"][:, :, None] - rot.thresholds), axis=2)
    np.testing.assert_array_equal(e["code_flags"], gap < 1e-5)
