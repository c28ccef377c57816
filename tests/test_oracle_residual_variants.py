"""Residual-correction variants at equal bits, and the NSN pre-transform
([NSNQuant] §1) ahead of the codec (CPU, oracle only).

Three reconstructions of a d-dimensional vector at 3 bits per coordinate plus
two floats:
  qjl   2-bit codes + m = d QJL sign bits of S r + ||r||   (the codec as built)
  sign  2-bit codes + d sign bits of r itself + e_bar      ([TurboESM] §2.D)
  mse3  3-bit codes, no residual term
Pins: the closed forms of the sign variant's error and of the codes-alone
error; e_bar is the least-squares scale of the sign vector; the QJL form's
reconstruction error is (pi/2 - 1/d) times the codes-alone error at m = d.
The comparison itself (printed with -s) has no pinned values: it is a
measurement."""
import numpy as np

import synth
from oracle import codec, rotation as ro


def _rot(d, bits, seed):
    return ro.build_rotation(d, bits, synth.rotation_randomness(d, seed), "hadamard")


def test_sign_residual_error_closed_form():
    # ||r - e_bar s||^2 = ||r||^2 - 2 e_bar ||r||_1 + d e_bar^2 = ||r||^2 - d e_bar^2
    d = 128
    rot = _rot(d, 2, 71)
    x = synth.heavy_tailed((1, 1, 64, d), 72).reshape(64, d).astype(np.float64)
    e = codec.encode_sign_residual(rot, x)
    xt = codec.dequantize_sign_residual(rot, e["codes"], e["signs"], e["norm"], e["ebar"])
    err = np.sum((x - xt) ** 2, axis=1)
    r2 = np.sum(e["r"] ** 2, axis=1)
    np.testing.assert_allclose(err, r2 - d * e["ebar"] ** 2, rtol=1e-9, atol=1e-9)
    assert np.all(err <= r2 + 1e-9)              # never worse than the codes alone


def test_ebar_is_the_least_squares_scale():
    d = 64
    rot = _rot(d, 1, 73)
    x = synth.heavy_tailed((1, 1, 16, d), 74).reshape(16, d).astype(np.float64)
    e = codec.encode_sign_residual(rot, x)
    s = np.where(e["signs"], 1.0, -1.0)
    for a in (0.97, 1.03):
        worse = np.sum((e["r"] - a * e["ebar"][:, None] * s) ** 2, axis=1)
        best = np.sum((e["r"] - e["ebar"][:, None] * s) ** 2, axis=1)
        assert np.all(best < worse)


def test_codes_alone_error_is_the_residual_norm():
    d = 128
    rot = _rot(d, 3, 75)
    x = synth.heavy_tailed((1, 1, 32, d), 76).reshape(32, d).astype(np.float64)
    e = codec.encode(rot, x)
    xt = codec.dequantize_mse_only(rot, e["codes"], e["norm"])
    np.testing.assert_allclose(np.sqrt(np.sum((x - xt) ** 2, axis=1)), e["rnorm"], rtol=1e-10)


def _attention(q, k, v, scale):
    s = (q @ k.T) * scale
    s -= s.max(axis=1, keepdims=True)
    p = np.exp(s)
    return (p / p.sum(axis=1, keepdims=True)) @ v


def _compare(n_outliers, seed):
    d, n, nq = 128, 2048, 64
    k = synth.heavy_tailed((1, 1, n, d), seed, n_outliers=n_outliers).reshape(n, d).astype(np.float64)
    v = synth.heavy_tailed((1, 1, n, d), seed + 1, n_outliers=n_outliers).reshape(n, d).astype(np.float64)
    q = synth.heavy_tailed((1, 1, nq, d), seed + 2, n_outliers=n_outliers).reshape(nq, d).astype(np.float64)
    r2, r3 = _rot(d, 2, seed + 3), _rot(d, 3, seed + 3)

    def qjl(x):
        e = codec.encode(r2, x)
        return codec.dequantize(r2, e["codes"], e["signs"], e["norm"], e["rnorm"])

    def sign(x):
        e = codec.encode_sign_residual(r2, x)
        return codec.dequantize_sign_residual(r2, e["codes"], e["signs"], e["norm"], e["ebar"])

    def mse3(x):
        e = codec.encode(r3, x)
        return codec.dequantize_mse_only(r3, e["codes"], e["norm"])

    def mse2(x):
        e = codec.encode(r2, x)
        return codec.dequantize_mse_only(r2, e["codes"], e["norm"])

    exact_ip = q @ k.T
    exact_out = _attention(q, k, v, 1 / np.sqrt(d))
    rows = {}
    for name, f in (("qjl 2+1", qjl), ("sign 2+1", sign), ("mse 3", mse3), ("mse 2 (2 bits only)", mse2)):
        kt, vt = f(k), f(v)
        umse = float(np.mean(np.sum((k - kt) ** 2, axis=1) / np.sum(k * k, axis=1)))
        dip = (q @ kt.T - exact_ip) / np.sqrt(np.mean(exact_ip ** 2))
        out = _attention(q, kt, vt, 1 / np.sqrt(d))
        cos = np.sum(out * exact_out, axis=1) / (np.linalg.norm(out, axis=1) * np.linalg.norm(exact_out, axis=1))
        rows[name] = (umse, float(np.mean(dip)), float(np.sqrt(np.mean(dip ** 2))), float(np.mean(cos)),
                      float(np.min(cos)))
    print(f"\n{'with 4 outlier channels x20' if n_outliers else 'N(0, 1), no outliers'}")
    print("variant               unit MSE   ip bias / rms   ip err / rms   attn cos mean   attn cos min")
    for name, (a, b, c, m, mn) in rows.items():
        print(f"{name:20s} {a:9.5f} {b:+14.5f} {c:14.5f} {m:14.6f} {mn:14.6f}")
    return rows


def test_compare_at_equal_bits():
    """Unit-vector MSE, inner-product bias and error against exact products
    (both relative to the rms exact product), and attention-output cosine
    against exact attention, for keys and values of d = 128 (2048 vectors,
    64 queries of the same law), with and without the workloads' outlier
    channels.  Printed; only invariants and one closed form are asserted."""
    d = 128
    for n_outliers in (4, 0):
        rows = _compare(n_outliers, 81 + n_outliers)
        # more code bits, and the sign correction, both beat 2-bit codes alone
        assert rows["mse 3"][0] < rows["mse 2 (2 bits only)"][0]
        assert rows["sign 2+1"][0] < rows["mse 2 (2 bits only)"][0]
        # the QJL estimate of r is unbiased with E||r - r~||^2 = (pi/2 d/m - 1/m) ||r||^2, so at m = d
        # its error is (pi/2 - 1/d) times that of the codes alone
        ratio = rows["qjl 2+1"][0] / rows["mse 2 (2 bits only)"][0]
        assert abs(ratio - (np.pi / 2 - 1 / d)) < 0.05, ratio


# ---------------------------------------------------------------------------
# Normalize-Shift-Normalize ([NSNQuant] §1) ahead of the codec
# ---------------------------------------------------------------------------
def _offset_law(n, d, seed, n_offset=8, offset=4.0, n_outliers=4):
    """heavy_tailed rows plus a fixed per-channel offset on n_offset seeded
    channels (channels whose mean is far from zero in every token)."""
    x = synth.heavy_tailed((1, 1, n, d), seed, n_outliers=n_outliers).reshape(n, d).astype(np.float64)
    rng = np.random.default_rng(seed + 1)
    ch = rng.choice(d, n_offset, replace=False)
    x[:, ch] += offset * np.where(rng.random(n_offset) < 0.5, -1.0, 1.0)
    return x


def test_nsn_round_trip_and_invariants():
    d = 128
    x = _offset_law(300, d, 91)
    x3, s1, o, s2 = codec.nsn_forward(x)
    np.testing.assert_allclose(codec.nsn_inverse(x3, s1, o, s2), x, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(np.sum(x3 * x3, axis=1), d, rtol=1e-12)              # norm sqrt(d)
    np.testing.assert_allclose(np.mean(x3 * s2[:, None], axis=0), 0.0, atol=1e-12)   # centred channels
    np.testing.assert_allclose(np.sum((x / s1[:, None]) ** 2, axis=1), d, rtol=1e-12)


def test_nsn_comparison():
    """The codec (2+1 bits) on x directly and on NSN's x3, for rows with 8
    channels offset by +-4 in every token, over heavy_tailed rows (with the
    x20 outlier channels) and over N(0, 1) rows: unit MSE and attention
    cosine against exact attention.  Printed; the NSN route must not lose on
    the MSE of these laws, where the shift removes the offsets."""
    d, n, nq = 128, 2048, 64
    rot = _rot(d, 2, 106)

    def direct(x):
        e = codec.encode(rot, x)
        return codec.dequantize(rot, e["codes"], e["signs"], e["norm"], e["rnorm"])

    def nsn(x):
        x3, s1, o, s2 = codec.nsn_forward(x)
        return codec.nsn_inverse(direct(x3), s1, o, s2)

    for n_outliers in (4, 0):
        k = _offset_law(n, d, 101, n_outliers=n_outliers)
        v = _offset_law(n, d, 103, n_outliers=n_outliers)
        q = synth.heavy_tailed((1, 1, nq, d), 105, n_outliers=n_outliers).reshape(nq, d).astype(np.float64)
        exact = _attention(q, k, v, 1 / np.sqrt(d))
        res = {}
        print(f"\noffsets +-4 on 8 channels, {'with 4 outlier channels x20' if n_outliers else 'N(0, 1) otherwise'}")
        for name, f in (("codec on x", direct), ("codec on NSN(x)", nsn)):
            kt, vt = f(k), f(v)
            umse = float(np.mean(np.sum((k - kt) ** 2, axis=1) / np.sum(k * k, axis=1)))
            out = _attention(q, kt, vt, 1 / np.sqrt(d))
            cos = np.sum(out * exact, axis=1) / (np.linalg.norm(out, axis=1) * np.linalg.norm(exact, axis=1))
            res[name] = (umse, float(np.mean(cos)))
            print(f"{name:18s} unit MSE {umse:.5f}  attention cosine {np.mean(cos):.6f}")
        assert res["codec on NSN(x)"][0] < res["codec on x"][0]
