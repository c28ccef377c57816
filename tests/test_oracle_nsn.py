"""Pins of the oracle's NSN record mode ([NSNQuant] §1, §4): the encode of a
block and decode attention over its records."""
import math

import numpy as np
import pytest

import synth
from helpers import oracle_rotation
from oracle import attention as at
from oracle import codec
from oracle.rotation import apply_rope


def _block(l, d, seed, offset=4.0):
    """Rows N(0, 1) with 8 channels offset by +-offset in every token (the
    case NSN's shift removes)."""
    g = np.random.default_rng(seed)
    x = g.standard_normal((l, d))
    ch = g.choice(d, 8, replace=False)
    x[:, ch] += offset * np.where(g.random(8) < 0.5, -1.0, 1.0)
    return x


def test_nsn_encode_invariants():
    d, l = 128, 300
    rot, _ = oracle_rotation(d, 2, 5, rope=10000.0)
    x = _block(l, d, 1)
    pos = np.arange(l) + 17
    e = codec.nsn_encode(rot, x, pos)
    xr = apply_rope(x, pos, 10000.0)
    np.testing.assert_allclose(e["x_nsn"], xr, rtol=1e-12, atol=1e-12)
    # s1 = ||x~|| / sqrt(d); the shifted records have unit-free directions
    np.testing.assert_allclose(e["s1"], np.linalg.norm(xr, axis=1) / math.sqrt(d), rtol=1e-12)
    # inverse: x' + s1 o = x~, and the normalised shifted tokens have zero channel mean
    np.testing.assert_allclose(e["x_shift"] + e["s1"][:, None] * e["o"][None, :], xr, rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(np.mean(e["x_shift"] / e["s1"][:, None], axis=0), 0.0, atol=1e-12)
    # ||x'|| / s1 = ||x1 - o|| = s2 sqrt(d): the codec's norm of x' against nsn_forward's s2
    _, _, _, s2 = codec.nsn_forward(xr)
    np.testing.assert_allclose(e["norm"], e["s1"] * s2 * math.sqrt(d), rtol=1e-12)
    # the codec is scale-invariant: x' and x3 = x' / (s1 s2) get the same codes and signs
    e3 = codec.encode(rot, e["x_shift"] / (e["s1"] * s2)[:, None], None)
    assert np.array_equal(e3["codes"], e["codes"]) and np.array_equal(e3["signs"], e["signs"])
    np.testing.assert_allclose(e3["rnorm"] * e["s1"] * s2, e["rnorm"], rtol=1e-10)


def test_nsn_reduces_error_on_offset_channels():
    """On rows with offset channels the NSN records reconstruct x~ with a
    smaller relative error than the plain codec at the same bits."""
    d, l = 128, 2048
    rot, _ = oracle_rotation(d, 2, 6)
    x = _block(l, d, 2)
    e = codec.nsn_encode(rot, x)
    xh = codec.dequantize_nsn(rot, e["codes"], e["signs"], e["norm"], e["rnorm"], e["s1"], e["o"])
    ep = codec.encode(rot, x)
    xp = codec.dequantize(rot, ep["codes"], ep["signs"], ep["norm"], ep["rnorm"])
    err_nsn = np.sum((xh - x) ** 2) / np.sum(x * x)
    err_plain = np.sum((xp - x) ** 2) / np.sum(x * x)
    assert err_nsn < 0.8 * err_plain, (err_nsn, err_plain)


def _nsn_cache(rot, x, pos):
    """[B, H, T, d] blocks -> records, s1 [B, H, T], o [B, H, d]."""
    B, H, T, d = x.shape
    codes, signs, norms, s1, o = [], [], [], [], []
    for b in range(B):
        for h in range(H):
            e = codec.nsn_encode(rot, x[b, h], pos)
            codes.append(codec.pack_planes(e["codes"], rot.bits))
            signs.append(codec.pack_bits(e["signs"]))
            norms.append(np.stack([e["norm"], e["rnorm"]], axis=1))
            s1.append(e["s1"])
            o.append(e["o"])
    sh = lambda a: np.stack(a).reshape(B, H, T, *np.stack(a).shape[2:])
    return (sh(codes), sh(signs), sh(norms)), np.stack(s1).reshape(B, H, T), np.stack(o).reshape(B, H, d)


@pytest.mark.parametrize("G", [1, 4])
def test_nsn_decode_equals_attention_over_dequantized_rows(G):
    """Two routes: decode_attention_nsn (scores through the codes plus the
    s1 <q', o> term) against softmax attention over keys and values fully
    dequantized by dequantize_nsn."""
    d, T, B, Hkv = 128, 200, 2, 2
    Hq = G * Hkv
    rk, _ = oracle_rotation(d, 2, 11, rope=10000.0)
    rv, _ = oracle_rotation(d, 2, 12)
    k = np.stack([np.stack([_block(T, d, 100 + 10 * b + j) for j in range(Hkv)]) for b in range(B)])
    v = np.stack([np.stack([_block(T, d, 200 + 10 * b + j) for j in range(Hkv)]) for b in range(B)])
    pos = np.arange(T)
    kc, ks1, ko = _nsn_cache(rk, k, pos)
    vc, vs1, vo = _nsn_cache(rv, v, None)
    q = synth.heavy_tailed((B, Hq, d), 7).astype(np.float64)
    scale = 1 / math.sqrt(d)
    out = at.decode_attention_nsn(rk, rv, q, [T - 1] * B, kc, vc, ks1, ko, vs1, vo, scale)
    for b in range(B):
        qr = apply_rope(q[b], np.full(Hq, T - 1), 10000.0)
        for h in range(Hq):
            j = h // G
            unpack = lambda rot, c: (codec.unpack_planes(c[0][b, j], rot.bits, d), codec.unpack_bits(c[1][b, j], rot.m),
                                     c[2][b, j][:, 0], c[2][b, j][:, 1])
            kh = codec.dequantize_nsn(rk, *unpack(rk, kc), ks1[b, j], ko[b, j])
            vh = codec.dequantize_nsn(rv, *unpack(rv, vc), vs1[b, j], vo[b, j])
            sc = scale * (kh @ qr[h])
            p = np.exp(sc - sc.max())
            p /= p.sum()
            np.testing.assert_allclose(out[b, h], p @ vh, rtol=1e-9, atol=1e-9)


def test_nsn_decode_with_zero_shift_is_decode_attention():
    """o = 0 (any s1): the NSN decode is the plain decode over the same records."""
    d, T = 128, 150
    rk, _ = oracle_rotation(d, 3, 21, rope=10000.0)
    rv, _ = oracle_rotation(d, 3, 22)
    k = synth.heavy_tailed((1, 1, T, d), 3)
    v = synth.heavy_tailed((1, 1, T, d), 4)
    from helpers import oracle_records
    kc = tuple(a.reshape(1, 1, T, -1) for a in oracle_records(rk, k.reshape(-1, d), np.arange(T))[:3])
    vc = tuple(a.reshape(1, 1, T, -1) for a in oracle_records(rv, v.reshape(-1, d))[:3])
    q = synth.heavy_tailed((1, 4, d), 5)
    s1 = np.random.default_rng(0).random((1, 1, T)) + 0.5
    zero = np.zeros((1, 1, d))
    a = at.decode_attention_nsn(rk, rv, q, [T - 1], kc, vc, s1, zero, s1, zero, 1 / math.sqrt(d))
    b = at.decode_attention(rk, rv, q, [T - 1], kc, vc, 1 / math.sqrt(d))
    np.testing.assert_allclose(a, b, rtol=1e-11, atol=1e-11)


def test_nsn_append_matches_block_encode():
    """A token appended to a block with the block's own shift o is encoded as
    the block encode does for it: appending block token t (its raw row and
    position) reproduces token t's record and s1 exactly, and x' + s1 o
    gives back the token after RoPE."""
    d, l = 128, 257
    rot, _ = oracle_rotation(d, 2, 7, rope=10000.0)
    x = _block(l, d, 3)
    pos = np.arange(l) + 11
    e = codec.nsn_encode(rot, x, pos)
    pick = np.array([0, 100, l - 1])
    a = codec.nsn_append(rot, x[pick], pos[pick], e["o"])
    for key in ("codes", "signs"):
        assert np.array_equal(a[key], e[key][pick])
    for key in ("norm", "rnorm", "s1"):
        np.testing.assert_allclose(a[key], e[key][pick], rtol=1e-12, atol=0)
    np.testing.assert_allclose(a["x_shift"] + a["s1"][:, None] * e["o"][None, :],
                               apply_rope(x[pick], pos[pick], 10000.0), rtol=1e-12, atol=1e-12)


def test_nsn_append_zero_shift_is_plain_encode():
    """With o = 0 the appended record is the plain codec's record of x~."""
    d = 64
    rot, _ = oracle_rotation(d, 3, 8, rope=10000.0)
    x = _block(5, d, 4)
    pos = np.array([0, 3, 9, 1000, 65535])
    a = codec.nsn_append(rot, x, pos, np.zeros(d))
    p = codec.encode(rot, x, pos)
    assert np.array_equal(a["codes"], p["codes"]) and np.array_equal(a["signs"], p["signs"])
    np.testing.assert_allclose(a["norm"], p["norm"], rtol=1e-12)
    np.testing.assert_allclose(a["s1"], np.linalg.norm(x, axis=1) / math.sqrt(d), rtol=1e-12)
