"""Pins for the oracle's decode over a packed cache plus a full-precision
window ([NSNQuant] §4, "Résidus"), CPU only."""
import numpy as np
from scipy.special import softmax

import synth
from oracle import attention as at
from oracle import codec, rotation as ro


def _rot(d, bits, seed, rope=0.0):
    return ro.build_rotation(d, bits, synth.rotation_randomness(d, seed), "hadamard", rope_base=rope)


def _cache(rot, x, pos=None):
    """x [B, H, T, d] -> packed (codes, signs, norms)."""
    B, H, T, d = x.shape
    flat = x.reshape(-1, d)
    p = None if pos is None else np.tile(pos, B * H)
    e = codec.encode(rot, flat, p)
    codes = codec.pack_planes(e["codes"], rot.bits).reshape(B, H, T, -1)
    signs = codec.pack_bits(e["signs"]).reshape(B, H, T, -1)
    norms = np.stack([e["norm"], e["rnorm"]], axis=1).astype(np.float32).reshape(B, H, T, 2)
    return codes, signs, norms


def _empty_cache(rot, B, H):
    return (np.zeros((B, H, 0, rot.bits * rot.d // 8), np.uint8), np.zeros((B, H, 0, rot.m // 8), np.uint8),
            np.zeros((B, H, 0, 2), np.float32))


def _rope_matrix(pos, d, base):
    """RoPE as an explicit d x d matrix: plane (i, i + d/2) turned by pos * base^(-2i/d)."""
    M = np.zeros((d, d))
    for i in range(d // 2):
        a = pos * base ** (-2.0 * i / d)
        c, s = np.cos(a), np.sin(a)
        M[i, i], M[i, i + d // 2] = c, -s
        M[i + d // 2, i], M[i + d // 2, i + d // 2] = s, c
    return M


def test_empty_window_equals_decode():
    # R = 0: the window route (dequantized keys) against the code route of decode_attention
    d, B, Hq, Hkv, T = 64, 2, 4, 2, 11
    rk, rv = _rot(d, 2, 21, rope=10000.0), _rot(d, 2, 22)
    kc = _cache(rk, synth.heavy_tailed((B, Hkv, T, d), 23), np.arange(T))
    vc = _cache(rv, synth.heavy_tailed((B, Hkv, T, d), 24))
    q = synth.heavy_tailed((B, Hq, d), 25)
    qpos = [T, T + 3]
    empty = np.zeros((B, Hkv, 0, d))
    ref = at.decode_attention(rk, rv, q, qpos, kc, vc, 0.125)
    out = at.decode_attention_window(rk, rv, q, qpos, kc, vc, empty, empty, 0.125)
    np.testing.assert_allclose(out, ref, rtol=1e-11, atol=1e-11)


def test_window_only_equals_textbook_attention():
    # T = 0: plain softmax attention with RoPE written as rotation matrices
    d, R, base = 64, 7, 10000.0
    rk, rv = _rot(d, 2, 31, rope=base), _rot(d, 2, 32)
    kw = synth.heavy_tailed((1, 1, R, d), 33)
    vw = synth.heavy_tailed((1, 1, R, d), 34)
    q = synth.heavy_tailed((1, 1, d), 35)
    qpos = R + 2
    scale = 1 / np.sqrt(d)
    qr = _rope_matrix(qpos, d, base) @ q[0, 0]
    kr = np.stack([_rope_matrix(i, d, base) @ kw[0, 0, i] for i in range(R)])
    ref = softmax(kr @ qr * scale) @ vw[0, 0]
    out = at.decode_attention_window(rk, rv, q, [qpos], _empty_cache(rk, 1, 1), _empty_cache(rv, 1, 1),
                                     kw, vw, scale)
    np.testing.assert_allclose(out[0, 0], ref, rtol=1e-12, atol=1e-12)


def test_single_window_token_returns_its_value():
    d = 128
    rk, rv = _rot(d, 3, 41, rope=10000.0), _rot(d, 3, 42)
    kw = synth.heavy_tailed((1, 1, 1, d), 43)
    vw = synth.heavy_tailed((1, 1, 1, d), 44)
    q = synth.heavy_tailed((1, 2, d), 45)
    out = at.decode_attention_window(rk, rv, q, [5], _empty_cache(rk, 1, 1), _empty_cache(rv, 1, 1), kw, vw, 0.1)
    np.testing.assert_allclose(out[0, 0], vw[0, 0, 0], rtol=1e-14, atol=1e-14)
    np.testing.assert_allclose(out[0, 1], vw[0, 0, 0], rtol=1e-14, atol=1e-14)


def test_zero_query_gives_mean_of_both_parts():
    d, T, R = 64, 6, 5
    rk, rv = _rot(d, 2, 51, rope=10000.0), _rot(d, 2, 52)
    kc = _cache(rk, synth.heavy_tailed((1, 1, T, d), 53), np.arange(T))
    vx = synth.heavy_tailed((1, 1, T, d), 54)
    vc = _cache(rv, vx)
    kw = synth.heavy_tailed((1, 1, R, d), 55)
    vw = synth.heavy_tailed((1, 1, R, d), 56)
    codes, signs, norms = vc
    vdeq = codec.dequantize(rv, codec.unpack_planes(codes[0, 0], 2, d), codec.unpack_bits(signs[0, 0], d),
                            norms[0, 0, :, 0], norms[0, 0, :, 1])
    ref = (vdeq.sum(axis=0) + vw[0, 0].astype(np.float64).sum(axis=0)) / (T + R)
    out = at.decode_attention_window(rk, rv, np.zeros((1, 1, d)), [T + R], kc, vc, kw, vw, 0.125)
    np.testing.assert_allclose(out[0, 0], ref, rtol=1e-11, atol=1e-11)


def test_window_sits_after_the_packed_part():
    # Packed keys pointing away from the query carry zero weight (exp underflows), so
    # only the window counts.  Moving every position by T (query and window keys) keeps
    # the relative positions and so the output; placing the window keys at 0..R-1
    # instead of T..T+R-1 would change it.
    d, T, R, base = 64, 9, 6, 10000.0
    rk, rv = _rot(d, 2, 61, rope=base), _rot(d, 2, 62)
    q = synth.heavy_tailed((1, 1, d), 63)
    kw = synth.heavy_tailed((1, 1, R, d), 64)
    vw = synth.heavy_tailed((1, 1, R, d), 65)
    qpos = T + R
    away = -1e3 * ro.apply_rope(q[0, 0], qpos, base)
    kc = _cache(rk, np.tile(away, (1, 1, T, 1)))          # stored as is: already at the query's frame
    vc = _cache(rv, synth.heavy_tailed((1, 1, T, d), 66))
    out = at.decode_attention_window(rk, rv, q, [qpos], kc, vc, kw, vw, 1 / np.sqrt(d))
    shifted = at.decode_attention_window(rk, rv, q, [R], _empty_cache(rk, 1, 1), _empty_cache(rv, 1, 1), kw, vw,
                                         1 / np.sqrt(d))
    np.testing.assert_allclose(out, shifted, rtol=1e-10, atol=1e-10)
    # and the pin has teeth: the same window with the query moved by T differs
    moved = at.decode_attention_window(rk, rv, q, [R + T], _empty_cache(rk, 1, 1), _empty_cache(rv, 1, 1), kw, vw,
                                       1 / np.sqrt(d))
    assert np.max(np.abs(moved - shifted)) > 1e-3
