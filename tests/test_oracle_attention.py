"""Pins for the oracle's attention from packed codes (CPU only)."""
import numpy as np
import pytest

import synth
from oracle import attention as at
from oracle import codec, rotation as ro


def _rot(d, bits, seed, rope=0.0):
    return ro.build_rotation(d, bits, synth.rotation_randomness(d, seed), "hadamard", rope_base=rope)


def _cache(rot, x, pos=None):
    """x [B, H, T, d] -> packed (codes, signs, norms) and the encode dict."""
    B, H, T, d = x.shape
    flat = x.reshape(-1, d)
    p = None if pos is None else np.tile(pos, B * H)
    e = codec.encode(rot, flat, p)
    codes = codec.pack_planes(e["codes"], rot.bits).reshape(B, H, T, -1)
    signs = codec.pack_bits(e["signs"]).reshape(B, H, T, -1)
    norms = np.stack([e["norm"], e["rnorm"]], axis=1).astype(np.float32).reshape(B, H, T, 2)
    return (codes, signs, norms), e


def _dequant(rot, cache):
    codes, signs, norms = cache
    c = codec.unpack_planes(codes.reshape(-1, codes.shape[-1]), rot.bits, rot.d)
    z = codec.unpack_bits(signs.reshape(-1, signs.shape[-1]), rot.m)
    n = norms.reshape(-1, 2).astype(np.float64)
    return codec.dequantize(rot, c, z, n[:, 0], n[:, 1])


def test_single_token_returns_dequantized_value():
    d = 128
    rk, rv = _rot(d, 2, 1, rope=10000.0), _rot(d, 2, 2)
    k = synth.heavy_tailed((1, 1, 1, d), 3)
    v = synth.heavy_tailed((1, 1, 1, d), 4)
    kc, _ = _cache(rk, k, np.arange(1))
    vc, _ = _cache(rv, v)
    q = synth.heavy_tailed((1, 1, d), 5)
    out = at.decode_attention(rk, rv, q, [0], kc, vc, 1 / np.sqrt(d))
    np.testing.assert_allclose(out[0, 0], _dequant(rv, vc)[0], rtol=1e-12, atol=1e-12)


def test_zero_query_gives_mean_value():
    d, T = 64, 13
    rk, rv = _rot(d, 2, 1, rope=10000.0), _rot(d, 3, 2)
    kc, _ = _cache(rk, synth.heavy_tailed((1, 1, T, d), 6), np.arange(T))
    vc, _ = _cache(rv, synth.heavy_tailed((1, 1, T, d), 7))
    out = at.decode_attention(rk, rv, np.zeros((1, 1, d)), [T - 1], kc, vc, 0.125)
    np.testing.assert_allclose(out[0, 0], _dequant(rv, vc).mean(axis=0), rtol=1e-11, atol=1e-11)


def test_brute_force_loops_tiny():
    # token-by-token loop on dequantized vectors (score = <RoPE(q), k~_t>)
    d, T = 64, 9
    rk, rv = _rot(d, 2, 3, rope=10000.0), _rot(d, 2, 4)
    kc, _ = _cache(rk, synth.heavy_tailed((1, 1, T, d), 8), np.arange(T))
    vc, _ = _cache(rv, synth.heavy_tailed((1, 1, T, d), 9))
    q = synth.heavy_tailed((1, 1, d), 10)
    kt, vt = _dequant(rk, kc), _dequant(rv, vc)
    qr = ro.apply_rope(q[0, 0], T - 1, 10000.0)
    scale = 1 / np.sqrt(d)
    sc = [float(qr @ kt[t]) * scale for t in range(T)]
    mx = max(sc)
    w = [np.exp(s - mx) for s in sc]
    ref = sum(w[t] * vt[t] for t in range(T)) / sum(w)
    out = at.decode_attention(rk, rv, q, [T - 1], kc, vc, scale)
    np.testing.assert_allclose(out[0, 0], ref, rtol=1e-10, atol=1e-10)


def test_token_permutation_invariance():
    d, T = 64, 16
    rk, rv = _rot(d, 2, 5), _rot(d, 2, 6)       # no RoPE: positions do not move with tokens
    kc, _ = _cache(rk, synth.heavy_tailed((1, 1, T, d), 11))
    vc, _ = _cache(rv, synth.heavy_tailed((1, 1, T, d), 12))
    perm = np.random.default_rng(0).permutation(T)
    kp = tuple(a[:, :, perm] for a in kc)
    vp = tuple(a[:, :, perm] for a in vc)
    q = synth.heavy_tailed((1, 1, d), 13)
    a = at.decode_attention(rk, rv, q, [0], kc, vc, 0.1)
    b = at.decode_attention(rk, rv, q, [0], kp, vp, 0.1)
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-12)


def test_gqa_mapping():
    d, T, B, Hq, Hkv = 64, 8, 2, 4, 2
    rk, rv = _rot(d, 2, 7, rope=10000.0), _rot(d, 2, 8)
    kc, _ = _cache(rk, synth.heavy_tailed((B, Hkv, T, d), 14), np.arange(T))
    vc, _ = _cache(rv, synth.heavy_tailed((B, Hkv, T, d), 15))
    q = synth.heavy_tailed((B, Hq, d), 16)
    out = at.decode_attention(rk, rv, q, [T - 1, T - 1], kc, vc, 0.125)
    for h in range(Hq):
        kv = h // 2
        one = at.decode_attention(rk, rv, q[:, h:h + 1], [T - 1, T - 1],
                                  tuple(a[:, kv:kv + 1] for a in kc),
                                  tuple(a[:, kv:kv + 1] for a in vc), 0.125)
        np.testing.assert_allclose(out[:, h], one[:, 0], rtol=1e-13)


def test_encoder_equals_decode_per_query():
    d, T = 64, 12
    rk, rv = _rot(d, 2, 9, rope=10000.0), _rot(d, 2, 10)
    kc, _ = _cache(rk, synth.heavy_tailed((1, 1, T, d), 17), np.arange(T))
    vc, _ = _cache(rv, synth.heavy_tailed((1, 1, T, d), 18))
    q = synth.heavy_tailed((1, 1, 5, d), 19)
    enc = at.encoder_attention(rk, rv, q, kc, vc, 0.125)
    for s in range(5):
        dec = at.decode_attention(rk, rv, q[:, :, s], [s], kc, vc, 0.125)
        np.testing.assert_allclose(enc[:, :, s], dec, rtol=1e-12)


def test_empty_cache_gives_zero():
    d = 64
    rk, rv = _rot(d, 2, 1), _rot(d, 2, 2)
    empty = (np.zeros((1, 1, 0, 16), np.uint8), np.zeros((1, 1, 0, 8), np.uint8), np.zeros((1, 1, 0, 2), np.float32))
    out = at.decode_attention(rk, rv, np.ones((1, 1, d)), [0], empty, empty, 0.1)
    assert np.all(out == 0)


def test_converges_to_exact_attention_with_bits():
    # Quantized attention approaches exact RoPE attention as bits grow (quality
    # statistic in the sense of the cosine similarity TurboESM reports, §3).
    d, T = 128, 256
    k = synth.heavy_tailed((1, 1, T, d), 20)
    v = synth.heavy_tailed((1, 1, T, d), 21)
    q = synth.heavy_tailed((1, 1, d), 22) * 0.05
    ref = at.exact_attention(q[0], k[0, 0], v[0, 0], 1 / np.sqrt(d), 10000.0, [T - 1], np.arange(T))[0]
    cos = []
    for bits in (1, 2, 3, 5):
        rk, rv = _rot(d, bits, 30, rope=10000.0), _rot(d, bits, 31)
        kc, _ = _cache(rk, k, np.arange(T))
        vc, _ = _cache(rv, v)
        out = at.decode_attention(rk, rv, q, [T - 1], kc, vc, 1 / np.sqrt(d))[0, 0]
        cos.append(out @ ref / np.linalg.norm(out) / np.linalg.norm(ref))
    assert all(a < b for a, b in zip(cos, cos[1:]))
    assert cos[-1] > 0.99


def test_unquantized_rotated_path_is_exact():
    # With the rotation alone (no quantization), attention is unchanged:
    # scores use (Pi R_i q)^T (Pi R_j k) = (R_i q)^T (R_j k).
    d, T = 64, 10
    rot = _rot(d, 2, 40)
    k = np.random.default_rng(1).standard_normal((T, d))
    v = np.random.default_rng(2).standard_normal((T, d))
    q = np.random.default_rng(3).standard_normal((1, d))
    qr, kr = ro.apply_rope(q, [T - 1], 1e4), ro.apply_rope(k, np.arange(T), 1e4)
    s_rot = (qr @ rot.pi.T) @ (kr @ rot.pi.T).T
    np.testing.assert_allclose(s_rot, qr @ kr.T, rtol=1e-12, atol=1e-12)
