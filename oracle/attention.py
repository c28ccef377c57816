"""Attention scored straight from the packed cache (float64 oracle).

TEST INFRASTRUCTURE ONLY (see the package header).

Definitions ([TurboESM] §2.A and §2.E; [TurboQuant] "QJL"):

  q' = RoPE(q, q_pos); q~ = Pi_K q'; s = S_K q~
  score_t = scale * ( ||k_t|| <q~, c_K[idx_t]>
                      + ||r_t|| sqrt(pi/2)/m <s, 2 z_t - 1> )
  p = softmax(score) over all cached tokens (no mask; two-pass formula)
  out = Pi_V^T ( sum_t p_t ||v_t|| c_V[idx^v_t]
                 + sqrt(pi/2)/m S_V^T sum_t p_t ||r^v_t|| (2 z^v_t - 1) )

i.e. attention over the dequantized keys and values; the inverse rotation
Pi^T is applied once after the weighted sum ([TurboESM] §2.E fuses
dequantization, residual correction, inverse rotation and the softmax).
Grouped-query attention maps query head h to KV head h // (Hq / Hkv).
An empty cache (T = 0) gives an all-zero output.

Pins (tests/test_oracle_attention.py): score route equals the dot product of
q' with the fully dequantized key (two independent routes); T = 1 returns the
dequantized value; q = 0 returns the mean value; token permutation
invariance; convergence to exact attention as bits grow; the unquantized
rotated path equals exact RoPE attention ([TurboESM] §2.A).
"""
from __future__ import annotations

import numpy as np

from .codec import QJL_CONST, unpack_bits, unpack_planes
from .rotation import Rotation, apply_rope


def _unpack_cache(rot: Rotation, codes, signs, norms):
    lead = codes.shape[:-1]
    c = unpack_planes(codes.reshape(-1, codes.shape[-1]), rot.bits, rot.d).reshape(*lead, rot.d)
    z = unpack_bits(signs.reshape(-1, signs.shape[-1]), rot.m).reshape(*lead, rot.m)
    nrm = np.asarray(norms, dtype=np.float64)
    return c, z, nrm[..., 0], nrm[..., 1]


def _attend(rot_k, rot_v, qrope, kc, kz, kn, kr, vc, vz, vn, vr, scale):
    """qrope [S, d] roped queries against one head's cache [T, ...] -> [S, d]."""
    S = qrope.shape[0]
    T = kc.shape[0]
    if T == 0:
        return np.zeros((S, rot_v.d))
    qt = qrope @ rot_k.pi.T
    sq = qt @ rot_k.s.T
    kyhat = rot_k.levels[kc]
    kzs = np.where(kz, 1.0, -1.0)
    score = (qt @ kyhat.T) * kn[None, :] + (sq @ kzs.T) * (QJL_CONST / rot_k.m) * kr[None, :]
    score = score * scale
    mx = np.max(score, axis=1, keepdims=True)
    e = np.exp(score - mx)
    p = e / np.sum(e, axis=1, keepdims=True)
    vyhat = rot_v.levels[vc]
    vzs = np.where(vz, 1.0, -1.0)
    acc = (p * vn[None, :]) @ vyhat
    acc_s = (p * vr[None, :]) @ vzs
    rotated = acc + (QJL_CONST / rot_v.m) * (acc_s @ rot_v.s)
    return rotated @ rot_v.pi


def decode_attention(rot_k: Rotation, rot_v: Rotation, q, q_pos, k_cache, v_cache,
                     scale: float) -> np.ndarray:
    """One decode step: q [B, Hq, d], q_pos [B]; caches are (codes, signs, norms)
    with shapes [B, Hkv, T, bits*d/8], [B, Hkv, T, m/8], [B, Hkv, T, 2].
    Returns out [B, Hq, d] float64."""
    q = np.asarray(q, dtype=np.float64)
    B, Hq, d = q.shape
    kc, kz, kn, kr = _unpack_cache(rot_k, *k_cache)
    vc, vz, vn, vr = _unpack_cache(rot_v, *v_cache)
    Hkv = kc.shape[1]
    g = Hq // Hkv
    out = np.zeros((B, Hq, rot_v.d))
    for b in range(B):
        qr = q[b]
        if rot_k.rope_base:
            qr = apply_rope(qr, np.full(Hq, q_pos[b]), rot_k.rope_base)
        for h in range(Hq):
            kv = h // g
            out[b, h] = _attend(rot_k, rot_v, qr[h:h + 1], kc[b, kv], kz[b, kv], kn[b, kv],
                                kr[b, kv], vc[b, kv], vz[b, kv], vn[b, kv], vr[b, kv], scale)[0]
    return out


def encoder_attention(rot_k: Rotation, rot_v: Rotation, q, k_cache, v_cache, scale: float,
                      q_pos_offset: int = 0) -> np.ndarray:
    """Bidirectional attention of S queries per head over the whole cache.

    q [B, Hq, S, d] with query s at position q_pos_offset + s; caches as in
    :func:`decode_attention` ([B, Hkv, T, ...]).  Returns [B, Hq, S, d]."""
    q = np.asarray(q, dtype=np.float64)
    B, Hq, S, d = q.shape
    kc, kz, kn, kr = _unpack_cache(rot_k, *k_cache)
    vc, vz, vn, vr = _unpack_cache(rot_v, *v_cache)
    Hkv = kc.shape[1]
    g = Hq // Hkv
    out = np.zeros((B, Hq, S, rot_v.d))
    pos = q_pos_offset + np.arange(S)
    for b in range(B):
        for h in range(Hq):
            kv = h // g
            qr = apply_rope(q[b, h], pos, rot_k.rope_base) if rot_k.rope_base else q[b, h]
            out[b, h] = _attend(rot_k, rot_v, qr, kc[b, kv], kz[b, kv], kn[b, kv], kr[b, kv],
                                vc[b, kv], vz[b, kv], vn[b, kv], vr[b, kv], scale)
    return out


def exact_attention(q, k, v, scale: float, rope_base: float = 0.0, q_pos=None, k_pos=None):
    """Unquantized softmax attention of q [S, d] over k, v [T, d] (float64)."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    if rope_base:
        q = apply_rope(q, q_pos, rope_base)
        k = apply_rope(k, k_pos, rope_base)
    s = (q @ k.T) * scale
    s = s - np.max(s, axis=1, keepdims=True)
    e = np.exp(s)
    return (e / np.sum(e, axis=1, keepdims=True)) @ v
