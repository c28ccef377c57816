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

Full-precision window ([NSNQuant] §4, "Résidus", after KIVI): the cache is a
quantized part of T tokens plus a residual of the R most recent tokens kept
as the model produced them; when the residual is full it is quantized and
appended to the packed part.  Decode attends to both: window token i sits at
position T + i, so its key gets RoPE there, and the softmax runs over the
union.  Pins (tests/test_oracle_window.py): R = 0 equals decode_attention
(whose scores take the other route, through the codes); T = 0 equals textbook
softmax attention; one window token and no packed part returns its value; a
shift of every position by the same amount leaves the output unchanged,
which fails if the window keys are not placed after the packed part.
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


def decode_attention_nsn(rot_k: Rotation, rot_v: Rotation, q, q_pos, k_cache, v_cache, k_s1, k_o, v_s1, v_o,
                         scale: float) -> np.ndarray:
    """decode_attention over NSN records ([NSNQuant] §1, §4; codec.nsn_encode):
    key t of sequence (b, j) is k'^_t + s1k_t o_k[b, j] and value t is
    v'^_t + s1v_t o_v[b, j], so

      score_t = scale * ( <q', k'^_t> + s1k_t <q', o_k> )
      out     = sum_t p_t v'^_t + o_v sum_t p_t s1v_t

    with q' = RoPE(q) and k'^, v'^ the codec's estimates of the shifted
    records (scored as in decode_attention).  k_s1, v_s1 [B, Hkv, T];
    k_o, v_o [B, Hkv, d].  Returns out [B, Hq, d] float64."""
    q = np.asarray(q, dtype=np.float64)
    B, Hq, d = q.shape
    kc, kz, kn, kr = _unpack_cache(rot_k, *k_cache)
    vc, vz, vn, vr = _unpack_cache(rot_v, *v_cache)
    k_s1, k_o = np.asarray(k_s1, dtype=np.float64), np.asarray(k_o, dtype=np.float64)
    v_s1, v_o = np.asarray(v_s1, dtype=np.float64), np.asarray(v_o, dtype=np.float64)
    Hkv, T = kc.shape[1], kc.shape[2]
    g = Hq // Hkv
    out = np.zeros((B, Hq, rot_v.d))
    if T == 0:
        return out
    for b in range(B):
        qr = q[b]
        if rot_k.rope_base:
            qr = apply_rope(qr, np.full(Hq, q_pos[b]), rot_k.rope_base)
        for h in range(Hq):
            j = h // g
            qt = qr[h] @ rot_k.pi.T
            sq = rot_k.s @ qt
            kzs = np.where(kz[b, j], 1.0, -1.0)
            score = (rot_k.levels[kc[b, j]] @ qt) * kn[b, j] + (kzs @ sq) * (QJL_CONST / rot_k.m) * kr[b, j]
            score = scale * (score + k_s1[b, j] * (qr[h] @ k_o[b, j]))
            p = np.exp(score - np.max(score))
            p = p / np.sum(p)
            vzs = np.where(vz[b, j], 1.0, -1.0)
            rotated = (p * vn[b, j]) @ rot_v.levels[vc[b, j]] + \
                (QJL_CONST / rot_v.m) * (((p * vr[b, j]) @ vzs) @ rot_v.s)
            out[b, h] = rotated @ rot_v.pi + v_o[b, j] * (p @ v_s1[b, j])
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


def decode_attention_window(rot_k: Rotation, rot_v: Rotation, q, q_pos, k_cache, v_cache, k_window,
                            v_window, scale: float) -> np.ndarray:
    """One decode step over a packed cache plus a full-precision window
    ([NSNQuant] §4, "Résidus").

    q [B, Hq, d], q_pos [B]; packed caches (codes, signs, norms) of shape
    [B, Hkv, T, ...] as in :func:`decode_attention`; k_window, v_window
    [B, Hkv, R, d] the raw keys (before RoPE) and values of the R most recent
    tokens, window token i at position T + i.  The keys are the dequantized
    packed keys followed by RoPE(k_window); the values the dequantized packed
    values followed by v_window; softmax attention over all T + R of them.
    Returns out [B, Hq, d] float64."""
    from .codec import dequantize
    q = np.asarray(q, dtype=np.float64)
    kw = np.asarray(k_window, dtype=np.float64)
    vw = np.asarray(v_window, dtype=np.float64)
    B, Hq, d = q.shape
    kc, kz, kn, kr = _unpack_cache(rot_k, *k_cache)
    vc, vz, vn, vr = _unpack_cache(rot_v, *v_cache)
    Hkv, T = kc.shape[1], kc.shape[2]
    R = kw.shape[2]
    g = Hq // Hkv
    out = np.zeros((B, Hq, rot_v.d))
    for b in range(B):
        for h in range(Hq):
            kv = h // g
            keys = [dequantize(rot_k, kc[b, kv], kz[b, kv], kn[b, kv], kr[b, kv])]
            vals = [dequantize(rot_v, vc[b, kv], vz[b, kv], vn[b, kv], vr[b, kv])]
            kwin = kw[b, kv]
            qh = q[b, h]
            if rot_k.rope_base:
                kwin = apply_rope(kwin, T + np.arange(R), rot_k.rope_base)
                qh = apply_rope(qh, q_pos[b], rot_k.rope_base)
            keys.append(kwin)
            vals.append(vw[b, kv])
            K = np.concatenate(keys, axis=0)
            V = np.concatenate(vals, axis=0)
            if K.shape[0] == 0:
                continue
            score = (K @ qh) * scale
            e = np.exp(score - np.max(score))
            out[b, h] = (e / np.sum(e)) @ V
    return out


LOG2E = 1.4426950408889634


def decode_partials(rot_k: Rotation, rot_v: Rotation, q, q_pos, k_cache, v_cache, scale: float) -> np.ndarray:
    """Per query head, the partial record of the softmax over this cache's
    tokens (a shard of a longer context), [B, Hq, 2 + 2d]:
      m    = max_t s_t, with s_t = score_t * log2(e) (scores as in
             decode_attention, scale included),
      l    = sum_t 2^(s_t - m),
      A    = sum_t 2^(s_t - m) ||v_t|| c_V[idx^v_t]        (rotated space, d),
      A_s  = sum_t 2^(s_t - m) ||r^v_t|| (2 z^v_t - 1)     (m entries).
    An empty cache gives m = -inf, l = 0 and zeros.  The same definitions as
    decode_attention before its normalisation and inverse rotation
    ([TurboESM] §2.E)."""
    q = np.asarray(q, dtype=np.float64)
    B, Hq, d = q.shape
    kc, kz, kn, kr = _unpack_cache(rot_k, *k_cache)
    vc, vz, vn, vr = _unpack_cache(rot_v, *v_cache)
    Hkv, T = kc.shape[1], kc.shape[2]
    g = Hq // Hkv
    out = np.zeros((B, Hq, 2 + 2 * rot_v.d))
    for b in range(B):
        qr = q[b]
        if rot_k.rope_base:
            qr = apply_rope(qr, np.full(Hq, q_pos[b]), rot_k.rope_base)
        for h in range(Hq):
            kv = h // g
            if T == 0:
                out[b, h, 0] = -np.inf
                continue
            qt = qr[h] @ rot_k.pi.T
            sq = rot_k.s @ qt
            score = (rot_k.levels[kc[b, kv]] @ qt) * kn[b, kv] \
                + (np.where(kz[b, kv], 1.0, -1.0) @ sq) * (QJL_CONST / rot_k.m) * kr[b, kv]
            s2 = score * scale * LOG2E
            m = np.max(s2)
            w = np.exp2(s2 - m)
            out[b, h, 0] = m
            out[b, h, 1] = np.sum(w)
            out[b, h, 2:2 + rot_v.d] = (w * vn[b, kv]) @ rot_v.levels[vc[b, kv]]
            out[b, h, 2 + rot_v.d:] = (w * vr[b, kv]) @ np.where(vz[b, kv], 1.0, -1.0)
    return out


def merge_partials(rot_v: Rotation, parts) -> np.ndarray:
    """Attention output [B, Hq, d] from partial records [P, B, Hq, 2 + 2d] of
    disjoint token ranges: with M = max_p m_p and f_p = 2^(m_p - M),
      out = Pi_V^T (sum_p f_p A_p + sqrt(pi/2)/m S_V^T sum_p f_p A_s,p)
            / sum_p f_p l_p,
    zeros when every part is empty."""
    parts = np.asarray(parts, dtype=np.float64)
    P, B, Hq, rec = parts.shape
    d = rot_v.d
    out = np.zeros((B, Hq, d))
    for b in range(B):
        for h in range(Hq):
            m = parts[:, b, h, 0]
            if np.all(np.isneginf(m)):
                continue
            M = np.max(m)
            f = np.where(np.isneginf(m), 0.0, np.exp2(m - M))
            L = np.sum(f * parts[:, b, h, 1])
            A = f @ parts[:, b, h, 2:2 + d]
            As = f @ parts[:, b, h, 2 + d:]
            out[b, h] = ((A + (QJL_CONST / rot_v.m) * (As @ rot_v.s)) / L) @ rot_v.pi
    return out
