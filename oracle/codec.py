"""Encode, pack, unpack and dequantize vectors (float64 oracle).

TEST INFRASTRUCTURE ONLY (see the package header).

Encoding of one vector x in R^d (steps in the pages' order):

 1. RoPE at the vector's position when the handle has a RoPE base, before
    any rotation ([TurboESM] §2.A).
 2. Norm ||x|| and direction u = x / ||x|| ([TurboQuant] "Principe",
    Étape 1: the stage keeps "the intensity of the original vector").
 3. Rotation y = Pi u ([TurboQuant] Étape 1; [NSNQuant] §2).
 4. Per-coordinate Lloyd-Max code idx_i = #{j : t_j <= y_i} (a value on a
    threshold takes the upper code; [TurboESM] §2.C, [TurboQuant] Étape 1).
 5. Residual r = ||x|| (y - c[idx]) = Pi (x - x_hat), and ||r||
    ([TurboESM] §2.D: the residual x - x_hat).
 6. QJL sign sketch z_j = [(S r)_j >= 0], j < m ([TurboQuant] "QJL": each
    value of the Johnson-Lindenstrauss transform reduced to one sign bit).
 7. Bit packing (below).

Dequantization (rotated space):  ||x|| c[idx] + sqrt(pi/2)/m ||r|| S^T (2z - 1),
then Pi^T back to the original space.  The QJL term is the unbiased estimate
of r from its sign sketch: for s ~ N(0, I), E[sign(<s, r>) s] = sqrt(2/pi)
r/||r|| ([TurboQuant] "QJL": the estimator that removes the bias).

Packed record layout (the format the CUDA path reads and writes):
  codes: ``bits`` bit-planes of d bits each, plane k holding bit k of every
         code, coordinate i at byte i//8, bit i%8 (LSB first); planes stored
         in order k = 0 .. bits-1, so a record is bits*d/8 bytes.
  signs: one plane of m bits, same bit order (bit = 1 means (S r)_j >= 0).
  norms: two float32 per vector, (||x||, ||r||).

Boundary flags (the tolerance the parity tests grant):
  code flag  |y_i - t_j| < 1e-5 for some threshold t_j (unit coordinates);
  sign flag  |(S r)_j| < 1e-5 ||S_j|| ||r||.
"""
from __future__ import annotations

import math

import numpy as np

from .rotation import Rotation, apply_rope

QJL_CONST = math.sqrt(math.pi / 2.0)
CODE_FLAG_EPS = 1e-5
SIGN_FLAG_EPS = 1e-5


def encode(rot: Rotation, x, pos=None) -> dict:
    """Encode rows of x [n, d]; ``pos`` [n] positions for RoPE (or None)."""
    x = np.asarray(x, dtype=np.float64)
    if x.ndim == 1:
        x = x[None, :]
    n, d = x.shape
    assert d == rot.d
    if rot.rope_base and pos is not None:
        x = apply_rope(x, np.asarray(pos), rot.rope_base)
    norm = np.sqrt(np.sum(x * x, axis=1))
    safe = np.where(norm > 0, norm, 1.0)
    u = np.where(norm[:, None] > 0, x / safe[:, None], 0.0)
    y = u @ rot.pi.T
    codes = np.searchsorted(rot.thresholds, y, side="right")
    yhat = rot.levels[codes]
    r = norm[:, None] * (y - yhat)
    rnorm = np.sqrt(np.sum(r * r, axis=1))
    proj = r @ rot.s.T
    signs = proj >= 0.0
    code_flags = np.min(np.abs(y[:, :, None] - rot.thresholds[None, None, :]), axis=2) < CODE_FLAG_EPS
    srow = np.sqrt(np.sum(rot.s * rot.s, axis=1))
    sign_flags = np.abs(proj) < SIGN_FLAG_EPS * srow[None, :] * rnorm[:, None]
    return dict(codes=codes.astype(np.int64), signs=signs, norm=norm, rnorm=rnorm,
                y=y, proj=proj, code_flags=code_flags, sign_flags=sign_flags,
                x_rope=x)


def pack_bits(bits_2d) -> np.ndarray:
    """[n, L] booleans -> [n, L/8] uint8, element i at byte i//8 bit i%8."""
    b = np.asarray(bits_2d, dtype=np.uint8)
    n, L = b.shape
    assert L % 8 == 0
    out = np.zeros((n, L // 8), dtype=np.uint8)
    for i in range(L):
        out[:, i // 8] |= (b[:, i] & 1) << (i % 8)
    return out


def unpack_bits(packed, L: int) -> np.ndarray:
    """Inverse of :func:`pack_bits`: [n, L/8] uint8 -> [n, L] bool."""
    p = np.asarray(packed, dtype=np.uint8)
    out = np.zeros((p.shape[0], L), dtype=bool)
    for i in range(L):
        out[:, i] = (p[:, i // 8] >> (i % 8)) & 1
    return out


def pack_planes(codes, bits: int) -> np.ndarray:
    """[n, d] integer codes -> [n, bits*d/8] uint8 bit-planes (plane 0 first)."""
    codes = np.asarray(codes, dtype=np.int64)
    return np.concatenate([pack_bits((codes >> k) & 1) for k in range(bits)], axis=1)


def unpack_planes(packed, bits: int, d: int) -> np.ndarray:
    """Inverse of :func:`pack_planes`."""
    p = np.asarray(packed, dtype=np.uint8)
    w = d // 8
    codes = np.zeros((p.shape[0], d), dtype=np.int64)
    for k in range(bits):
        codes |= unpack_bits(p[:, k * w:(k + 1) * w], d).astype(np.int64) << k
    return codes


def dequantize(rot: Rotation, codes, signs, norm, rnorm, rotated: bool = False) -> np.ndarray:
    """Reconstruction x_tilde [n, d] (original space unless ``rotated``)."""
    codes = np.asarray(codes)
    z = np.where(np.asarray(signs, dtype=bool), 1.0, -1.0)
    norm = np.asarray(norm, dtype=np.float64)
    rnorm = np.asarray(rnorm, dtype=np.float64)
    mse_part = norm[:, None] * rot.levels[codes]
    qjl_part = (QJL_CONST / rot.m) * rnorm[:, None] * (z @ rot.s)
    xr = mse_part + qjl_part
    return xr if rotated else xr @ rot.pi


def score_from_codes(rot: Rotation, q, codes, signs, norm, rnorm) -> np.ndarray:
    """Inner-product estimates <q, x_n> from the codes, q [d] or [nq, d].

    <Pi q, ||x|| c[idx]> + ||r|| sqrt(pi/2)/m <S Pi q, 2z - 1>, the estimator
    of [TurboQuant] "QJL" (high-precision query, sign-bit data).
    Returns [n] for a single query, else [nq, n].
    """
    q = np.asarray(q, dtype=np.float64)
    single = q.ndim == 1
    q2 = q[None, :] if single else q
    qt = q2 @ rot.pi.T                      # rotated queries [nq, d]
    sq = qt @ rot.s.T                        # S Pi q          [nq, m]
    yhat = rot.levels[np.asarray(codes)]     # [n, d]
    z = np.where(np.asarray(signs, dtype=bool), 1.0, -1.0)
    mse = (qt @ yhat.T) * np.asarray(norm, dtype=np.float64)[None, :]
    qjl = (sq @ z.T) * (QJL_CONST / rot.m) * np.asarray(rnorm, dtype=np.float64)[None, :]
    out = mse + qjl
    return out[0] if single else out


# ---------------------------------------------------------------------------
# Residual-correction variants, for comparison at equal bits (test
# infrastructure; the CUDA path implements the QJL form above only).
#
# [TurboESM] §2.D keeps only the sign of the residual (1 bit) and rebuilds
# x_tilde = x_hat + sign * e_bar, e_bar a mean residual magnitude the page
# calibrates beforehand.  Calibration data is out of scope here, so e_bar is
# read as the mean magnitude of this vector's own residual,
# e_bar = ||r||_1 / d, stored in place of ||r|| (same bytes as the QJL form
# with m = d: d code bits per plane, d sign bits, two floats).  Signs are of
# the rotated residual, coordinate by coordinate (no projection).
# The MSE-only form drops the residual term: x_tilde = Pi^T ||x|| c[idx].
# ---------------------------------------------------------------------------
def encode_sign_residual(rot: Rotation, x, pos=None) -> dict:
    """Codes as :func:`encode`; sign bits z_i = [r_i >= 0] of the rotated
    residual r = ||x|| (y - c[idx]) and e_bar = ||r||_1 / d per vector."""
    e = encode(rot, x, pos)
    r = e["norm"][:, None] * (e["y"] - rot.levels[e["codes"]])
    return dict(codes=e["codes"], signs=r >= 0.0, norm=e["norm"], ebar=np.mean(np.abs(r), axis=1), r=r)


def dequantize_sign_residual(rot: Rotation, codes, signs, norm, ebar, rotated: bool = False) -> np.ndarray:
    """x_tilde = Pi^T (||x|| c[idx] + e_bar (2z - 1)) ([TurboESM] §2.D)."""
    z = np.where(np.asarray(signs, dtype=bool), 1.0, -1.0)
    xr = np.asarray(norm, dtype=np.float64)[:, None] * rot.levels[np.asarray(codes)] \
        + np.asarray(ebar, dtype=np.float64)[:, None] * z
    return xr if rotated else xr @ rot.pi


def dequantize_mse_only(rot: Rotation, codes, norm, rotated: bool = False) -> np.ndarray:
    """x_tilde = Pi^T ||x|| c[idx]: the codes alone, no residual term."""
    xr = np.asarray(norm, dtype=np.float64)[:, None] * rot.levels[np.asarray(codes)]
    return xr if rotated else xr @ rot.pi


# ---------------------------------------------------------------------------
# Normalize-Shift-Normalize pre-transform ([NSNQuant] §1).  For a block of l
# tokens x [l, d]:
#   x1 = x sqrt(d) / ||x||           per token, s1 = ||x|| / sqrt(d)
#   o  = mean over the block's tokens of x1, per channel
#   x3 = (x1 - o) sqrt(d) / ||x1 - o||  per token, s2 = ||x1 - o|| / sqrt(d)
# so that x = s1 (s2 x3 + o).  x3 then goes through the codec as any vector.
# ---------------------------------------------------------------------------
def nsn_forward(x):
    """Returns (x3 [l, d], s1 [l], o [d], s2 [l]) of [NSNQuant] §1."""
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[1]
    s1 = np.sqrt(np.sum(x * x, axis=1)) / math.sqrt(d)
    x1 = x / np.where(s1 > 0, s1, 1.0)[:, None]
    o = np.mean(x1, axis=0)
    x2 = x1 - o
    s2 = np.sqrt(np.sum(x2 * x2, axis=1)) / math.sqrt(d)
    x3 = x2 / np.where(s2 > 0, s2, 1.0)[:, None]
    return x3, s1, o, s2


def nsn_inverse(x3, s1, o, s2):
    """x = s1 (s2 x3 + o)."""
    return np.asarray(s1)[:, None] * (np.asarray(s2)[:, None] * np.asarray(x3) + np.asarray(o)[None, :])


# ---------------------------------------------------------------------------
# NSN as a record mode of the codec ([NSNQuant] §1 and §4).  For one block of
# tokens (one sequence and head), RoPE first (the codec's codes live in the
# space after RoPE, [TurboESM] §2.A), then (x3, s1, o, s2) = nsn_forward(x~).
# The codec encodes x' = s1 s2 x3 = x~ - s1 o without RoPE, so its record
# holds the direction of x3 and the norms ||x'|| = s1 s2 sqrt(d) and
# ||r'|| = s1 s2 ||r3||; s1 per token and o per block are kept beside it.
# Dequantization: x^ = x'^ + s1 o, the inverse of the page's transform with
# x3 replaced by its reconstruction.  (NSNQuant applies NSN before RoPE; with
# the shift after RoPE the score term s1 <q', o> needs one dot product per
# query and block instead of one per token.)
# ---------------------------------------------------------------------------
def nsn_encode(rot: Rotation, x, pos=None) -> dict:
    """Encode one block x [l, d] with NSN: the codec dict of x' plus the
    per-token s1 [l] and the block shift o [d] (both in the space after
    RoPE)."""
    x = np.asarray(x, dtype=np.float64)
    if rot.rope_base and pos is not None:
        x = apply_rope(x, np.asarray(pos), rot.rope_base)
    x3, s1, o, s2 = nsn_forward(x)
    xp = (s1 * s2)[:, None] * x3
    e = encode(rot, xp, None)
    e["s1"] = s1
    e["o"] = o
    e["x_nsn"] = x
    e["x_shift"] = xp
    return e


def nsn_append(rot: Rotation, x, pos, o) -> dict:
    """Encode tokens x [n, d] appended to a block whose shift o [d] is already
    fixed ([NSNQuant] §4: tokens after the block keep its statistics): RoPE
    at pos when the handle has it, s1 = ||x~|| / sqrt(d), x' = x~ - s1 o, and
    the codec's record of x'.  Returns the codec dict of x' plus s1 [n]."""
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[1]
    if rot.rope_base and pos is not None:
        x = apply_rope(x, np.asarray(pos), rot.rope_base)
    s1 = np.sqrt(np.sum(x * x, axis=1)) / math.sqrt(d)
    xp = x - s1[:, None] * np.asarray(o, dtype=np.float64)[None, :]
    e = encode(rot, xp, None)
    e["s1"] = s1
    e["x_shift"] = xp
    return e


def dequantize_nsn(rot: Rotation, codes, signs, norm, rnorm, s1, o) -> np.ndarray:
    """x^ [n, d] = dequantize(record of x') + s1 o (space after RoPE)."""
    xp = dequantize(rot, codes, signs, norm, rnorm)
    return xp + np.asarray(s1, dtype=np.float64)[:, None] * np.asarray(o, dtype=np.float64)[None, :]
