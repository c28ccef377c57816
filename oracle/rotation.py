"""Rotations, RoPE and the QJL projection for the oracle (float64).

TEST INFRASTRUCTURE ONLY (see the package header).

* Randomized Hadamard rotation  Pi = H_d diag(D) / sqrt(d)  with H_d the
  Sylvester (natural-order) Hadamard matrix, H[i, j] = (-1)^popcount(i & j),
  and D a random +-1 diagonal ([NSNQuant] §2: the randomized Hadamard
  transform; [TurboQuant] "Principe", Étape 1: a data-oblivious random
  rotation).  Used for power-of-two head dimensions.
* Dense seeded rotation  Pi = Q diag(sign(diag R))  from the QR factorization
  G = QR of a seeded Gaussian matrix (Haar distributed; the sign fix makes it
  unique).  Used where d is not a power of two.
* RoPE, half-split ("rotate-half") pairing of coordinates i and i + d/2 with
  angle pos * base^(-2i/d), applied before the rotation ([TurboESM] §2.A:
  RoPE first, then Pi; the order keeps (Pi R_i q)^T (Pi R_j k) = (R_i q)^T
  (R_j k) because Pi^T Pi = I).
* QJL projection S: m x d i.i.d. N(0, 1) entries ([TurboQuant] "QJL"),
  rounded to the nearest bf16-representable value (reading: lets the GPU hold
  S exactly in 16 bits; the oracle uses the same rounded matrix).

Pins (tests/test_oracle_rotation.py): H_d against scipy.linalg.hadamard and
the closed forms of H_2 and H_4; Pi^T Pi = I; the QR sign convention; RoPE
against its complex-number form, its norm preservation and its dependence on
i - j only; the rotation-invariance identity of [TurboESM] §2.A; bf16 rounding
against torch's conversion.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

from .codebook import lloyd_max


def sylvester_hadamard(d: int) -> np.ndarray:
    """Unnormalised Sylvester Hadamard matrix of order d (d a power of two)."""
    if d < 1 or d & (d - 1):
        raise ValueError("d must be a power of two")
    i = np.arange(d)
    pc = np.vectorize(lambda v: bin(int(v)).count("1"))(i[:, None] & i[None, :])
    return np.where(pc % 2 == 0, 1.0, -1.0)


def hadamard_rotation(signs: np.ndarray) -> np.ndarray:
    """Pi = H_d diag(signs) / sqrt(d) (float64 [d, d])."""
    d = len(signs)
    return sylvester_hadamard(d) * np.asarray(signs, dtype=np.float64)[None, :] / np.sqrt(d)


def dense_rotation(gauss: np.ndarray) -> np.ndarray:
    """Haar rotation from a Gaussian matrix: Q diag(sign(diag R)) with G = QR."""
    q, r = np.linalg.qr(np.asarray(gauss, dtype=np.float64))
    s = np.sign(np.diag(r))
    s[s == 0] = 1.0
    return q * s[None, :]


def round_to_bf16(x) -> np.ndarray:
    """Round float32 values to the nearest bf16-representable value
    (ties to even), returned as float32."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16) << 16
    nan = np.isnan(np.asarray(x, dtype=np.float32))
    out = (r & 0xFFFFFFFF).astype(np.uint32).view(np.float32)
    return np.where(nan, np.float32(np.nan), out)


def rope_angles(pos, d: int, base: float) -> np.ndarray:
    """Angles pos * base^(-2i/d), i < d/2, float64 [..., d/2]."""
    i = np.arange(d // 2, dtype=np.float64)
    theta = base ** (-2.0 * i / d)
    return np.asarray(pos, dtype=np.float64)[..., None] * theta


def apply_rope(x, pos, base: float) -> np.ndarray:
    """Rotate-half RoPE: (x_i, x_{i+d/2}) -> rotation by pos * theta_i."""
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    ang = rope_angles(pos, d, base)
    c, s = np.cos(ang), np.sin(ang)
    x1, x2 = x[..., : d // 2], x[..., d // 2:]
    return np.concatenate((x1 * c - x2 * s, x2 * c + x1 * s), axis=-1)


@dataclass
class Rotation:
    """Everything one codec handle fixes: Pi, S, codebook and RoPE base."""
    d: int
    m: int
    bits: int
    kind: str                      # "hadamard" or "dense"
    pi: np.ndarray                 # [d, d] float64, y = pi @ u
    s: np.ndarray                  # [m, d] float64 (bf16-representable)
    levels: np.ndarray             # [2**bits] ascending
    thresholds: np.ndarray         # [2**bits - 1]
    rope_base: float = 0.0         # 0 -> no RoPE
    signs: np.ndarray | None = field(default=None, repr=False)


def build_rotation(d: int, bits: int, randomness: dict, kind: str = "hadamard",
                   rope_base: float = 0.0) -> Rotation:
    """Build the oracle's handle from the seeded draws of ``synth``."""
    if kind == "hadamard":
        pi = hadamard_rotation(randomness["signs"])
    elif kind == "dense":
        pi = dense_rotation(randomness["gauss_pi"])
    else:
        raise ValueError(kind)
    s = round_to_bf16(randomness["gauss_s"]).astype(np.float64)
    levels, thresholds = lloyd_max(d, bits)
    return Rotation(d=d, m=s.shape[0], bits=bits, kind=kind, pi=pi, s=s,
                    levels=levels, thresholds=thresholds, rope_base=rope_base,
                    signs=np.asarray(randomness["signs"]))
