"""Counter-based random draws of a seeded codec handle (oracle side).

TEST INFRASTRUCTURE ONLY (see the package header).

The codec draws three random objects ([TurboQuant] "Principe", Étape 1 and
"QJL"; [NSNQuant] §2; [TurboESM] §2.B builds a rotation per layer and head,
which is reproducible only from a seed): the +-1 sign diagonal D of a
randomized Hadamard rotation, the m x d Gaussian QJL matrix S, and the d x d
Gaussian matrix whose QR factor is a dense rotation.  The pages name no
generator.  Both sides of the parity tests implement the same published
counter-based generator, Philox4x32-10 (J. K. Salmon, M. A. Moraes,
R. O. Dror, D. E. Shaw, "Parallel random numbers: as easy as 1, 2, 3",
SC 2011), each from that definition and sharing no code:

* one Philox4x32 round maps the counter (c0, c1, c2, c3) and key (k0, k1) to
  (hi(M1 c2) ^ c1 ^ k0, lo(M1 c2), hi(M0 c0) ^ c3 ^ k1, lo(M0 c0)) with the
  multipliers M0 = 0xD2511F53, M1 = 0xCD9E8D57 (hi/lo: the upper/lower 32
  bits of the 64-bit product); the key is bumped by the Weyl constants
  W0 = 0x9E3779B9, W1 = 0xBB67AE85 between rounds; ten rounds.

How a handle's draws use it (this library's own convention, the same on both
sides):

* key = (seed mod 2^32, seed >> 32) for a 64-bit seed;
* counter = (i mod 2^32, i >> 32, stream, 0), with stream 0 for D, 1 for S and
  2 for the dense Gaussian;
* D_i = -1 when the top bit of word 0 of block i is set, else +1;
* Gaussians come in pairs: block p gives two 52-bit uniforms
  u = ((w0 >> 6) 2^26 + (w1 >> 6) + 1/2) / 2^52 from words (0, 1) and (2, 3)
  (every step exact in float64, so u lies strictly inside (0, 1)),
  then Box-Muller: r = sqrt(-2 ln u1), z_{2p} = r cos(2 pi u2),
  z_{2p+1} = r sin(2 pi u2); the row-major element k of S (or of the dense
  Gaussian) is z_k.

Pins (tests/test_oracle_philox.py): the known-answer vectors published with
the Random123 distribution of the generator; a scalar pure-Python round
function against the vectorised one; the law of the uniforms and normals
(moments and a Kolmogorov-Smirnov test).
"""
from __future__ import annotations

import numpy as np

M0, M1 = 0xD2511F53, 0xCD9E8D57
W0, W1 = 0x9E3779B9, 0xBB67AE85
MASK32 = 0xFFFFFFFF
ROUNDS = 10

STREAM_SIGNS, STREAM_S, STREAM_DENSE = 0, 1, 2


def philox4x32_scalar(counter, key, rounds: int = ROUNDS):
    """Philox4x32 of one counter (4 ints) and key (2 ints), plain Python ints."""
    c0, c1, c2, c3 = (int(v) & MASK32 for v in counter)
    k0, k1 = (int(v) & MASK32 for v in key)
    for r in range(rounds):
        if r:
            k0 = (k0 + W0) & MASK32
            k1 = (k1 + W1) & MASK32
        p0 = M0 * c0
        p1 = M1 * c2
        c0, c1, c2, c3 = ((p1 >> 32) ^ c1 ^ k0, p1 & MASK32, (p0 >> 32) ^ c3 ^ k1, p0 & MASK32)
    return c0, c1, c2, c3


def philox4x32(c0, c1, c2, c3, k0: int, k1: int, rounds: int = ROUNDS):
    """Vectorised Philox4x32 over arrays of counters (uint64 arithmetic)."""
    c = [np.asarray(v, dtype=np.uint64) & np.uint64(MASK32) for v in (c0, c1, c2, c3)]
    c0, c1, c2, c3 = np.broadcast_arrays(*c)
    c0, c1, c2, c3 = (v.copy() for v in (c0, c1, c2, c3))
    k0, k1 = int(k0) & MASK32, int(k1) & MASK32
    m32 = np.uint64(MASK32)
    for r in range(rounds):
        if r:
            k0 = (k0 + W0) & MASK32
            k1 = (k1 + W1) & MASK32
        p0 = np.uint64(M0) * c0          # < 2^64: exact in uint64
        p1 = np.uint64(M1) * c2
        c0, c1, c2, c3 = ((p1 >> np.uint64(32)) ^ c1 ^ np.uint64(k0), p1 & m32,
                          (p0 >> np.uint64(32)) ^ c3 ^ np.uint64(k1), p0 & m32)
    return c0, c1, c2, c3


def _key(seed: int):
    seed = int(seed) & ((1 << 64) - 1)
    return seed & MASK32, seed >> 32


def _blocks(seed: int, stream: int, n: int):
    idx = np.arange(n, dtype=np.uint64)
    k0, k1 = _key(seed)
    return philox4x32(idx & np.uint64(MASK32), idx >> np.uint64(32), np.uint64(stream), np.uint64(0), k0, k1)


def uniform52(wa, wb) -> np.ndarray:
    """(0, 1) uniforms from two 32-bit words: 52 bits, centred on the grid.
    The integer part is below 2^52, so adding 1/2 and scaling are exact."""
    a = (np.asarray(wa, dtype=np.uint64) >> np.uint64(6)).astype(np.float64)
    b = (np.asarray(wb, dtype=np.uint64) >> np.uint64(6)).astype(np.float64)
    return (a * 67108864.0 + b + 0.5) / 4503599627370496.0


def gaussians(seed: int, stream: int, count: int) -> np.ndarray:
    """The first `count` N(0, 1) draws of a stream (Box-Muller pairs), float64."""
    n_pairs = (count + 1) // 2
    w0, w1, w2, w3 = _blocks(seed, stream, n_pairs)
    u1 = uniform52(w0, w1)
    u2 = uniform52(w2, w3)
    r = np.sqrt(-2.0 * np.log(u1))
    z = np.empty(2 * n_pairs, dtype=np.float64)
    z[0::2] = r * np.cos(2.0 * np.pi * u2)
    z[1::2] = r * np.sin(2.0 * np.pi * u2)
    return z[:count]


def sign_diagonal(seed: int, d: int) -> np.ndarray:
    """D: int8 [d] of +-1."""
    w0, _, _, _ = _blocks(seed, STREAM_SIGNS, d)
    return np.where((w0 >> np.uint64(31)) & np.uint64(1), -1, 1).astype(np.int8)


def rotation_draws(d: int, seed: int, dense: bool = False, m: int | None = None) -> dict:
    """All draws of a seeded handle, in the layout `build_rotation` takes:
    signs int8 [d], gauss_s float32 [m, d] (the float64 draws rounded to
    float32, the type in which a handle receives its QJL Gaussians),
    gauss_pi float64 [d, d] or None."""
    m = d if m is None else m
    return {
        "signs": sign_diagonal(seed, d),
        "gauss_s": gaussians(seed, STREAM_S, m * d).reshape(m, d).astype(np.float32),
        "gauss_pi": gaussians(seed, STREAM_DENSE, d * d).reshape(d, d) if dense else None,
    }
