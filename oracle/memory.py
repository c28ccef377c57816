"""Byte arithmetic of the packed cache (oracle).

TEST INFRASTRUCTURE ONLY (see the package header).

A packed vector costs bits*d/8 code bytes + m/8 sign bytes + two float32
norms.  [TurboESM] §3 quotes the KV cache of ESM-2 650M (33 layers, 20 heads)
at 1024 tokens going from 330 MB to 47 MB (7.1x) at 3 bits with QJL, and §2.D
an effective 3.125 bits per element.  330 MiB is exactly the float32 K+V
cache of that model (head_dim 64); the tests pin that figure and report this
layout's own ratio next to the quoted one (the three quoted figures are not
mutually consistent; the reading is recorded with the design notes).
"""
from __future__ import annotations


def record_bytes(d: int, bits: int, m: int | None = None, norm_bytes: int = 8) -> int:
    """Bytes of one packed vector: codes + signs + norms."""
    m = d if m is None else m
    return bits * d // 8 + m // 8 + norm_bytes


def cache_bytes(layers: int, heads: int, tokens: int, d: int, bits: int,
                m: int | None = None, kv: int = 2) -> int:
    """Bytes of a packed K+V cache."""
    return layers * heads * tokens * kv * record_bytes(d, bits, m)
