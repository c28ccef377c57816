"""Pins of the oracle's partial records and their merge (oracle/attention.py:
decode_partials, merge_partials), the algebra of a sequence-sharded decode.

The merge of the partials of any split of the tokens into disjoint ranges
must equal decode_attention over all of them, whose two-pass softmax is
pinned on its own (tests/test_oracle_attention.py); the ranges include empty
ones, single tokens and an unequal split.  A dropped 2^(m_p - M) factor, a
natural-log/log2 mix-up, a missing QJL term or a wrong normalisation all fail
it."""
import numpy as np
import pytest

import synth
from helpers import oracle_records, oracle_rotation
from oracle import attention as at

D = 128


def _cache(orot, x, pos=None):
    B, H, T, d = x.shape
    if T == 0:
        return (np.zeros((B, H, 0, orot.bits * d // 8), np.uint8), np.zeros((B, H, 0, orot.m // 8), np.uint8),
                np.zeros((B, H, 0, 2), np.float32))
    c, s, n, _ = oracle_records(orot, x.reshape(-1, d), None if pos is None else np.tile(pos, B * H))
    return tuple(a.reshape(B, H, T, -1) for a in (c, s, n))


@pytest.mark.parametrize("cuts", [[0, 300], [0, 1, 300], [0, 0, 150, 300], [0, 37, 38, 200, 300]])
def test_merge_of_partials_equals_decode(cuts):
    B, Hkv, G, T = 2, 2, 2, 300
    rk, _ = oracle_rotation(D, 2, 31, rope=10000.0)
    rv, _ = oracle_rotation(D, 2, 32)
    k = synth.heavy_tailed((B, Hkv, T, D), 33)
    v = synth.heavy_tailed((B, Hkv, T, D), 34)
    q = synth.heavy_tailed((B, Hkv * G, D), 35)
    qpos = [T - 1] * B
    kc, vc = _cache(rk, k, np.arange(T)), _cache(rv, v)
    ref = at.decode_attention(rk, rv, q, qpos, kc, vc, 1 / np.sqrt(D))
    parts = np.stack([at.decode_partials(rk, rv, q, qpos, tuple(a[:, :, s:e] for a in kc),
                                         tuple(a[:, :, s:e] for a in vc), 1 / np.sqrt(D))
                      for s, e in zip(cuts[:-1], cuts[1:])])
    np.testing.assert_allclose(at.merge_partials(rv, parts), ref, rtol=1e-10, atol=1e-12)


def test_empty_partials_merge_to_zero_and_one_token_gives_its_value():
    rk, _ = oracle_rotation(D, 2, 41, rope=10000.0)
    rv, _ = oracle_rotation(D, 2, 42)
    q = synth.heavy_tailed((1, 1, D), 43)
    empty = _cache(rk, np.zeros((1, 1, 0, D)))
    p0 = at.decode_partials(rk, rv, q, [0], empty, empty, 0.1)
    assert np.isneginf(p0[0, 0, 0]) and p0[0, 0, 1] == 0 and not p0[0, 0, 2:].any()
    assert not at.merge_partials(rv, p0[None]).any()
    v = synth.heavy_tailed((1, 1, 1, D), 44)
    kc, vc = _cache(rk, synth.heavy_tailed((1, 1, 1, D), 45), np.arange(1)), _cache(rv, v)
    p1 = at.decode_partials(rk, rv, q, [0], kc, vc, 0.1)
    assert p1[0, 0, 1] == 1.0
    out = at.merge_partials(rv, np.stack([p0, p1]))
    np.testing.assert_allclose(out, at.decode_attention(rk, rv, q, [0], kc, vc, 0.1), rtol=1e-12, atol=1e-12)
