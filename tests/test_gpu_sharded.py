"""The library's kernels of the sharded paths on one GPU: shards processed one
after the other stand in for the ranks (no kernel waits on another).

* tq_decode_partials over disjoint token ranges, then
  tq_decode_merge_partials, against tq_decode_attention over all tokens and
  against the oracle; the partial records themselves against the oracle's
  (their invariants: the normalised sums and m + log2 l, since the kernel's
  running maximum may lag the true one).
* tq_search_merge_topk of per-shard top-k lists (ids shifted by the shard's
  first row) against tq_search_topk over the whole database: the scores of a
  row do not depend on the sharding, so the results are identical."""
import numpy as np
import pytest
import torch

import synth
from helpers import assert_close, oracle_records, oracle_rotation
from oracle import attention as at

pytestmark = pytest.mark.gpu
D = 128


def _gpu_rot(bits, seed, rope=0.0, kind="hadamard", d=D):
    from vector_quantization_b200 import tq
    return tq.Rotation(d, bits, synth.rotation_randomness(d, seed, dense=(kind == "dense")), kind,
                       rope_base=rope, rope_max_pos=(1 << 20) + 8)


@pytest.mark.parametrize("cuts,G", [([0, 1000, 2000, 3001], 4), ([0, 0, 17, 500], 8), ([0, 64], 1)])
def test_partials_merge_equals_whole_decode(cuda_device, cuts, G):
    from vector_quantization_b200 import tq
    dev = cuda_device
    B, Hkv, bits = 2, 2, 2
    T = cuts[-1]
    rk_o, _ = oracle_rotation(D, bits, 301, rope=10000.0)
    rv_o, _ = oracle_rotation(D, bits, 302)
    rk, rv = _gpu_rot(bits, 301, 10000.0), _gpu_rot(bits, 302)
    k = synth.heavy_tailed((B, Hkv, T, D), 303)
    v = synth.heavy_tailed((B, Hkv, T, D), 304)
    kc = tuple(a.reshape(B, Hkv, T, -1) for a in oracle_records(rk_o, k.reshape(-1, D), np.tile(np.arange(T), B * Hkv))[:3])
    vc = tuple(a.reshape(B, Hkv, T, -1) for a in oracle_records(rv_o, v.reshape(-1, D))[:3])
    q = torch.from_numpy(synth.heavy_tailed((B, Hkv * G, D), 305)).to(dev)
    qpos = torch.full((B,), T - 1, dtype=torch.int64, device=dev)
    parts, oparts = [], []
    def shard(cache, s, e):
        # the shard's records in arrays of even capacity (the cache stride must be even)
        cap = max(2, (e - s + 1) & ~1)
        out = []
        for a in cache:
            b = np.zeros((B, Hkv, cap) + a.shape[3:], dtype=a.dtype)
            b[:, :, :e - s] = a[:, :, s:e]
            out.append(torch.from_numpy(b).to(dev))
        return tuple(out)

    for s, e in zip(cuts[:-1], cuts[1:]):
        parts.append(tq.decode_partials(rk, rv, q, qpos, shard(kc, s, e), shard(vc, s, e), e - s))
        oparts.append(at.decode_partials(rk_o, rv_o, q.cpu().numpy(), [T - 1] * B, tuple(a[:, :, s:e] for a in kc),
                                         tuple(a[:, :, s:e] for a in vc), 1 / np.sqrt(D)))
    stacked = torch.stack(parts)
    out = tq.decode_merge_partials(rv, stacked, Hkv)
    whole = tq.decode_attention(rk, rv, q, qpos, shard(kc, 0, T), shard(vc, 0, T), T)
    torch.cuda.synchronize()
    ref = at.decode_attention(rk_o, rv_o, q.cpu().numpy(), [T - 1] * B, kc, vc, 1 / np.sqrt(D))
    assert_close(out.cpu().numpy(), ref, what="merged partials vs oracle")
    assert_close(out.cpu().numpy(), whole.cpu().numpy(), what="merged partials vs whole decode")
    # record invariants against the oracle's partials
    for g, o in zip(stacked.cpu().numpy().astype(np.float64), oparts):
        empty = np.isneginf(o[..., 0])
        assert np.all(np.isneginf(g[..., 0][empty])) and np.all(g[..., 1][empty] == 0)
        live = ~empty
        gl, ol = g[live], o[live]   # empty records (sum 0) take no log or division
        np.testing.assert_allclose(gl[:, 0] + np.log2(gl[:, 1]), ol[:, 0] + np.log2(ol[:, 1]), rtol=0, atol=2e-4)
        assert_close(gl[:, 2:] / gl[:, 1:2], ol[:, 2:] / ol[:, 1:2], what="normalised sums")


def test_search_merge_of_shards_equals_whole_search(cuda_device):
    from vector_quantization_b200 import tq
    dev = cuda_device
    d, N, nq, k = 256, 5000, 40, 10
    rot = _gpu_rot(1, 311, kind="dense", d=d)
    o, _ = oracle_rotation(d, 1, 311, kind="dense")
    U = synth.haar_basis(d, 312)
    c, s, n, _ = oracle_records(o, synth.anisotropic(N, d, 313, basis=U))
    qs = torch.from_numpy(synth.anisotropic(nq, d, 314, basis=U)).to(dev)
    whole = tq.search_topk(rot, qs, tuple(torch.from_numpy(a).to(dev) for a in (c, s, n)), k)
    cuts = [0, 1700, 1701, 5000]
    lists = [tq.search_topk(rot, qs, tuple(torch.from_numpy(np.ascontiguousarray(a[a0:a1])).to(dev)
                                           for a in (c, s, n)), k) for a0, a1 in zip(cuts[:-1], cuts[1:])]
    sc, ids = tq.search_merge_topk(torch.stack([l[0] for l in lists]), torch.stack([l[1] for l in lists]), k,
                                   id_offsets=cuts[:-1])
    torch.cuda.synchronize()
    np.testing.assert_array_equal(ids.cpu().numpy(), whole[1].cpu().numpy())
    np.testing.assert_array_equal(sc.cpu().numpy(), whole[0].cpu().numpy())
