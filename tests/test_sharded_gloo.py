"""The sequence-sharded decode and the database-sharded search across ranks,
on CPU with two gloo ranks: each rank computes its shard's result with the
oracle (partial softmax records; top-k lists), the package's plumbing
(vector_quantization_b200.sharded: shard_range, gather_rows) moves them between
ranks, and the oracle's merge must reproduce the single-rank oracle result on
every rank.  The library's own partial, merge and list-merge kernels are
checked against the unsharded calls on one GPU (tests/test_gpu_sharded.py)."""
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
D = 128


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _decode_case():
    import synth
    from helpers import oracle_records, oracle_rotation
    B, Hkv, G, T = 2, 2, 4, 203
    rk, _ = oracle_rotation(D, 2, 61, rope=10000.0)
    rv, _ = oracle_rotation(D, 2, 62)
    k = synth.heavy_tailed((B, Hkv, T, D), 63)
    v = synth.heavy_tailed((B, Hkv, T, D), 64)
    q = synth.heavy_tailed((B, Hkv * G, D), 65)

    def pack(rot, x, pos):
        c, s, n, _ = oracle_records(rot, x.reshape(-1, D), None if pos is None else np.tile(pos, B * Hkv))
        return tuple(a.reshape(B, Hkv, T, -1) for a in (c, s, n))
    return rk, rv, q, [T - 1] * B, pack(rk, k, np.arange(T)), pack(rv, v, None), T


def _rank_main(rank, world, port, out):
    import datetime
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from oracle import attention as at
    from oracle import search as osearch
    from vector_quantization_b200 import sharded
    import synth
    from helpers import oracle_records, oracle_rotation
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        # ---- sequence-sharded decode
        rk, rv, q, qpos, kc, vc, T = _decode_case()
        s, e = sharded.shard_range(T, rank, world)
        part = at.decode_partials(rk, rv, q, qpos, tuple(a[:, :, s:e] for a in kc),
                                  tuple(a[:, :, s:e] for a in vc), 1 / np.sqrt(D))
        parts = sharded.gather_rows(torch.from_numpy(part), None).numpy()
        dec = at.merge_partials(rv, parts)
        # ---- database-sharded search
        d, N, nq, k = 128, 900, 5, 10
        rot, _ = oracle_rotation(d, 1, 66, kind="dense")
        U = synth.haar_basis(d, 67)
        db = synth.anisotropic(N, d, 68, basis=U)
        qs = synth.anisotropic(nq, d, 69, basis=U)
        s2, e2 = sharded.shard_range(N, rank, world)
        c, sg, n, _ = oracle_records(rot, db[s2:e2])
        sc = osearch.search_scores(rot, qs, c, sg, n)
        ls, li = osearch.topk_desc(sc, k)
        all_s = sharded.gather_rows(torch.from_numpy(ls), None).numpy()
        all_i = sharded.gather_rows(torch.from_numpy(li + s2), None).numpy()
        # merge of the lists: descending score, ties to the lower global id
        cand_s = all_s.transpose(1, 0, 2).reshape(nq, -1)
        cand_i = all_i.transpose(1, 0, 2).reshape(nq, -1)
        order = np.lexsort((cand_i, -cand_s), axis=1)[:, :k]
        merged = np.take_along_axis(cand_i, order, axis=1)
        dist.barrier()
        out.put((rank, dec, merged))
    finally:
        dist.destroy_process_group()


def test_shard_range_covers_in_order_with_tile_boundaries():
    from vector_quantization_b200.sharded import shard_range
    for n in (0, 1, 15, 16, 17, 203, 1 << 20):
        for world in (1, 2, 3, 8):
            spans = [shard_range(n, r, world) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == n
            for (a, b), (c, d) in zip(spans, spans[1:]):
                assert b == c and a <= b
            for a, b in spans[:-1]:
                assert a % 16 == 0 and b % 16 == 0 or b == n
            sizes = [b - a for a, b in spans if b < n]
            assert not sizes or max(sizes) - min(sizes) <= 16
    with pytest.raises(ValueError):
        shard_range(10, 2, 2)


def test_sharded_decode_and_search_gloo_two_ranks():
    from oracle import attention as at
    from oracle import search as osearch
    import synth
    from helpers import oracle_records, oracle_rotation
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    res = [out.get(timeout=240) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    rk, rv, q, qpos, kc, vc, T = _decode_case()
    ref = at.decode_attention(rk, rv, q, qpos, kc, vc, 1 / np.sqrt(D))
    d, N, nq, k = 128, 900, 5, 10
    rot, _ = oracle_rotation(d, 1, 66, kind="dense")
    U = synth.haar_basis(d, 67)
    c, sg, n, _ = oracle_records(rot, synth.anisotropic(N, d, 68, basis=U))
    _, ref_ids = osearch.topk_desc(osearch.search_scores(rot, synth.anisotropic(nq, d, 69, basis=U), c, sg, n), k)
    for rank, dec, merged in res:
        np.testing.assert_allclose(dec, ref, rtol=1e-10, atol=1e-12, err_msg=f"rank {rank}")
        np.testing.assert_array_equal(merged, ref_ids, err_msg=f"rank {rank}")
