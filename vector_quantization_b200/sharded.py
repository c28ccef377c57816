"""Decode and search over data split across the ranks of a process group.

One process per GPU (``torch.distributed``, NCCL on NVLink); every rank holds
a shard of the data and runs the library's kernels on it, and one all-gather
carries the small per-shard results:

* sequence-sharded decode ([TurboESM] §2.E's online softmax, split by token
  range): rank r holds tokens ``shard_range(T, r, world)`` of every sequence's
  packed cache.  Each rank writes one partial record per query head
  (``tq_decode_partials``: max, sum of weights, O_code, O_z; 2 + 2d floats),
  the ranks all-gather them ([world, B, Hq, 2 + 2d], e.g. 8 x 64 x 258 floats
  = 528 KB for a 64-head long-context slice on 8 GPUs), and every rank merges
  them (``tq_decode_merge_partials``: log-sum-exp, QJL value correction,
  inverse rotation).  The long-context motivation is the multi-hundred-GB KV
  cache of million-token contexts (technoexpress, "TurboQuant vs OSCAR vs
  EpiCache").
* database-sharded search ([TurboQuant] "Performances en recherche
  vectorielle"): rank r holds rows ``shard_range(N, r, world)``; each rank's
  top-k lists are all-gathered and merged (``tq_search_merge_topk``, ties to
  the lower global id).

Data lands in each rank's own memory before any kernel reads it: the
collectives copy into local buffers, and no kernel takes a peer's memory as
an operand.
"""
from __future__ import annotations


def shard_range(n: int, rank: int, world: int, align: int = 16):
    """[start, end) of rank's share of n items: contiguous, in rank order,
    boundaries on multiples of `align` (a decode tile), sizes differing by at
    most one `align` block; trailing ranks may get nothing when n is small."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("rank must lie in [0, world)")
    blocks = -(-n // align)
    base, extra = divmod(blocks, world)
    start_blk = rank * base + min(rank, extra)
    count = base + (1 if rank < extra else 0)
    start = min(n, start_blk * align)
    end = min(n, (start_blk + count) * align)
    return start, end


def gather_rows(local, group=None):
    """All-gather of one tensor per rank: returns [world, *local.shape] in
    rank order (every rank's `local` must have the same shape and dtype)."""
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    out = torch.empty((world,) + tuple(local.shape), dtype=local.dtype, device=local.device)
    dist.all_gather(list(out.unbind(0)), local.contiguous(), group=group)
    return out


def sharded_decode_attention(rot_k, rot_v, q, q_pos, k_shard, v_shard, T_shard: int, *, seq_lens=None,
                             scale: float | None = None, group=None):
    """One decode step of attention over a context whose tokens are split
    across the ranks of `group`: q [B, Hq, d] and q_pos [B] are the same on
    every rank; k_shard/v_shard are this rank's packed caches
    [B, Hkv, cap, ...] holding T_shard tokens (or seq_lens[b] for sequence
    b).  Returns out [B, Hq, d] float32 on every rank."""
    from . import tq
    Hkv = k_shard[0].shape[1]
    part = tq.decode_partials(rot_k, rot_v, q, q_pos, k_shard, v_shard, T_shard, seq_lens=seq_lens, scale=scale)
    parts = gather_rows(part, group)
    return tq.decode_merge_partials(rot_v, parts, Hkv)


def sharded_search_topk(rot, queries, db_shard, row_offset: int, k: int, group=None):
    """Top-k inner-product search over a database split by rows across the
    ranks of `group`: queries [nq, d] are the same on every rank; db_shard is
    this rank's packed rows (codes, signs, norms), the first of which is
    global row `row_offset`.  Returns (scores [nq, k], global ids [nq, k]) on
    every rank."""
    import torch
    from . import tq
    scores, ids = tq.search_topk(rot, queries, db_shard, k)
    offs = gather_rows(torch.tensor([int(row_offset)], dtype=torch.int64, device=queries.device), group).view(-1)
    return tq.search_merge_topk(gather_rows(scores, group), gather_rows(ids, group), k, id_offsets=offs)
