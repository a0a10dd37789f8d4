"""One long sequence's indexer top-k split over the GPUs of a process group.

The lightning indexer scores every visible compressed entry of a sequence and keeps the k best
([notes] Sec. 2.3, Eq. 16 and the Indexer listing).  At 1M tokens one sequence has 262,144 entries
(17.8 MB of FP4 index keys); this module splits them over the ranks of a torch.distributed group
(one process per GPU): rank g keeps entries [base_g, base_g + count_g) of every sequence, scores
them and returns its own k best (indexer_topk with score_out), the ranks exchange those lists
(all_gather over NCCL: k (score, index) pairs per query, 8 KB at k = 1024), and every rank merges
them (csa_topk_merge).  The union of the shards' k best contains the sequence's k best, so the
result equals the unsharded top-k exactly, ties to the lower index included.

Every step runs in the library's kernels; this module only places the slices and moves the lists.
"""
from __future__ import annotations

import torch

from . import csa_topk_merge, indexer_topk


def shard_bounds(n_entries: int, world: int, rank: int) -> tuple[int, int]:
    """(base, count) of rank's contiguous slice of n_entries entries split over world ranks."""
    per = -(-n_entries // world)
    base = min(rank * per, n_entries)
    return base, max(0, min(per, n_entries - base))


def local_positions(q_pos: torch.Tensor, m: int, base: int) -> torch.Tensor:
    """Positions that make the shard's entries visible exactly as in the whole sequence: the shard
    holds entries base.., so a query at t sees its first N_vis(t) - base of them (none when
    negative).  Integer bookkeeping on the caller's positions."""
    return ((q_pos + 1) // m - base) * m - 1


def indexer_topk_shard(q, w, keys_local, m: int, k: int, q_pos: torch.Tensor, base: int, count: int,
                       workspace=None, stream=None):
    """This rank's part: the k best of its slice (entry indices relative to the slice, -1 padded)
    and their scores."""
    Nq = w.shape[0]
    sc = torch.empty((Nq, k), dtype=torch.float32, device=w.device)
    idx = indexer_topk(q, w, keys_local, m, k, max_nvis=max(count, 1), q_pos=local_positions(q_pos, m, base),
                       n_keys=count, score_out=sc, workspace=workspace, stream=stream)
    return sc, idx


def merge_shards(sc_all: torch.Tensor, idx_all: torch.Tensor, bases: torch.Tensor, k: int, stream=None):
    """The exact top-k of the gathered lists ([world, Nq, k] each; list g offset by bases[g])."""
    return csa_topk_merge(sc_all, idx_all, k, bases=bases, stream=stream)


def indexer_topk_sharded(q, w, keys_local, m: int, k: int, q_pos: torch.Tensor, n_entries: int, group=None,
                         workspace=None, shard_fn=None, merge_fn=None):
    """The top-k of each query over all n_entries of its sequence, with this rank holding the
    keys of its slice (shard_bounds(n_entries, world, rank)) in keys_local.  Collective: every rank
    of `group` calls it with the same queries; every rank returns the same [Nq, k] indices.
    shard_fn / merge_fn default to this library's kernels (indexer_topk_shard, merge_shards)."""
    import torch.distributed as dist
    shard_fn = shard_fn or indexer_topk_shard
    merge_fn = merge_fn or merge_shards
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    base, count = shard_bounds(n_entries, world, rank)
    sc, idx = shard_fn(q, w, keys_local, m, k, q_pos, base, count, workspace=workspace)
    sc_all = [torch.empty_like(sc) for _ in range(world)]
    idx_all = [torch.empty_like(idx) for _ in range(world)]
    dist.all_gather(sc_all, sc, group=group)
    dist.all_gather(idx_all, idx, group=group)
    bases = torch.tensor([shard_bounds(n_entries, world, g)[0] for g in range(world)], dtype=torch.int64,
                         device=sc.device)
    return merge_fn(torch.stack(sc_all), torch.stack(idx_all), bases, k)
