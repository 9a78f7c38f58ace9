"""Cluster-sharded selection over several GPUs (one process per GPU).

Every rank holds the same index (appends, seals and refits are
deterministic, so replicas stay identical) and, for each query, builds the
same candidate list.  Rank r rescores only its share of the list (a
contiguous range of 128-slot tiles, `AttentionIndex.route_refine_shard`),
so the gather traffic of one request is split across the GPUs.  The
partial top-k results are exchanged with one all-gather (NCCL over NVLink)
and merged by the library's merge kernel: the result equals the
single-GPU `route_refine` exactly.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def exchange_and_merge(ids: torch.Tensor, scores: torch.Tensor, k: int, merge, group=None):
    """All-gather the [T, k] partial results of every rank (rank order) and
    merge them: `merge(all_ids [P, T, k], all_scores [P, T, k], k)`."""
    world = dist.get_world_size(group)
    all_ids = torch.empty((world,) + tuple(ids.shape), dtype=ids.dtype, device=ids.device)
    all_sc = torch.empty((world,) + tuple(scores.shape), dtype=scores.dtype, device=scores.device)
    if dist.get_backend(group) == "nccl":
        dist.all_gather_into_tensor(all_ids, ids.contiguous(), group=group)
        dist.all_gather_into_tensor(all_sc, scores.contiguous(), group=group)
    else:  # gloo has only the list form
        dist.all_gather(list(all_ids.unbind(0)), ids.contiguous(), group=group)
        dist.all_gather(list(all_sc.unbind(0)), scores.contiguous(), group=group)
    return merge(all_ids, all_sc, k)


def sharded_route_refine(index, q, w, pos0: int, k: int, C_budget: int, group=None):
    """Route + refine of one chunk with the rescore split over the ranks of
    `group`; every rank returns the full [T, k] result."""
    from . import merge_topk
    rank, world = dist.get_rank(group), dist.get_world_size(group)
    ids, sc = index.route_refine_shard(q, w, pos0, k, C_budget, rank, world)
    return exchange_and_merge(ids, sc, k, lambda a, b, kk: merge_topk(a, b, kk), group=group)
