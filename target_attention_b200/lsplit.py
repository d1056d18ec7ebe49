"""Sequence-parallel (L-split) STCA forward across ranks.

Attention over a user's history is the exact merge of attention over disjoint slices of
it (WeChat TA article, §1.1: each slice keeps its running max, sum of weights and weighted
sum of V; the slices combine without approximation).  So one very long history can be
split across GPUs: every rank holds slice r of each user's history and all of the user's
targets, computes the history side and the attention state of its slice, and per layer the
ranks exchange one state per (target, head) -- an all-gather -- after which each rank
merges them and computes the (small) target side redundantly.

The phases themselves run in the library (``stca_lsplit_begin / _partial / _merge``);
this module holds the host side: how histories are sliced and the per-layer exchange loop.
"""
from __future__ import annotations

import numpy as np


def slice_bounds(lengths, ranks: int, rank: int):
    """Token range [lo, hi) of user u's slice ``rank`` of ``ranks``: floor(L r / R) ..
    floor(L (r+1) / R), so the slices of a user are contiguous, disjoint, in rank order and
    cover its history (a user shorter than R has empty slices)."""
    L = np.asarray(lengths, dtype=np.int64)
    return (L * rank) // ranks, (L * (rank + 1)) // ranks


def slice_histories(lengths, ids, dt, ranks: int, rank: int):
    """This rank's slice of every user's history: (slice lengths, ids, dt) with the users'
    slices back to back (dt None stays None)."""
    L = np.asarray(lengths, dtype=np.int64)
    off = np.concatenate([[0], np.cumsum(L)])
    lo, hi = slice_bounds(L, ranks, rank)
    take = np.concatenate([np.arange(off[u] + lo[u], off[u] + hi[u]) for u in range(len(L))]) if len(L) else \
        np.zeros(0, np.int64)
    take = take.astype(np.int64)
    ids = np.asarray(ids)[take]
    dt = None if dt is None else np.asarray(dt)[take]
    return (hi - lo).astype(np.int32), ids, dt


def all_gather_fn(group=None):
    """gather(t) -> [R, *t.shape], the ranks' tensors in rank order, over torch.distributed
    (NCCL for CUDA tensors; gloo on CPU)."""
    import torch
    import torch.distributed as dist

    def gather(t):
        t = t.contiguous()
        R = dist.get_world_size(group)
        if t.is_cuda:
            out = torch.empty((R,) + tuple(t.shape), dtype=t.dtype, device=t.device)
            dist.all_gather_into_tensor(out, t, group=group)
            return out
        parts = [torch.empty_like(t) for _ in range(R)]
        dist.all_gather(parts, t, group=group)
        return torch.stack(parts)

    return gather


def run_phases(engine, layers: int, gather):
    """The exchange loop: ``engine.begin()``; per layer ``(acc, ml) = engine.partial(i)``,
    then ``engine.merge(i, gather(acc), gather(ml))``; returns ``engine.result()``.  Every
    rank makes the same calls in the same order, so the collectives match."""
    engine.begin()
    for i in range(layers):
        acc, ml = engine.partial(i)
        engine.merge(i, gather(acc), gather(ml))
    return engine.result()
