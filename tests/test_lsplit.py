"""Sequence-parallel (L-split) forward, host side: history slicing and the per-layer
exchange loop, on CPU with world-size-2 gloo process groups.  The merge across ranks is
checked against the oracle's unsplit attention (the WeChat TA article §1.1: attention over
disjoint key slices merges exactly)."""
import math
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import stca_ref as R
from target_attention_b200.lsplit import all_gather_fn, run_phases, slice_bounds, slice_histories


def test_slices_cover_each_history_in_rank_order():
    rng = np.random.default_rng(5)
    lengths = np.array([0, 1, 2, 3, 7, 100, 1001], np.int32)
    n = int(lengths.sum())
    ids = rng.integers(0, 1000, n).astype(np.int32)
    dt = rng.integers(0, 1 << 16, n).astype(np.int32)
    off = np.concatenate([[0], np.cumsum(lengths)])
    for ranks in (1, 2, 3, 8):
        parts = [slice_histories(lengths, ids, dt, ranks, r) for r in range(ranks)]
        assert sum(p[0] for p in parts).tolist() == lengths.tolist()
        for u in range(len(lengths)):
            got_ids, got_dt = [], []
            for (lens, pi, pd) in parts:
                o = np.concatenate([[0], np.cumsum(lens)])
                got_ids.append(pi[o[u]:o[u + 1]])
                got_dt.append(pd[o[u]:o[u + 1]])
            np.testing.assert_array_equal(np.concatenate(got_ids), ids[off[u]:off[u + 1]])
            np.testing.assert_array_equal(np.concatenate(got_dt), dt[off[u]:off[u + 1]])
        # slice sizes differ by at most one token per user
        sizes = np.stack([p[0] for p in parts])
        assert (sizes.max(0) - sizes.min(0) <= 1).all()
    lo, hi = slice_bounds([5], 3, 2)
    assert (lo[0], hi[0]) == (3, 5)
    lens, ids2, dt2 = slice_histories(lengths, ids, None, 2, 1)
    assert dt2 is None and len(ids2) == lens.sum()


class _OracleEngine:
    """A rank's side of the exchange loop with the oracle's slice states: per layer, its
    slice of the keys of every (target, head), states as (acc, (max, sum)) tensors."""

    def __init__(self, q, K, V, score, ranks, rank):
        self.q, self.K, self.V, self.score = q, K, V, score
        self.ranks, self.rank = ranks, rank
        self.out = []

    def begin(self):
        self.out = []

    def partial(self, i):
        q, K, V = self.q[i], self.K[i], self.V[i]          # [T, H, dh], [L, H, dh], [L, H, dh]
        T, H, dh = q.shape
        lo, hi = slice_bounds([K.shape[0]], self.ranks, self.rank)
        acc = torch.zeros((T, H, dh), dtype=torch.float64)
        ml = torch.zeros((T, H, 2), dtype=torch.float64)
        for t in range(T):
            for h in range(H):
                m, l, a = R.attention_partial(q[t, h], K[lo[0]:hi[0], h], V[lo[0]:hi[0], h], self.score,
                                              1 / math.sqrt(dh))
                acc[t, h] = torch.from_numpy(np.asarray(a, np.float64))
                ml[t, h] = torch.tensor([m if m is not None else 0.0, l if l is not None else 0.0])
        return acc, ml

    def merge(self, i, all_acc, all_ml):
        T, H, dh = all_acc.shape[1:]
        o = np.zeros((T, H, dh))
        for t in range(T):
            for h in range(H):
                parts = [(float(all_ml[r, t, h, 0]), float(all_ml[r, t, h, 1]), all_acc[r, t, h].numpy())
                         for r in range(all_acc.shape[0])]
                o[t, h] = R.merge_partials(parts, self.score)
        self.out.append(o)

    def result(self):
        return self.out


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, score, q, K, V, results):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        eng = _OracleEngine(q, K, V, score, world, rank)
        outs = run_phases(eng, len(q), all_gather_fn())
        results[rank] = [o.tolist() for o in outs]
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("score", ["softmax", "relu"])
def test_gloo_two_ranks_merge_equals_unsplit_attention(score):
    rng = np.random.default_rng(11 if score == "softmax" else 12)
    layers, T, H, dh, L = 2, 3, 2, 4, 9
    q = [rng.normal(size=(T, H, dh)) for _ in range(layers)]
    K = [rng.normal(size=(L, H, dh)) for _ in range(layers)]
    V = [rng.normal(size=(L, H, dh)) for _ in range(layers)]
    world = 2
    with mp.Manager() as man:
        results = man.dict()
        mp.spawn(_rank_main, args=(world, _free_port(), score, q, K, V, results), nprocs=world, join=True)
        got = [np.array(results[r]) for r in range(world)]
    np.testing.assert_array_equal(got[0], got[1])        # every rank merged the same states
    want = np.array([[[R.head_attention(q[i][t, h], K[i][:, h], V[i][:, h], score, 1 / math.sqrt(dh))
                       for h in range(H)] for t in range(T)] for i in range(layers)])
    np.testing.assert_allclose(got[0], want, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- bench's rank logic


def _bench_rank_main(rank, world, port, results):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        from workloads import make_stca
        wl = make_stca(2, users=3, data_seed=bench.rank_data_seed(2, rank))
        n_tok = int(wl["lengths"].sum())
        results[rank] = dict(
            n_tok=n_tok, ids_head=wl["ids"][:16].tolist(),
            total=bench.reduce_over_ranks(n_tok, world, "sum", device="cpu"),
            slowest=bench.reduce_over_ranks(10.0 + rank, world, "max", device="cpu"))
    finally:
        dist.destroy_process_group()


def test_gloo_two_ranks_bench_shards_users_and_reduces():
    """bench.py at N > 1: each rank draws its own users (different ids and lengths), the
    step time is the max over ranks and the work the sum over ranks."""
    world = 2
    with mp.Manager() as man:
        results = man.dict()
        mp.spawn(_bench_rank_main, args=(world, _free_port(), results), nprocs=world, join=True)
        r = [dict(results[i]) for i in range(world)]
    assert r[0]["ids_head"] != r[1]["ids_head"]
    assert r[0]["total"] == r[1]["total"] == r[0]["n_tok"] + r[1]["n_tok"]
    assert r[0]["slowest"] == r[1]["slowest"] == 11.0
