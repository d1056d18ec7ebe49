"""Sequence-parallel (L-split) forward through the library's phases on one GPU.

R ranks are emulated by R handles that run one after another; their per-layer attention
states are stacked in rank order, which is what the all-gather between GPUs delivers
(no rank waits on another inside a kernel).  Every rank's z must be identical, equal the
whole forward up to the order of summation, and match the fp64 oracle."""
import numpy as np
import pytest
import torch

from oracle import stca_ref as R
from target_attention_b200 import binding as B
from target_attention_b200.device import StcaModel
from workloads import make_stca

pytestmark = pytest.mark.gpu
dev = "cuda"
TOL_BF16, TOL_F32 = 2e-2, 1e-4


def _emulate(wl, ranks, dedup=None):
    models = [StcaModel(wl, dedup=dedup) for _ in range(ranks)]
    xs = [m.slice_inputs(wl, ranks, r) for r, m in enumerate(models)]
    T, d = xs[0]["t_tot"], wl["cfg"]["d"]
    zs = [torch.full((T, d), float("nan"), device=dev) for _ in range(ranks)]
    engines = [m.lsplit_engine(x, z) for m, x, z in zip(models, xs, zs)]
    for e in engines:
        e.begin()
    for i in range(wl["cfg"]["M"]):
        states = [e.partial(i) for e in engines]
        all_acc = torch.stack([s[0] for s in states])
        all_ml = torch.stack([s[1] for s in states])
        for e in engines:
            e.merge(i, all_acc, all_ml)
    torch.cuda.synchronize()
    for m in models:
        assert B.stca_sync_status(m.handle) == B.OK
    whole = torch.empty((T, d), device=dev)
    B.check(models[0].forward(models[0].inputs(wl), whole))
    torch.cuda.synchronize()
    got = [z.cpu().numpy() for z in zs]
    for m in models:
        m.close()
    return got, whole.cpu().numpy()


@pytest.mark.parametrize("cfg,kw,ranks,tol", [
    (2, dict(users=5, lengths=[1, 2, 700, 1500, 333]), 3, TOL_BF16),       # some slices empty
    (3, dict(users=3, L=900, n_items=20_000), 2, TOL_BF16),                  # time buckets, 3 layers
    (3, dict(users=2, L=600, n_items=10_000, M=2, score="relu"), 4, TOL_BF16),
    (1, dict(), 2, TOL_F32),                                                 # fp32, SIMT path
])
def test_lsplit_ranks_match_whole_forward_and_oracle(cfg, kw, ranks, tol):
    wl = make_stca(cfg, **kw)
    got, whole = _emulate(wl, ranks)
    for g in got[1:]:
        np.testing.assert_array_equal(g, got[0])           # every rank computes the same z
    assert np.isfinite(got[0]).all()
    err_whole = R.row_rel_err(got[0], whole)
    err_ref = R.row_rel_err(got[0], R.stca_forward(wl)[0])
    print(f"lsplit R={ranks}: vs whole forward {err_whole:.2e}, vs oracle {err_ref:.2e}")
    # the slices see a user's repeated keys in other groups than the whole history does,
    # so the bf16 weights of the P V product round differently: a quarter of the bar
    assert err_whole <= tol / 4
    assert err_ref <= tol


def test_lsplit_one_rank_is_the_whole_forward_up_to_merge():
    wl = make_stca(2, users=4, L=800)
    got, whole = _emulate(wl, 1)
    assert R.row_rel_err(got[0], whole) <= 1e-5


def test_lsplit_phase_order_is_checked():
    wl = make_stca(2, users=2, L=300)
    m = StcaModel(wl)
    x = m.inputs(wl)
    T, d, H = x["t_tot"], wl["cfg"]["d"], wl["cfg"]["H"]
    acc = torch.empty((T, d), device=dev)
    ml = torch.empty((T, H, 2), device=dev)
    z = torch.empty((T, d), device=dev)
    h = m.handle
    assert B.stca_lsplit_partial(h, 0, acc, ml) == B.ERR_INVALID_ARG          # no begin
    B.check(B.stca_lsplit_begin(h, x["ids"], x["lengths"], x["dt"], x["x_t"], x["targets_per_user"], x["B"],
                                x["n_tok"], x["t_tot"], m.weights))
    assert B.stca_lsplit_merge(h, 0, 1, acc[None], ml[None], z) == B.ERR_INVALID_ARG   # no partial yet
    assert B.stca_lsplit_partial(h, 1, acc, ml) == B.ERR_INVALID_ARG          # wrong layer
    assert B.stca_lsplit_partial(h, 0, acc, None) == B.ERR_INVALID_ARG        # softmax needs ml
    B.check(B.stca_lsplit_partial(h, 0, acc, ml))
    assert B.stca_lsplit_partial(h, 0, acc, ml) == B.ERR_INVALID_ARG          # twice
    assert B.stca_lsplit_merge(h, 0, 0, acc[None], ml[None], z) == B.ERR_INVALID_ARG
    assert B.stca_lsplit_merge(h, 0, 33, acc[None], ml[None], z) == B.ERR_INVALID_ARG
    B.check(B.stca_lsplit_merge(h, 0, 1, acc[None], ml[None], None))        # not the last layer
    B.check(B.stca_lsplit_partial(h, 1, acc, ml))
    assert B.stca_lsplit_merge(h, 1, 1, acc[None], ml[None], None) == B.ERR_INVALID_ARG  # last needs z
    B.check(B.stca_lsplit_merge(h, 1, 1, acc[None], ml[None], z))
    assert B.stca_lsplit_partial(h, 0, acc, ml) == B.ERR_INVALID_ARG          # closed
    torch.cuda.synchronize()
    assert B.stca_sync_status(h) == B.OK
    want = torch.empty((T, d), device=dev)
    B.check(m.forward(x, want))
    torch.cuda.synchronize()
    assert R.row_rel_err(z.cpu().numpy(), want.cpu().numpy()) <= 1e-5
    m.close()


def test_lsplit_without_targets_runs_every_phase():
    """Ranks whose request has no targets still make every call (the collectives must match
    across ranks); the phases do no work."""
    wl = make_stca(2, users=2, L=300, m=0)
    m = StcaModel(wl, max_targets=1)
    x = m.slice_inputs(wl, 2, 1)
    z = torch.empty((1, wl["cfg"]["d"]), device=dev)
    e = m.lsplit_engine(x, z)
    e.begin()
    for i in range(wl["cfg"]["M"]):
        acc, ml = e.partial(i)
        assert acc.shape[0] == 0
        e.merge(i, torch.stack([acc, acc]), torch.stack([ml, ml]))
    torch.cuda.synchronize()
    assert B.stca_sync_status(m.handle) == B.OK
    m.close()
