"""The allocation-free pointwise entry point (for callers that cannot call cudaMalloc:
plugins inside a runtime that owns the device memory pool, or request paths where an
allocation is not allowed) must give the same result as the handle-based entry point.

This file is collected last on purpose, and its checks hold both in a fresh process and
after every other test has run in the same process."""
import numpy as np
import pytest
import torch

from target_attention_b200 import binding as B
from target_attention_b200.device import PointwiseModel, to_device
from workloads import make_pointwise

pytestmark = pytest.mark.gpu
dev = "cuda"


def _via_handle(wl):
    m = PointwiseModel(wl)
    x = m.inputs(wl)
    out = torch.full((x["B"], 128), float("nan"), device=dev)
    B.check(m.forward(x, out), "stca_pointwise_forward")
    assert B.stca_sync_status(m.handle) == B.OK
    m.close()
    return out.cpu().numpy()


def _via_noalloc(wl, table, n_tok=None, expect_err=0):
    ids, lengths, q = (to_device(wl[k], dev) for k in ("ids", "lengths", "q"))
    out = torch.full((len(wl["lengths"]), 128), float("nan"), device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    n_tok = int(wl["lengths"].sum()) if n_tok is None else n_tok
    B.check(B.stca_pointwise_forward_noalloc(ids, lengths, q, table, table.shape[0], len(wl["lengths"]),
                                             n_tok, out, err), "stca_pointwise_forward_noalloc")
    torch.cuda.synchronize()
    assert err.item() == expect_err
    return out.cpu().numpy()


def _close(got, ref):
    scale = np.maximum(np.abs(ref).max(axis=1, keepdims=True), 1e-6)
    return (np.abs(got - ref) / scale).max() <= 1e-4


def test_noalloc_matches_handle_entry_on_two_calls_in_a_row():
    # two different batches back to back: the shared scratch keeps the first call's
    # contents, which must not leak into the second
    wl1 = make_pointwise(users=300, L=6000, L_lo=1, n_items=100_000, seed=77)
    wl2 = make_pointwise(users=57, L=9000, L_lo=1000, n_items=100_000, seed=78)
    table = to_device(wl1["table"], dev)
    for wl in (wl1, wl2):
        wl = dict(wl, table=wl1["table"])
        ref = _via_handle(wl)
        got = _via_noalloc(wl, table)
        assert _close(got, ref)


def test_noalloc_reports_a_bad_id_and_the_next_call_starts_clean():
    # the shared error word must not carry one call's error into the next call
    wl = make_pointwise(users=40, L=3000, L_lo=100, n_items=50_000, seed=79)
    table = to_device(wl["table"], dev)
    bad = dict(wl, ids=wl["ids"].copy())
    bad["ids"][17] = 50_000  # one past the last row
    _via_noalloc(bad, table, expect_err=B.ERR_ID_OUT_OF_RANGE)
    ref = _via_handle(wl)
    got = _via_noalloc(wl, table)
    assert _close(got, ref)


def test_noalloc_cuts_lengths_at_n_tok():
    # lengths that add up to more than n_tok are reported, and the histories are cut at
    # n_tok: the ids past n_tok (valid rows here, inside the buffer) are never read, so
    # the result equals that of the last sample's history ending at n_tok
    wl = make_pointwise(users=33, L=2500, L_lo=500, n_items=50_000, seed=80)
    table = to_device(wl["table"], dev)
    n_tok = int(wl["lengths"].sum())
    extra = 64
    over = dict(wl, lengths=wl["lengths"].copy(),
                ids=np.concatenate([wl["ids"], np.arange(extra, dtype=np.int32) + 123]))
    over["lengths"][-1] += extra
    ref = _via_handle(wl)
    got = _via_noalloc(over, table, n_tok=n_tok, expect_err=B.ERR_BAD_LENGTHS)
    assert _close(got, ref)


def test_noalloc_rejects_batches_above_its_limit():
    x = torch.zeros(1, dtype=torch.int32, device=dev)
    rc = B.stca_pointwise_forward_noalloc(x, x, x, x, 1, B.NOALLOC_MAX_USERS + 1, 0, x)
    assert rc == B.ERR_CAPACITY
