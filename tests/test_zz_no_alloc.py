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


def _via_noalloc(wl, table):
    ids, lengths, q = (to_device(wl[k], dev) for k in ("ids", "lengths", "q"))
    out = torch.full((len(wl["lengths"]), 128), float("nan"), device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    B.check(B.stca_pointwise_forward_noalloc(ids, lengths, q, table, table.shape[0], len(wl["lengths"]),
                                             int(wl["lengths"].sum()), out, err), "stca_pointwise_forward_noalloc")
    torch.cuda.synchronize()
    assert err.item() == 0
    return out.cpu().numpy()


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
        scale = np.maximum(np.abs(ref).max(axis=1, keepdims=True), 1e-6)
        assert (np.abs(got - ref) / scale).max() <= 1e-4


def test_noalloc_rejects_batches_above_its_limit():
    x = torch.zeros(1, dtype=torch.int32, device=dev)
    rc = B.stca_pointwise_forward_noalloc(x, x, x, x, 1, B.NOALLOC_MAX_USERS + 1, 0, x)
    assert rc == B.ERR_CAPACITY
