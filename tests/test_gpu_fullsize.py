"""Parity at the benchmark's full sizes, in the configuration bench.py times.

Each test builds the same seeded workload bench.py builds (rank 0), converts the weights
once as bench.py does (``pin``), runs one forward on the device, and checks the outputs
of a seeded sample of users against the fp64 oracle computed for those users alone (the
oracle takes a few seconds per user at these lengths).  Every other output is checked for
the properties that hold at any size: finite, and no device-side error."""
import types

import numpy as np
import pytest
import torch

import bench
from oracle import stca_ref as R
from target_attention_b200 import binding as B
from target_attention_b200.device import HyformerModel, PointwiseModel, StcaModel

pytestmark = [pytest.mark.gpu, pytest.mark.slow]
dev = "cuda"
TOL_BF16 = 2e-2


def _bench_workload(workload):
    args = types.SimpleNamespace(workload=workload, users=None, n_items=None, length=None)
    return bench.make_workload(args, data_seed=bench.rank_data_seed(workload, 0))


def _sample(n_users, k, seed):
    rng = np.random.default_rng(seed)
    picks = {0, n_users - 1} | set(rng.choice(n_users, size=k, replace=False).tolist())
    return sorted(picks)


def _target_rows(wl, users):
    toff = R.exclusive_offsets(wl["targets_per_user"])
    return np.concatenate([np.arange(toff[u], toff[u + 1]) for u in users])


@pytest.mark.parametrize("workload", [2, 3])
def test_stca_full_size_sampled_users(workload):
    wl = _bench_workload(workload)
    m = StcaModel(wl, dedup=2)
    m.pin()
    x = m.inputs(wl)
    T, d, M = x["t_tot"], wl["cfg"]["d"], wl["cfg"]["M"]
    z = torch.full((T, d), float("nan"), device=dev)
    o = torch.full((M, T, d), float("nan"), device=dev)
    B.check(m.forward(x, z, o))
    torch.cuda.synchronize()
    assert B.stca_sync_status(m.handle) == B.OK
    z, o = z.cpu().numpy(), o.cpu().numpy()
    m.close()
    assert np.isfinite(z).all() and np.isfinite(o).all()
    users = _sample(len(wl["lengths"]), 2 if workload == 3 else 6, 100 + workload)
    zr, orr = R.stca_forward(wl, users=users)
    rows = _target_rows(wl, users)
    for i in range(M):
        e = R.row_rel_err(o[i][rows], orr[i])
        print(f"config {workload} full size, users {users}: o^({i + 1}) row-relative error {e:.3e}")
        assert e <= TOL_BF16
    e = R.row_rel_err(z[rows], zr)
    print(f"config {workload} full size, users {users}: z row-relative error {e:.3e}")
    assert e <= TOL_BF16


def test_pointwise_full_size_sampled_users():
    wl = _bench_workload(4)
    m = PointwiseModel(wl)
    x = m.inputs(wl)
    out = torch.full((x["B"], wl["cfg"]["d"]), float("nan"), device=dev)
    B.check(m.forward(x, out))
    torch.cuda.synchronize()
    assert B.stca_sync_status(m.handle) == B.OK
    out = out.cpu().numpy()
    m.close()
    assert np.isfinite(out).all()
    users = _sample(x["B"], 14, 104)
    ref = R.pointwise_relu_ta(wl, users=users)
    e = R.row_rel_err(out[users], ref)
    print(f"config 4 full size, {len(users)} users: row-relative error {e:.3e}")
    assert e <= 1e-4


def test_hyformer_full_size_sampled_users():
    wl = _bench_workload(5)
    m = HyformerModel(wl, dedup=2)
    m.pin()
    x = m.inputs(wl)
    out = torch.full((x["B"], 2 * x["n_query"], wl["cfg"]["d"]), float("nan"), device=dev)
    B.check(m.forward(x, out))
    torch.cuda.synchronize()
    assert B.stca_sync_status(m.handle) == B.OK
    out = out.cpu().numpy()
    m.close()
    assert np.isfinite(out).all()
    users = _sample(x["B"], 1, 105)
    ref = R.hyformer_forward(wl, users=users)
    e = R.row_rel_err(out[users].reshape(-1, out.shape[-1]), ref.reshape(-1, ref.shape[-1]))
    print(f"config 5 full size, users {users}: row-relative error {e:.3e}")
    assert e <= TOL_BF16
