"""W_K / W_V folded into the queries (stca_config.kv_fold): the same forward computed
without any K/V row, checked against the fp64 oracle (bar 2e-2) and against the unfolded
path on the same handle weights, through the C ABI."""
import numpy as np
import pytest
import torch

from oracle import stca_ref as R
from target_attention_b200 import binding as B
from target_attention_b200.device import StcaModel
from workloads import make_stca

pytestmark = pytest.mark.gpu
dev = "cuda"
TOL = 2e-2


def _z(m, x, handle, T, d):
    z = torch.full((max(T, 1), d), float("nan"), device=dev)
    o = torch.full((m.cfg["M"], max(T, 1), d), float("nan"), device=dev)
    B.check(m.forward(x, z, o, handle=handle), "stca_forward")
    assert B.stca_sync_status(handle) == B.OK
    return z.cpu().numpy()[:T], o.cpu().numpy()[:, :T]


@pytest.mark.parametrize("score", ["softmax", "relu"])
@pytest.mark.parametrize("dedup", [0, 2])
def test_fold_matches_oracle_and_unfolded(score, dedup):
    wl = make_stca(2, users=6, n_items=20_000, score=score)
    m = StcaModel(wl, dedup=dedup)
    hf = m.other_handle(kv_fold=1)
    x = m.inputs(wl)
    T, d = x["t_tot"], wl["cfg"]["d"]
    z_fold, o_fold = _z(m, x, hf, T, d)
    z_plain, _ = _z(m, x, m.handle, T, d)
    B.stca_destroy(hf)
    m.close()
    zr, orr = R.stca_forward(wl)
    for i in range(wl["cfg"]["M"]):
        e = R.row_rel_err(o_fold[i], orr[i])
        print(f"fold o^({i + 1}) row-relative error {e:.3e}")
        assert e <= TOL
    e = R.row_rel_err(z_fold, zr)
    e_plain = R.row_rel_err(z_plain, zr)
    print(f"fold z row-relative error {e:.3e} (unfolded path {e_plain:.3e})")
    assert e <= TOL and e_plain <= TOL
    # two results each within the bar of the oracle are within twice the bar of each other
    assert R.row_rel_err(z_fold, z_plain) <= 2 * TOL


def test_fold_edge_cases():
    """Empty histories, one token, users without targets, ragged tails, a user with more
    than 32 (target, head) rows (two query chunks), several L-slices (merge)."""
    lengths = np.array([0, 1, 129, 0, 2600, 40], np.int32)
    wl = make_stca(2, lengths=lengths, n_items=3000, m=9)
    wl["targets_per_user"] = np.array([3, 2, 0, 1, 9, 0], np.int32)
    wl["x_t"] = wl["x_t"][:15]
    m = StcaModel(wl)
    hf = m.other_handle(kv_fold=1)
    x = m.inputs(wl)
    z, o = _z(m, x, hf, 15, 256)
    B.stca_destroy(hf)
    m.close()
    zr, orr = R.stca_forward(wl)
    assert R.row_rel_err(z, zr) <= TOL
    for i in range(wl["cfg"]["M"]):
        assert R.row_rel_err(o[i], orr[i]) <= TOL


def test_fold_rejected_where_it_does_not_apply():
    wl = make_stca(3, users=1, L=50, n_items=1000)
    m = StcaModel(wl)
    with pytest.raises(B.StcaError):
        m.other_handle(kv_fold=1)   # d = 512
    m.close()
    wl = make_stca(2, users=2, L=50, n_items=1000)
    m = StcaModel(wl)
    hf = m.other_handle(kv_fold=1)
    x = m.inputs(wl)
    assert B.stca_lsplit_begin(hf, x["ids"], x["lengths"], x["dt"], x["x_t"], x["targets_per_user"], x["B"],
                               x["n_tok"], x["t_tot"], m.weights) == B.ERR_UNSUPPORTED
    B.stca_destroy(hf)
    m.close()
