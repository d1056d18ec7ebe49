"""Weights converted once (stca_pin_weights): the same results as converting on every
call, and a changed weight struct is noticed."""
import numpy as np
import pytest
import torch

from oracle import stca_ref as R
from target_attention_b200 import binding as B
from target_attention_b200.device import HyformerModel, StcaModel
from workloads import make_hyformer, make_stca

pytestmark = pytest.mark.gpu
dev = "cuda"


def _z(m, x, weights=None):
    z = torch.full((x["t_tot"], m.cfg["d"]), float("nan"), device=dev)
    w = weights or m.weights
    B.check(B.stca_forward(m.handle, x["ids"], x["lengths"], x["dt"], x["x_t"], x["targets_per_user"], x["B"],
                           x["n_tok"], x["t_tot"], w, z, None, None))
    assert B.stca_sync_status(m.handle) == B.OK
    return z.cpu().numpy()


def test_stca_pinned_equals_per_call_conversion():
    wl = make_stca(3, users=3, L=700, n_items=2_000)
    m = StcaModel(wl)
    x = m.inputs(wl)
    z0 = _z(m, x)
    m.pin()
    z1 = _z(m, x)
    np.testing.assert_array_equal(z0, z1)
    # a different struct with the same pointers converts again, with the same result
    other = B.StcaWeights.from_buffer_copy(m.weights)
    np.testing.assert_array_equal(_z(m, x, other), z0)
    # a changed struct (another W_O for layer 0) is noticed, not served from the pin
    wo2 = (torch.randn(512, 512, device=dev) * 0.05).to(torch.bfloat16)
    m.keep.append(wo2)
    saved = m.weights.WO[0]
    m.weights.WO[0] = wo2.data_ptr()
    z_changed = _z(m, x)
    B.stca_unpin_weights(m.handle)
    z_ref = _z(m, x)
    np.testing.assert_array_equal(z_changed, z_ref)
    assert not np.array_equal(z_changed, z0)
    m.weights.WO[0] = saved
    m.close()


def test_hyformer_pinned_matches_oracle():
    wl = make_hyformer(users=3, L_feed=700, L_search=130, n_items=300)
    m = HyformerModel(wl)
    x = m.inputs(wl)
    outs = []
    for pin in (False, True):
        if pin:
            m.pin()
        out = torch.full((x["B"], 32, 512), float("nan"), device=dev)
        B.check(m.forward(x, out))
        assert B.stca_sync_status(m.handle) == B.OK
        outs.append(out.cpu().numpy().reshape(-1, 512))
    m.close()
    ref = R.hyformer_forward(wl).reshape(-1, 512)
    e_pin, e_call = R.row_rel_err(outs[1], ref), R.row_rel_err(outs[0], ref)
    print(f"hyformer pinned err {e_pin:.2e}, per-call {e_call:.2e}")
    assert e_pin <= 2e-2 and e_call <= 2e-2
    assert R.row_rel_err(outs[1], outs[0]) <= 1e-2
