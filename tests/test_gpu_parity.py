"""End-to-end parity of the three forward entry points against the fp64 oracle, on the
same seeded inputs, through the C ABI.  Tolerances (row-normwise max relative error):
2e-2 for bf16 storage with fp32 accumulation, 1e-4 for the fp32 configuration."""
import numpy as np
import pytest
import torch

from oracle import stca_ref as R
from target_attention_b200 import binding as B
from target_attention_b200.device import HyformerModel, PointwiseModel, StcaModel
from workloads import make_hyformer, make_pointwise, make_stca

pytestmark = pytest.mark.gpu
dev = "cuda"
TOL_BF16, TOL_FP32 = 2e-2, 1e-4


def _run_stca(wl, with_o=True, model=None):
    m = model or StcaModel(wl)
    x = m.inputs(wl)
    T, d, M = x["t_tot"], wl["cfg"]["d"], wl["cfg"]["M"]
    z = torch.full((max(T, 1), d), float("nan"), device=dev)
    o = torch.full((M, max(T, 1), d), float("nan"), device=dev) if with_o else None
    B.check(m.forward(x, z, o), "stca_forward")
    assert B.stca_sync_status(m.handle) == B.OK
    res = (z.cpu().numpy()[:T], None if o is None else o.cpu().numpy()[:, :T])
    if model is None:
        m.close()
    return res


def _check_stca(wl, tol, users=None):
    z, o = _run_stca(wl)
    zr, orr = R.stca_forward(wl, users=users)
    if users is not None:
        toff = R.exclusive_offsets(wl["targets_per_user"])
        rows = np.concatenate([np.arange(toff[u], toff[u + 1]) for u in users])
        z, o = z[rows], o[:, rows]
    for i in range(wl["cfg"]["M"]):
        e = R.row_rel_err(o[i], orr[i])
        print(f"parity o^({i + 1}) row-relative error {e:.3e}")
        assert e <= tol, f"o^({i + 1}) err {e}"
    e = R.row_rel_err(z, zr)
    print(f"parity z row-relative error {e:.3e}")
    assert e <= tol, f"z err {e}"
    return z


def test_config1_fp32_full():
    _check_stca(make_stca(1), TOL_FP32)


def test_config2_bf16_small():
    _check_stca(make_stca(2, users=6, n_items=20_000), TOL_BF16)


def test_config3_bf16_small_time_feature():
    _check_stca(make_stca(3, users=3, L=600, n_items=50_000), TOL_BF16)


def test_config3_relu_scores():
    _check_stca(make_stca(3, users=2, L=300, n_items=10_000, M=2, score="relu"), TOL_BF16)


def test_config2_relu_scores():
    """ReLU scores on the d = 256 shape (Beta-ragged ~1.4K histories, M = 2): unnormalised,
    so the queries' rounding is not cancelled by a softmax denominator."""
    _check_stca(make_stca(2, users=6, n_items=20_000, score="relu"), TOL_BF16)


def test_ragged_edge_cases():
    """Empty histories, a single-token history, users without targets, ragged tails."""
    lengths = np.array([0, 1, 129, 0, 257, 40], np.int32)
    wl = make_stca(2, lengths=lengths, n_items=3000)
    wl["targets_per_user"] = np.array([3, 2, 0, 1, 5, 0], np.int32)
    wl["x_t"] = wl["x_t"][:11]
    _check_stca(wl, TOL_BF16)


def test_fp32_ragged_edge_cases():
    lengths = np.array([0, 3, 70], np.int32)
    wl = make_stca(1, lengths=lengths)
    wl["targets_per_user"] = np.array([2, 0, 3], np.int32)
    wl["x_t"] = wl["x_t"][:5]
    _check_stca(wl, TOL_FP32)


def test_rlb_batched_equals_single_target_runs():
    """The m targets of a user, run together, give bit-for-bit the same z as m runs with
    one target each: the per-user K/V is shared, never mixed between targets."""
    wl = make_stca(3, users=1, L=500, n_items=20_000, m=5)
    z_all, _ = _run_stca(wl, with_o=False)
    m = StcaModel(wl)
    for k in range(5):
        one = dict(wl, x_t=wl["x_t"][k:k + 1], targets_per_user=np.array([1], np.int32))
        z1, _ = _run_stca(one, with_o=False, model=m)
        np.testing.assert_array_equal(z1[0], z_all[k])
    m.close()


def test_bad_ids_reported_not_faulting():
    wl = make_stca(2, users=2, L=50, n_items=1000)
    wl["ids"] = wl["ids"].copy()
    wl["ids"][7] = 1000
    m = StcaModel(wl)
    x = m.inputs(wl)
    z = torch.empty((x["t_tot"], 256), device=dev)
    B.check(m.forward(x, z))
    assert B.stca_sync_status(m.handle) == B.ERR_ID_OUT_OF_RANGE
    assert B.stca_sync_status(m.handle) == B.OK          # read-and-clear
    m.close()


def test_capacity_and_argument_errors():
    wl = make_stca(2, users=2, L=50, n_items=1000)
    m = StcaModel(wl)
    x = m.inputs(wl)
    z = torch.empty((x["t_tot"], 256), device=dev)
    assert B.stca_forward(m.handle, x["ids"], x["lengths"], None, x["x_t"], x["targets_per_user"], 3, x["n_tok"],
                          x["t_tot"], m.weights, z) == B.ERR_CAPACITY
    assert B.stca_forward(m.handle, None, x["lengths"], None, x["x_t"], x["targets_per_user"], 2, x["n_tok"],
                          x["t_tot"], m.weights, z) == B.ERR_INVALID_ARG
    # lengths that do not add up to n_tok are detected on the device
    B.check(B.stca_forward(m.handle, x["ids"], x["lengths"], None, x["x_t"], x["targets_per_user"], 2,
                           x["n_tok"] - 1, x["t_tot"], m.weights, z))
    assert B.stca_sync_status(m.handle) == B.ERR_BAD_LENGTHS
    m.close()


def test_host_buffer_entry_matches_device_entry():
    wl = make_stca(3, users=2, L=300, n_items=10_000)
    m = StcaModel(wl)
    x = m.inputs(wl)
    z_dev = torch.empty((x["t_tot"], 512), device=dev)
    B.check(m.forward(x, z_dev))
    xh = {k: (v.cpu().pin_memory() if torch.is_tensor(v) else v) for k, v in x.items()}
    z_host = torch.empty((x["t_tot"], 512), pin_memory=True)
    B.check(m.forward_host(xh, z_host))
    torch.cuda.synchronize()
    np.testing.assert_array_equal(z_host.numpy(), z_dev.cpu().numpy())
    m.close()


def test_host_buffer_entry_back_to_back_calls():
    """Host-buffer calls with different inputs, enqueued back to back with no synchronisation
    between them (the inputs alternate between two staging slots while the previous forward
    runs): each result equals the device entry's for the same inputs."""
    wl = make_stca(3, users=3, L=400, n_items=10_000)
    m = StcaModel(wl)
    inputs = [m.inputs(make_stca(3, users=3, L=400, n_items=10_000, data_seed=100 + i)) for i in range(5)]
    want = []
    for x in inputs:
        z = torch.empty((x["t_tot"], 512), device=dev)
        B.check(m.forward(x, z))
        want.append(z.cpu().numpy())
    hosts = [{k: (v.cpu().pin_memory() if torch.is_tensor(v) else v) for k, v in x.items()} for x in inputs]
    outs = [torch.full((x["t_tot"], 512), float("nan"), pin_memory=True) for x in inputs]
    torch.cuda.synchronize()
    for xh, zh in zip(hosts, outs):
        B.check(m.forward_host(xh, zh))
    torch.cuda.synchronize()
    assert B.stca_sync_status(m.handle) == B.OK
    for zh, w in zip(outs, want):
        np.testing.assert_array_equal(zh.numpy(), w)
    m.close()


def test_host_buffer_entry_fence_on_caller_stream():
    """Back-to-back host-buffer calls on a side stream, completed by stca_host_fence on that
    stream and a synchronisation of that stream alone (no device-wide synchronise): every
    z read-back has landed, each equal to the device entry's result."""
    wl = make_stca(3, users=2, L=350, n_items=10_000)
    m = StcaModel(wl)
    side = torch.cuda.Stream()
    assert m.host_fence(side) == B.OK  # nothing enqueued yet
    inputs = [m.inputs(make_stca(3, users=2, L=350, n_items=10_000, data_seed=200 + i)) for i in range(4)]
    want = []
    for x in inputs:
        z = torch.empty((x["t_tot"], 512), device=dev)
        B.check(m.forward(x, z))
        want.append(z.cpu().numpy())
    hosts = [{k: (v.cpu().pin_memory() if torch.is_tensor(v) else v) for k, v in x.items()} for x in inputs]
    outs = [torch.full((x["t_tot"], 512), float("nan"), pin_memory=True) for x in inputs]
    torch.cuda.synchronize()
    for xh, zh in zip(hosts, outs):
        B.check(m.forward_host(xh, zh, stream=side))
    B.check(m.host_fence(side))
    side.synchronize()
    for zh, w in zip(outs, want):
        np.testing.assert_array_equal(zh.numpy(), w)
    assert B.stca_sync_status(m.handle) == B.OK
    m.close()


def test_lengths_above_the_totals_are_cut_at_them():
    """History lengths that add up to more than n_tok and target counts that add up to
    more than t_tot are reported (ERR_BAD_LENGTHS) and cut at the declared totals: the
    extra ids and target rows (valid, inside padded buffers here) are never used and no
    z row past t_tot is written, so the result equals the run with consistent counts.
    The handle has room for the extra tokens and targets, so the check stays inside every
    buffer whatever the kernels do."""
    wl = make_stca(2, users=5, n_items=20_000)
    extra_tok, extra_tgt = 48, 3
    m = StcaModel(wl, max_tokens=int(wl["lengths"].sum()) + extra_tok,
                  max_targets=int(wl["targets_per_user"].sum()) + extra_tgt)
    z_ok, _ = _run_stca(wl, with_o=False, model=m)
    over = dict(wl, lengths=wl["lengths"].copy(), targets_per_user=wl["targets_per_user"].copy(),
                ids=np.concatenate([wl["ids"], np.arange(extra_tok, dtype=np.int32) + 5]),
                dt=None if wl["dt"] is None else np.concatenate([wl["dt"], np.zeros(extra_tok, np.int32)]),
                x_t=np.concatenate([wl["x_t"], wl["x_t"][:extra_tgt]]))
    over["lengths"][-1] += extra_tok
    over["targets_per_user"][-1] += extra_tgt
    x = m.inputs(over)
    x["n_tok"], x["t_tot"] = int(wl["lengths"].sum()), int(wl["targets_per_user"].sum())
    T, d = x["t_tot"], wl["cfg"]["d"]
    z = torch.full((T + extra_tgt, d), float("nan"), device=dev)
    B.check(m.forward(x, z), "stca_forward")
    assert B.stca_sync_status(m.handle) == B.ERR_BAD_LENGTHS
    m.close()
    zc = z.cpu().numpy()
    assert np.isnan(zc[T:]).all()
    assert R.row_rel_err(zc[:T], z_ok) <= 1e-6


def test_pointwise_lengths_above_n_tok_are_cut():
    wl = make_pointwise(users=33, L=2500, L_lo=500, n_items=50_000, seed=81)
    ref = _run_pointwise(wl)
    n_tok, extra = int(wl["lengths"].sum()), 64
    over = dict(wl, lengths=wl["lengths"].copy(),
                ids=np.concatenate([wl["ids"], np.arange(extra, dtype=np.int32) + 7]))
    over["lengths"][-1] += extra
    m = PointwiseModel(over, max_tokens=n_tok + extra)
    x = m.inputs(over)
    x["n_tok"] = n_tok
    out = torch.full((x["B"], 128), float("nan"), device=dev)
    B.check(m.forward(x, out))
    assert B.stca_sync_status(m.handle) == B.ERR_BAD_LENGTHS
    m.close()
    assert R.row_rel_err(out.cpu().numpy(), ref) <= 1e-6


# ---------------------------------------------------------------- pointwise ReLU TA


def _run_pointwise(wl):
    m = PointwiseModel(wl)
    x = m.inputs(wl)
    out = torch.full((x["B"], 128), float("nan"), device=dev)
    B.check(m.forward(x, out))
    assert B.stca_sync_status(m.handle) == B.OK
    m.close()
    return out.cpu().numpy()


def test_pointwise_small():
    wl = make_pointwise(users=40, L=3000, L_lo=1, n_items=50_000)
    wl["lengths"] = wl["lengths"].copy()
    got = _run_pointwise(wl)
    ref = R.pointwise_relu_ta(wl)
    print(f"parity pointwise row-relative error {R.row_rel_err(got, ref):.3e}")
    assert R.row_rel_err(got, ref) <= 1e-4


def test_pointwise_empty_rows():
    wl = make_pointwise(users=4, L=10, L_lo=1, n_items=100, lengths=np.array([0, 5, 0, 1], np.int32))
    got = _run_pointwise(wl)
    assert (got[0] == 0).all() and (got[2] == 0).all()
    assert R.row_rel_err(got, R.pointwise_relu_ta(wl)) <= 1e-4


def test_pointwise_ragged_extremes():
    """Ragged extremes in one batch: one sample 20K rows long (cut into several slices),
    runs of empty samples, samples shorter than a ring stage and samples ending exactly on
    a stage boundary."""
    lengths = np.array([0, 1, 0, 0, 127, 128, 129, 20_000, 3, 0, 0, 0, 5000, 0, 256, 1], np.int32)
    wl = make_pointwise(users=len(lengths), L=10, L_lo=1, n_items=30_000, lengths=lengths, seed=17)
    got = _run_pointwise(wl)
    for b in np.flatnonzero(lengths == 0):
        assert (got[b] == 0).all()
    e = R.row_rel_err(got, R.pointwise_relu_ta(wl))
    print(f"parity pointwise (ragged extremes) row-relative error {e:.3e}")
    assert e <= 1e-4


def test_pointwise_all_histories_empty():
    wl = make_pointwise(users=3, L=10, L_lo=1, n_items=100, lengths=np.zeros(3, np.int32))
    m = PointwiseModel(wl, max_tokens=1)
    x = m.inputs(wl)
    out = torch.full((3, 128), float("nan"), device=dev)
    B.check(m.forward(x, out))
    assert B.stca_sync_status(m.handle) == B.OK
    m.close()
    assert (out.cpu().numpy() == 0).all()


# ---------------------------------------------------------------- multi-sequence decode


def test_hyformer_small():
    wl = make_hyformer(users=3, L_feed=700, L_search=130, n_items=20_000)
    m = HyformerModel(wl)
    x = m.inputs(wl)
    out = torch.full((x["B"], 32, 512), float("nan"), device=dev)
    B.check(m.forward(x, out))
    assert B.stca_sync_status(m.handle) == B.OK
    m.close()
    ref = R.hyformer_forward(wl)
    e = R.row_rel_err(out.cpu().numpy(), ref)
    print(f"parity hyformer row-relative error {e:.3e}")
    assert e <= TOL_BF16, e
