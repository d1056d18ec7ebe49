"""Randomised shapes against the oracle: seeded draws of users, ragged history lengths
(zeros included), ragged target counts (zeros included), score form, distinct-key mode and
a few layer counts, through the device and host-buffer entries and the sequence-parallel
phases.  Each case is small enough for the fp64 oracle to finish in well under a second."""
import numpy as np
import pytest
import torch

from oracle import stca_ref as R
from target_attention_b200 import binding as B
from target_attention_b200.device import StcaModel
from workloads import make_stca

pytestmark = pytest.mark.gpu
dev = "cuda"
TOL_BF16, TOL_FP32 = 2e-2, 1e-4


def _case(seed):
    rng = np.random.default_rng(seed)
    cfg = int(rng.choice([1, 2, 3]))
    users = int(rng.integers(1, 6))
    hi = 600 if cfg != 1 else 300
    lengths = rng.integers(0, hi, users).astype(np.int32)
    lengths[rng.random(users) < 0.2] = 0
    if lengths.sum() == 0:
        lengths[0] = 1
    kw = dict(lengths=lengths, data_seed=seed)
    if cfg != 1:
        kw.update(n_items=int(rng.choice([500, 20_000])), M=int(rng.integers(1, 4)))
        if rng.random() < 0.3:
            kw["score"] = "relu"
    wl = make_stca(cfg, **kw)
    m_max = wl["cfg"]["m"]
    tpu = rng.integers(0, m_max + 1, users).astype(np.int32)
    if tpu.sum() == 0:
        tpu[0] = 1
    wl["targets_per_user"] = tpu
    wl["x_t"] = np.ascontiguousarray(wl["x_t"][: int(tpu.sum())])
    dedup = 0 if cfg == 1 else int(rng.choice([0, 1, 2]))
    return wl, dedup, rng


@pytest.mark.parametrize("seed", range(12))
def test_random_shapes_match_oracle(seed):
    wl, dedup, rng = _case(1000 + seed)
    tol = TOL_FP32 if wl["cfg"]["dtype"] == "fp32" else TOL_BF16
    m = StcaModel(wl, dedup=dedup)
    x = m.inputs(wl)
    T, d = x["t_tot"], wl["cfg"]["d"]
    zr, _ = R.stca_forward(wl)

    z = torch.full((T, d), float("nan"), device=dev)
    B.check(m.forward(x, z))
    torch.cuda.synchronize()
    assert B.stca_sync_status(m.handle) == B.OK
    e = R.row_rel_err(z.cpu().numpy(), zr)
    print(f"seed {seed}: config {wl['cfg']} dedup {dedup}: device entry {e:.2e}")
    assert e <= tol

    # host-buffer entry on the same handle
    xh = {k: (v.cpu().pin_memory() if torch.is_tensor(v) else v) for k, v in x.items()}
    zh = torch.full((T, d), float("nan"), pin_memory=True)
    B.check(m.forward_host(xh, zh))
    torch.cuda.synchronize()
    np.testing.assert_array_equal(zh.numpy(), z.cpu().numpy())

    # sequence-parallel phases over 2 or 3 emulated ranks on the same handle, one after another
    ranks = int(rng.integers(2, 4))
    parts = [m.slice_inputs(wl, ranks, r) for r in range(ranks)]
    models = [m] + [StcaModel(wl, dedup=dedup) for _ in range(ranks - 1)]
    zs = [torch.full((max(T, 1), d), float("nan"), device=dev) for _ in range(ranks)]
    engines = [mm.lsplit_engine(p, zz) for mm, p, zz in zip(models, parts, zs)]
    for eng in engines:
        eng.begin()
    for i in range(wl["cfg"]["M"]):
        st = [eng.partial(i) for eng in engines]
        all_acc = torch.stack([s_[0] for s_ in st])
        all_ml = torch.stack([s_[1] for s_ in st])
        for eng in engines:
            eng.merge(i, all_acc, all_ml)
    torch.cuda.synchronize()
    for mm in models:
        assert B.stca_sync_status(mm.handle) == B.OK
    el = R.row_rel_err(zs[0][:T].cpu().numpy(), zr)
    print(f"seed {seed}: sequence-parallel over {ranks} ranks {el:.2e}")
    assert el <= tol
    for mm in models:
        mm.close()
