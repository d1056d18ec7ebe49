"""Distinct-row form of the history side (HyFormer page §3.8.1, GPU pooling): the key
(item id, time bucket) fixes X~, K and V of a token, so running the history GEMMs once
per distinct key must reproduce the per-token results bit for bit."""
import numpy as np
import pytest
import torch

from oracle import stca_ref as R
from target_attention_b200 import binding as B
from target_attention_b200.device import HyformerModel, StcaModel
from workloads import make_hyformer, make_stca

pytestmark = pytest.mark.gpu
dev = "cuda"


def _keys(ids, dt):
    b = np.zeros_like(ids, dtype=np.int64) if dt is None else R.dt_bucket(dt).astype(np.int64)
    return ids.astype(np.int64) * 16 + b


@pytest.mark.parametrize("case", ["zipf_dt", "all_same", "all_distinct", "empty"])
def test_dedup_map_is_consistent(case):
    g = np.random.default_rng(3)
    n = {"zipf_dt": 300_000, "all_same": 5000, "all_distinct": 70_000, "empty": 0}[case]
    if case == "zipf_dt":
        ids = np.minimum(g.zipf(1.3, size=n), 10**6).astype(np.int32)
        dt = (np.floor(np.exp2(g.uniform(0, 16, size=n))) - 1).astype(np.int32)
    elif case == "all_same":
        ids, dt = np.full(n, 7, np.int32), None
    else:
        ids, dt = g.permutation(10**6)[:n].astype(np.int32), None
    ws = torch.empty(B.stca_k_dedup_workspace_bytes(max(n, 1)), dtype=torch.uint8, device=dev)
    uidx = torch.full((max(n, 1),), -1, dtype=torch.int32, device=dev)
    utok = torch.full((max(n, 1),), -1, dtype=torch.int32, device=dev)
    count = torch.zeros(1, dtype=torch.int32, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    t_ids = torch.from_numpy(ids).to(dev) if n else None
    t_dt = torch.from_numpy(dt).to(dev) if (n and dt is not None) else None
    B.check(B.stca_k_dedup(t_ids, t_dt, n, ws, uidx, utok, count, err))
    torch.cuda.synchronize()
    assert err.item() == 0
    keys = _keys(ids, dt)
    U = count.item()
    assert U == len(np.unique(keys))
    if n == 0:
        return
    ui, ut = uidx.cpu().numpy(), utok.cpu().numpy()[:U]
    assert ((ui >= 0) & (ui < U)).all()
    assert ((ut >= 0) & (ut < n)).all()
    np.testing.assert_array_equal(keys[ut[ui]], keys)        # each token maps to a row of its key
    assert len(np.unique(keys[ut])) == U                       # distinct rows have distinct keys


def _z(model, x, T, d, handle=None):
    z = torch.full((T, d), float("nan"), device=dev)
    B.check(model.forward(x, z, handle=handle))
    assert B.stca_sync_status(handle or model.handle) == B.OK
    return z.cpu().numpy()


@pytest.mark.parametrize("config, kw", [(2, dict(users=6, n_items=5_000)),
                                        (3, dict(users=3, L=900, n_items=2_000))])
def test_dedup_equals_per_token_bitwise(config, kw):
    wl = make_stca(config, **kw)
    m = StcaModel(wl, dedup=1)
    x = m.inputs(wl)
    T, d = x["t_tot"], wl["cfg"]["d"]
    h0 = m.other_handle(dedup=0)
    z_dedup = _z(m, x, T, d)
    z_plain = _z(m, x, T, d, handle=h0)
    B.stca_destroy(h0)
    m.close()
    np.testing.assert_array_equal(z_dedup, z_plain)


def test_dedup_edge_cases_match_oracle():
    lengths = np.array([0, 1, 300, 0, 5], np.int32)
    wl = make_stca(3, lengths=lengths, n_items=50, m=3)
    wl["ids"] = wl["ids"].copy()
    wl["ids"][1:301] = 11           # one user whose whole history is a single item
    m = StcaModel(wl, dedup=1)
    x = m.inputs(wl)
    z = _z(m, x, x["t_tot"], 512)
    m.close()
    zr, _ = R.stca_forward(wl)
    assert R.row_rel_err(z, zr) <= 2e-2


def test_hyformer_dedup_equals_per_token_bitwise():
    wl = make_hyformer(users=3, L_feed=700, L_search=130, n_items=3_000)
    m = HyformerModel(wl, dedup=1)
    x = m.inputs(wl)
    h0 = m.other_handle(dedup=0)
    outs = []
    for h in (None, h0):
        out = torch.full((x["B"], 32, 512), float("nan"), device=dev)
        B.check(m.forward(x, out, handle=h))
        assert B.stca_sync_status(h or m.handle) == B.OK
        outs.append(out.cpu().numpy())
    B.stca_destroy(h0)
    m.close()
    np.testing.assert_array_equal(outs[0], outs[1])


# ---------------------------------------------------------------- per-user compaction


def _expected_compaction(rows, hoff):
    """Each user's distinct rows in order of first token, with their token counts."""
    out = []
    for u in range(len(hoff) - 1):
        seg = rows[hoff[u]:hoff[u + 1]]
        if len(seg) >= 16384:                      # kept per token
            out.append((seg, np.ones(len(seg), np.int64)))
            continue
        _, first, cnt = np.unique(seg, return_index=True, return_counts=True)
        order = np.argsort(first)
        out.append((seg[first[order]], cnt[order]))
    return out


@pytest.mark.parametrize("case", ["zipf", "edges", "long_users"])
def test_compact_user_rows_is_exact(case):
    g = np.random.default_rng(31)
    if case == "zipf":
        lengths = g.integers(0, 3000, size=40)
        n = int(lengths.sum())
        rows = np.minimum(g.zipf(1.3, size=n) - 1, 5000).astype(np.int32)
    elif case == "edges":
        lengths = np.array([0, 1, 2, 700, 0, 64, 65, 5])
        n = int(lengths.sum())
        rows = g.integers(0, 50, size=n).astype(np.int32)
        rows[3:703] = 17                           # one row for a whole user
    else:
        lengths = np.array([16383, 16384, 20000, 3])  # full table, first per-token user, larger
        n = int(lengths.sum())
        rows = g.permutation(n).astype(np.int32)   # all distinct
        rows[16383 + 16384:16383 + 16384 + 100] = 7
    hoff = R.exclusive_offsets(lengths.astype(np.int32))
    Bu = len(lengths)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a, np.int32)).to(dev)
    out_rows = torch.full((max(n, 1),), -7, dtype=torch.int32, device=dev)
    out_mult = torch.full((max(n, 1),), -7, dtype=torch.int32, device=dev)
    out_len = torch.full((Bu,), -7, dtype=torch.int32, device=dev)
    B.check(B.stca_k_compact_user_rows(t(hoff), Bu, t(rows), out_rows, out_mult, out_len))
    torch.cuda.synchronize()
    got_r, got_m, got_l = out_rows.cpu().numpy(), out_mult.cpu().numpy(), out_len.cpu().numpy()
    for u, (er, em) in enumerate(_expected_compaction(rows, hoff)):
        assert got_l[u] == len(er), u
        np.testing.assert_array_equal(got_r[hoff[u]:hoff[u] + len(er)], er)
        np.testing.assert_array_equal(got_m[hoff[u]:hoff[u] + len(er)], em)


@pytest.mark.parametrize("config, kw", [(2, dict(users=6, n_items=5_000)),
                                        (3, dict(users=3, L=900, n_items=2_000)),
                                        (3, dict(users=3, L=900, n_items=300, score="relu"))])
def test_compacted_attention_matches_per_token(config, kw):
    """Attending once per distinct key of a user, weighted by its token count, is the same
    function as attending per token: equal up to summation order, and within the bf16 bar
    of the oracle."""
    wl = make_stca(config, **kw)
    m = StcaModel(wl, dedup=2)
    x = m.inputs(wl)
    T, d = x["t_tot"], wl["cfg"]["d"]
    h0 = m.other_handle(dedup=0)
    z_c = _z(m, x, T, d)
    z_p = _z(m, x, T, d, handle=h0)
    B.stca_destroy(h0)
    m.close()
    zr, _ = R.stca_forward(wl)
    e_cp, e_or = R.row_rel_err(z_c, z_p), R.row_rel_err(z_c, zr)
    print(f"compacted vs per-token {e_cp:.2e}, vs oracle {e_or:.2e}")
    assert e_cp <= 1e-2 and e_or <= 2e-2


def test_compacted_edge_cases_match_oracle():
    lengths = np.array([0, 1, 300, 0, 5, 16400], np.int32)   # the last user is kept per token
    wl = make_stca(3, lengths=lengths, n_items=50, m=3)
    wl["ids"] = wl["ids"].copy()
    wl["ids"][1:301] = 11
    m = StcaModel(wl, dedup=2)
    x = m.inputs(wl)
    z = _z(m, x, x["t_tot"], 512)
    m.close()
    zr, _ = R.stca_forward(wl)
    assert R.row_rel_err(z, zr) <= 2e-2


def test_hyformer_compacted_matches_oracle():
    wl = make_hyformer(users=3, L_feed=700, L_search=130, n_items=300)
    m = HyformerModel(wl, dedup=2)
    x = m.inputs(wl)
    out = torch.full((x["B"], 32, 512), float("nan"), device=dev)
    B.check(m.forward(x, out))
    assert B.stca_sync_status(m.handle) == B.OK
    m.close()
    ref = R.hyformer_forward(wl)
    assert R.row_rel_err(out.cpu().numpy().reshape(-1, 512), ref.reshape(-1, 512)) <= 2e-2
