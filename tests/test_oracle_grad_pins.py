"""Pins for the fp64 backward oracle (``oracle/stca_grad.py``): each step's backward
against torch.autograd in fp64, closed forms of the attention gradient, the split-L
backward against the unsplit one, and central finite differences of the whole forward
(``oracle/stca_ref.py``) for every gradient tensor.  CPU only."""
import copy
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import stca_grad as G
from oracle import stca_ref as R
from workloads import make_stca

t64 = lambda a: torch.tensor(np.asarray(a, dtype=np.float64), requires_grad=True)


def _rng(seed):
    return np.random.default_rng(seed)


# ---------------------------------------------------------------- steps vs torch.autograd


def test_swiglu_bwd_vs_autograd():
    g = _rng(1)
    x, dy = g.standard_normal((5, 6)), g.standard_normal((5, 6))
    f = {"W1": g.standard_normal((6, 9)), "W3": g.standard_normal((6, 9)), "W2": g.standard_normal((9, 6))}
    tx, tw = t64(x), {k: t64(v) for k, v in f.items()}
    y = (F.silu(tx @ tw["W1"]) * (tx @ tw["W3"])) @ tw["W2"]
    y.backward(torch.from_numpy(dy))
    dx, gw = G.swiglu_bwd(x, f, dy)
    np.testing.assert_allclose(dx, tx.grad.numpy(), rtol=1e-12, atol=1e-12)
    for k in f:
        np.testing.assert_allclose(gw[k], tw[k].grad.numpy(), rtol=1e-12, atol=1e-12)


def test_layer_norm_bwd_vs_autograd():
    g = _rng(2)
    x, dy = g.standard_normal((4, 10)) * 3 + 1, g.standard_normal((4, 10))
    gamma, beta = g.standard_normal(10), g.standard_normal(10)
    tx, tg, tb = t64(x), t64(gamma), t64(beta)
    F.layer_norm(tx, (10,), tg, tb, 1e-5).backward(torch.from_numpy(dy))
    dx, dg, db = G.layer_norm_bwd(x, gamma, beta, 1e-5, dy)
    np.testing.assert_allclose(dx, tx.grad.numpy(), rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(dg, tg.grad.numpy(), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(db, tb.grad.numpy(), rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("L", [1, 2, 8])
def test_softmax_attention_bwd_vs_autograd_sdpa(L):
    """torch's scaled_dot_product_attention (scale 1/sqrt(d_h)) differentiated by autograd."""
    g = _rng(3 + L)
    dh = 8
    q, K, V, do = g.standard_normal(dh), g.standard_normal((L, dh)), g.standard_normal((L, dh)), g.standard_normal(dh)
    tq, tK, tV = t64(q), t64(K), t64(V)
    o = F.scaled_dot_product_attention(tq[None, None, None], tK[None, None], tV[None, None])[0, 0, 0]
    o.backward(torch.from_numpy(do))
    dq, dK, dV = G.head_attention_bwd(q, K, V, "softmax", 1 / math.sqrt(dh), do)
    np.testing.assert_allclose(dq, tq.grad.numpy(), rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(dK, tK.grad.numpy(), rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(dV, tV.grad.numpy(), rtol=1e-11, atol=1e-13)


def test_relu_attention_bwd_vs_autograd():
    g = _rng(7)
    dh, L = 8, 7
    q, K, V, do = g.standard_normal(dh), g.standard_normal((L, dh)), g.standard_normal((L, dh)), g.standard_normal(dh)
    tq, tK, tV = t64(q), t64(K), t64(V)
    o = torch.relu(tK @ tq / math.sqrt(dh)) @ tV
    o.backward(torch.from_numpy(do))
    dq, dK, dV = G.head_attention_bwd(q, K, V, "relu", 1 / math.sqrt(dh), do)
    assert ((K @ q) > 0).any() and ((K @ q) < 0).any()
    np.testing.assert_allclose(dq, tq.grad.numpy(), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(dK, tK.grad.numpy(), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(dV, tV.grad.numpy(), rtol=1e-12, atol=1e-13)


# ---------------------------------------------------------------- closed forms


def test_single_key_and_identical_keys_give_zero_query_gradient():
    """With one key, or with all keys equal, the softmax weights do not depend on q or K:
    dq = 0 and dK = 0 exactly (up to rounding), and dV_j = p_j do."""
    g = _rng(8)
    dh = 16
    q, do = g.standard_normal(dh), g.standard_normal(dh)
    K1, V1 = g.standard_normal((1, dh)), g.standard_normal((1, dh))
    dq, dK, dV = G.head_attention_bwd(q, K1, V1, "softmax", 0.25, do)
    assert np.abs(dq).max() == 0 and np.abs(dK).max() == 0
    np.testing.assert_array_equal(dV[0], do)
    K = np.tile(g.standard_normal(dh), (5, 1))
    V = g.standard_normal((5, dh))
    dq, dK, dV = G.head_attention_bwd(q, K, V, "softmax", 0.25, do)
    assert np.abs(dq).max() < 1e-14
    np.testing.assert_allclose(dV, np.tile(do / 5, (5, 1)), rtol=1e-14)


def test_relu_closed_forms():
    g = _rng(9)
    dh = 16
    q, do = g.standard_normal(dh), g.standard_normal(dh)
    K = -np.abs(g.standard_normal((6, dh))) * np.sign(q)  # every score negative
    V = g.standard_normal((6, dh))
    dq, dK, dV = G.head_attention_bwd(q, K, V, "relu", 0.25, do)
    assert not dq.any() and not dK.any() and not dV.any()
    K = np.abs(g.standard_normal((6, dh))) * np.sign(q)   # every score positive: linear in V
    dq, dK, dV = G.head_attention_bwd(q, K, V, "relu", 0.25, do)
    np.testing.assert_allclose(dV, np.outer(0.25 * K @ q, do), rtol=1e-14)
    np.testing.assert_allclose(dq, 0.25 * K.T @ (V @ do), rtol=1e-13)


@pytest.mark.parametrize("score", ["softmax", "relu"])
@pytest.mark.parametrize("chunk", [1, 3, 7, 20])
def test_sliced_backward_equals_unsplit(score, chunk):
    g = _rng(10)
    dh, L = 8, 20
    q, K, V, do = g.standard_normal(dh), g.standard_normal((L, dh)), g.standard_normal((L, dh)), g.standard_normal(dh)
    sc = 1 / math.sqrt(dh)
    o = R.head_attention(q, K, V, score, sc)
    lse = G.softmax_lse(q, K, sc)
    bounds = [(b, min(L, b + chunk)) for b in range(0, L, chunk)] + [(L, L)]
    ref = G.head_attention_bwd(q, K, V, score, sc, do)
    got = G.head_attention_bwd_sliced(q, K, V, score, sc, do, o, lse, bounds)
    for a, b in zip(got, ref):
        np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-13)


def test_softmax_lse_definition():
    s = np.array([0.5, -2.0, 3.0])
    K = np.diag([1.0, 1.0, 1.0])
    assert abs(G.softmax_lse(s, K, 1.0) - math.log(sum(math.exp(v) for v in s))) < 1e-14


# ---------------------------------------------------------------- whole model: finite differences


def _as_f64_workload(wl):
    """The same workload with every float tensor decoded to float64 (exact), so that
    perturbed copies can be fed to the forward."""
    out = dict(wl)
    out["weights"] = copy.deepcopy(wl["weights"])
    out["table"] = R.to_f64(wl["table"])
    out["x_t"] = R.to_f64(wl["x_t"])
    if wl.get("dt_table") is not None:
        out["dt_table"] = R.to_f64(wl["dt_table"])

    def conv(o):
        if isinstance(o, dict):
            return {k: conv(v) for k, v in o.items()}
        if isinstance(o, list):
            return [conv(v) for v in o]
        if o is None:
            return None
        return R.to_f64(o)

    out["weights"] = conv(out["weights"])
    return out


def _leaves(grads, wl):
    """(name, gradient array, getter/setter of the parameter array) for every tensor."""
    out = []

    def walk(g, w, name):
        if isinstance(g, dict):
            for k in g:
                walk(g[k], w[k], f"{name}.{k}")
        elif isinstance(g, list):
            for i, (gi, wi) in enumerate(zip(g, w)):
                if gi is not None:
                    walk(gi, wi, f"{name}[{i}]")
        else:
            out.append((name, g, w))

    walk(grads, wl["weights"], "w")
    return out


def _loss(wl, dZ):
    z, _ = R.stca_forward(wl)
    return float((z * dZ).sum())


@pytest.mark.parametrize("case", ["softmax_M2", "relu_M2", "softmax_M3_time"])
def test_whole_model_gradients_vs_central_differences(case):
    """For every gradient tensor: <grad, v> equals (L(theta + e v) - L(theta - e v)) / 2e
    for a random direction v (central differences of the oracle's own forward)."""
    if case == "softmax_M3_time":
        wl = make_stca(3, users=2, lengths=np.array([6, 3], np.int32), n_items=40, d=16, H=2, hidden=32, m=2, M=3)
    else:
        wl = make_stca(2, users=2, lengths=np.array([5, 8], np.int32), n_items=40, d=16, H=4, hidden=32, m=3, M=2,
                       score="relu" if case.startswith("relu") else "softmax")
    wl = _as_f64_workload(wl)
    g = _rng(11)
    T, d = len(wl["x_t"]), wl["cfg"]["d"]
    dZ = g.standard_normal((T, d))
    grads, dtable, ddt, dxt = G.stca_backward(wl, dZ)
    eps = 1e-6
    checks = [(n, gr, arr) for n, gr, arr in _leaves(grads, wl)]
    checks.append(("table", dtable, wl["table"]))
    checks.append(("x_t", dxt, wl["x_t"]))
    if ddt is not None:
        checks.append(("dt_table", ddt, wl["dt_table"]))
    for name, gr, arr in checks:
        v = g.standard_normal(arr.shape)
        base = arr.copy()
        arr[...] = base + eps * v
        lp = _loss(wl, dZ)
        arr[...] = base - eps * v
        lm = _loss(wl, dZ)
        arr[...] = base
        fd = (lp - lm) / (2 * eps)
        an = float((gr * v).sum())
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, fd, an)


def test_history_layer_bwd_vs_autograd():
    """X -> LN(SwiGLU(X)) -> [K | V]: every gradient of the composed layer against
    torch.autograd in fp64, random LayerNorm affine."""
    g = _rng(7)
    n, d, h = 6, 8, 12
    X = g.standard_normal((n, d))
    f = {"W1": g.standard_normal((d, h)), "W3": g.standard_normal((d, h)), "W2": g.standard_normal((h, d)),
         "gamma": g.standard_normal(d), "beta": g.standard_normal(d)}
    WK, WV = g.standard_normal((d, d)), g.standard_normal((d, d))
    dK, dV = g.standard_normal((n, d)), g.standard_normal((n, d))
    tX, tf, tK, tV = t64(X), {k: t64(v) for k, v in f.items()}, t64(WK), t64(WV)
    y = (F.silu(tX @ tf["W1"]) * (tX @ tf["W3"])) @ tf["W2"]
    xt = F.layer_norm(y, (d,), tf["gamma"], tf["beta"], eps=1e-5)
    loss = ((xt @ tK) * torch.from_numpy(dK)).sum() + ((xt @ tV) * torch.from_numpy(dV)).sum()
    loss.backward()
    dX, gw = G.history_layer_bwd(X, f, WK, WV, 1e-5, dK, dV)
    np.testing.assert_allclose(dX, tX.grad.numpy(), rtol=1e-10, atol=1e-10)
    for k in f:
        np.testing.assert_allclose(gw[k], tf[k].grad.numpy(), rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(gw["WK"], tK.grad.numpy(), rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(gw["WV"], tV.grad.numpy(), rtol=1e-10, atol=1e-10)


def test_table_rows_bwd_adds_each_token_to_its_rows():
    dtab, ddt = np.zeros((5, 3)), np.zeros((16, 3))
    ids = np.array([4, 0, 4, 2], np.int32)
    dt = np.array([0, 1, 3, 100000], np.int32)       # buckets 0, 1, 2, 15
    dX = np.arange(12, dtype=np.float64).reshape(4, 3)
    G.table_rows_bwd(dtab, ddt, ids, dt, dX)
    np.testing.assert_array_equal(dtab[4], dX[0] + dX[2])
    np.testing.assert_array_equal(dtab[0], dX[1])
    np.testing.assert_array_equal(dtab[[1, 3]], 0)
    np.testing.assert_array_equal(ddt[[0, 1, 2, 15]], dX)
