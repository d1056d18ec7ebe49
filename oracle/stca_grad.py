"""Plain fp64 CPU gradients of the STCA forward pass (the backward pass of training).

TEST INFRASTRUCTURE.  Only the tests, ``__graft_entry__.smoke()`` and the bench's CPU
baseline leg may import this module.  It shares no code with the CUDA library.

The pages train STCA on short histories and serve long ones: [notes] section
"短序列训练，长序列推理" (train at about 2K items, infer at 10K) and the [review]
architecture tree, branch (C) "Extrapolation Aware Training".  Training needs the
gradient of a loss through the forward pass of ``stca_ref``; this module computes it by
the chain rule, step by step in reverse order of the forward, per user and per target,
in float64 with no intermediate rounding.

The loss is L = sum_t dZ[t] . z[t] for a given upstream gradient dZ [T, d] (any loss
reduces to this form at its linearisation point).  Every gradient is returned: every
weight tensor, the embedding table and time-bucket table (rows scatter-added from the
tokens that looked them up) and the target embeddings x_t.

Attention backward (one head, one query q against keys K and values V, scale c):
    softmax: s = c K q, p = softmax(s), o = p V
        dV = p (x) do,  dp = V do,  ds = p * (dp - do . o),  dq = c K^T ds,  dK = c ds (x) q
    relu:    s = c K q, r = relu(s), o = r V
        dV = r (x) do,  dp = V do,  ds = dp * [s > 0],  dq = c K^T ds,  dK = c ds (x) q
A history that is split along L ([wechat] §1.1: local attention over slices, then a merge)
has the same backward slice by slice once the final statistics of the forward are known:
p_j = exp(s_j - lse) with lse = log sum_j exp(s_j) over the whole history and
do . o from the merged output; each slice then gives its keys' dK, dV and a part of dq,
and the parts of dq add up (``head_attention_bwd_sliced``).
"""
from __future__ import annotations

import math

import numpy as np

from .stca_ref import dt_bucket, exclusive_offsets, gather_history, head_attention, layer_norm, silu, swiglu, to_f64

# --------------------------------------------------------------------------------------
# building blocks: each returns the input gradient and the parameter gradients of one
# forward step given the gradient of its output


def silu_grad(x):
    """d SiLU(x) / dx = sigma(x) (1 + x (1 - sigma(x)))."""
    sg = 1.0 / (1.0 + np.exp(-x))
    return sg * (1.0 + x * (1.0 - sg))


def swiglu_bwd(x, ffn, dy):
    """y = (SiLU(x W1) * (x W3)) W2; x [n, d] or [d].  Returns dx, {W1, W3, W2}."""
    W1, W3, W2 = to_f64(ffn["W1"]), to_f64(ffn["W3"]), to_f64(ffn["W2"])
    x2, dy2 = np.atleast_2d(x), np.atleast_2d(dy)
    a, b = x2 @ W1, x2 @ W3
    g = silu(a)
    hid = g * b
    dhid = dy2 @ W2.T
    da = dhid * b * silu_grad(a)
    db = dhid * g
    dx = da @ W1.T + db @ W3.T
    grads = {"W1": x2.T @ da, "W3": x2.T @ db, "W2": hid.T @ dy2}
    return dx.reshape(np.shape(x)), grads


def layer_norm_bwd(x, gamma, beta, eps, dy):
    """y = (x - mean) / sqrt(var + eps) * gamma + beta over the last axis (biased
    variance).  Returns dx, dgamma, dbeta."""
    x2, dy2 = np.atleast_2d(x), np.atleast_2d(dy)
    mu = x2.mean(axis=-1, keepdims=True)
    rstd = 1.0 / np.sqrt(((x2 - mu) ** 2).mean(axis=-1, keepdims=True) + eps)
    xhat = (x2 - mu) * rstd
    dxhat = dy2 * to_f64(gamma)
    dx = rstd * (dxhat - dxhat.mean(axis=-1, keepdims=True) - xhat * (dxhat * xhat).mean(axis=-1, keepdims=True))
    return dx.reshape(np.shape(x)), (dy2 * xhat).sum(axis=0), dy2.sum(axis=0)


def ffn_ln_bwd(x, ffn, eps, dy):
    """LN(SwiGLU(x)) backward.  Returns dx and {W1, W3, W2, gamma, beta}."""
    y = swiglu(x, ffn)
    dy_sw, dgamma, dbeta = layer_norm_bwd(y, ffn["gamma"], ffn["beta"], eps, dy)
    dx, g = swiglu_bwd(x, ffn, dy_sw)
    g.update(gamma=dgamma, beta=dbeta)
    return dx, g


def head_attention_bwd(q_h, K_h, V_h, score, scale, do):
    """Backward of ``stca_ref.head_attention`` for one query.  Returns dq, dK, dV."""
    if K_h.shape[0] == 0:
        return np.zeros_like(q_h), np.zeros_like(K_h), np.zeros_like(V_h)
    s = (K_h @ q_h) * scale
    dp = V_h @ do
    if score == "softmax":
        p = np.exp(s - s.max())
        p /= p.sum()
        o = p @ V_h
        ds = p * (dp - do @ o)
        w = p
    elif score == "relu":
        w = np.maximum(s, 0.0)
        ds = dp * (s > 0)
    else:
        raise ValueError(score)
    return scale * (K_h.T @ ds), scale * np.outer(ds, q_h), np.outer(w, do)


def softmax_lse(q_h, K_h, scale):
    """lse = log sum_j exp(s_j) of one query over all its keys: the statistic a training
    forward keeps so that the backward can form p_j = exp(s_j - lse) slice by slice."""
    s = (K_h @ q_h) * scale
    if s.size == 0:
        return -math.inf
    m = s.max()
    return m + math.log(np.exp(s - m).sum())


def head_attention_bwd_sliced(q_h, K_h, V_h, score, scale, do, o, lse, bounds):
    """The same backward computed slice by slice along the keys, as a split-L kernel does:
    slice [b0, b1) uses only its own keys plus the forward's final lse (softmax) and output
    o; it returns its keys' dK, dV and its share of dq.  Returns (dq, dK, dV) with dq the
    sum of the slices' shares."""
    dq = np.zeros_like(q_h)
    dK = np.zeros_like(K_h)
    dV = np.zeros_like(V_h)
    D = do @ o
    for b0, b1 in bounds:
        Kc, Vc = K_h[b0:b1], V_h[b0:b1]
        if Kc.shape[0] == 0:
            continue
        s = (Kc @ q_h) * scale
        dp = Vc @ do
        if score == "softmax":
            w = np.exp(s - lse)
            ds = w * (dp - D)
        else:
            w = np.maximum(s, 0.0)
            ds = dp * (s > 0)
        dq += scale * (Kc.T @ ds)
        dK[b0:b1] = scale * np.outer(ds, q_h)
        dV[b0:b1] = np.outer(w, do)
    return dq, dK, dV


# --------------------------------------------------------------------------------------
# whole forward


def _zeros_like_weights(w, M):
    def ffn0(f, ln=True):
        g = {k: np.zeros(np.shape(f[k])) for k in ("W1", "W3", "W2")}
        if ln:
            g["gamma"], g["beta"] = np.zeros(np.shape(f["gamma"])), np.zeros(np.shape(f["beta"]))
        return g

    z = lambda a: np.zeros(np.shape(a))
    return {
        "hist": [ffn0(w["hist"][i]) for i in range(M)],
        "WQ": [z(w["WQ"][i]) for i in range(M)], "WK": [z(w["WK"][i]) for i in range(M)],
        "WV": [z(w["WV"][i]) for i in range(M)], "WO": [z(w["WO"][i]) for i in range(M)],
        "WC": [None] + [z(w["WC"][i]) for i in range(1, M)],
        "fuse": [None] + [ffn0(w["fuse"][i]) for i in range(1, M)],
        "tgt": ffn0(w["tgt"]), "WZ": z(w["WZ"]), "zffn": ffn0(w["zffn"], ln=False),
    }


def _add_ffn(acc, g):
    for k, v in g.items():
        acc[k] += v


def stca_backward(wl, dZ):
    """Gradients of L = sum_t dZ[t] . z[t] for the STCA workload ``wl`` (as in
    ``stca_ref.stca_forward``).  Returns (grads of the weights in the structure of
    wl["weights"], d table [n_items, d], d dt_table [16, d] or None, d x_t [T, d])."""
    cfg, w = wl["cfg"], wl["weights"]
    d, H, M, eps, score = cfg["d"], cfg["H"], cfg["M"], cfg.get("ln_eps", 1e-5), cfg["score"]
    dh = d // H
    scale = 1.0 / math.sqrt(dh)
    f64 = to_f64
    G = _zeros_like_weights(w, M)
    table = np.asarray(wl["table"])
    dtable = np.zeros((table.shape[0], d))
    has_dt = wl.get("dt") is not None
    ddt_table = np.zeros((16, d)) if has_dt else None
    dxt_all = np.zeros((len(wl["x_t"]), d))
    dZ = np.asarray(dZ, dtype=np.float64)
    hoff = exclusive_offsets(wl["lengths"])
    toff = exclusive_offsets(wl["targets_per_user"])
    for u in range(len(wl["lengths"])):
        sl = slice(hoff[u], hoff[u + 1])
        dt = wl["dt"][sl] if has_dt else None
        X = gather_history(wl["table"], wl["ids"][sl], dt, wl.get("dt_table"))
        # history side, forward (kept for the backward)
        Y = [swiglu(X, w["hist"][i]) for i in range(M)]
        Xt = [layer_norm(Y[i], w["hist"][i]["gamma"], w["hist"][i]["beta"], eps) for i in range(M)]
        K = [Xt[i] @ f64(w["WK"][i]) for i in range(M)]
        V = [Xt[i] @ f64(w["WV"][i]) for i in range(M)]
        dK = [np.zeros_like(K[i]) for i in range(M)]
        dV = [np.zeros_like(V[i]) for i in range(M)]
        for t in range(toff[u], toff[u + 1]):
            x_t = f64(wl["x_t"][t])
            # target side, forward
            q = [layer_norm(swiglu(x_t, w["tgt"]), w["tgt"]["gamma"], w["tgt"]["beta"], eps)]
            Qp, obar, outs, cats, fused_in = [], [], [], [], [None]
            for i in range(M):
                Qp.append(q[i] @ f64(w["WQ"][i]))
                heads = []
                for hh in range(H):
                    c = slice(hh * dh, (hh + 1) * dh)
                    heads.append(head_attention(Qp[i][c], K[i][:, c], V[i][:, c], score, scale))
                obar.append(np.concatenate(heads))
                outs.append(obar[i] @ f64(w["WO"][i]))
                cats.append(np.concatenate(outs + [x_t]))
                if i + 1 < M:
                    ui = cats[i] @ f64(w["WC"][i + 1])
                    fused_in.append(ui)
                    q.append(layer_norm(swiglu(ui, w["fuse"][i + 1]), w["fuse"][i + 1]["gamma"],
                                        w["fuse"][i + 1]["beta"], eps))
            # z = SwiGLU_Z(cat_M W_Z)
            zin = cats[M - 1] @ f64(w["WZ"])
            dzin, gz = swiglu_bwd(zin, w["zffn"], dZ[t])
            _add_ffn(G["zffn"], gz)
            G["WZ"] += np.outer(cats[M - 1], dzin)
            dcat = dzin @ f64(w["WZ"]).T              # gradient of [o1 .. oM | x_t]
            dout = [dcat[i * d:(i + 1) * d].copy() for i in range(M)]
            dxt = dcat[M * d:].copy()
            for i in reversed(range(M)):
                # o^(i) = obar W_O, then per-head attention of Q = q W_Q
                G["WO"][i] += np.outer(obar[i], dout[i])
                dobar = dout[i] @ f64(w["WO"][i]).T
                dQ = np.zeros(d)
                for hh in range(H):
                    c = slice(hh * dh, (hh + 1) * dh)
                    dq_h, dK_h, dV_h = head_attention_bwd(Qp[i][c], K[i][:, c], V[i][:, c], score, scale,
                                                          dobar[c])
                    dQ[c] = dq_h
                    dK[i][:, c] += dK_h      # the user's K/V serve all its targets (RLB)
                    dV[i][:, c] += dV_h
                G["WQ"][i] += np.outer(q[i], dQ)
                dq = dQ @ f64(w["WQ"][i]).T
                if i == 0:   # q1 = LN(SwiGLU_t(x_t))
                    dx, g = ffn_ln_bwd(x_t, w["tgt"], eps, dq)
                    _add_ffn(G["tgt"], g)
                    dxt += dx
                else:        # q^(i) = LN(SwiGLU^(i)(cat_{i-1} W_C^(i)))
                    du, g = ffn_ln_bwd(fused_in[i], w["fuse"][i], eps, dq)
                    _add_ffn(G["fuse"][i], g)
                    G["WC"][i] += np.outer(cats[i - 1], du)
                    dc = du @ f64(w["WC"][i]).T
                    for j in range(i):
                        dout[j] += dc[j * d:(j + 1) * d]
                    dxt += dc[i * d:]
            dxt_all[t] = dxt
        # history side, backward: K = Xt W_K, V = Xt W_V, Xt = LN(SwiGLU(X))
        dX = np.zeros_like(X)
        for i in range(M):
            dx, g = history_layer_bwd(X, w["hist"][i], w["WK"][i], w["WV"][i], eps, dK[i], dV[i])
            G["WK"][i] += g.pop("WK")
            G["WV"][i] += g.pop("WV")
            _add_ffn(G["hist"][i], g)
            dX += dx
        table_rows_bwd(dtable, ddt_table, wl["ids"][sl], dt, dX)
    return G, dtable, ddt_table, dxt_all


def history_layer_bwd(X, ffn, WK, WV, eps, dK, dV):
    """One layer's history side, X -> Xt = LN(SwiGLU(X)) -> K = Xt W_K, V = Xt W_V
    ([notes] section "STCA"; [review] 核心公式), backward from dK, dV [n, d]: returns dX and
    {W1, W3, W2, gamma, beta, WK, WV}."""
    Xt = layer_norm(swiglu(X, ffn), ffn["gamma"], ffn["beta"], eps)
    dK, dV = np.asarray(dK, np.float64), np.asarray(dV, np.float64)
    dXt = dK @ to_f64(WK).T + dV @ to_f64(WV).T
    dX, g = ffn_ln_bwd(X, ffn, eps, dXt)
    g.update(WK=Xt.T @ dK, WV=Xt.T @ dV)
    return dX, g


def table_rows_bwd(dtable, ddt_table, ids, dt, dX):
    """The lookup x_n = E[ids_n] (+ T[bucket(dt_n)]) backward: every token's gradient row is
    added to the table rows it read (in place)."""
    np.add.at(dtable, np.asarray(ids, dtype=np.int64), dX)
    if ddt_table is not None and dt is not None:
        np.add.at(ddt_table, dt_bucket(dt), dX)
