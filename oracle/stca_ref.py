"""Plain fp64 CPU oracle for the STCA forward pass and its two variants.

TEST INFRASTRUCTURE.  Only the tests, ``__graft_entry__.smoke()`` and the bench's CPU
baseline leg may import this module.  It shares no code with the CUDA library and is
deliberately slow: per-user and per-target Python loops around numpy float64 matmuls,
with no request-level sharing, blocking, fusion or reordering beyond what the formulas
state.

Sources (cited by page title and section or equation):

* [notes]  "超长序列建模 —— STCA 精读笔记" (wln20.github.io), sections "STCA" and
  "Request Level Batching（RLB）": problem statement, layer-1 encoders, per-layer K/V
  source, query fusion, z.
* [review] "Make It Long, Keep It Fast: End-to-End 10K Long User Behavior Sequence
  Modeling for Billion-Scale Douyin Recommendation" paper review (xllm-io.github.io),
  §三 "核心公式" and architecture tree: per-head attention, fusion, z; §四 table
  (SwiGLU FFN, time-delta feature).
* [wechat] "视频号推荐超长序列技术演进：从端到端到 Cross-Mask Transformer"
  (dingyadong.top), §1.1 (distributed TA: local attention then merge; low-memory TA
  operator with fused lookup) and §1.2 (element-wise ReLU scores).
* [hyformer] "HyFormer：重新审视序列建模和特征交互在 CTR 预测中的作用"
  (gitcode.csdn.net), §3.4.1 eq (7)-(8), §3.4.2 eq (9), §3.5 eq (10)-(15),
  §3.6 eq (16), §3.7 (multi-sequence).

Readings where the pages are silent or garbled (each also listed in the design notes):

* SwiGLU(x) = (SiLU(x W1) * (x W3)) W2, no biases, d -> hidden -> d.
* No residual around the FFN blocks; LayerNorm uses the biased variance and eps.
* z = SwiGLU_Z([o1 | ... | oM | x_t] W_Z) without LayerNorm (the review's formula).
* Softmax over the user's own tokens only, scale 1/sqrt(d_h); an empty history gives o = 0.
* ReLU scores are not normalised: o = sum_j relu(s_j) v_j.
* Time feature: x_j = E[id_j] + T[b_j], b_j = min(15, floor(log2(dt_j + 1))).
* HyFormer: standard multi-head cross attention with its own W_Q/W_K/W_V/W_O per sequence,
  no LayerNorm in the SwiGLU encoder, per-token SwiGLU per token index, residual Q + Q~.

Stored inputs are fp32 arrays or bf16 bit patterns (``uint16``); both decode exactly to
float64 here, and every step after that runs in float64 with no intermediate rounding.
"""
from __future__ import annotations

import math

import numpy as np

# --------------------------------------------------------------------------------------
# storage decoding


def to_f64(x) -> np.ndarray:
    """Decode a stored tensor (float32/float64, or bf16 bit patterns in uint16) exactly."""
    x = np.asarray(x)
    if x.dtype == np.uint16:
        return (x.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    return x.astype(np.float64)


# --------------------------------------------------------------------------------------
# ragged layout ([notes] STCA: one history H of length L per user; RLB: targets grouped
# per user)


def exclusive_offsets(lengths) -> np.ndarray:
    """offsets[u] = sum of lengths[:u]; offsets has B+1 entries (int64)."""
    lengths = [int(v) for v in lengths]
    out = [0]
    for v in lengths:
        out.append(out[-1] + v)
    return np.asarray(out, dtype=np.int64)


def dt_bucket(dt) -> np.ndarray:
    """Time-difference bucket min(15, floor(log2(dt + 1))) for dt >= 0, in integers.

    [review] §四 lists the interaction time gap as an extra per-token feature; the
    16-bin log2 bucketing is this library's reading of it.
    """
    out = []
    for v in np.asarray(dt).reshape(-1):
        v = int(v)
        if v < 0:
            raise ValueError("negative time difference")
        out.append(min(15, (v + 1).bit_length() - 1))
    return np.asarray(out, dtype=np.int32)


def gather_history(table, ids, dt=None, dt_table=None) -> np.ndarray:
    """X[n] = E[ids[n]] (+ T[bucket(dt[n])]) in float64.  [wechat] §1.1 (KV lookup)."""
    ids = np.asarray(ids, dtype=np.int64)
    X = to_f64(np.asarray(table)[ids])
    if dt is not None:
        X = X + to_f64(np.asarray(dt_table))[dt_bucket(dt)]
    return X


# --------------------------------------------------------------------------------------
# building blocks


def silu(x):
    return x / (1.0 + np.exp(-x))


def layer_norm(x, gamma, beta, eps):
    """LayerNorm over the last axis: biased variance, learnable gamma/beta."""
    x = np.asarray(x, dtype=np.float64)
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    return (x - mu) / np.sqrt(var + eps) * to_f64(gamma) + to_f64(beta)


def swiglu(x, ffn):
    """SwiGLU FFN (dimension preserving, [review] §四): (SiLU(x W1) * (x W3)) W2."""
    W1, W3, W2 = to_f64(ffn["W1"]), to_f64(ffn["W3"]), to_f64(ffn["W2"])
    return (silu(x @ W1) * (x @ W3)) @ W2


def ffn_ln(x, ffn, eps):
    """LN(SwiGLU(x)): the per-layer encoder of [notes] STCA (history and target sides)."""
    return layer_norm(swiglu(x, ffn), ffn["gamma"], ffn["beta"], eps)


def attention_weights(q_h, K_h, scale):
    """Softmax weights of one query against all keys ([review] 核心公式, alpha^(i,j))."""
    s = (K_h @ q_h) * scale
    e = np.exp(s - s.max())
    return e / e.sum()


def head_attention(q_h, K_h, V_h, score, scale):
    """One head of single-query cross attention.

    softmax: o = softmax(q K^T * scale) V   ([review] 核心公式)
    relu:    o = sum_j relu(q.k_j * scale) v_j   ([wechat] §1.2, unnormalised)
    An empty key set gives o = 0.
    """
    if K_h.shape[0] == 0:
        return np.zeros(V_h.shape[1])
    if score == "softmax":
        return attention_weights(q_h, K_h, scale) @ V_h
    if score == "relu":
        return np.maximum((K_h @ q_h) * scale, 0.0) @ V_h
    raise ValueError(score)


def attention_partial(q_h, K_h, V_h, score, scale):
    """Local attention state over one slice of the keys ([wechat] §1.1 distributed TA).

    softmax: (max score, sum of exp(s - max), sum of exp(s - max) v); relu: (-, -, sum).
    """
    if score == "relu":
        return None, None, np.maximum((K_h @ q_h) * scale, 0.0) @ V_h
    if K_h.shape[0] == 0:
        return -math.inf, 0.0, np.zeros(V_h.shape[1])
    s = (K_h @ q_h) * scale
    mx = s.max()
    e = np.exp(s - mx)
    return mx, e.sum(), e @ V_h


def merge_partials(parts, score):
    """Combine local states of disjoint key slices into the full attention output."""
    if score == "relu":
        return sum(p[2] for p in parts)
    mxs = [p[0] for p in parts if p[1] > 0]
    if not mxs:
        return np.zeros_like(parts[0][2])
    M = max(mxs)
    num = sum(p[2] * math.exp(p[0] - M) for p in parts if p[1] > 0)
    den = sum(p[1] * math.exp(p[0] - M) for p in parts if p[1] > 0)
    return num / den


# --------------------------------------------------------------------------------------
# STCA forward (configs 1-3)


def stca_user_kv(X, w, layer, eps):
    """K^(i), V^(i) of one user from the ORIGINAL history X ([notes] STCA: every layer's
    X~ comes from X through that layer's own SwiGLU-FFN + LN)."""
    Xt = ffn_ln(X, w["hist"][layer], eps)
    return Xt @ to_f64(w["WK"][layer]), Xt @ to_f64(w["WV"][layer])


def stca_target(x_t, KV, w, cfg, return_queries=False):
    """All M layers for one target against one user's per-layer K/V.

    q1 = LN(SwiGLU_t(x_t))                                  [notes] STCA layer 1
    o_h^(i) = attention(q^(i) W_Q^(i)[:,h], K^(i)_h, V^(i)_h)  [review] 核心公式
    o^(i) = [o_1 | ... | o_H] W_O^(i)                       [notes] STCA
    q^(i+1) = LN(SwiGLU^(i+1)([o^(1)|...|o^(i)|x_t] W_C^(i+1)))  [review] 层间融合
    z = SwiGLU_Z([o^(1)|...|o^(M)|x_t] W_Z)                  [review] architecture tree
    """
    d, H, M, eps = cfg["d"], cfg["H"], cfg["M"], cfg.get("ln_eps", 1e-5)
    dh = d // H
    scale = 1.0 / math.sqrt(dh)
    x_t = to_f64(x_t)
    q = ffn_ln(x_t, w["tgt"], eps)
    queries = [q]
    outs = []
    for i in range(M):
        K, V = KV[i]
        Q = q @ to_f64(w["WQ"][i])
        heads = []
        for h in range(H):
            cols = slice(h * dh, (h + 1) * dh)
            heads.append(head_attention(Q[cols], K[:, cols], V[:, cols], cfg["score"], scale))
        outs.append(np.concatenate(heads) @ to_f64(w["WO"][i]))
        if i + 1 < M:
            cat = np.concatenate(outs + [x_t])
            q = ffn_ln(cat @ to_f64(w["WC"][i + 1]), w["fuse"][i + 1], eps)
            queries.append(q)
    cat = np.concatenate(outs + [x_t])
    z = swiglu(cat @ to_f64(w["WZ"]), w["zffn"])
    if return_queries:
        return z, outs, queries
    return z, outs


def stca_forward(wl, users=None):
    """STCA forward for the workload dict ``wl`` (see ``workloads.make_stca``).

    Returns (z [T, d], o [M, T, d]) for the targets of ``users`` (all users by default),
    rows in target order.  Each target is computed on its own; the only thing shared per
    user is the user's K/V, which is a pure function of the user's history.
    """
    cfg, w = wl["cfg"], wl["weights"]
    eps = cfg.get("ln_eps", 1e-5)
    B = len(wl["lengths"])
    hoff = exclusive_offsets(wl["lengths"])
    toff = exclusive_offsets(wl["targets_per_user"])
    users = range(B) if users is None else users
    zs, os_ = [], []
    for u in users:
        sl = slice(hoff[u], hoff[u + 1])
        dt = None if wl.get("dt") is None else wl["dt"][sl]
        X = gather_history(wl["table"], wl["ids"][sl], dt, wl.get("dt_table"))
        KV = [stca_user_kv(X, w, i, eps) for i in range(cfg["M"])]
        for t in range(toff[u], toff[u + 1]):
            z, outs = stca_target(wl["x_t"][t], KV, w, cfg)
            zs.append(z)
            os_.append(np.stack(outs))
    d = cfg["d"]
    if not zs:
        return np.zeros((0, d)), np.zeros((cfg["M"], 0, d))
    return np.stack(zs), np.stack(os_, axis=1)


# --------------------------------------------------------------------------------------
# pointwise ReLU target attention with fused lookup (config 4)


def pointwise_relu_ta(wl, users=None):
    """o_b = sum_j relu(q_b . e_j / sqrt(D)) e_j with k_j = v_j = E[id_j].

    [wechat] §1.1 low-memory TA operator (lookup fused with attention; the gathered
    [B, L, D] matrix is the thing it avoids) and §1.2 (element-wise ReLU scores).
    """
    hoff = exclusive_offsets(wl["lengths"])
    D = wl["cfg"]["d"]
    scale = 1.0 / math.sqrt(D)
    users = range(len(wl["lengths"])) if users is None else users
    out = []
    for b in users:
        E = gather_history(wl["table"], wl["ids"][hoff[b]:hoff[b + 1]])
        q = to_f64(wl["q"][b])
        out.append(head_attention(q, E, E, "relu", scale))
    return np.stack(out) if out else np.zeros((0, D))


# --------------------------------------------------------------------------------------
# multi-query multi-sequence decode (config 5)


def token_mix(Q):
    """[hyformer] eq (11)-(13): split each of the T tokens into T sub-spaces of width D/T,
    then token h of the result concatenates sub-space h of tokens 1..T in order."""
    T, D = Q.shape
    sub = D // T
    out = np.empty_like(Q)
    for h in range(T):
        for t in range(T):
            out[h, t * sub:(t + 1) * sub] = Q[t, h * sub:(h + 1) * sub]
    return out


def cross_attention(Qin, K, V, WQ, WO, H):
    """Standard multi-head cross attention of several queries ([hyformer] eq (9)),
    queries projected by W_Q, keys/values already projected, heads joined by W_O."""
    d = Qin.shape[1]
    dh = d // H
    scale = 1.0 / math.sqrt(dh)
    Qp = Qin @ WQ
    rows = []
    for n in range(Qin.shape[0]):
        heads = []
        for h in range(H):
            cols = slice(h * dh, (h + 1) * dh)
            heads.append(head_attention(Qp[n, cols], K[:, cols], V[:, cols], "softmax", scale))
        rows.append(np.concatenate(heads))
    return np.stack(rows) @ WO


def hyformer_user(Q0, Xs, w, cfg):
    """All blocks for one user: Q0 [2*nq, d] queries, Xs = [X_feed, X_search].

    Per block and per sequence s ([hyformer] §3.4, §3.7):
        H = SwiGLU(X_s)                 eq (7), recomputed from the raw sequence
        K, V = H W_K, H W_V              eq (8)
        Q^_s = CrossAttn(Q_s, K, V)      eq (9)/(16)
    then query boosting ([hyformer] §3.5):
        Q = [Q^_feed; Q^_search]         eq (10), no non-sequential tokens
        Q~ = PerToken-FFN(mix(Q))        eq (11)-(14)
        Q_next = Q + Q~                  eq (15)
    """
    nq, H = cfg["n_query"], cfg["H"]
    Q = to_f64(Q0)
    for blk in w["blocks"]:
        Qhat = np.empty_like(Q)
        for s, X in enumerate(Xs):
            f = blk["seq"][s]
            Hs = swiglu(X, f)
            K, V = Hs @ to_f64(f["WK"]), Hs @ to_f64(f["WV"])
            rows = slice(s * nq, (s + 1) * nq)
            Qhat[rows] = cross_attention(Q[rows], K, V, to_f64(f["WQ"]), to_f64(f["WO"]), H)
        mixed = token_mix(Qhat)
        boost = np.stack([swiglu(mixed[k], blk["tok"][k]) for k in range(mixed.shape[0])])
        Q = Qhat + boost
    return Q


def hyformer_forward(wl, users=None):
    """Output queries [len(users), 2*nq, d] for the workload dict ``wl``."""
    cfg, w = wl["cfg"], wl["weights"]
    offs = [exclusive_offsets(wl["lengths"][s]) for s in range(2)]
    B = len(wl["lengths"][0])
    users = range(B) if users is None else users
    out = []
    for b in users:
        Xs = [gather_history(wl["table"], wl["ids"][s][offs[s][b]:offs[s][b + 1]])
              for s in range(2)]
        out.append(hyformer_user(wl["q0"][b], Xs, w, cfg))
    return np.stack(out)


# --------------------------------------------------------------------------------------
# error metric


def row_rel_err(got, ref) -> float:
    """max over rows of max_k |g - r| / max(||r||_inf, 1e-6)."""
    got = np.asarray(got, dtype=np.float64).reshape(-1, np.shape(ref)[-1])
    ref = np.asarray(ref, dtype=np.float64).reshape(-1, np.shape(ref)[-1])
    if ref.shape[0] == 0:
        return 0.0
    den = np.maximum(np.abs(ref).max(axis=1), 1e-6)
    return float((np.abs(got - ref).max(axis=1) / den).max())
