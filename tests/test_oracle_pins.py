"""Pins for the fp64 oracle: hand-derived worked examples, closed forms, library
special cases and invariants the STCA/HyFormer formulas fix.  CPU only."""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import stca_ref as R
from workloads import make_hyformer, make_pointwise, make_stca


def _load(golden_dir, name):
    with open(os.path.join(golden_dir, name)) as f:
        return json.load(f)


def _rng(seed=0):
    return np.random.default_rng(seed)


# ---------------------------------------------------------------- golden worked examples


def test_golden_attention(golden_dir):
    g = _load(golden_dir, "attention_two_keys.json")
    q = np.array(g["q"])
    scale = 1 / math.sqrt(2)
    K, V = np.array(g["k_softmax"]), np.array(g["v_softmax"])
    np.testing.assert_allclose(R.attention_weights(q, K, scale), g["weights_softmax"], atol=1e-15)
    np.testing.assert_allclose(R.head_attention(q, K, V, "softmax", scale), g["o_softmax"], atol=1e-14)
    K, V = np.array(g["k_relu"]), np.array(g["v_relu"])
    np.testing.assert_allclose(R.head_attention(q, K, V, "relu", scale), g["o_relu"], atol=1e-14)


def test_golden_dt_buckets(golden_dir):
    g = _load(golden_dir, "dt_buckets.json")
    assert R.dt_bucket(g["dt"]).tolist() == g["bucket"]


def test_golden_token_mix(golden_dir):
    g = _load(golden_dir, "token_mix_T2.json")
    np.testing.assert_array_equal(R.token_mix(np.array(g["Q"], float)), g["mixed"])


def test_golden_layer_norm_swiglu(golden_dir):
    g = _load(golden_dir, "layer_norm_swiglu.json")
    x = np.array(g["ln_x"])
    np.testing.assert_allclose(R.layer_norm(x, np.ones(4), np.zeros(4), 0.0), g["ln_out"], atol=1e-15)
    np.testing.assert_allclose(R.layer_norm(x, np.array(g["ln_gamma"]), np.array(g["ln_beta"]), 0.0),
                               g["ln_out_affine"], atol=1e-15)
    ffn = dict(W1=np.array([[1.0]]), W3=np.array([[2.0]]), W2=np.array([[3.0]]))
    assert abs(R.swiglu(np.array([1.0]), ffn)[0] - g["swiglu_out"]) < 1e-14


# ---------------------------------------------------------------- integer bookkeeping


def test_offsets_match_cumsum():
    lengths = _rng(1).integers(0, 50, size=37)
    off = R.exclusive_offsets(lengths)
    assert off[0] == 0 and len(off) == 38
    np.testing.assert_array_equal(off[1:], np.cumsum(lengths))


def test_dt_bucket_bracketing():
    dt = np.concatenate([np.arange(0, 70000), _rng(2).integers(0, 2**31 - 2, size=5000)])
    b = R.dt_bucket(dt).astype(np.int64)
    v = dt.astype(np.int64) + 1
    assert ((b >= 0) & (b <= 15)).all()
    lo_ok = (np.left_shift(1, b) <= v)
    hi_ok = (v < np.left_shift(1, b + 1)) | (b == 15)
    assert lo_ok.all() and hi_ok.all()


def test_gather_matches_indexing_bitwise():
    wl = make_stca(3, users=2, L=50, n_items=1000)
    X = R.gather_history(wl["table"], wl["ids"][:100], wl["dt"][:100], wl["dt_table"])
    E = torch.from_numpy(wl["table"].view(np.int16)).view(torch.bfloat16).double().numpy()
    T = torch.from_numpy(wl["dt_table"].view(np.int16)).view(torch.bfloat16).double().numpy()
    b = np.minimum(15, np.floor(np.log2(wl["dt"][:100].astype(np.float64) + 1))).astype(int)
    np.testing.assert_array_equal(X, E[wl["ids"][:100]] + T[b])


# ---------------------------------------------------------------- building blocks vs torch


def test_layer_norm_and_silu_vs_torch():
    g = _rng(3)
    x = g.standard_normal((7, 33)) * 3 + 1
    gamma, beta = g.standard_normal(33), g.standard_normal(33)
    ref = F.layer_norm(torch.from_numpy(x), (33,), torch.from_numpy(gamma), torch.from_numpy(beta), 1e-5)
    np.testing.assert_allclose(R.layer_norm(x, gamma, beta, 1e-5), ref.numpy(), rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(R.silu(x), F.silu(torch.from_numpy(x)).numpy(), rtol=1e-14, atol=1e-15)


def test_layer_norm_identity_moments():
    x = _rng(4).standard_normal((5, 64)) * 10 + 3
    y = R.layer_norm(x, np.ones(64), np.zeros(64), 0.0)
    np.testing.assert_allclose(y.mean(axis=1), 0, atol=1e-14)
    np.testing.assert_allclose(y.var(axis=1), 1, atol=1e-13)


def test_swiglu_zero_gate_and_shapes():
    g = _rng(5)
    x = g.standard_normal((3, 8))
    ffn = dict(W1=np.zeros((8, 16)), W3=g.standard_normal((8, 16)), W2=g.standard_normal((16, 8)))
    np.testing.assert_array_equal(R.swiglu(x, ffn), 0)
    ffn["W1"] = g.standard_normal((8, 16))
    assert R.swiglu(x, ffn).shape == (3, 8)


# ---------------------------------------------------------------- attention pins


def test_softmax_weights_sum_to_one():
    g = _rng(6)
    for L in (1, 2, 17, 1000):
        w = R.attention_weights(g.standard_normal(32) * 4, g.standard_normal((L, 32)), 1 / math.sqrt(32))
        assert abs(w.sum() - 1) < 1e-12 and (w >= 0).all()


def test_identical_keys_give_mean_of_values():
    g = _rng(7)
    k = g.standard_normal(16)
    K = np.tile(k, (9, 1))
    V = g.standard_normal((9, 16))
    o = R.head_attention(g.standard_normal(16), K, V, "softmax", 0.25)
    np.testing.assert_allclose(o, V.mean(axis=0), atol=1e-14)


def test_head_attention_vs_torch_sdpa():
    g = _rng(8)
    for L, dh in ((1, 8), (5, 32), (300, 64)):
        q, K, V = g.standard_normal(dh), g.standard_normal((L, dh)), g.standard_normal((L, dh))
        ref = F.scaled_dot_product_attention(torch.from_numpy(q)[None, None, None],
                                             torch.from_numpy(K)[None, None],
                                             torch.from_numpy(V)[None, None])
        o = R.head_attention(q, K, V, "softmax", 1 / math.sqrt(dh))
        np.testing.assert_allclose(o, ref.reshape(-1).numpy(), rtol=1e-12, atol=1e-13)


def test_bruteforce_small_L():
    """Unshifted exponentials and exactly rounded sums, element by element."""
    g = _rng(9)
    for L in range(1, 9):
        q, K, V = g.standard_normal(4), g.standard_normal((L, 4)), g.standard_normal((L, 4))
        s = [sum(q[c] * K[j, c] for c in range(4)) * 0.5 for j in range(L)]
        e = [math.exp(v) for v in s]
        den = math.fsum(e)
        ref = [math.fsum(e[j] * V[j, c] for j in range(L)) / den for c in range(4)]
        np.testing.assert_allclose(R.head_attention(q, K, V, "softmax", 0.5), ref, rtol=1e-13)
        ref_r = [math.fsum(max(s[j], 0.0) * V[j, c] for j in range(L)) for c in range(4)]
        np.testing.assert_allclose(R.head_attention(q, K, V, "relu", 0.5), ref_r, rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("score", ["softmax", "relu"])
def test_split_merge_equals_unsplit(score):
    g = _rng(10)
    L = 23
    q, K, V = g.standard_normal(16) * 2, g.standard_normal((L, 16)), g.standard_normal((L, 16))
    full = R.head_attention(q, K, V, score, 0.25)
    for C in (1, 3, 7, L):
        parts = [R.attention_partial(q, K[s:s + C], V[s:s + C], score, 0.25) for s in range(0, L, C)]
        np.testing.assert_allclose(R.merge_partials(parts, score), full, rtol=1e-12, atol=1e-13)
    # an empty slice contributes nothing
    parts = [R.attention_partial(q, K[:0], V[:0], score, 0.25), R.attention_partial(q, K, V, score, 0.25)]
    np.testing.assert_allclose(R.merge_partials(parts, score), full, rtol=1e-12, atol=1e-13)


def test_relu_special_cases():
    g = _rng(11)
    q = g.standard_normal(8)
    K = -np.sign(q) * np.abs(g.standard_normal((6, 8)))      # every score negative
    V = g.standard_normal((6, 8))
    np.testing.assert_array_equal(R.head_attention(q, K, V, "relu", 0.3), 0)
    np.testing.assert_array_equal(R.head_attention(np.zeros(8), g.standard_normal((6, 8)), V, "relu", 0.3), 0)
    e = g.standard_normal(8)
    s = q @ e * 0.3
    np.testing.assert_allclose(R.head_attention(q, e[None], e[None], "relu", 0.3), max(s, 0) * e, atol=1e-15)


@pytest.mark.parametrize("score", ["softmax", "relu"])
def test_empty_history_gives_zero(score):
    o = R.head_attention(np.ones(4), np.zeros((0, 4)), np.zeros((0, 4)), score, 0.5)
    np.testing.assert_array_equal(o, 0)


# ---------------------------------------------------------------- whole-STCA pins


def _small_stca(config_id=2, **kw):
    base = dict(users=3, L=20, n_items=500)
    base.update(kw)
    return make_stca(config_id, **base)


def _f64(x):
    return R.to_f64(x)


def test_single_token_history_closed_form():
    """L = 1: every head's softmax weight is 1, so o^(i) = ((LN(SwiGLU(x_1))) W_V) W_O."""
    wl = _small_stca(3, users=2, L=1, d=64, H=4, hidden=128, m=3)
    z, o = R.stca_forward(wl)
    w, cfg = wl["weights"], wl["cfg"]
    for u in range(2):
        x1 = R.gather_history(wl["table"], wl["ids"][u:u + 1], wl["dt"][u:u + 1], wl["dt_table"])[0]
        for i in range(cfg["M"]):
            xt = R.layer_norm(R.swiglu(x1, w["hist"][i]), w["hist"][i]["gamma"], w["hist"][i]["beta"], 1e-5)
            expect = (xt @ _f64(w["WV"][i])) @ _f64(w["WO"][i])
            for t in range(3 * u, 3 * u + 3):
                np.testing.assert_allclose(o[i, t], expect, rtol=1e-11, atol=1e-12)


def _torch_mha(d, H, WQ, WK, WV, WO):
    """torch's own multi-head attention module in fp64, bias-free, holding the weights
    given in the pages' [in, out] convention (torch stores [out, in])."""
    mha = torch.nn.MultiheadAttention(d, H, bias=False, batch_first=True, dtype=torch.float64)
    with torch.no_grad():
        mha.in_proj_weight.copy_(torch.cat([torch.from_numpy(_f64(W)).T for W in (WQ, WK, WV)]))
        mha.out_proj.weight.copy_(torch.from_numpy(_f64(WO)).T)
    return mha


@pytest.mark.parametrize("score_layers", [1, 2, 3])
def test_stca_score_path_vs_torch_multihead_attention(score_layers):
    """Each layer's o^(i) is standard multi-head attention of the one query q^(i) over the
    user's X~^(i) ([review] 核心公式: alpha = softmax(q W_Q (X~ W_K)^T / sqrt(d_h)),
    o = alpha X~ W_V, heads joined by W_O).  torch.nn.MultiheadAttention does the
    projections, the head split and the 1/sqrt(d_h) scale itself, so a wrong scale, a
    swapped W_Q/W_K or a wrong head slice in the oracle fails here.  LayerNorm and SiLU
    come from torch's functional ops.  The chain is followed to the model's output z
    ([review] architecture tree: z from [o^(1) | ... | o^(M) | x_t] W_Z through the z
    SwiGLU), so with three layers the order of several o blocks in the concatenations,
    the fusion of each layer and W_Z are pinned too."""
    d, H, L = 64, 4, 7
    wl = make_stca(2, users=1, lengths=np.array([L], np.int32), n_items=100, d=d, H=H, hidden=128, m=2,
                   M=score_layers)
    cfg, w = wl["cfg"], wl["weights"]
    z, o = R.stca_forward(wl)
    t = lambda a: torch.from_numpy(_f64(a))

    def ln_swiglu(x, f, ln=True):
        y = (F.silu(x @ t(f["W1"])) * (x @ t(f["W3"]))) @ t(f["W2"])
        return F.layer_norm(y, (d,), t(f["gamma"]), t(f["beta"]), 1e-5) if ln else y

    X = t(wl["table"])[torch.from_numpy(wl["ids"].astype(np.int64))]
    for k in range(2):
        x_t = t(wl["x_t"][k])
        q = ln_swiglu(x_t, w["tgt"])
        outs = []
        for i in range(score_layers):
            Xt = ln_swiglu(X, w["hist"][i])
            mha = _torch_mha(d, H, w["WQ"][i], w["WK"][i], w["WV"][i], w["WO"][i])
            oi, _ = mha(q[None, None], Xt[None], Xt[None], need_weights=False)
            outs.append(oi[0, 0].detach())
            np.testing.assert_allclose(o[i, k], outs[-1].numpy(), rtol=1e-11, atol=1e-12)
            if i + 1 < score_layers:
                q = ln_swiglu(torch.cat(outs + [x_t]) @ t(w["WC"][i + 1]), w["fuse"][i + 1])
        zk = ln_swiglu(torch.cat(outs + [x_t]) @ t(w["WZ"]), w["zffn"], ln=False)
        np.testing.assert_allclose(z[k], zk.numpy(), rtol=1e-11, atol=1e-12)


def test_rlb_batched_equals_independent_targets():
    wl = _small_stca(2, users=2, m=5)
    z, o = R.stca_forward(wl)
    for u in range(2):
        for k in range(5):
            t = 5 * u + k
            single = dict(wl, x_t=wl["x_t"][t:t + 1], targets_per_user=np.array([1], np.int32),
                          lengths=wl["lengths"][u:u + 1],
                          ids=wl["ids"][wl["lengths"][:u].sum():wl["lengths"][:u + 1].sum()])
            z1, o1 = R.stca_forward(single)
            np.testing.assert_array_equal(z1[0], z[t])
            np.testing.assert_array_equal(o1[:, 0], o[:, t])


def test_history_permutation_invariance():
    wl = _small_stca(3, users=2, L=30, d=64, H=4, hidden=128, m=2)
    z, o = R.stca_forward(wl)
    perm = np.concatenate([np.random.default_rng(12).permutation(30), 30 + np.random.default_rng(13).permutation(30)])
    wl2 = dict(wl, ids=wl["ids"][perm], dt=wl["dt"][perm])
    z2, o2 = R.stca_forward(wl2)
    np.testing.assert_allclose(z2, z, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(o2, o, rtol=1e-11, atol=1e-12)


def test_earlier_layers_do_not_see_later_layers():
    """o^(1) of a 2-layer model equals o^(1) of the 1-layer model with the same layer-1 weights."""
    wl = _small_stca(2)
    _, o = R.stca_forward(wl)
    w = wl["weights"]
    d = wl["cfg"]["d"]
    g = _rng(14)
    w1 = dict(hist=w["hist"][:1], WQ=w["WQ"][:1], WK=w["WK"][:1], WV=w["WV"][:1], WO=w["WO"][:1],
              tgt=w["tgt"], WC=[None], fuse=[None], WZ=g.standard_normal((2 * d, d)) * 0.05,
              zffn=w["zffn"])
    _, o1 = R.stca_forward(dict(wl, cfg=dict(wl["cfg"], M=1), weights=w1))
    np.testing.assert_array_equal(o1[0], o[0])


def test_concat_order_puts_target_last():
    """[o^(1)|...|o^(i)|x_t]: with only the last d rows of W_C / W_Z nonzero, q^(2) and z
    depend on x_t alone, so changing the history leaves them unchanged."""
    wl = _small_stca(2)
    w = dict(wl["weights"])
    d = wl["cfg"]["d"]
    WZ = _f64(w["WZ"]).copy()
    WZ[:-d] = 0
    WC = _f64(w["WC"][1]).copy()
    WC[:-d] = 0
    w.update(WZ=WZ, WC=[None, WC])
    wl_a = dict(wl, weights=w)
    wl_b = dict(wl_a, ids=(wl["ids"] + 7) % 500)
    za, oa = R.stca_forward(wl_a)
    zb, ob = R.stca_forward(wl_b)
    np.testing.assert_allclose(za, zb, rtol=1e-12, atol=1e-13)
    assert np.abs(oa[1] - ob[1]).max() > 1e-3      # the history still moves o^(2) through K/V
    # and the opposite block assignment does depend on the history
    WZ2 = _f64(wl["weights"]["WZ"]).copy()
    WZ2[-d:] = 0
    w2 = dict(wl["weights"], WZ=WZ2)
    zc, _ = R.stca_forward(dict(wl, weights=w2))
    zd, _ = R.stca_forward(dict(wl, weights=w2, ids=(wl["ids"] + 7) % 500))
    assert np.abs(zc - zd).max() > 1e-4


def test_fused_query_is_layer_normed():
    wl = _small_stca(2, ln_affine="identity")
    cfg = wl["cfg"]
    X = R.gather_history(wl["table"], wl["ids"][:wl["lengths"][0]])
    KV = [R.stca_user_kv(X, wl["weights"], i, 1e-5) for i in range(cfg["M"])]
    _, _, qs = R.stca_target(wl["x_t"][0], KV, wl["weights"], cfg, return_queries=True)
    for q in qs:
        assert abs(q.mean()) < 1e-12 and abs(q.var() - 1) < 1e-3


def test_fp32_config_shapes():
    wl = make_stca(1)
    z, o = R.stca_forward(wl)
    assert z.shape == (4, 64) and o.shape == (1, 4, 64)
    assert np.isfinite(z).all()


# ---------------------------------------------------------------- pointwise ReLU TA


def test_pointwise_matches_definition_elementwise():
    wl = make_pointwise(users=3, L=40, L_lo=1, n_items=300)
    o = R.pointwise_relu_ta(wl)
    off = np.concatenate([[0], np.cumsum(wl["lengths"])])
    for b in range(3):
        E = R.to_f64(wl["table"][wl["ids"][off[b]:off[b + 1]]])
        q = R.to_f64(wl["q"][b])
        ref = [math.fsum(max(float(q @ E[j]) / math.sqrt(128), 0.0) * E[j, c] for j in range(len(E)))
               for c in range(128)]
        np.testing.assert_allclose(o[b], ref, rtol=1e-11, atol=1e-15)


# ---------------------------------------------------------------- HyFormer


def test_token_mix_involution_and_reshape():
    Q = _rng(15).standard_normal((32, 512))
    m = R.token_mix(Q)
    np.testing.assert_array_equal(R.token_mix(m), Q)
    np.testing.assert_array_equal(m, Q.reshape(32, 32, 16).transpose(1, 0, 2).reshape(32, 512))


def test_cross_attention_vs_torch_mha():
    g = _rng(16)
    d, H, L = 32, 4, 11
    Q, K, V = g.standard_normal((5, d)), g.standard_normal((L, d)), g.standard_normal((L, d))
    WQ, WO = g.standard_normal((d, d)), g.standard_normal((d, d))
    t = lambda a: torch.from_numpy(a)
    q = (t(Q) @ t(WQ)).reshape(5, H, d // H).transpose(0, 1)
    k = t(K).reshape(L, H, d // H).transpose(0, 1)
    v = t(V).reshape(L, H, d // H).transpose(0, 1)
    ref = F.scaled_dot_product_attention(q, k, v).transpose(0, 1).reshape(5, d) @ t(WO)
    np.testing.assert_allclose(R.cross_attention(Q, K, V, WQ, WO, H), ref.numpy(), rtol=1e-11, atol=1e-12)


def test_hyformer_zero_ffn_leaves_decoded_queries():
    """Per-token W2 = 0 makes the boost zero, so one block returns Q^ = CrossAttn(Q0, K, V);
    with a single repeated item per sequence, every query decodes to (SwiGLU(e) W_V) W_O."""
    wl = make_hyformer(users=2, L_feed=6, L_search=3, n_items=50, d=64, hidden=128, H=4,
                       blocks=1)
    wl["ids"] = [np.full_like(wl["ids"][0], 3), np.full_like(wl["ids"][1], 9)]
    for tok in wl["weights"]["blocks"][0]["tok"]:
        tok["W2"] = np.zeros_like(R.to_f64(tok["W2"]))
    out = R.hyformer_forward(wl)
    for s, item in enumerate((3, 9)):
        f = wl["weights"]["blocks"][0]["seq"][s]
        e = R.to_f64(wl["table"][item])
        expect = (R.swiglu(e, f) @ R.to_f64(f["WV"])) @ R.to_f64(f["WO"])
        for b in range(2):
            np.testing.assert_allclose(out[b, 16 * s:16 * s + 16], np.tile(expect, (16, 1)),
                                       rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("k", [5, 30])
def test_hyformer_per_token_ffn_index(k):
    """[hyformer] eq (14): mixed token k goes through its own SwiGLU (the k-th of T).  With
    every per-token W2 zero except token k's, the boost is zero on every row but k, so
    those rows equal the decoded queries Q^ exactly (eq 15), and row k differs from Q^ by
    the SwiGLU of mixed token k (eq 11-13) through token k's weights."""
    wl = make_hyformer(users=1, L_feed=9, L_search=4, n_items=60, d=64, hidden=128, H=4, blocks=1)
    wl["table"] = R.to_f64(wl["table"]) * 50.0   # rows of norm ~8, so the boost is not tiny
    tok = wl["weights"]["blocks"][0]["tok"]
    keep = {key: R.to_f64(v) for key, v in tok[k].items()}
    for f in tok:
        f["W2"] = np.zeros_like(R.to_f64(f["W2"]))
    qhat = R.hyformer_forward(wl)[0]          # all boosts zero: the decoded queries
    tok[k]["W2"] = keep["W2"]
    out = R.hyformer_forward(wl)[0]
    others = np.arange(32) != k
    np.testing.assert_array_equal(out[others], qhat[others])
    boost = R.swiglu(R.token_mix(qhat)[k], keep)
    assert np.abs(boost).max() > 1e-2 * np.abs(qhat[k]).max()
    np.testing.assert_allclose(out[k] - qhat[k], boost, rtol=1e-10, atol=1e-14)


def test_hyformer_residual_adds_boost():
    """With W_O = 0 the decoded queries are zero and the boost of zero is SwiGLU(0) = 0."""
    wl = make_hyformer(users=1, L_feed=5, L_search=4, n_items=50, d=64, hidden=128, H=4, blocks=2)
    for blk in wl["weights"]["blocks"]:
        for f in blk["seq"]:
            f["WO"] = np.zeros_like(R.to_f64(f["WO"]))
    np.testing.assert_array_equal(R.hyformer_forward(wl), 0)


def test_row_rel_err_metric():
    ref = np.array([[1.0, -4.0], [0.0, 0.0]])
    got = np.array([[1.1, -4.0], [1e-7, 0.0]])
    assert abs(R.row_rel_err(got, ref) - 0.1) < 1e-12
