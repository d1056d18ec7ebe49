"""Seeded generators for the five STCA workloads.

Shapes and distributions follow the workloads the STCA and HyFormer pages describe:
ultra-long histories (10K at inference, ~2K Beta-distributed lengths in training), Zipf
item popularity, many targets per request, and a 16-bin time-difference feature.  The
pages' own data (Douyin logs) is proprietary; these synthetic inputs stand in for it.

Every tensor comes from its own ``numpy.random.SeedSequence`` child, spawned in a fixed
order (lengths, ids, dt, targets/queries, table, dt table, weights in layer order), so a
size change in one tensor never shifts the draws of another.

Storage formats: ``fp32`` tensors are ``float32`` arrays; ``bf16`` tensors are ``uint16``
arrays holding bf16 bit patterns (round-to-nearest-even from a float32 draw).  LayerNorm
gamma/beta are always ``float32``.
"""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

# The five workloads, by number.  "hidden" is the SwiGLU hidden width.
STCA_CONFIGS = {
    1: dict(kind="stca", dtype="fp32", users=1, length="fixed", L=512, n_items=10_000,
            id_dist="uniform", d=64, H=2, hidden=128, m=4, M=1, score="softmax",
            time_buckets=0),
    2: dict(kind="stca", dtype="bf16", users=64, length="beta", L=2048, beta_a=2.0,
            n_items=1_000_000, id_dist="zipf", zipf_s=1.1, d=256, H=4, hidden=512, m=8,
            M=2, score="softmax", time_buckets=0),
    3: dict(kind="stca", dtype="bf16", users=256, length="fixed", L=10_000,
            n_items=4_000_000, id_dist="zipf", zipf_s=1.1, d=512, H=8, hidden=1024, m=32,
            M=3, score="softmax", time_buckets=16),
    4: dict(kind="pointwise", dtype="bf16", users=1024, length="uniform", L_lo=1000,
            L=10_000, n_items=2_000_000, id_dist="zipf", zipf_s=1.2, d=128),
    5: dict(kind="hyformer", dtype="bf16", users=128, L_feed=8192, L_search=1024,
            n_items=2_000_000, id_dist="zipf", zipf_s=1.1, d=512, H=8, hidden=1024,
            n_query=16, blocks=3),
}

_CHUNK_ROWS = 1 << 18


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Encode float32 values as bf16 bit patterns, rounding to nearest even."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounded = u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return (rounded >> np.uint32(16)).astype(np.uint16)


def _store(x: np.ndarray, dtype: str) -> np.ndarray:
    return bf16_bits(x) if dtype == "bf16" else np.ascontiguousarray(x, dtype=np.float32)


def _rng(ss: np.random.SeedSequence) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(ss))


def _normal_table(ss, rows: int, cols: int, std: float, dtype: str) -> np.ndarray:
    """N(0, std^2) table, drawn in fixed row chunks (one child seed each) on threads."""
    n_chunks = max(1, (rows + _CHUNK_ROWS - 1) // _CHUNK_ROWS)
    children = ss.spawn(n_chunks)
    out = np.empty((rows, cols), dtype=np.uint16 if dtype == "bf16" else np.float32)

    def fill(c):
        r0 = c * _CHUNK_ROWS
        r1 = min(rows, r0 + _CHUNK_ROWS)
        g = _rng(children[c])
        block = g.standard_normal((r1 - r0, cols), dtype=np.float32)
        block *= np.float32(std)
        out[r0:r1] = _store(block, dtype)

    workers = min(n_chunks, os.cpu_count() or 1, 16)
    if workers > 1:
        with ThreadPoolExecutor(workers) as ex:
            list(ex.map(fill, range(n_chunks)))
    else:
        for c in range(n_chunks):
            fill(c)
    return out


def _xavier(g: np.random.Generator, fan_in: int, fan_out: int, dtype: str) -> np.ndarray:
    a = math.sqrt(6.0 / (fan_in + fan_out))
    w = g.uniform(-a, a, size=(fan_in, fan_out)).astype(np.float32)
    return _store(w, dtype)


def _ln_params(g: np.random.Generator, d: int, affine: str):
    if affine == "identity":
        return np.ones(d, np.float32), np.zeros(d, np.float32)
    gamma = (1.0 + 0.1 * g.standard_normal(d)).astype(np.float32)
    beta = (0.1 * g.standard_normal(d)).astype(np.float32)
    return gamma, beta


def _zipf_ids(g: np.random.Generator, n: int, n_items: int, s: float) -> np.ndarray:
    """Bounded Zipf: P(rank r) proportional to r^-s over r = 1..n_items; id = r - 1."""
    ranks = np.arange(1, n_items + 1, dtype=np.float64)
    cdf = np.cumsum(ranks ** (-s))
    u = g.random(n) * cdf[-1]
    ids = np.searchsorted(cdf, u, side="right")
    return np.minimum(ids, n_items - 1).astype(np.int32)


def _ids(g, n, cfg):
    if cfg["id_dist"] == "uniform":
        return g.integers(0, cfg["n_items"], size=n, dtype=np.int64).astype(np.int32)
    return _zipf_ids(g, n, cfg["n_items"], cfg["zipf_s"])


def _lengths(g, cfg, users):
    kind = cfg["length"]
    if kind == "fixed":
        return np.full(users, cfg["L"], dtype=np.int32)
    if kind == "beta":
        x = g.beta(cfg["beta_a"], 1.0, size=users)
        return np.maximum(1, np.ceil(x * cfg["L"])).astype(np.int32)
    if kind == "uniform":
        return g.integers(cfg["L_lo"], cfg["L"] + 1, size=users, dtype=np.int64).astype(np.int32)
    raise ValueError(kind)


def _config(config_id: int, **over) -> dict:
    cfg = dict(STCA_CONFIGS[config_id])
    for k, v in over.items():
        if v is not None:
            cfg[k] = v
    return cfg


def _ffn(g, d, hidden, dtype, affine=None, ln=True):
    f = dict(W1=_xavier(g, d, hidden, dtype), W3=_xavier(g, d, hidden, dtype),
             W2=_xavier(g, hidden, d, dtype))
    if ln:
        f["gamma"], f["beta"] = _ln_params(g, d, affine)
    return f


def _stca_streams(config_id, seed, data_seed):
    ss = np.random.SeedSequence(1000 + config_id if seed is None else seed)
    streams = list(ss.spawn(7))  # lengths, ids, dt, x_t, table, dt table, weights
    if data_seed is not None:
        streams[:4] = np.random.SeedSequence(data_seed).spawn(4)
    return streams


def _stca_history(cfg, lengths, s_len, s_ids, s_dt):
    if lengths is None:
        lengths = _lengths(_rng(s_len), cfg, cfg["users"])
    lengths = np.asarray(lengths, dtype=np.int32)
    n_tok = int(lengths.sum())
    ids = _ids(_rng(s_ids), n_tok, cfg)
    dt = None
    if cfg["time_buckets"]:
        # seconds since the interaction: floor(2^U[0,16)) - 1
        e = _rng(s_dt).uniform(0.0, 16.0, size=n_tok)
        dt = (np.floor(np.exp2(e)) - 1).astype(np.int32)
    return lengths, ids, dt


def make_stca_history(config_id: int, *, users=None, L=None, n_items=None, seed=None, data_seed=None,
                      **over) -> dict:
    """The history side of ``make_stca`` alone (lengths, ids, dt: the same draws), without
    the table, targets and weights, for probes that only need the key lists."""
    cfg = _config(config_id, users=users, L=L, n_items=n_items, **over)
    assert cfg["kind"] == "stca"
    s_len, s_ids, s_dt = _stca_streams(config_id, seed, data_seed)[:3]
    lengths, ids, dt = _stca_history(cfg, None, s_len, s_ids, s_dt)
    return dict(cfg=cfg, lengths=lengths, ids=ids, dt=dt)


def make_stca(config_id: int, *, users=None, L=None, n_items=None, m=None, lengths=None,
              seed=None, data_seed=None, ln_affine="random", **over) -> dict:
    """Inputs and random-init weights for an STCA workload (configs 1-3 and variants).

    ``data_seed``, when given, draws the per-request inputs (lengths, ids, dt, x_t) from
    its own seed while the table and weights keep ``seed``: several replicas then serve
    different users with the same model.
    """
    cfg = _config(config_id, users=users, L=L, n_items=n_items, m=m, **over)
    assert cfg["kind"] == "stca"
    s_len, s_ids, s_dt, s_xt, s_tab, s_dtab, s_w = _stca_streams(config_id, seed, data_seed)
    dtype, d, hidden, M = cfg["dtype"], cfg["d"], cfg["hidden"], cfg["M"]
    lengths, ids, dt = _stca_history(cfg, lengths, s_len, s_ids, s_dt)
    B = len(lengths)
    tpu = np.full(B, cfg["m"], dtype=np.int32)
    t_tot = int(tpu.sum())
    x_t = _store(_rng(s_xt).standard_normal((t_tot, d), dtype=np.float32), dtype)
    table = _normal_table(s_tab, cfg["n_items"], d, 0.02, dtype)
    dt_table = None
    if cfg["time_buckets"]:
        dt_table = _normal_table(s_dtab, cfg["time_buckets"], d, 0.02, dtype)
    g = _rng(s_w)
    w = dict(hist=[], WQ=[], WK=[], WV=[], WO=[], WC=[None], fuse=[None])
    for _ in range(M):
        w["hist"].append(_ffn(g, d, hidden, dtype, ln_affine))
        for k in ("WQ", "WK", "WV", "WO"):
            w[k].append(_xavier(g, d, d, dtype))
    w["tgt"] = _ffn(g, d, hidden, dtype, ln_affine)
    for i in range(1, M):
        w["WC"].append(_xavier(g, (i + 1) * d, d, dtype))
        w["fuse"].append(_ffn(g, d, hidden, dtype, ln_affine))
    w["WZ"] = _xavier(g, (M + 1) * d, d, dtype)
    w["zffn"] = _ffn(g, d, hidden, dtype, ln=False)
    return dict(cfg=cfg, lengths=lengths, ids=ids, dt=dt, targets_per_user=tpu, x_t=x_t,
                table=table, dt_table=dt_table, weights=w)


def make_pointwise(config_id: int = 4, *, users=None, L=None, L_lo=None, n_items=None,
                   lengths=None, seed=None, **over) -> dict:
    """Inputs for pointwise ReLU target attention with fused lookup (config 4)."""
    cfg = _config(config_id, users=users, L=L, L_lo=L_lo, n_items=n_items, **over)
    assert cfg["kind"] == "pointwise"
    ss = np.random.SeedSequence(1000 + config_id if seed is None else seed)
    s_len, s_ids, s_q, s_tab = ss.spawn(4)
    if lengths is None:
        lengths = _lengths(_rng(s_len), cfg, cfg["users"])
    lengths = np.asarray(lengths, dtype=np.int32)
    ids = _ids(_rng(s_ids), int(lengths.sum()), cfg)
    q = _store(_rng(s_q).standard_normal((len(lengths), cfg["d"]), dtype=np.float32),
               cfg["dtype"])
    table = _normal_table(s_tab, cfg["n_items"], cfg["d"], 0.02, cfg["dtype"])
    return dict(cfg=cfg, lengths=lengths, ids=ids, q=q, table=table)


def make_hyformer(config_id: int = 5, *, users=None, L_feed=None, L_search=None,
                  n_items=None, seed=None, **over) -> dict:
    """Inputs and random-init weights for the multi-sequence query decoding workload."""
    cfg = _config(config_id, users=users, L_feed=L_feed, L_search=L_search,
                  n_items=n_items, **over)
    assert cfg["kind"] == "hyformer"
    ss = np.random.SeedSequence(1000 + config_id if seed is None else seed)
    s_len, s_ids, s_q, s_tab, s_w = ss.spawn(5)
    B, d, hidden, nq = cfg["users"], cfg["d"], cfg["hidden"], cfg["n_query"]
    dtype = cfg["dtype"]
    lengths = [np.full(B, cfg["L_feed"], np.int32), np.full(B, cfg["L_search"], np.int32)]
    gi = _rng(s_ids)
    ids = [_ids(gi, int(lengths[0].sum()), cfg), _ids(gi, int(lengths[1].sum()), cfg)]
    n_tokens = 2 * nq
    q0 = _store(_rng(s_q).standard_normal((B, n_tokens, d), dtype=np.float32), dtype)
    table = _normal_table(s_tab, cfg["n_items"], d, 0.02, dtype)
    g = _rng(s_w)
    blocks = []
    for _ in range(cfg["blocks"]):
        seqs = []
        for _s in range(2):
            f = _ffn(g, d, hidden, dtype, ln=False)
            for k in ("WQ", "WK", "WV", "WO"):
                f[k] = _xavier(g, d, d, dtype)
            seqs.append(f)
        tok = [_ffn(g, d, hidden, dtype, ln=False) for _t in range(n_tokens)]
        blocks.append(dict(seq=seqs, tok=tok))
    return dict(cfg=cfg, lengths=lengths, ids=ids, q0=q0, table=table,
                weights=dict(blocks=blocks))
