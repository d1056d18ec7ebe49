"""Per-kernel parity of libstca's steps against the fp64 oracle's component functions,
called through the kernel-level C entry points (include/stca_kernels.h)."""
import math

import numpy as np
import pytest
import torch

from oracle import stca_ref as R
from target_attention_b200 import binding as B
from tests._util import bf16_to_f64, bits_of, zeros_err

pytestmark = pytest.mark.gpu
dev = "cuda"


def _bf16(a64, seed=None):
    return torch.from_numpy(np.asarray(a64, np.float32)).to(torch.bfloat16).to(dev)


def _rng(seed):
    return np.random.default_rng(seed)


def _pack(W, mode, rows, row_offset=0, dst=None):
    """W: bf16 [K, N] device tensor -> packed [rows, K] via the library."""
    K, N = W.shape
    if dst is None:
        dst = torch.zeros(rows, K, dtype=torch.bfloat16, device=dev)
    B.check(B.stca_k_pack_weight(W, K, N, dst, mode, row_offset))
    return dst


# ---------------------------------------------------------------- a1: ragged offsets


def test_offsets_bit_exact_and_checks():
    lengths = _rng(0).integers(0, 3000, size=2500).astype(np.int32)
    lengths[[0, 7, 2499]] = 0
    L = torch.from_numpy(lengths).to(dev)
    off = torch.full((2501,), -1, dtype=torch.int32, device=dev)
    err = zeros_err()
    B.check(B.stca_k_offsets(L, 2500, off, int(lengths.sum()), err))
    torch.cuda.synchronize()
    np.testing.assert_array_equal(off.cpu().numpy(), R.exclusive_offsets(lengths))
    assert err.item() == 0
    # a total that does not match is reported, as is a negative length
    B.check(B.stca_k_offsets(L, 2500, off, int(lengths.sum()) + 1, err))
    torch.cuda.synchronize()
    assert err.item() == B.ERR_BAD_LENGTHS
    err.zero_()
    lengths[5] = -3
    B.check(B.stca_k_offsets(torch.from_numpy(lengths).to(dev), 2500, off, 0, err))
    torch.cuda.synchronize()
    assert err.item() == B.ERR_BAD_LENGTHS


def _clamped_offsets(lengths, expected):
    """Exclusive prefix sums with negative lengths counted as 0, each cut at `expected`."""
    return np.minimum(R.exclusive_offsets(np.maximum(lengths, 0)), max(expected, 0))


@pytest.mark.parametrize("case", ["far_above", "below", "negative", "zero_total"])
def test_offsets_are_clamped_to_the_declared_total(case):
    """Lengths that disagree with the declared total are reported and the offsets are cut
    at that total, so that no later kernel leaves buffers sized by it."""
    lengths = _rng(3).integers(0, 3000, size=2500).astype(np.int32)
    total = int(lengths.sum())
    if case == "far_above":
        lengths[1234] = 1_000_000_000  # the sum is ~1e9 above the declared total
        expected = total
    elif case == "below":
        expected = total + 777
    elif case == "negative":
        lengths[[3, 1800]] = [-5, -2_000_000_000]
        expected = total // 2
    else:
        expected = 0
    off = torch.full((2501,), -1, dtype=torch.int32, device=dev)
    err = zeros_err()
    B.check(B.stca_k_offsets(torch.from_numpy(lengths).to(dev), 2500, off, expected, err))
    torch.cuda.synchronize()
    got = off.cpu().numpy().astype(np.int64)
    np.testing.assert_array_equal(got, _clamped_offsets(lengths, expected))
    assert got[-1] <= expected and (np.diff(got) >= 0).all()
    assert err.item() == B.ERR_BAD_LENGTHS


# ---------------------------------------------------------------- weight packing


def test_pack_weight_layouts():
    W = _bf16(_rng(1).standard_normal((256, 384)))
    Wb = bits_of(W)
    p0 = _pack(W, 0, 384 + 5, row_offset=5)
    np.testing.assert_array_equal(bits_of(p0)[5:], Wb.T)
    p1 = _pack(W, 1, 768)
    p1 = _pack(W, 2, 768, dst=p1)
    pb = bits_of(p1)
    for n in range(384):
        g = (n // 128) * 256 + n % 128
        np.testing.assert_array_equal(pb[g], Wb[:, n])
        np.testing.assert_array_equal(pb[g + 128], Wb[:, n])


# ---------------------------------------------------------------- a2: fused gather (bit exact)


@pytest.mark.parametrize("K, with_dt", [(256, False), (512, True), (512, False)])
def test_fused_gather_is_bit_exact(K, with_dt):
    """Identity weights make the tensor-core GEMM copy its A operand, so the output rows
    are exactly the gathered rows: bf16(E[id] (+ T[bucket(dt)])), rounded from fp32."""
    g = _rng(2)
    n_items, M = 5000, 389                      # 4 tiles, ragged tail
    E = _bf16(g.standard_normal((n_items, K)) * 0.02)
    T = _bf16(g.standard_normal((16, K)) * 0.02) if with_dt else None
    ids = g.integers(0, n_items, size=M).astype(np.int32)
    dt = (np.floor(np.exp2(g.uniform(0, 16, size=M))) - 1).astype(np.int32) if with_dt else None
    Wp = torch.eye(K, dtype=torch.bfloat16, device=dev)           # packed identity [K, K]
    C = torch.full((M, K), float("nan"), dtype=torch.bfloat16, device=dev)
    X = torch.full((M, K), float("nan"), dtype=torch.bfloat16, device=dev)
    err = zeros_err()
    ids_t = torch.from_numpy(ids).to(dev)
    dt_t = torch.from_numpy(dt).to(dev) if with_dt else None
    B.check(B.stca_k_gemm_resident(1, 0, None, ids_t, dt_t, E, T, n_items, M, K, Wp, K, C, K, err, x_out=X))
    torch.cuda.synchronize()
    assert err.item() == 0
    Ef = E.float().cpu().numpy()[ids]
    if with_dt:
        Ef = Ef + T.float().cpu().numpy()[R.dt_bucket(dt)]    # fp32 sum, as the kernel
    expect = torch.from_numpy(Ef.astype(np.float32)).to(torch.bfloat16)
    np.testing.assert_array_equal(bits_of(C), bits_of(expect))
    # the written-through rows are the same bits, and a dense GEMM over them matches
    np.testing.assert_array_equal(bits_of(X), bits_of(expect))
    C2 = torch.full((M, K), float("nan"), dtype=torch.bfloat16, device=dev)
    B.check(B.stca_k_gemm_resident(0, 0, X, None, None, None, None, 0, M, K, Wp, K, C2, K, err))
    torch.cuda.synchronize()
    np.testing.assert_array_equal(bits_of(C2), bits_of(expect))


def test_fused_gather_flags_bad_ids():
    K, n_items, M = 256, 100, 130
    E = _bf16(_rng(3).standard_normal((n_items, K)))
    ids = np.arange(M, dtype=np.int32) % n_items
    ids[17] = n_items           # out of range
    ids[129] = -1
    Wp = torch.eye(K, dtype=torch.bfloat16, device=dev)
    C = torch.empty((M, K), dtype=torch.bfloat16, device=dev)
    err = zeros_err()
    B.check(B.stca_k_gemm_resident(1, 0, None, torch.from_numpy(ids).to(dev), None, E, None, n_items, M, K, Wp, K, C,
                                   K, err))
    torch.cuda.synchronize()
    assert err.item() == B.ERR_ID_OUT_OF_RANGE
    c = C.float().cpu().numpy()
    assert (c[17] == 0).all() and (c[129] == 0).all()
    np.testing.assert_array_equal(c[18], E.float().cpu().numpy()[18])


# ---------------------------------------------------------------- a3/a4: tensor-core GEMMs


def _close_bf16(got, ref, tol=1e-2):
    err = R.row_rel_err(got, ref)
    assert err <= tol, err


@pytest.mark.parametrize("K, N, M", [(256, 512, 300), (512, 1024, 257), (512, 256, 1)])
def test_gemm_resident_plain(K, N, M):
    g = _rng(4)
    A = _bf16(g.standard_normal((M, K)))
    W = _bf16(g.standard_normal((K, N)) / math.sqrt(K))
    Wp = _pack(W, 0, N)
    C = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    err = zeros_err()
    B.check(B.stca_k_gemm_resident(0, 0, A, None, None, None, None, 0, M, K, Wp, N, C, N, err))
    torch.cuda.synchronize()
    assert err.item() == 0
    _close_bf16(bf16_to_f64(C), bf16_to_f64(A) @ bf16_to_f64(W))


@pytest.mark.parametrize("K, hidden, M", [(256, 512, 200), (512, 1024, 390)])
def test_gemm_gather_swiglu(K, hidden, M):
    g = _rng(5)
    n_items = 3000
    E = _bf16(g.standard_normal((n_items, K)) * 0.5)
    ids = g.integers(0, n_items, size=M).astype(np.int32)
    W1 = _bf16(g.standard_normal((K, hidden)) / math.sqrt(K))
    W3 = _bf16(g.standard_normal((K, hidden)) / math.sqrt(K))
    Wp = _pack(W1, 1, 2 * hidden)
    _pack(W3, 2, 2 * hidden, dst=Wp)
    C = torch.empty((M, hidden), dtype=torch.bfloat16, device=dev)
    err = zeros_err()
    B.check(B.stca_k_gemm_resident(1, 1, None, torch.from_numpy(ids).to(dev), None, E, None, n_items, M, K, Wp,
                                   hidden, C, hidden, err))
    torch.cuda.synchronize()
    assert err.item() == 0
    X = bf16_to_f64(E)[ids]
    ref = R.silu(X @ bf16_to_f64(W1)) * (X @ bf16_to_f64(W3))
    _close_bf16(bf16_to_f64(C), ref)


@pytest.mark.parametrize("K, N, M, ln", [(1024, 512, 333, True), (512, 256, 129, True), (1024, 512, 200, False)])
def test_gemm_rowwise(K, N, M, ln):
    g = _rng(6)
    A = _bf16(g.standard_normal((M, K)))
    W = _bf16(g.standard_normal((K, N)) / math.sqrt(K))
    Wp = _pack(W, 0, N)
    gamma = torch.from_numpy((1 + 0.1 * g.standard_normal(N)).astype(np.float32)).to(dev)
    beta = torch.from_numpy((0.1 * g.standard_normal(N)).astype(np.float32)).to(dev)
    C = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    err = zeros_err()
    B.check(B.stca_k_gemm_rowwise(2 if ln else 0, A, M, K, Wp, N, gamma if ln else None, beta if ln else None, 1e-5,
                                  C, N, err))
    torch.cuda.synchronize()
    assert err.item() == 0
    Y = bf16_to_f64(A) @ bf16_to_f64(W)
    if ln:
        Y = R.layer_norm(Y, gamma.cpu().numpy(), beta.cpu().numpy(), 1e-5)
    _close_bf16(bf16_to_f64(C), Y)


@pytest.mark.parametrize("M, layers, hidden, with_dt", [(700, 2, 512, False), (3000 + 77, 3, 256, True),
                                                         (130, 1, 512, False)])
def test_ffn_fused_layernorm_rows(M, layers, hidden, with_dt):
    """The fused history FFN (d = 256): per layer, rstd (y' - mean gamma) + beta against the
    oracle's LN(SwiGLU(X)) of the gathered rows; several row tiles per CTA pair, a ragged
    tail, one to three layers, with and without the time-bucket row."""
    g = _rng(12)
    d, n_items = 256, 5000
    E = _bf16(g.standard_normal((n_items, d)) * 0.5)
    ids = g.integers(0, n_items, size=M).astype(np.int32)
    dt = np.floor(2.0 ** g.uniform(0, 16, M)).astype(np.int32) - 1 if with_dt else None
    T = _bf16(g.standard_normal((16, d)) * 0.5) if with_dt else None
    W1s, W3s, W2s, gam, bet = [], [], [], [], []
    W13p = torch.zeros((layers * 2 * hidden, d), dtype=torch.bfloat16, device=dev)
    W2p = torch.zeros((layers * d, hidden), dtype=torch.bfloat16, device=dev)
    for l in range(layers):
        W1s.append(_bf16(g.standard_normal((d, hidden)) / math.sqrt(d)))
        W3s.append(_bf16(g.standard_normal((d, hidden)) / math.sqrt(d)))
        W2s.append(_bf16(g.standard_normal((hidden, d)) / math.sqrt(hidden)))
        _pack(W1s[-1], 1, 2 * hidden, dst=W13p[l * 2 * hidden:(l + 1) * 2 * hidden])
        _pack(W3s[-1], 2, 2 * hidden, dst=W13p[l * 2 * hidden:(l + 1) * 2 * hidden])
        _pack(W2s[-1], 0, d, dst=W2p[l * d:(l + 1) * d])
        gam.append(torch.from_numpy((1 + 0.1 * g.standard_normal(d)).astype(np.float32)).to(dev))
        bet.append(0.1 * g.standard_normal(d))
    stride = (M + 255) // 256 * 256
    Y = torch.full((layers * stride, d), float("nan"), dtype=torch.bfloat16, device=dev)
    stats = torch.full((layers * stride, 2), float("nan"), dtype=torch.float32, device=dev)
    err = zeros_err()
    B.check(B.stca_k_ffn_fused(torch.from_numpy(ids).to(dev), None if dt is None else torch.from_numpy(dt).to(dev),
                               E, T, n_items, M, layers, hidden, W13p, W2p, gam, 1e-5, Y, stride, stats, err))
    torch.cuda.synchronize()
    assert err.item() == 0
    X = R.gather_history(E.cpu().view(torch.int16).numpy().view(np.uint16), ids, dt,
                         None if T is None else T.cpu().view(torch.int16).numpy().view(np.uint16))
    Yh, st = bf16_to_f64(Y), stats.cpu().numpy().astype(np.float64)
    for l in range(layers):
        ffn = dict(W1=bf16_to_f64(W1s[l]), W3=bf16_to_f64(W3s[l]), W2=bf16_to_f64(W2s[l]),
                   gamma=gam[l].cpu().numpy(), beta=bet[l])
        ref = R.ffn_ln(X, ffn, 1e-5)
        rows = slice(l * stride, l * stride + M)
        mean, rstd = st[rows, :1], st[rows, 1:]
        got = rstd * (Yh[rows] - mean * ffn["gamma"]) + bet[l]
        e = R.row_rel_err(got, ref)
        print(f"fused FFN layer {l}: row-relative error {e:.2e}")
        assert e <= 2e-2, (l, e)


# ---------------------------------------------------------------- a5/a8/a9: target-side GEMMs


def _f32(a):
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(dev)


@pytest.mark.parametrize("M, K, N, dual, split, resid", [
    (8192 + 77, 512, 512, False, False, False),   # many row tiles and a ragged tail
    (4096, 512, 512, False, False, True),         # 128-column tiles (a 256-wide grid fills too few SMs)
    (512, 256, 256, False, False, False),         # 64-column tiles
    (300, 1536, 512, False, True, True),          # two concatenated A blocks, residual
    (129, 512, 1024, True, False, False),         # SwiGLU pair
    (1, 1024, 96, False, False, False),           # one row; N not a multiple of the tile
])
def test_query_gemm_keeps_fp32_accuracy(M, K, N, dual, split, resid):
    """The tensor-core target-side GEMM splits fp32 activations into two bf16 terms, so the
    result matches the fp64 product of the fp32 inputs far more closely than one bf16
    rounding of A would (2^-9)."""
    g = _rng(21 + M)
    lda = K + (512 if split else 0)
    A = g.standard_normal((M, lda)).astype(np.float32)
    ksplit, kshift = ((K // 3) // 64 * 64, 512) if split else (K, 0)
    Al = np.concatenate([A[:, :ksplit], A[:, ksplit + kshift:K + kshift]], axis=1) if split else A[:, :K]
    Al = Al.astype(np.float64)
    W1 = _bf16(g.standard_normal((K, N)) / math.sqrt(K))
    if dual:
        W3 = _bf16(g.standard_normal((K, N)) / math.sqrt(K))
        Wp = _pack(W1, 1, 2 * N)
        _pack(W3, 2, 2 * N, dst=Wp)
        ref = R.silu(Al @ bf16_to_f64(W1)) * (Al @ bf16_to_f64(W3))
    else:
        Wp = _pack(W1, 0, N)
        ref = Al @ bf16_to_f64(W1)
    Rt = None
    if resid:
        Rm = g.standard_normal((M, N)).astype(np.float32)
        Rt = _f32(Rm)
        ref = ref + Rm
    C = torch.full((M, N), float("nan"), dtype=torch.float32, device=dev)
    err = zeros_err()
    B.check(B.stca_k_gemm_query(_f32(A), lda, M, K, ksplit, kshift, Wp, N, dual, Rt, N, C, N, err))
    torch.cuda.synchronize()
    assert err.item() == 0
    got = C.cpu().numpy().astype(np.float64)
    rel = np.abs(got - ref).max(axis=1) / np.maximum(np.abs(ref).max(axis=1), 1e-30)
    print(f"query GEMM M={M} K={K} N={N} dual={dual}: max row rel err {rel.max():.2e}")
    assert rel.max() < 3e-5


# ---------------------------------------------------------------- a6/a7: attention + merge


def _attention_case(kv_bf16, d, H, lengths, targets, splits, score, seed):
    g = _rng(seed)
    n_tok, T = int(sum(lengths)), int(sum(targets))
    KV = g.standard_normal((max(n_tok, 1), 2 * d))
    Q = g.standard_normal((max(T, 1), d)).astype(np.float32)
    if kv_bf16:
        KVt = _bf16(KV)
        KV64 = bf16_to_f64(KVt)
    else:
        KVt = torch.from_numpy(KV.astype(np.float32)).to(dev)
        KV64 = KV.astype(np.float32).astype(np.float64)
    hoff = R.exclusive_offsets(lengths)
    toff = R.exclusive_offsets(targets)
    Bu = len(lengths)
    part_acc = torch.empty((splits, max(T, 1), d), dtype=torch.float32, device=dev)
    part_ml = torch.empty((splits, max(T, 1), H, 2), dtype=torch.float32, device=dev)
    out = torch.full((max(T, 1), d), float("nan"), dtype=torch.float32, device=dev)
    err = zeros_err()
    B.check(B.stca_k_attention(1 if kv_bf16 else 0, torch.from_numpy(Q).to(dev), KVt,
                               torch.from_numpy(hoff.astype(np.int32)).to(dev),
                               torch.from_numpy(toff.astype(np.int32)).to(dev), Bu, T, d, H, splits, score,
                               part_acc, part_ml, out, err))
    torch.cuda.synchronize()
    assert err.item() == 0
    dh = d // H
    ref = np.zeros((T, d))
    for u in range(Bu):
        rows = KV64[hoff[u]:hoff[u + 1]]
        for t in range(toff[u], toff[u + 1]):
            for h in range(H):
                cols = slice(h * dh, (h + 1) * dh)
                if kv_bf16:  # [N, H, 2 d_h]: head h's K then V in one segment
                    K_h, V_h = rows[:, 2 * h * dh:(2 * h + 1) * dh], rows[:, (2 * h + 1) * dh:(2 * h + 2) * dh]
                else:        # [N, 2d]: K in [0, d), V in [d, 2d)
                    K_h, V_h = rows[:, cols], rows[:, d:][:, cols]
                ref[t, cols] = R.head_attention(Q[t, cols].astype(np.float64), K_h, V_h,
                                                "softmax" if score == 0 else "relu", 1 / math.sqrt(dh))
    return out.cpu().numpy()[:T], ref


@pytest.mark.parametrize("score", [0, 1])
@pytest.mark.parametrize("splits", [1, 3, 16])
def test_attention_bf16(score, splits):
    lengths = [0, 1, 31, 33, 700, 2049, 5]
    targets = [2, 1, 16, 17, 33, 40, 0]
    got, ref = _attention_case(True, 256, 4, lengths, targets, splits, score, seed=7 + score)
    # per-head rows: compare each (target, head) block on its own scale
    err = R.row_rel_err(got.reshape(-1, 64), ref.reshape(-1, 64))
    assert err <= 2e-2, err
    # the empty history gives exactly zero
    assert (got[:2] == 0).all()


@pytest.mark.parametrize("score", [0, 1])
@pytest.mark.parametrize("splits", [1, 3])
def test_attention_bf16_gathered_weighted_keys(score, splits):
    """Keys gathered by row index with multiplicities (the compacted form): a key that
    stands for c tokens must act like c copies of itself.  Each user's slot range is longer
    than its key count (kv_len < allotted), rows repeat across users, and the reference
    expands every key into its copies."""
    g = _rng(13 + score)
    d, H, dh, U = 256, 4, 64, 3000
    lengths = np.array([0, 1, 33, 700, 2049, 5], np.int32)     # keys per user
    slack = np.array([3, 0, 7, 1, 0, 2], np.int32)             # unused slots after them
    targets = np.array([2, 1, 17, 33, 40, 3], np.int32)
    hoff = R.exclusive_offsets(lengths + slack)
    toff = R.exclusive_offsets(targets)
    n_slots, T = int(hoff[-1]), int(toff[-1])
    rows = g.integers(0, U, size=n_slots).astype(np.int32)
    mult = g.integers(1, 6, size=n_slots).astype(np.int32)
    KVt = _bf16(g.standard_normal((U, 2 * d)))
    KV64 = bf16_to_f64(KVt)
    Q = g.standard_normal((T, d)).astype(np.float32)
    part_acc = torch.empty((splits, T, d), dtype=torch.float32, device=dev)
    part_ml = torch.empty((splits, T, H, 2), dtype=torch.float32, device=dev)
    out = torch.full((T, d), float("nan"), dtype=torch.float32, device=dev)
    err = zeros_err()
    i32 = lambda x: torch.from_numpy(np.ascontiguousarray(x, np.int32)).to(dev)
    B.check(B.stca_k_attention_rows(1, torch.from_numpy(Q).to(dev), KVt, i32(hoff), i32(toff), i32(rows),
                                    i32(lengths), i32(mult), len(lengths), T, d, H, splits, score, part_acc, part_ml,
                                    out, err))
    torch.cuda.synchronize()
    assert err.item() == 0
    got = out.cpu().numpy()
    ref = np.zeros((T, d))
    for u in range(len(lengths)):
        ent = slice(hoff[u], hoff[u] + lengths[u])
        expanded = KV64[np.repeat(rows[ent], mult[ent])]
        for t in range(toff[u], toff[u + 1]):
            for h in range(H):
                K_h, V_h = expanded[:, 2 * h * dh:(2 * h + 1) * dh], expanded[:, (2 * h + 1) * dh:(2 * h + 2) * dh]
                cols = slice(h * dh, (h + 1) * dh)
                ref[t, cols] = R.head_attention(Q[t, cols].astype(np.float64), K_h, V_h,
                                                "softmax" if score == 0 else "relu", 1 / math.sqrt(dh))
    e = R.row_rel_err(got.reshape(-1, dh), ref.reshape(-1, dh))
    print(f"gathered weighted keys: row-relative error {e:.2e}")
    assert e <= 2e-2, e
    assert (got[:2] == 0).all()


@pytest.mark.parametrize("score", [0, 1])
def test_attention_f32(score):
    lengths = [0, 1, 9, 600]
    targets = [1, 3, 4, 4]
    got, ref = _attention_case(False, 64, 2, lengths, targets, 2, score, seed=9)
    err = R.row_rel_err(got.reshape(-1, 32), ref.reshape(-1, 32))
    assert err <= 1e-5, err
    assert (got[:1] == 0).all()


# ---------------------------------------------------------------- persistent tile walks


def _rows_sample(M):
    return np.unique(np.concatenate([np.arange(0, M, 97), np.arange(max(0, M - 300), M)]))


@pytest.mark.parametrize("with_dt", [False, True])
def test_gather_swiglu_many_tiles_per_pair(with_dt):
    """M spans several 256-row tiles per CTA pair, so every barrier phase wraps."""
    g = _rng(11)
    K, hidden, n_items, M = 512, 1024, 200_000, 41_000
    E = _bf16(g.standard_normal((n_items, K)) * 0.5)
    T = _bf16(g.standard_normal((16, K)) * 0.5) if with_dt else None
    ids = g.integers(0, n_items, size=M).astype(np.int32)
    dt = (np.floor(np.exp2(g.uniform(0, 16, size=M))) - 1).astype(np.int32) if with_dt else None
    W1 = _bf16(g.standard_normal((K, hidden)) / math.sqrt(K))
    W3 = _bf16(g.standard_normal((K, hidden)) / math.sqrt(K))
    Wp = _pack(W1, 1, 2 * hidden)
    _pack(W3, 2, 2 * hidden, dst=Wp)
    C = torch.empty((M, hidden), dtype=torch.bfloat16, device=dev)
    Xw = torch.empty((M, K), dtype=torch.bfloat16, device=dev)
    err = zeros_err()
    P = torch.empty((M, 2 * hidden), dtype=torch.bfloat16, device=dev)
    B.check(B.stca_k_gemm_resident(1, 1, None, torch.from_numpy(ids).to(dev),
                                   torch.from_numpy(dt).to(dev) if with_dt else None, E, T, n_items, M, K, Wp,
                                   hidden, C, hidden, err, x_out=Xw, p_out=P))
    torch.cuda.synchronize()
    assert err.item() == 0
    # the pre-activations [X W1 | X W3]: the plain GEMM over the written-through rows gives
    # the same fp32 accumulators (same K order), so the same bits
    Pp = _pack(W1, 0, 2 * hidden)
    _pack(W3, 0, 2 * hidden, dst=Pp, row_offset=hidden)
    P2 = torch.empty_like(P)
    B.check(B.stca_k_gemm_resident(0, 0, Xw, None, None, None, None, 0, M, K, Pp, 2 * hidden, P2, 2 * hidden, err))
    torch.cuda.synchronize()
    np.testing.assert_array_equal(bits_of(P), bits_of(P2))
    # every written-through row, bit for bit (fp32 sum rounded once to bf16)
    Ef = E.float().cpu().numpy()[ids]
    if with_dt:
        Ef = Ef + T.float().cpu().numpy()[R.dt_bucket(dt)]
    np.testing.assert_array_equal(bits_of(Xw), bits_of(torch.from_numpy(Ef.astype(np.float32)).to(torch.bfloat16)))
    rows = _rows_sample(M)
    X = bf16_to_f64(E)[ids[rows]]
    if with_dt:
        X = X + bf16_to_f64(T)[R.dt_bucket(dt[rows])]
    ref = R.silu(X @ bf16_to_f64(W1)) * (X @ bf16_to_f64(W3))
    _close_bf16(bf16_to_f64(C)[rows], ref)


def test_resident_plain_many_tiles_per_pair():
    g = _rng(12)
    K, N, M = 512, 1024, 45_123
    A = _bf16(g.standard_normal((M, K)))
    W = _bf16(g.standard_normal((K, N)) / math.sqrt(K))
    Wp = _pack(W, 0, N)
    C = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    err = zeros_err()
    B.check(B.stca_k_gemm_resident(0, 0, A, None, None, None, None, 0, M, K, Wp, N, C, N, err))
    torch.cuda.synchronize()
    assert err.item() == 0
    rows = _rows_sample(M)
    _close_bf16(bf16_to_f64(C)[rows], bf16_to_f64(A)[rows] @ bf16_to_f64(W))


@pytest.mark.parametrize("N", [256, 512])
def test_rowwise_ln_many_tiles_per_pair(N):
    g = _rng(13)
    K, M = 1024, 40_007
    A = _bf16(g.standard_normal((M, K)))
    W = _bf16(g.standard_normal((K, N)) / math.sqrt(K))
    Wp = _pack(W, 0, N)
    gamma = torch.from_numpy((1 + 0.1 * g.standard_normal(N)).astype(np.float32)).to(dev)
    beta = torch.from_numpy((0.1 * g.standard_normal(N)).astype(np.float32)).to(dev)
    C = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    err = zeros_err()
    B.check(B.stca_k_gemm_rowwise(2, A, M, K, Wp, N, gamma, beta, 1e-5, C, N, err))
    torch.cuda.synchronize()
    assert err.item() == 0
    rows = _rows_sample(M)
    Y = R.layer_norm(bf16_to_f64(A)[rows] @ bf16_to_f64(W), gamma.cpu().numpy(), beta.cpu().numpy(), 1e-5)
    _close_bf16(bf16_to_f64(C)[rows], Y)
