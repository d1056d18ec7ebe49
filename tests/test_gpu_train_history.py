"""Backward of one layer's history side on the GPU (X -> LN(SwiGLU(X)) -> [K | V], then the
lookup), as ``target_attention_b200.training.HistoryLayerBackward`` composes it from the
library's kernel-level entries, against the fp64 oracle
(``stca_grad.history_layer_bwd`` and ``table_rows_bwd``) on the same bf16 inputs.

The forward values the backward needs are recomputed on the GPU the way a training step
would (the gathered rows X, x W1 | x W3, the SwiGLU output A and y = A W2); the upstream
dK, dV are random, rounded to bf16 as the attention backward would hand them over.
Gradients are compared normwise per tensor: max |g - r| / max |r| <= 2e-2 (bf16 operands
and intermediates, fp32 accumulation).  The weight-gradient GEMM and the LayerNorm
backward are also checked alone against float64 on their exact bf16 inputs."""
import numpy as np
import pytest
import torch

from oracle import stca_grad as G
from oracle import stca_ref as R
from target_attention_b200 import binding as B
from target_attention_b200.training import HistoryLayerBackward
from tests._util import bf16_to_f64
from workloads import make_stca

pytestmark = pytest.mark.gpu
dev = "cuda"
TOL = 2e-2


def up16(bits):
    """bf16 bit patterns (uint16) -> device bf16 tensor."""
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)


def to_bf16(x):
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.bfloat16).to(dev)


def ws(nbytes):
    return torch.empty(max(int(nbytes), 16), dtype=torch.uint8, device=dev)


def normwise(got, ref):
    ref = np.asarray(ref, np.float64)
    return float(np.abs(np.asarray(got, np.float64) - ref).max() / max(np.abs(ref).max(), 1e-30))


@pytest.mark.parametrize("impl", [0, 1])
@pytest.mark.parametrize("M, K, N, lda_pad", [(1000, 128, 128, 0), (5003, 256, 512, 8), (77, 512, 256, 0),
                                               (40_000, 128, 768, 0), (300, 384, 256, 16), (64, 256, 1024, 0),
                                               (200_000, 256, 1024, 0), (3, 128, 256, 0)])
def test_gemm_wgrad_matches_float64(M, K, N, lda_pad, impl):
    """C = A^T G over ragged token counts (a partial last stage, several token slices, one
    stage, fewer tokens than one stage), padded leading dimensions, N a multiple of 128 but
    not of 256, and C += A^T G with accumulate; impl 0 the tcgen05 kernel, 1 mma.sync.

    The bar is elementwise against the magnitude of the sum's terms, |C - ref| <= 1e-6
    sum_t |a_t| |g_t|: fp32 accumulation of n terms errs by at most about n_adds 2^-24
    times that sum, so this is the scale its rounding lives on (random data: the sum
    itself is ~sqrt(M) times smaller, and a fixed bar on it would tighten as M grows).
    Both kernels measure about 2e-7 at 200K tokens (11K-token slices)."""
    g = np.random.default_rng(M)
    A = to_bf16(g.standard_normal((M, K + lda_pad)))
    Gm = to_bf16(g.standard_normal((M, N)))
    C = torch.full((K, N), float("nan"), device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    w = ws(B.stca_k_gemm_wgrad_workspace_bytes(M, K, N))
    B.check(B.stca_k_gemm_wgrad(A, K + lda_pad, Gm, N, M, K, N, C, N, 0, w, w.numel(), impl=impl, err=err))
    a64, g64 = A[:, :K].double(), Gm.double()
    ref = (a64.T @ g64).cpu().numpy()
    mag = (a64.abs().T @ g64.abs()).cpu().numpy()
    got = C.cpu().numpy()
    assert err.item() == 0
    assert (np.abs(got - ref) <= 1e-6 * mag).all(), float((np.abs(got - ref) / mag).max())
    B.check(B.stca_k_gemm_wgrad(A, K + lda_pad, Gm, N, M, K, N, C, N, 1, w, w.numel(), impl=impl, err=err))
    assert (np.abs(C.cpu().numpy() - 2 * ref) <= 2e-6 * mag).all()
    # the partials are added in a fixed order: the same bits every run
    C2 = torch.empty_like(C)
    B.check(B.stca_k_gemm_wgrad(A, K + lda_pad, Gm, N, M, K, N, C2, N, 0, w, w.numel(), impl=impl, err=err))
    assert torch.equal(C2.cpu(), torch.from_numpy(got))
    assert err.item() == 0


@pytest.mark.parametrize("d", [256, 512])
@pytest.mark.parametrize("fp32", [0, 1])
def test_layer_norm_bwd_and_fwd_match_oracle(d, fp32):
    """LayerNorm backward (bf16 history rows, fp32 target rows) and the forward the training
    step recomputes with."""
    g = np.random.default_rng(d + fp32)
    M, eps = 333, 1e-5
    cast = (lambda x: torch.from_numpy(np.asarray(x, np.float32)).to(dev)) if fp32 else to_bf16
    y = cast(g.standard_normal((M, d)) * 2 + 0.5)
    dxt = cast(g.standard_normal((M, d)))
    gamma = torch.from_numpy(g.standard_normal(d).astype(np.float32)).to(dev)
    beta = torch.from_numpy(g.standard_normal(d).astype(np.float32)).to(dev)
    dy, xt, xf = torch.empty_like(y), torch.empty_like(y), torch.empty_like(y)
    dg = torch.empty(d, device=dev)
    db = torch.empty(d, device=dev)
    w = ws(B.stca_k_layer_norm_bwd_workspace_bytes(M, d))
    B.check(B.stca_k_layer_norm_bwd(y, dxt, M, d, gamma, beta, eps, dy, xt, dg, db, 0, w, w.numel(), fp32=fp32))
    B.check(B.stca_k_layer_norm(y, d, fp32, M, d, gamma, beta, eps, xf, d, fp32))
    y64, dxt64 = bf16_to_f64(y), bf16_to_f64(dxt)
    rdy, rdg, rdb = G.layer_norm_bwd(y64, gamma.cpu().numpy(), beta.cpu().numpy(), eps, dxt64)
    bar = 1e-5 if fp32 else 1e-2
    assert normwise(bf16_to_f64(dy), rdy) < bar
    assert normwise(dg.cpu().numpy(), rdg) < 1e-4 and normwise(db.cpu().numpy(), rdb) < 1e-4
    rxt = R.layer_norm(y64, gamma.cpu().numpy(), beta.cpu().numpy(), eps)
    assert normwise(bf16_to_f64(xt), rxt) < bar
    assert normwise(bf16_to_f64(xf), rxt) < bar


def test_swiglu_bwd_fp32_and_bf16_copy():
    g = np.random.default_rng(9)
    M, h = 77, 64
    P = torch.from_numpy(g.standard_normal((M, 2 * h)).astype(np.float32)).to(dev)
    dA = torch.from_numpy(g.standard_normal((M, h)).astype(np.float32)).to(dev)
    dP, A = torch.empty_like(P), torch.empty_like(dA)
    B.check(B.stca_k_swiglu_bwd(P, dA, M, h, dP, A, fp32=1))
    p, da = P.cpu().double().numpy(), dA.cpu().double().numpy()
    a, b = p[:, :h], p[:, h:]
    sig = 1 / (1 + np.exp(-a))
    assert normwise(A.cpu().numpy(), a * sig * b) < 1e-5
    assert normwise(dP.cpu().numpy()[:, :h], da * b * G.silu_grad(a)) < 1e-5
    assert normwise(dP.cpu().numpy()[:, h:], da * a * sig) < 1e-5
    out = torch.empty((M, h), dtype=torch.bfloat16, device=dev)
    B.check(B.stca_k_f32_to_bf16(P, 2 * h, M, h, out, h))       # a strided block, rounded to bf16
    assert torch.equal(out, P[:, :h].to(torch.bfloat16))


@pytest.mark.parametrize("d", [128, 256, 512])
@pytest.mark.parametrize("ids_kind", ["hot", "single", "uniform"])
def test_table_rows_bwd_matches_oracle(d, ids_kind):
    """The lookup's backward dE[ids] += dX, dT[bucket] += dX (stca_grad.table_rows_bwd) on
    5003 tokens (ragged against the 1024-token groups): half the tokens on one id, or every
    token on one id, or uniform ids; with time buckets.  d = 128 runs the per-token kernel,
    256 and 512 the grouped one."""
    g = np.random.default_rng(d)
    M, n_items = 5003, 700
    ids = g.integers(0, n_items, M)
    if ids_kind == "hot":
        ids[g.random(M) < 0.5] = 17
    elif ids_kind == "single":
        ids[:] = 3
    dt = g.integers(0, 10 ** 6, M)
    dX16 = to_bf16(g.standard_normal((M, d)))
    ids_t = torch.from_numpy(ids.astype(np.int32)).to(dev)
    dt_t = torch.from_numpy(dt.astype(np.int32)).to(dev)
    dtab = torch.zeros((n_items, d), device=dev)
    ddt = torch.zeros((16, d), device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    B.check(B.stca_k_table_rows_bwd(dX16, M, d, ids_t, dt_t, n_items, dtab, ddt, err))
    rtab, rdt = np.zeros((n_items, d)), np.zeros((16, d))
    G.table_rows_bwd(rtab, rdt, ids, dt, bf16_to_f64(dX16))
    assert err.item() == 0
    assert normwise(dtab.cpu().numpy(), rtab) < 1e-5
    assert normwise(ddt.cpu().numpy(), rdt) < 1e-5
    # an id outside the table is reported and its row is skipped
    ids2 = ids.copy()
    ids2[100] = n_items
    B.check(B.stca_k_table_rows_bwd(dX16, M, d, torch.from_numpy(ids2.astype(np.int32)).to(dev), None, n_items,
                                    dtab.zero_(), None, err))
    assert err.item() == B.ERR_ID_OUT_OF_RANGE
    keep = np.ones(M, bool)
    keep[100] = False
    rtab = np.zeros((n_items, d))
    G.table_rows_bwd(rtab, None, ids[keep], None, bf16_to_f64(dX16)[keep])
    assert normwise(dtab.cpu().numpy(), rtab) < 1e-5


@pytest.mark.parametrize("config", [2, 3])
def test_history_layer_backward_matches_oracle(config):
    """config 2's shape (d = 256, h = 512, no time feature) and config 3's (d = 512,
    h = 1024, 16 time buckets), two users of ragged length, layer 0's weights."""
    wl = make_stca(config, users=2, L=1500 if config == 2 else 900, n_items=3000)
    cfg = wl["cfg"]
    d, h, eps = cfg["d"], cfg["hidden"], 1e-5
    w = wl["weights"]
    ffn, WK, WV = w["hist"][0], w["WK"][0], w["WV"][0]
    ids, dt = wl["ids"], wl["dt"]
    M = len(ids)
    g = np.random.default_rng(5)
    bf16_round = lambda x: torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).double().numpy()
    dK, dV = bf16_round(g.standard_normal((M, d))), bf16_round(g.standard_normal((M, d)))
    # device inputs
    table, W1, W3, W2 = up16(wl["table"]), up16(ffn["W1"]), up16(ffn["W3"]), up16(ffn["W2"])
    dtab = up16(wl["dt_table"]) if dt is not None else None
    ids_t = torch.from_numpy(ids.astype(np.int32)).to(dev)
    dt_t = torch.from_numpy(dt.astype(np.int32)).to(dev) if dt is not None else None
    gamma = torch.from_numpy(R.to_f64(ffn["gamma"]).astype(np.float32)).to(dev)
    beta = torch.from_numpy(R.to_f64(ffn["beta"]).astype(np.float32)).to(dev)
    n_items = int(wl["table"].shape[0])
    # ---- forward values recomputed, then the backward (target_attention_b200.training)
    layer = HistoryLayerBackward(M, d, h, W1, W3, W2, up16(WK), up16(WV), gamma, beta, eps)
    layer.recompute(ids_t, dt_t, table, dtab, n_items)
    dKV = np.zeros((M, 2 * d))
    for hh in range(d // 64):                            # the K/V rows' [K_h | V_h] columns
        dKV[:, 128 * hh:128 * hh + 64] = dK[:, 64 * hh:64 * hh + 64]
        dKV[:, 128 * hh + 64:128 * hh + 128] = dV[:, 64 * hh:64 * hh + 64]
    dtable = torch.zeros((n_items, d), device=dev)
    ddt = torch.zeros((16, d), device=dev) if dt is not None else None
    layer.backward(to_bf16(dKV), ids_t, dt_t, n_items, dtable, ddt)
    torch.cuda.synchronize()
    assert layer.err.item() == 0
    dWKV, dW2, dW13, dgamma, dbeta, dX = layer.dWKV, layer.dW2, layer.dW13, layer.dgamma, layer.dbeta, layer.dX
    # ---- oracle on the same stored values
    X64 = R.gather_history(wl["table"], ids, dt, wl.get("dt_table"))
    rdX, rg = G.history_layer_bwd(X64, ffn, WK, WV, eps, dK, dV)
    rtab = np.zeros((n_items, d))
    rdt = np.zeros((16, d)) if dt is not None else None
    G.table_rows_bwd(rtab, rdt, ids, dt, rdX)
    gKV = dWKV.cpu().numpy()
    gWK = np.concatenate([gKV[:, 128 * hh:128 * hh + 64] for hh in range(d // 64)], axis=1)
    gWV = np.concatenate([gKV[:, 128 * hh + 64:128 * hh + 128] for hh in range(d // 64)], axis=1)
    got = {"WK": gWK, "WV": gWV, "W2": dW2.cpu().numpy(), "W1": dW13.cpu().numpy()[:, :h],
           "W3": dW13.cpu().numpy()[:, h:], "gamma": dgamma.cpu().numpy(), "beta": dbeta.cpu().numpy()}
    errs = {k: normwise(got[k], rg[k]) for k in got}
    errs["X"] = normwise(bf16_to_f64(dX), rdX)
    errs["table"] = normwise(dtable.cpu().numpy(), rtab)
    if dt is not None:
        errs["dt_table"] = normwise(ddt.cpu().numpy(), rdt)
    print("history-side backward, normwise errors:", {k: f"{v:.1e}" for k, v in errs.items()})
    assert max(errs.values()) <= TOL, errs
