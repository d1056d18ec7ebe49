"""Training step of the attention: the forward with its softmax statistics and the
backward (stca_attention_train_forward / stca_attention_backward) against the fp64
backward oracle, through the C ABI, on inputs shaped like the pages' training workload
(d = 256, H = 4, ~2K Beta-ragged histories, several targets per user).

Gradients are compared normwise per (user, head) block: max |g - r| / max |r| over the
block <= 2e-2 (bf16 K/V, queries, output gradients and weights as MMA operands, fp32
accumulation).  dQ and dK are sums of signed terms ds_tj k_j and ds_tj q_t, with
ds_tj = p_tj (dp_tj - D_t), that can cancel (dK of a one-key history is exactly 0), so a
block is measured against the largest sum of its terms' magnitudes, p_tj (|dp_tj| + |D_t|)
|k_j| or |q_t| (the gradient's size before cancellation), when that is larger than the
block itself.  The ReLU form's mask
[s > 0] is a decision, so for it both sides get bf16-representable queries and output
gradients and take it on the same scores."""
import math

import numpy as np
import pytest
import torch

from oracle import stca_grad as G
from oracle import stca_ref as R
from target_attention_b200 import binding as B
from tests._util import bf16_to_f64, zeros_err
from workloads import make_stca

pytestmark = pytest.mark.gpu
dev = "cuda"
D, H, DH = 256, 4, 64
TOL = 2e-2


def _inputs(lengths, targets, seed, bf16_q=False):
    g = np.random.default_rng(seed)
    lengths, targets = np.asarray(lengths, np.int32), np.asarray(targets, np.int32)
    N, T = int(lengths.sum()), int(targets.sum())
    KV = torch.from_numpy(g.standard_normal((max(N, 1), 2 * D)).astype(np.float32)).to(torch.bfloat16).to(dev)
    Q = torch.from_numpy(g.standard_normal((max(T, 1), D)).astype(np.float32)).to(dev)
    dO = torch.from_numpy(g.standard_normal((max(T, 1), D)).astype(np.float32)).to(dev)
    if bf16_q:
        Q, dO = Q.to(torch.bfloat16).float(), dO.to(torch.bfloat16).float()
    return dict(lengths=lengths, targets=targets, N=N, T=T, B=len(lengths), KVt=KV, Qt=Q, dOt=dO,
                hoff=torch.from_numpy(R.exclusive_offsets(lengths).astype(np.int32)).to(dev),
                toff=torch.from_numpy(R.exclusive_offsets(targets).astype(np.int32)).to(dev))


def _forward(x, score, splits):
    T = max(x["T"], 1)
    out = torch.full((T, D), float("nan"), device=dev)
    lse = torch.full((T, H), float("nan"), device=dev) if score == 0 else None
    pa, pm = torch.empty((splits, T, D), device=dev), torch.empty((splits, T, H, 2), device=dev)
    err = zeros_err()
    B.check(B.stca_attention_train_forward(x["Qt"], x["KVt"], x["hoff"], x["toff"], x["B"], x["T"], D, H, splits,
                                           score, pa, pm, out, lse, err), "train forward")
    torch.cuda.synchronize()
    assert err.item() == 0
    return out, lse


def _backward(x, score, splits, out, lse):
    dQ = torch.full((max(x["T"], 1), D), float("nan"), device=dev)
    dKV = torch.full((max(x["N"], 1), 2 * D), float("nan"), device=dev)
    pdq = torch.empty((splits, max(x["T"], 1), D), device=dev)
    B.check(B.stca_attention_backward(x["Qt"], x["KVt"], x["hoff"], x["toff"], x["B"], x["T"], D, H, splits, score,
                                      out, lse, x["dOt"], dQ, dKV, pdq), "backward")
    # the bf16 form: the same fp32 sums rounded to nearest even, dKV only as scratch
    dQ2 = torch.empty_like(dQ)
    scratch = torch.full_like(dKV, float("nan"))
    dKV16 = torch.full(dKV.shape, float("nan"), dtype=torch.bfloat16, device=dev)
    B.check(B.stca_attention_backward(x["Qt"], x["KVt"], x["hoff"], x["toff"], x["B"], x["T"], D, H, splits, score,
                                      out, lse, x["dOt"], dQ2, scratch, pdq, dKV16=dKV16), "backward, bf16 K/V")
    torch.cuda.synchronize()
    n = x["N"]
    assert torch.equal(dKV16[:n], dKV[:n].to(torch.bfloat16))
    assert torch.equal(dQ2, dQ)
    return dQ.cpu().numpy()[:x["T"]], dKV.cpu().numpy()[:x["N"]]


def _case(lengths, targets, score, splits, seed):
    x = _inputs(lengths, targets, seed, bf16_q=score == 1)
    out, lse = _forward(x, score, splits)
    dQ, dKV = _backward(x, score, splits, out, lse)
    T = x["T"]
    return dict(lengths=x["lengths"], targets=x["targets"], KV=bf16_to_f64(x["KVt"]),
                Q=x["Qt"].cpu().numpy().astype(np.float64), dO=x["dOt"].cpu().numpy().astype(np.float64),
                out=out.cpu().numpy()[:T], lse=None if lse is None else lse.cpu().numpy()[:T], dQ=dQ, dKV=dKV)


def _reference(c, score):
    """Oracle per (target, head), K/V gradients summed over each user's targets."""
    hoff, toff = R.exclusive_offsets(c["lengths"]), R.exclusive_offsets(c["targets"])
    T, N = int(toff[-1]), int(hoff[-1])
    sc = 1 / math.sqrt(DH)
    out, lse, dQ = np.zeros((T, D)), np.full((T, H), -np.inf), np.zeros((T, D))
    dKV = np.zeros((N, 2 * D))
    dQ_mag, dK_mag = np.zeros((T, D)), np.zeros((N, D))  # sums of the terms' magnitudes
    for u in range(len(c["lengths"])):
        rows = c["KV"][hoff[u]:hoff[u + 1]]
        for h in range(H):
            K_h, V_h = rows[:, 2 * h * DH:(2 * h + 1) * DH], rows[:, (2 * h + 1) * DH:(2 * h + 2) * DH]
            cols = slice(h * DH, (h + 1) * DH)
            for t in range(toff[u], toff[u + 1]):
                q, do = c["Q"][t, cols], c["dO"][t, cols]
                out[t, cols] = R.head_attention(q, K_h, V_h, "softmax" if score == 0 else "relu", sc)
                if score == 0:
                    lse[t, h] = G.softmax_lse(q, K_h, sc)
                dq, dK, dV = G.head_attention_bwd(q, K_h, V_h, "softmax" if score == 0 else "relu", sc, do)
                dQ[t, cols] = dq
                dKV[hoff[u]:hoff[u + 1], 2 * h * DH:(2 * h + 1) * DH] += dK
                dKV[hoff[u]:hoff[u + 1], (2 * h + 1) * DH:(2 * h + 2) * DH] += dV
                if len(K_h):
                    s_ = K_h @ q * sc
                    dp = V_h @ do
                    if score == 0:
                        p = np.exp(s_ - s_.max())
                        p /= p.sum()
                        mag = p * (np.abs(dp) + abs(do @ (p @ V_h)))
                    else:
                        mag = np.abs(dp) * (s_ > 0)
                    dQ_mag[t, cols] = sc * (np.abs(K_h).T @ mag)
                    dK_mag[hoff[u]:hoff[u + 1], cols] += sc * np.outer(mag, np.abs(q))
    return dict(out=out, lse=lse, dQ=dQ, dKV=dKV, dQ_mag=dQ_mag, dK_mag=dK_mag)


def _block_err(got, ref, floor):
    if ref.size == 0:
        return 0.0
    return float(np.abs(got - ref).max() / max(np.abs(ref).max(), floor, 1e-30))


def _check(c, ref, score):
    hoff, toff = R.exclusive_offsets(c["lengths"]), R.exclusive_offsets(c["targets"])
    assert np.isfinite(c["dQ"]).all() and np.isfinite(c["dKV"]).all()
    e_out = R.row_rel_err(c["out"].reshape(-1, DH), ref["out"].reshape(-1, DH))
    assert e_out <= TOL, e_out
    if score == 0:
        fin = np.isfinite(ref["lse"])
        assert (np.isneginf(c["lse"]) == ~fin).all()
        assert np.abs(c["lse"][fin] - ref["lse"][fin]).max() <= TOL
    worst = 0.0
    for u in range(len(c["lengths"])):
        tq, kk = slice(toff[u], toff[u + 1]), slice(hoff[u], hoff[u + 1])
        for h in range(H):
            cq = slice(h * DH, (h + 1) * DH)
            ck, cv = slice(2 * h * DH, (2 * h + 1) * DH), slice((2 * h + 1) * DH, (2 * h + 2) * DH)
            blocks = ((c["dQ"][tq, cq], ref["dQ"][tq, cq], ref["dQ_mag"][tq, cq]),
                      (c["dKV"][kk, ck], ref["dKV"][kk, ck], ref["dK_mag"][kk, cq]),
                      (c["dKV"][kk, cv], ref["dKV"][kk, cv], None))
            for got, r, mag in blocks:
                worst = max(worst, _block_err(got, r, 0.0 if mag is None or not mag.size else np.abs(mag).max()))
    print(f"attention backward: worst block-normwise error {worst:.2e} (forward rows {e_out:.2e})")
    assert worst <= TOL, worst


@pytest.mark.parametrize("score", [0, 1])
@pytest.mark.parametrize("splits", [1, 3])
def test_backward_edge_cases(score, splits):
    """An empty history with targets (dQ = 0), a user without targets (its keys get zero
    gradients), one key, a ragged tile tail, 20 targets (two query chunks)."""
    lengths = [0, 1, 17, 700, 2048, 33]
    targets = [2, 3, 20, 8, 0, 1]
    c = _case(lengths, targets, score, splits, seed=21 + score)
    ref = _reference(c, score)
    _check(c, ref, score)
    assert (c["dQ"][:2] == 0).all()
    hoff = R.exclusive_offsets(lengths)
    assert (c["dKV"][hoff[4]:hoff[5]] == 0).all()


@pytest.mark.parametrize("score", [0, 1])
def test_backward_training_shape(score):
    """Beta(2, 1) x 2048 ragged histories, 8 targets per user, d = 256, H = 4."""
    wl = make_stca(2, users=10, n_items=1000)
    c = _case(wl["lengths"], wl["targets_per_user"], score, 2, seed=31)
    _check(c, _reference(c, score), score)


def test_backward_splits_agree():
    """One forward; the backward with one slice and with four: a key's gradient is
    complete inside its slice (bit for bit), and the slices' dQ shares add up."""
    x = _inputs([1200, 300, 5], [8, 8, 3], seed=41)
    out, lse = _forward(x, 0, 1)
    dQ1, dKV1 = _backward(x, 0, 1, out, lse)
    dQ4, dKV4 = _backward(x, 0, 4, out, lse)
    np.testing.assert_array_equal(dKV1, dKV4)
    assert np.abs(dQ1 - dQ4).max() <= 1e-5 * np.abs(dQ1).max()
