"""The whole STCA training step on the GPU (target_attention_b200.training.StcaTrainingStep:
forward recompute, then the backward through the z FFN, W_Z, every layer's W_O, attention,
W_Q, fusion FFN / W_C or target FFN, and history side, into the table rows and x_t), against
the fp64 oracle's gradients of the same loss (``stca_grad.stca_backward``), on the pages'
training shape (config 2: d = 256, H = 4, M = 2, Beta-ragged histories, 8 targets per user)
and on config 3's (d = 512, H = 8, M = 3, time buckets), small batches.

Every gradient tensor is compared normwise: max |g - r| / max |r| <= 3e-2.  The GPU keeps
K/V, the history activations and the weight-gradient GEMMs' operands in bf16 (fp32
accumulation); the target side's fp32 rows enter the tensor cores as hi + lo bf16 terms.
The bar sits above the forward's 2e-2 because each gradient is a chain of several such
products, most of them through bf16 copies of fp32 rows."""
import numpy as np
import pytest
import torch

from oracle import stca_grad as G
from target_attention_b200 import binding as B
from target_attention_b200.training import StcaTrainingStep, device_weights
from workloads import make_stca

pytestmark = pytest.mark.gpu
dev = "cuda"
TOL = 3e-2


def normwise(got, ref):
    ref = np.asarray(ref, np.float64)
    return float(np.abs(np.asarray(got, np.float64) - ref).max() / max(np.abs(ref).max(), 1e-30))


@pytest.mark.parametrize("config, kw", [(2, dict(users=3, L=700, n_items=2000)),
                                        (2, dict(users=2, L=500, n_items=2000, score="relu")),
                                        (3, dict(users=2, L=400, n_items=2000))])
def test_training_step_matches_oracle(config, kw):
    wl = make_stca(config, **kw)
    cfg = wl["cfg"]
    d, M = cfg["d"], cfg["M"]
    lengths, tpu = wl["lengths"], wl["targets_per_user"]
    Bu, N, T = len(lengths), int(lengths.sum()), int(tpu.sum())
    i32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, np.int32)).to(dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    hoff, toff = torch.empty(Bu + 1, dtype=torch.int32, device=dev), torch.empty(Bu + 1, dtype=torch.int32, device=dev)
    B.check(B.stca_k_offsets(i32(lengths), Bu, hoff, N, err))
    B.check(B.stca_k_offsets(i32(tpu), Bu, toff, T, err))
    w = device_weights(wl["weights"])
    up16 = lambda bits: torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)
    table = up16(wl["table"])
    dt_table = up16(wl["dt_table"]) if wl["dt"] is not None else None
    n_items = int(wl["table"].shape[0])
    step = StcaTrainingStep(cfg, w, Bu, N, T)
    step.x_t_slot().copy_(up16(wl["x_t"]).float())               # the input rows, staged
    dZ = np.random.default_rng(3).standard_normal((T, d))
    dtable = torch.zeros((n_items, d), device=dev)
    ddt = torch.zeros((16, d), device=dev) if dt_table is not None else None
    g = step.run(i32(wl["ids"]), i32(wl["dt"]) if wl["dt"] is not None else None, hoff, toff, table, dt_table,
                 n_items, torch.from_numpy(dZ.astype(np.float32)).to(dev), dtable, ddt)
    torch.cuda.synchronize()
    assert err.item() == 0 and step.err.item() == 0
    rG, rtab, rdt, rdxt = G.stca_backward(wl, dZ)
    errs = {}
    cpu = lambda t: t.detach().float().cpu().numpy()
    for i in range(M):
        for k in ("W1", "W3", "W2", "gamma", "beta"):
            errs[f"hist{i}.{k}"] = normwise(cpu(g["hist"][i][k]), rG["hist"][i][k])
        kv = cpu(g["WKV_interleaved"][i])
        gk = np.concatenate([kv[:, 128 * j:128 * j + 64] for j in range(d // 64)], axis=1)
        gv = np.concatenate([kv[:, 128 * j + 64:128 * j + 128] for j in range(d // 64)], axis=1)
        errs[f"WK{i}"], errs[f"WV{i}"] = normwise(gk, rG["WK"][i]), normwise(gv, rG["WV"][i])
        errs[f"WQ{i}"] = normwise(cpu(g["WQ"][i]), rG["WQ"][i])
        errs[f"WO{i}"] = normwise(cpu(g["WO"][i]), rG["WO"][i])
        if i > 0:
            errs[f"WC{i}"] = normwise(cpu(g["WC"][i]), rG["WC"][i])
            for k in ("W1", "W3", "W2", "gamma", "beta"):
                errs[f"fuse{i}.{k}"] = normwise(cpu(g["fuse"][i][k]), rG["fuse"][i][k])
    for k in ("W1", "W3", "W2", "gamma", "beta"):
        errs[f"tgt.{k}"] = normwise(cpu(g["tgt"][k]), rG["tgt"][k])
    for k in ("W1", "W3", "W2"):
        errs[f"zffn.{k}"] = normwise(cpu(g["zffn"][k]), rG["zffn"][k])
    errs["WZ"] = normwise(cpu(g["WZ"]), rG["WZ"])
    errs["table"] = normwise(cpu(dtable), rtab)
    if ddt is not None:
        errs["dt_table"] = normwise(cpu(ddt), rdt)
    errs["x_t"] = normwise(cpu(step.dx_t()), rdxt)
    worst = max(errs, key=errs.get)
    print(f"training step: worst {worst} {errs[worst]:.2e};", {k: f"{v:.1e}" for k, v in errs.items()})
    assert errs[worst] <= TOL, errs


def test_training_step_replays_as_one_cuda_graph():
    """The whole step captured as a CUDA graph (StcaTrainingStep.capture) gives the eager
    step's weight gradients bit for bit (every reduction runs in a fixed order) and its
    table gradient up to the order of the lookup scatter's atomics."""
    wl = make_stca(2, users=3, L=600, n_items=2000)
    cfg = wl["cfg"]
    d = cfg["d"]
    lengths, tpu = wl["lengths"], wl["targets_per_user"]
    Bu, N, T = len(lengths), int(lengths.sum()), int(tpu.sum())
    i32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, np.int32)).to(dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    hoff, toff = torch.empty(Bu + 1, dtype=torch.int32, device=dev), torch.empty(Bu + 1, dtype=torch.int32, device=dev)
    B.check(B.stca_k_offsets(i32(lengths), Bu, hoff, N, err))
    B.check(B.stca_k_offsets(i32(tpu), Bu, toff, T, err))
    up16 = lambda bits: torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)
    table = up16(wl["table"])
    n_items = int(wl["table"].shape[0])
    step = StcaTrainingStep(cfg, device_weights(wl["weights"]), Bu, N, T)
    step.x_t_slot().copy_(up16(wl["x_t"]).float())
    ids = i32(wl["ids"])
    dZ = torch.from_numpy(np.random.default_rng(4).standard_normal((T, d)).astype(np.float32)).to(dev)
    dtab = torch.zeros((n_items, d), device=dev)
    eager = step.run(ids, None, hoff, toff, table, None, n_items, dZ, dtab)
    flat = lambda g: [t.clone() for t in _leaves(g)]
    ref, ref_tab = flat(eager), dtab.clone()
    graph, grads = step.capture(ids, None, hoff, toff, table, None, n_items, dZ, dtab)
    dtab.zero_()
    graph.replay()
    torch.cuda.synchronize()
    assert step.err.item() == 0
    for a, b in zip(flat(grads), ref):
        assert torch.equal(a, b)
    assert torch.allclose(dtab, ref_tab, rtol=0, atol=1e-6 * float(ref_tab.abs().max()))


def _leaves(g):
    if isinstance(g, dict):
        return [t for k in sorted(g) for t in _leaves(g[k])]
    if isinstance(g, (list, tuple)):
        return [t for x in g for t in _leaves(x)]
    return [] if g is None else [g]
