"""Device-side holders for the three entry points: upload a workload's weights and
inputs (numpy arrays in the storage formats of ``workloads``) to torch tensors, fill the
ctypes weight structs, own the libstca handle.  Marshalling only."""
from __future__ import annotations

import numpy as np
import torch

from . import binding as B


def to_device(arr, device="cuda", pin=False):
    """numpy (float32, int32, or bf16 bit patterns in uint16) -> torch tensor."""
    if arr is None:
        return None
    a = np.ascontiguousarray(arr)
    if a.dtype == np.uint16:
        t = torch.from_numpy(a.view(np.int16)).view(torch.bfloat16)
    else:
        t = torch.from_numpy(a)
    if pin:
        return t.pin_memory()
    return t.to(device, non_blocking=False)


class _Holder:
    def __init__(self, device):
        self.device = device
        self.keep = []

    def up(self, arr):
        t = to_device(arr, self.device)
        if t is not None:
            self.keep.append(t)
        return t

    def p(self, arr):
        t = self.up(arr)
        return None if t is None else t.data_ptr()

    def ffn(self, f, ln=True):
        s = B.StcaFfn()
        s.W1, s.W3, s.W2 = self.p(f["W1"]), self.p(f["W3"]), self.p(f["W2"])
        if ln and "gamma" in f:
            s.gamma, s.beta = self.p(f["gamma"]), self.p(f["beta"])
        return s


class StcaModel(_Holder):
    """Weights of an STCA workload on the device plus a handle sized for it.  dedup
    (stca_config.dedup) defaults to 2 for bf16 workloads: the history GEMMs run once per
    distinct key of the call, attention once per distinct key of each user."""

    def __init__(self, wl, device="cuda", max_users=None, max_tokens=None, max_targets=None, dedup=None, kv_fold=0):
        super().__init__(device)
        c = wl["cfg"]
        self.cfg = c
        self.config = B.StcaConfig(
            mode=B.MODE_STCA, M=c["M"], d=c["d"], H=c["H"], hidden=c["hidden"],
            dtype=B.BF16 if c["dtype"] == "bf16" else B.FP32,
            score=B.RELU if c["score"] == "relu" else B.SOFTMAX, time_buckets=c["time_buckets"],
            max_users=max_users or len(wl["lengths"]), max_tokens=max_tokens or int(wl["lengths"].sum()),
            max_targets=max_targets or int(wl["targets_per_user"].sum()),
            dedup=int((2 if c["dtype"] == "bf16" else 0) if dedup is None else dedup), ln_eps=c.get("ln_eps", 1e-5),
            kv_fold=int(kv_fold))
        w = wl["weights"]
        ws = B.StcaWeights()
        ws.table = self.p(wl["table"])
        ws.n_items = wl["table"].shape[0]
        ws.dt_table = self.p(wl["dt_table"])
        for i in range(c["M"]):
            ws.hist[i] = self.ffn(w["hist"][i])
            ws.WQ[i], ws.WK[i] = self.p(w["WQ"][i]), self.p(w["WK"][i])
            ws.WV[i], ws.WO[i] = self.p(w["WV"][i]), self.p(w["WO"][i])
            if i > 0:
                ws.WC[i] = self.p(w["WC"][i])
                ws.fuse[i] = self.ffn(w["fuse"][i])
        ws.tgt = self.ffn(w["tgt"])
        ws.WZ = self.p(w["WZ"])
        ws.zffn = self.ffn(w["zffn"], ln=False)
        self.weights = ws
        self.handle = B.stca_create(self.config)

    def other_handle(self, **changes):
        """A second handle over the same device weights with some config fields changed."""
        cfg = B.StcaConfig.from_buffer_copy(self.config)
        for k, v in changes.items():
            setattr(cfg, k, v)
        return B.stca_create(cfg)

    def pin(self, stream=None):
        """Convert the weights to the tensor-core layout once (stca_pin_weights)."""
        B.check(B.stca_pin_weights(self.handle, self.weights, stream), "stca_pin_weights")

    def inputs(self, wl):
        d = {k: to_device(wl[k], self.device) for k in ("ids", "lengths", "dt", "x_t", "targets_per_user")}
        d["B"] = len(wl["lengths"])
        d["n_tok"] = int(wl["lengths"].sum())
        d["t_tot"] = int(wl["targets_per_user"].sum())
        return d

    def forward(self, x, z_out, o_out=None, stream=None, handle=None):
        return B.stca_forward(handle or self.handle, x["ids"], x["lengths"], x["dt"], x["x_t"], x["targets_per_user"],
                              x["B"], x["n_tok"], x["t_tot"], self.weights, z_out, o_out, stream)

    def slice_inputs(self, wl, ranks, rank):
        """Inputs of rank ``rank`` of a sequence-parallel forward: its slice of every user's
        history (``lsplit.slice_histories``) and all of the targets."""
        from .lsplit import slice_histories

        lens, ids, dt = slice_histories(wl["lengths"], wl["ids"], wl["dt"], ranks, rank)
        d = {"ids": to_device(ids, self.device), "lengths": to_device(lens, self.device),
             "dt": to_device(dt, self.device), "x_t": to_device(wl["x_t"], self.device),
             "targets_per_user": to_device(wl["targets_per_user"], self.device)}
        d["B"] = len(lens)
        d["n_tok"] = int(lens.sum())
        d["t_tot"] = int(wl["targets_per_user"].sum())
        return d

    def lsplit_engine(self, x, z_out, stream=None):
        """The library's sequence-parallel phases for this rank's inputs ``x`` (see
        ``lsplit.run_phases``)."""
        return _LsplitEngine(self, x, z_out, stream)

    def forward_lsplit(self, x, z_out, gather, stream=None):
        """Sequence-parallel forward of this rank's slice ``x``; ``gather`` exchanges the
        per-layer attention states (``lsplit.all_gather_fn``)."""
        from .lsplit import run_phases

        return run_phases(self.lsplit_engine(x, z_out, stream), self.cfg["M"], gather)

    def forward_host(self, x, z_out, stream=None):
        return B.stca_forward_host(self.handle, x["ids"], x["lengths"], x["dt"], x["x_t"], x["targets_per_user"],
                                   x["B"], x["n_tok"], x["t_tot"], self.weights, z_out, stream)

    def host_fence(self, stream=None):
        """`stream` waits for the z read-backs of the forward_host calls so far."""
        return B.stca_host_fence(self.handle, stream)

    def close(self):
        if getattr(self, "handle", None) is not None:
            B.stca_destroy(self.handle)
            self.handle = None

    __del__ = close


class _LsplitEngine:
    """One rank's side of a sequence-parallel forward: stca_lsplit_begin, then per layer
    stca_lsplit_partial into (acc [t_tot, d], ml [t_tot, H, 2]) and stca_lsplit_merge of
    all ranks' states; z lands in z_out after the last layer."""

    def __init__(self, model, x, z_out, stream):
        self.m, self.x, self.z, self.stream = model, x, z_out, stream
        c = model.cfg
        T = x["t_tot"]
        self.acc = torch.empty((T, c["d"]), device=model.device)
        self.ml = torch.empty((T, c["H"], 2), device=model.device)

    def begin(self):
        x = self.x
        B.check(B.stca_lsplit_begin(self.m.handle, x["ids"], x["lengths"], x["dt"], x["x_t"], x["targets_per_user"],
                                    x["B"], x["n_tok"], x["t_tot"], self.m.weights, self.stream), "stca_lsplit_begin")

    def partial(self, i):
        B.check(B.stca_lsplit_partial(self.m.handle, i, self.acc, self.ml, self.stream), "stca_lsplit_partial")
        return self.acc, self.ml

    def merge(self, i, all_acc, all_ml):
        last = i + 1 == self.m.cfg["M"]
        B.check(B.stca_lsplit_merge(self.m.handle, i, all_acc.shape[0], all_acc, all_ml, self.z if last else None,
                                    self.stream), "stca_lsplit_merge")

    def result(self):
        return self.z


class PointwiseModel(_Holder):
    def __init__(self, wl, device="cuda", max_users=None, max_tokens=None):
        super().__init__(device)
        c = wl["cfg"]
        self.cfg = c
        self.config = B.StcaConfig(mode=B.MODE_POINTWISE, M=1, d=c["d"], H=1, hidden=c["d"], dtype=B.BF16,
                                   score=B.RELU, time_buckets=0, max_users=max_users or len(wl["lengths"]),
                                   max_tokens=max_tokens or int(wl["lengths"].sum()), max_targets=0, dedup=0,
                                   ln_eps=1e-5)
        self.table = self.up(wl["table"])
        self.handle = B.stca_create(self.config)

    def inputs(self, wl):
        return dict(ids=to_device(wl["ids"], self.device), lengths=to_device(wl["lengths"], self.device),
                    q=to_device(wl["q"], self.device), B=len(wl["lengths"]), n_tok=int(wl["lengths"].sum()))

    def forward(self, x, out, stream=None):
        return B.stca_pointwise_forward(self.handle, x["ids"], x["lengths"], x["q"], self.table, self.table.shape[0],
                                        x["B"], x["n_tok"], out, stream)

    def close(self):
        if getattr(self, "handle", None) is not None:
            B.stca_destroy(self.handle)
            self.handle = None

    __del__ = close


class HyformerModel(_Holder):
    def __init__(self, wl, device="cuda", max_users=None, max_tokens=None, dedup=2):
        super().__init__(device)
        c = wl["cfg"]
        self.cfg = c
        nq = c["n_query"]
        Bu = len(wl["lengths"][0])
        self.config = B.StcaConfig(
            mode=B.MODE_HYFORMER, M=c["blocks"], d=c["d"], H=c["H"], hidden=c["hidden"], dtype=B.BF16,
            score=B.SOFTMAX, time_buckets=0, max_users=max_users or Bu,
            max_tokens=max_tokens or int(max(wl["lengths"][0].sum(), wl["lengths"][1].sum())),
            max_targets=(max_users or Bu) * 2 * nq, dedup=int(dedup), ln_eps=1e-5)
        ws = B.HyfWeights()
        ws.table = self.p(wl["table"])
        ws.n_items = wl["table"].shape[0]
        ws.blocks = c["blocks"]
        for l, blk in enumerate(wl["weights"]["blocks"]):
            for s in range(2):
                f = blk["seq"][s]
                sw = B.HyfSeqWeights()
                sw.ffn = self.ffn(f, ln=False)
                sw.WQ, sw.WK, sw.WV, sw.WO = (self.p(f[k]) for k in ("WQ", "WK", "WV", "WO"))
                ws.blk[l].seq[s] = sw
            for t, f in enumerate(blk["tok"]):
                ws.blk[l].tok[t] = self.ffn(f, ln=False)
        self.weights = ws
        self.handle = B.stca_create(self.config)

    def pin(self, stream=None):
        """Convert the weights (per-token FFNs included) to the tensor-core layout once."""
        B.check(B.stca_pin_weights(self.handle, self.weights, stream), "stca_pin_weights")

    def inputs(self, wl):
        return dict(ids_feed=to_device(wl["ids"][0], self.device), len_feed=to_device(wl["lengths"][0], self.device),
                    ids_search=to_device(wl["ids"][1], self.device),
                    len_search=to_device(wl["lengths"][1], self.device), q0=to_device(wl["q0"], self.device),
                    B=len(wl["lengths"][0]), n_feed=int(wl["lengths"][0].sum()),
                    n_search=int(wl["lengths"][1].sum()), n_query=self.cfg["n_query"])

    def other_handle(self, **changes):
        cfg = B.StcaConfig.from_buffer_copy(self.config)
        for k, v in changes.items():
            setattr(cfg, k, v)
        return B.stca_create(cfg)

    def forward(self, x, out, stream=None, handle=None):
        return B.hyformer_forward(handle or self.handle, x["ids_feed"], x["len_feed"], x["n_feed"], x["ids_search"],
                                  x["len_search"], x["n_search"], x["q0"], x["B"], x["n_query"], self.weights, out,
                                  stream)

    def close(self):
        if getattr(self, "handle", None) is not None:
            B.stca_destroy(self.handle)
            self.handle = None

    __del__ = close
