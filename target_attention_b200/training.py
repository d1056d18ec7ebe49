"""One layer's history-side backward, composed from the library's kernel-level entries.

The history side of STCA layer i maps the looked-up rows X to Xt = LN(SwiGLU(X)) and
K, V = Xt W_K, Xt W_V (STCA notes, section "STCA"); the pages train it at about 2K-long
histories (STCA notes, "短序列训练，长序列推理").  ``HistoryLayerBackward`` holds the
operand layouts and scratch for one layer shape and runs, given dK and dV (in the K/V
rows' head-interleaved column order, as the attention backward produces them):

  recompute   X (gathered), A = SiLU(X W1) * (X W3), P = [X W1 | X W3], y = A W2
  backward    dXt = dKV [W_K | W_V]^T;  dy, Xt, dgamma, dbeta = LN backward;
              dW_KV = Xt^T dKV;  dA = dy W2^T;  dW2 = A^T dy;  dP = SwiGLU backward;
              dX = dP [W1 | W3]^T;  [dW1 | dW3] = X^T dP;  dE[ids], dT[bucket] += dX

Every step runs in the CUDA library; this module only allocates buffers and passes
pointers.  All tensors are torch CUDA tensors; weights bf16 row-major as in the forward
(W1, W3 [d, h], W2 [h, d], W_K, W_V [d, d]), gamma / beta fp32 [d].
"""
import torch

from . import binding as B


class HistoryLayerBackward:
    def __init__(self, M, d, h, W1, W3, W2, WK, WV, gamma, beta, eps=1e-5, device="cuda"):
        self.M, self.d, self.h, self.eps = M, d, h, eps
        self.gamma, self.beta = gamma, beta
        bf = lambda *s: torch.empty(s, dtype=torch.bfloat16, device=device)
        f32 = lambda *s: torch.empty(s, dtype=torch.float32, device=device)
        self.W2 = W2
        # operand layouts: forward GEMMs take packed weights, backward GEMMs the weights
        # as they are or with their columns placed side by side / head-interleaved
        self.W13p, self.W2p = bf(2 * h, d), bf(d, h)
        self.WKVi, self.W13c = bf(d, 2 * d), bf(d, 2 * h)
        for args in ((W1, d, h, self.W13p, 1, 0), (W3, d, h, self.W13p, 2, 0), (W2, h, d, self.W2p, 0, 0),
                     (WK, d, d, self.WKVi, 3, 0),
                     (WV, d, d, self.WKVi, 3, 64), (W1, d, h, self.W13c, 4, 0), (W3, d, h, self.W13c, 4, h)):
            B.check(B.stca_k_pack_weight(*args), "pack")
        # activations and gradients of the rows
        self.X, self.A, self.P, self.y = bf(M, d), bf(M, h), bf(M, 2 * h), bf(M, d)
        self.dXt, self.dy, self.Xt, self.dA, self.dP, self.dX = bf(M, d), bf(M, d), bf(M, d), bf(M, h), bf(M, 2 * h), \
            bf(M, d)
        # weight gradients
        self.dWKV, self.dW2, self.dW13 = f32(d, 2 * d), f32(h, d), f32(d, 2 * h)
        self.dgamma, self.dbeta = f32(d), f32(d)
        wg = max(B.stca_k_gemm_wgrad_workspace_bytes(M, K, N) for K, N in ((d, 2 * d), (h, d), (d, 2 * h)))
        self.wg = torch.empty(max(wg, 16), dtype=torch.uint8, device=device)
        self.wln = torch.empty(max(B.stca_k_layer_norm_bwd_workspace_bytes(M, d), 16), dtype=torch.uint8,
                               device=device)
        self.err = torch.zeros(1, dtype=torch.int32, device=device)

    def recompute(self, ids, dt, table, dt_table, n_items, stream=None, on_step=None):
        M, d, h, e = self.M, self.d, self.h, self.err
        step = _stepper(on_step)
        # A = SiLU(X W1) * (X W3), with the gathered X and the pre-activations P = [X W1 | X W3]
        # written by the same GEMM
        step(B.stca_k_gemm_resident(1, 1, None, ids, dt, table, dt_table, n_items, M, d, self.W13p, h, self.A, h, e,
                                       stream, x_out=self.X, p_out=self.P), "SwiGLU GEMM")
        step(B.stca_k_gemm_rowwise(0, self.A, M, h, self.W2p, d, None, None, self.eps, self.y, d, e, stream),
                "A W2")

    def backward(self, dKV, ids, dt, n_items, dtable, ddt_table=None, stream=None, on_step=None, xt_ready=False):
        """dKV [M, 2d] bf16 (head-interleaved K | V columns).  Weight gradients land in
        dWKV (head-interleaved columns), dW2, dW13 ([dW1 | dW3]), dgamma, dbeta; the table
        rows' gradients are added into dtable (and ddt_table).  on_step(name), when given, is
        called after each step is enqueued (a profiler records events there).  xt_ready: Xt =
        LN(y) is already in ``Xt`` (the LayerNorm backward then does not write it again)."""
        M, d, h, e = self.M, self.d, self.h, self.err
        step = _stepper(on_step)
        step(B.stca_k_gemm_rowwise(0, dKV, M, 2 * d, self.WKVi, d, None, None, self.eps, self.dXt, d, e, stream),
                "dKV [W_K | W_V]^T")
        step(B.stca_k_layer_norm_bwd(self.y, self.dXt, M, d, self.gamma, self.beta, self.eps, self.dy,
                                        None if xt_ready else self.Xt, self.dgamma, self.dbeta, 0, self.wln,
                                        self.wln.numel(), stream), "LN backward")
        step(B.stca_k_gemm_wgrad(self.Xt, d, dKV, 2 * d, M, d, 2 * d, self.dWKV, 2 * d, 0, self.wg, self.wg.numel(),
                                    stream, err=e), "Xt^T dKV")
        step(B.stca_k_gemm_resident(0, 0, self.dy, None, None, None, None, 0, M, d, self.W2, h, self.dA, h, e,
                                       stream), "dy W2^T")
        step(B.stca_k_gemm_wgrad(self.A, h, self.dy, d, M, h, d, self.dW2, d, 0, self.wg, self.wg.numel(), stream,
                                    err=e), "A^T dy")
        step(B.stca_k_swiglu_bwd(self.P, self.dA, M, h, self.dP, None, stream), "SwiGLU backward")
        step(B.stca_k_gemm_rowwise(0, self.dP, M, 2 * h, self.W13c, d, None, None, self.eps, self.dX, d, e, stream),
                "dP [W1 | W3]^T")
        step(B.stca_k_gemm_wgrad(self.X, d, self.dP, 2 * h, M, d, 2 * h, self.dW13, 2 * h, 0, self.wg,
                                    self.wg.numel(), stream, err=e), "X^T dP")
        step(B.stca_k_table_rows_bwd(self.dX, M, d, ids, dt, n_items, dtable, ddt_table, e, stream),
                "table rows")

    def flops(self):
        """Multiply-add work of each GEMM of recompute() + backward(), in flop."""
        M, d, h = self.M, self.d, self.h
        return {"SwiGLU GEMM": 2 * M * d * 2 * h, "A W2": 2 * M * h * d,
                "dKV [W_K | W_V]^T": 2 * M * 2 * d * d, "Xt^T dKV": 2 * M * d * 2 * d, "dy W2^T": 2 * M * d * h,
                "A^T dy": 2 * M * h * d, "dP [W1 | W3]^T": 2 * M * 2 * h * d, "X^T dP": 2 * M * d * 2 * h}


def _stepper(on_step):
    def check(rc, what):
        B.check(rc, what)
        if on_step is not None:
            on_step(what)
    return check


class _Ffn:
    """One fp32-activation SwiGLU FFN of the target side (y = (SiLU(x W1) * (x W3)) W2, then
    an optional LayerNorm): the operand layouts its forward and backward GEMMs take."""

    def __init__(self, f, d, h, device):
        bf = lambda *s: torch.empty(s, dtype=torch.bfloat16, device=device)
        self.f, self.d, self.h = f, d, h
        self.P0, self.P12, self.W2p, self.W13c = bf(2 * h, d), bf(2 * h, d), bf(d, h), bf(d, 2 * h)
        for args in ((f["W1"], d, h, self.P0, 0, 0), (f["W3"], d, h, self.P0, 0, h), (f["W1"], d, h, self.P12, 1, 0),
                     (f["W3"], d, h, self.P12, 2, 0), (f["W2"], h, d, self.W2p, 0, 0),
                     (f["W1"], d, h, self.W13c, 4, 0), (f["W3"], d, h, self.W13c, 4, h)):
            B.check(B.stca_k_pack_weight(*args), "pack")


class StcaTrainingStep:
    """Gradients of L = sum_t dZ[t] . z[t] through the whole STCA forward (the pages train
    it at about 2K-long histories: STCA notes, "短序列训练，长序列推理"), every step on the
    library's kernels, one history row per token.

    Forward values are recomputed: the history side per layer (HistoryLayerBackward's
    recompute, then Xt = LN(y) and the K/V rows), the target side in fp32 rows (q^(1) =
    LN(SwiGLU_t(x_t)); per layer Q = q W_Q, the attention with its log-sum-exp, o = obar W_O
    written into the concatenation [o^(1) .. o^(M) | x_t]; q^(i+1) = LN(SwiGLU(cat W_C));
    z = SwiGLU_Z(cat W_Z)).  The backward then runs in reverse: the z FFN, W_Z, per layer
    W_O, the attention backward (dQ and the K/V rows' gradients), W_Q, the fusion FFN and W_C
    or the layer-1 target FFN, and the history side of the layer.  The target side's
    weight gradients reduce over the T target rows with the weight-gradient GEMM on bf16
    copies of the fp32 rows.

    w: the weights as device tensors in the structure of the workload's weights (bf16
    matrices, fp32 LayerNorm parameters).  The caller writes x_t (fp32 [T, d]) into
    ``x_t_slot()`` before ``run``.
    """

    def __init__(self, cfg, w, B_users, n_tok, T, device="cuda"):
        d, h, M, H = cfg["d"], cfg["hidden"], cfg["M"], cfg["H"]
        self.cfg, self.w, self.dev = cfg, w, device
        self.d, self.h, self.M, self.H, self.B, self.N, self.T = d, h, M, H, B_users, n_tok, T
        self.eps = float(cfg.get("ln_eps", 1e-5))
        self.score = 0 if cfg["score"] == "softmax" else 1
        f32 = lambda *s: torch.zeros(s, dtype=torch.float32, device=device)
        bf = lambda *s: torch.empty(s, dtype=torch.bfloat16, device=device)
        self.f32, self.bf = f32, bf
        pk = lambda W, K, N: self._pack0(W, K, N)
        # target side operands
        self.WQp = [pk(w["WQ"][i], d, d) for i in range(M)]
        self.WOp = [pk(w["WO"][i], d, d) for i in range(M)]
        self.WCp = [None] + [pk(w["WC"][i], (i + 1) * d, d) for i in range(1, M)]
        self.WZp = pk(w["WZ"], (M + 1) * d, d)
        self.tgt = _Ffn(w["tgt"], d, h, device)
        self.fuse = [None] + [_Ffn(w["fuse"][i], d, h, device) for i in range(1, M)]
        self.zffn = _Ffn(w["zffn"], d, h, device)
        # history side, one per layer, and the K/V rows' forward operand
        self.hist = [HistoryLayerBackward(n_tok, d, h, w["hist"][i]["W1"], w["hist"][i]["W3"], w["hist"][i]["W2"],
                                          w["WK"][i], w["WV"][i], w["hist"][i]["gamma"], w["hist"][i]["beta"],
                                          self.eps, device) for i in range(M)]
        self.KVp = [self._pack0(self.hist[i].WKVi, d, 2 * d) for i in range(M)]
        self.KV = [bf(max(n_tok, 1), 2 * d) for _ in range(M)]
        # target-side activations (fp32 rows) and their bf16 copies for the weight gradients
        C = (M + 1) * d
        self.cat, self.dcat = f32(max(T, 1), C), f32(max(T, 1), C)
        self.q = []  # q^(1) .. q^(M), set by run()
        self.Qp = [f32(max(T, 1), d) for _ in range(M)]
        self.obar = [f32(max(T, 1), d) for _ in range(M)]
        self.lse = [f32(max(T, 1), H) for _ in range(M)]
        self.u = [None] + [f32(max(T, 1), d) for _ in range(1, M)]
        self.zin = f32(max(T, 1), d)
        self.z = None  # z [T, d], set by run()
        self.ffn_state = {}
        self.err = torch.zeros(1, dtype=torch.int32, device=device)

    def x_t_slot(self):
        """The fp32 [T, d] block of the concatenation where x_t goes (written by the caller)."""
        return self.cat[:, self.M * self.d:]

    # ---------------------------------------------------------------- helpers
    def _pack0(self, W, K, N):
        dst = self.bf(N, K)
        B.check(B.stca_k_pack_weight(W, K, N, dst, 0, 0), "pack")
        return dst

    def _gq(self, A, lda, K, Wp, N, C, ldc, dual=0, ksplit=None, kshift=0, R=None, ldr=0):
        """C [T, N] = A W (+ R) with A fp32 rows (lda), Wp the K-major operand [N(or 2N), K]."""
        B.check(B.stca_k_gemm_query(A, lda, self.T, K, K if ksplit is None else ksplit, kshift, Wp, N, dual, R, ldr,
                                    C, ldc, self.err), "target-side GEMM")

    def _to_bf16(self, X, ld, cols):
        out = self.bf(max(self.T, 1), cols)
        B.check(B.stca_k_f32_to_bf16(X, ld, self.T, cols, out, cols), "bf16 copy")
        return out

    def _wgrad(self, A16, lda, G16, ldg, K, N, out=None):
        out = self.f32(K, N) if out is None else out
        wsz = B.stca_k_gemm_wgrad_workspace_bytes(self.T, K, N)
        ws = torch.empty(max(wsz, 16), dtype=torch.uint8, device=self.dev)
        B.check(B.stca_k_gemm_wgrad(A16, lda, G16, ldg, self.T, K, N, out, N, 0, ws, ws.numel(), err=self.err),
                "weight gradient")
        return out

    # ---------------------------------------------------------------- target-side FFNs
    def _ffn_fwd(self, key, ffn, x, ldx, K, ln):
        """y = SwiGLU(x) (then LN when ln): keeps x, P = [x W1 | x W3], A and y for the backward.
        x: fp32 rows [T, ldx] of which the first K columns are the input (K = d)."""
        d, h, T = self.d, self.h, self.T
        st = {"x": x, "ldx": ldx, "P": self.f32(max(T, 1), 2 * h), "A": self.f32(max(T, 1), h),
              "y": self.f32(max(T, 1), d), "out": self.f32(max(T, 1), d) if ln is not None else None}
        self._gq(x, ldx, K, ffn.P0, 2 * h, st["P"], 2 * h)
        self._gq(x, ldx, K, ffn.P12, h, st["A"], h, dual=1)
        self._gq(st["A"], h, h, ffn.W2p, d, st["y"], d)
        if ln is not None:
            B.check(B.stca_k_layer_norm(st["y"], d, 1, T, d, ln["gamma"], ln["beta"], self.eps, st["out"], d, 1),
                    "LayerNorm")
        self.ffn_state[key] = st
        return st["out"] if ln is not None else st["y"]

    def _ffn_bwd(self, key, ffn, ln, dout, ld_dout, dx, ld_dx, R=None, ldr=0):
        """Backward of _ffn_fwd[key] from dout [T, d]: writes dx (= dP [W1 | W3]^T (+ R)) and
        returns the FFN's weight gradients."""
        d, h, T = self.d, self.h, self.T
        st = self.ffn_state[key]
        g = {}
        dy = dout
        if ln is not None:
            dy = self.f32(max(T, 1), d)
            g["gamma"], g["beta"] = self.f32(d), self.f32(d)
            wsz = B.stca_k_layer_norm_bwd_workspace_bytes(T, d)
            ws = torch.empty(max(wsz, 16), dtype=torch.uint8, device=self.dev)
            assert ld_dout == d, "the LayerNorm backward takes dense rows"
            B.check(B.stca_k_layer_norm_bwd(st["y"], dout, T, d, ln["gamma"], ln["beta"], self.eps, dy, None,
                                            g["gamma"], g["beta"], 0, ws, ws.numel(), fp32=1), "LayerNorm backward")
            ld_dout = d
        dA = self.f32(max(T, 1), h)
        self._gq(dy, ld_dout, d, ffn.f["W2"], h, dA, h)               # dA = dy W2^T (W2 itself)
        g["W2"] = self._wgrad(self._to_bf16(st["A"], h, h), h, self._to_bf16(dy, ld_dout, d), d, h, d)
        dP = self.f32(max(T, 1), 2 * h)
        B.check(B.stca_k_swiglu_bwd(st["P"], dA, T, h, dP, None, fp32=1), "SwiGLU backward")
        W13 = self._wgrad(self._to_bf16(st["x"], st["ldx"], d), d, self._to_bf16(dP, 2 * h, 2 * h), 2 * h, d, 2 * h)
        g["W1"], g["W3"] = W13[:, :h], W13[:, h:]
        self._gq(dP, 2 * h, 2 * h, ffn.W13c, d, dx, ld_dx, R=R, ldr=ldr)  # dx = dP [W1 | W3]^T (+ R)
        return g

    # ---------------------------------------------------------------- the step
    def run(self, ids, dt, hoff, toff, table, dt_table, n_items, dZ, dtable, ddt_table=None):
        """Forward recompute and backward for upstream dZ [T, d] (fp32).  Returns the weight
        gradients in the workload's structure (fp32 device tensors), except that W_K and W_V
        of layer i come as one [d, 2d] matrix "WKV_interleaved"[i] in the K/V rows' column
        order (head j's W_K columns at 128 j, its W_V columns at 128 j + 64); the table rows'
        gradients are added into dtable (and ddt_table); d x_t is ``dx_t()``."""
        self.forward_history(ids, dt, table, dt_table, n_items)
        self.forward_target(hoff, toff)
        return self.backward(ids, dt, hoff, toff, n_items, dZ, dtable, ddt_table)

    def capture(self, ids, dt, hoff, toff, table, dt_table, n_items, dZ, dtable, ddt_table=None):
        """Records one whole step (``run`` on the same buffers) as a CUDA graph: the step is a
        few hundred launches, most of them small on the target side, and replaying them as
        one graph removes the per-launch host work.  One eager step runs first, on the
        capture stream (so the caching allocator has every buffer).  Returns (graph, grads):
        ``graph.replay()`` recomputes ``grads`` in place; like ``run`` it adds the table rows'
        gradients into dtable (and ddt_table) on every replay."""
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            self.run(ids, dt, hoff, toff, table, dt_table, n_items, dZ, dtable, ddt_table)
        torch.cuda.current_stream().wait_stream(s)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            grads = self.run(ids, dt, hoff, toff, table, dt_table, n_items, dZ, dtable, ddt_table)
        return graph, grads

    def forward_history(self, ids, dt, table, dt_table, n_items):
        """Every layer's history side recomputed: the rows X, A, P, y, Xt = LN(y) and the K/V rows."""
        d, M, N, w = self.d, self.M, self.N, self.w
        for i in range(M):
            L = self.hist[i]
            L.recompute(ids, dt, table, dt_table, n_items)
            B.check(B.stca_k_layer_norm(L.y, d, 0, N, d, w["hist"][i]["gamma"], w["hist"][i]["beta"], self.eps, L.Xt,
                                        d, 0), "history LayerNorm")
            B.check(B.stca_k_gemm_resident(0, 0, L.Xt, None, None, None, None, 0, N, d, self.KVp[i], 2 * d, self.KV[i],
                                           2 * d, self.err), "K/V rows")

    def forward_target(self, hoff, toff):
        """The target side in fp32 rows, from x_t (in ``x_t_slot()``) and the K/V rows."""
        d, M, H, T = self.d, self.M, self.H, self.T
        C = (M + 1) * d
        w, sc = self.w, self.score
        pa = self.f32(1, max(T, 1), d)
        pm = self.f32(1, max(T, 1), H, 2)
        xt = self.x_t_slot()
        q0 = self._ffn_fwd("tgt", self.tgt, xt, C, d, w["tgt"])
        q = [q0]
        for i in range(M):
            self._gq(q[i], d, d, self.WQp[i], d, self.Qp[i], d)
            B.check(B.stca_attention_train_forward(self.Qp[i], self.KV[i], hoff, toff, self.B, T, d, H, 1, sc, pa, pm,
                                                   self.obar[i], self.lse[i] if sc == 0 else None, self.err),
                    "attention")
            self._gq(self.obar[i], d, d, self.WOp[i], d, self.cat[:, i * d:], C)  # o^(i+1) into the concatenation
            if i + 1 < M:
                # u = [o^(1) .. o^(i+1) | x_t] W_C^(i+2): two column blocks of the concatenation
                self._gq(self.cat, C, (i + 2) * d, self.WCp[i + 1], d, self.u[i + 1], d, ksplit=(i + 1) * d,
                         kshift=(M - i - 1) * d)
                q.append(self._ffn_fwd(("fuse", i + 1), self.fuse[i + 1], self.u[i + 1], d, d, w["fuse"][i + 1]))
        self.q = q
        self._gq(self.cat, C, C, self.WZp, d, self.zin, d)
        self.z = self._ffn_fwd("z", self.zffn, self.zin, d, d, None)

    def backward(self, ids, dt, hoff, toff, n_items, dZ, dtable, ddt_table=None):
        """The backward after forward_history and forward_target (see ``run``)."""
        d, h, M, H, T, N = self.d, self.h, self.M, self.H, self.T, self.N
        C = (M + 1) * d
        w, sc = self.w, self.score
        g = {"hist": [None] * M, "WQ": [None] * M, "WKV_interleaved": [None] * M, "WO": [None] * M,
             "WC": [None] * M, "fuse": [None] * M}
        # z = SwiGLU_Z(cat W_Z)
        dzin = self.f32(max(T, 1), d)
        g["zffn"] = self._ffn_bwd("z", self.zffn, None, dZ, d, dzin, d)
        cat16 = self._to_bf16(self.cat, C, C)
        g["WZ"] = self._wgrad(cat16, C, self._to_bf16(dzin, d, d), d, C, d)
        self._gq(dzin, d, d, w["WZ"], C, self.dcat, C)                    # d cat = dzin W_Z^T (every block)
        dobar, dQ, dq = self.f32(max(T, 1), d), self.f32(max(T, 1), d), self.f32(max(T, 1), d)
        dKV = self.f32(max(N, 1), 2 * d)        # fp32 partial sums of users with more than 16 targets
        dKV16 = self.bf(max(N, 1), 2 * d)
        for i in reversed(range(M)):
            dout = self.dcat[:, i * d:]
            g["WO"][i] = self._wgrad(self._to_bf16(self.obar[i], d, d), d, self._to_bf16(dout, C, d), d, d, d)
            self._gq(dout, C, d, w["WO"][i], d, dobar, d)                 # d obar = d o W_O^T
            B.check(B.stca_attention_backward(self.Qp[i], self.KV[i], hoff, toff, self.B, T, d, H, 1, sc, self.obar[i],
                                              self.lse[i] if sc == 0 else None, dobar, dQ, dKV, None, dKV16=dKV16),
                    "attention backward")
            g["WQ"][i] = self._wgrad(self._to_bf16(self.q[i], d, d), d, self._to_bf16(dQ, d, d), d, d, d)
            self._gq(dQ, d, d, w["WQ"][i], d, dq, d)                      # dq = dQ W_Q^T
            xt_blk = self.dcat[:, M * d:]
            if i == 0:   # q^(1) = LN(SwiGLU_t(x_t)): d x_t gathers into the concatenation's x_t block
                g["tgt"] = self._ffn_bwd("tgt", self.tgt, w["tgt"], dq, d, xt_blk, C, R=xt_blk, ldr=C)
            else:        # q^(i+1) = LN(SwiGLU(u)), u = [o^(1) .. o^(i) | x_t] W_C^(i+1)
                du = self.f32(max(T, 1), d)
                g["fuse"][i] = self._ffn_bwd(("fuse", i), self.fuse[i], w["fuse"][i], dq, d, du, d)
                du16 = self._to_bf16(du, d, d)
                gWC = self.f32((i + 1) * d, d)
                self._wgrad(cat16, C, du16, d, i * d, d, out=gWC[:i * d])
                self._wgrad(cat16[:, M * d:], C, du16, d, d, d, out=gWC[i * d:])
                g["WC"][i] = gWC
                # the o^(j) blocks and x_t take du W_C^T (added to what they already hold)
                self._gq(du, d, d, w["WC"][i][:i * d], i * d, self.dcat, C, R=self.dcat, ldr=C)
                self._gq(du, d, d, w["WC"][i][i * d:], d, xt_blk, C, R=xt_blk, ldr=C)
            # the history side of layer i from its K/V rows' gradients
            L = self.hist[i]
            L.backward(dKV16, ids, dt, n_items, dtable, ddt_table, xt_ready=True)
            # [dW_K | dW_V] in the K/V rows' head-interleaved columns: head j's K at 128 j, V at 128 j + 64
            g["WKV_interleaved"][i] = L.dWKV
            g["hist"][i] = {"W1": L.dW13[:, :h], "W3": L.dW13[:, h:], "W2": L.dW2, "gamma": L.dgamma,
                            "beta": L.dbeta}
        return g

    def flops(self, lengths, targets_per_user):
        """Multiply-add work of one step in flop: every history-side GEMM (recompute, the K/V
        rows and the backward) and the attention products (forward q.k and p v; backward the
        scores again, dP, dV, dK and dQ: 14 d flop per (target, key) pair).  The target
        side's T-row GEMMs are not counted."""
        import numpy as np
        pairs = float(np.dot(np.asarray(lengths, np.float64), np.asarray(targets_per_user, np.float64)))
        hist = sum(self.hist[0].flops().values()) + 2 * self.N * self.d * 2 * self.d
        return {"history": self.M * hist, "attention": self.M * 14 * self.d * pairs}

    def dx_t(self):
        """d x_t [T, d] fp32 (a view of the concatenation's gradient) after ``run``."""
        return self.dcat[:, self.M * self.d:]


def device_weights(w, device="cuda"):
    """The workload's weights (bf16 bit patterns as uint16, fp32 LayerNorm parameters) as
    device tensors in the same structure (bf16 and fp32), for StcaTrainingStep."""
    import numpy as np

    def up(a):
        if a is None:
            return None
        a = np.ascontiguousarray(a)
        if a.dtype == np.uint16:
            return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(device)
        return torch.from_numpy(a.astype(np.float32)).to(device)

    def walk(x):
        if isinstance(x, dict):
            return {k: walk(v) for k, v in x.items()}
        if isinstance(x, list):
            return [walk(v) for v in x]
        return up(x)

    return walk(w)
