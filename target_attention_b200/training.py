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
        self.W13p, self.Pp, self.W2p = bf(2 * h, d), bf(2 * h, d), bf(d, h)
        self.WKVi, self.W13c = bf(d, 2 * d), bf(d, 2 * h)
        for args in ((W1, d, h, self.W13p, 1, 0), (W3, d, h, self.W13p, 2, 0), (W1, d, h, self.Pp, 0, 0),
                     (W3, d, h, self.Pp, 0, h), (W2, h, d, self.W2p, 0, 0), (WK, d, d, self.WKVi, 3, 0),
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
        step(B.stca_k_gemm_resident(1, 1, None, ids, dt, table, dt_table, n_items, M, d, self.W13p, h, self.A, h, e,
                                       stream, x_out=self.X), "SwiGLU GEMM")
        step(B.stca_k_gemm_resident(0, 0, self.X, None, None, None, None, 0, M, d, self.Pp, 2 * h, self.P, 2 * h, e,
                                       stream), "X [W1 | W3]")
        step(B.stca_k_gemm_rowwise(0, self.A, M, h, self.W2p, d, None, None, self.eps, self.y, d, e, stream),
                "A W2")

    def backward(self, dKV, ids, dt, n_items, dtable, ddt_table=None, stream=None, on_step=None):
        """dKV [M, 2d] bf16 (head-interleaved K | V columns).  Weight gradients land in
        dWKV (head-interleaved columns), dW2, dW13 ([dW1 | dW3]), dgamma, dbeta; the table
        rows' gradients are added into dtable (and ddt_table).  on_step(name), when given, is
        called after each step is enqueued (a profiler records events there)."""
        M, d, h, e = self.M, self.d, self.h, self.err
        step = _stepper(on_step)
        step(B.stca_k_gemm_rowwise(0, dKV, M, 2 * d, self.WKVi, d, None, None, self.eps, self.dXt, d, e, stream),
                "dKV [W_K | W_V]^T")
        step(B.stca_k_layer_norm_bwd(self.y, self.dXt, M, d, self.gamma, self.beta, self.eps, self.dy, self.Xt,
                                        self.dgamma, self.dbeta, 0, self.wln, self.wln.numel(), stream), "LN backward")
        step(B.stca_k_gemm_wgrad(self.Xt, d, dKV, 2 * d, M, d, 2 * d, self.dWKV, 2 * d, 0, self.wg, self.wg.numel(),
                                    stream), "Xt^T dKV")
        step(B.stca_k_gemm_resident(0, 0, self.dy, None, None, None, None, 0, M, d, self.W2, h, self.dA, h, e,
                                       stream), "dy W2^T")
        step(B.stca_k_gemm_wgrad(self.A, h, self.dy, d, M, h, d, self.dW2, d, 0, self.wg, self.wg.numel(), stream),
                "A^T dy")
        step(B.stca_k_swiglu_bwd(self.P, self.dA, M, h, self.dP, None, stream), "SwiGLU backward")
        step(B.stca_k_gemm_rowwise(0, self.dP, M, 2 * h, self.W13c, d, None, None, self.eps, self.dX, d, e, stream),
                "dP [W1 | W3]^T")
        step(B.stca_k_gemm_wgrad(self.X, d, self.dP, 2 * h, M, d, 2 * h, self.dW13, 2 * h, 0, self.wg,
                                    self.wg.numel(), stream), "X^T dP")
        step(B.stca_k_table_rows_bwd(self.dX, M, d, ids, dt, n_items, dtable, ddt_table, e, stream),
                "table rows")

    def flops(self):
        """Multiply-add work of each GEMM of recompute() + backward(), in flop."""
        M, d, h = self.M, self.d, self.h
        return {"SwiGLU GEMM": 2 * M * d * 2 * h, "X [W1 | W3]": 2 * M * d * 2 * h, "A W2": 2 * M * h * d,
                "dKV [W_K | W_V]^T": 2 * M * 2 * d * d, "Xt^T dKV": 2 * M * d * 2 * d, "dy W2^T": 2 * M * d * h,
                "A^T dy": 2 * M * h * d, "dP [W1 | W3]^T": 2 * M * 2 * h * d, "X^T dP": 2 * M * d * 2 * h}


def _stepper(on_step):
    def check(rc, what):
        B.check(rc, what)
        if on_step is not None:
            on_step(what)
    return check
