"""ctypes binding of libstca (include/stca.h, include/stca_kernels.h).

Argument marshalling only: every computation runs inside libstca's CUDA kernels.  The
functions keep the C names and take torch tensors (device pointers) plus a CUDA stream;
they return the C status code.  Loading fails loudly when libstca.so is missing: there
is no other implementation to fall back to.
"""
from __future__ import annotations

import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libstca.so")

MAX_LAYERS = 8
MAX_QUERY_TOKENS = 64
NOALLOC_MAX_USERS = 2048

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CAPACITY, ERR_CUDA, ERR_ID_OUT_OF_RANGE, ERR_TIMEOUT, \
    ERR_BAD_LENGTHS = range(8)
FP32, BF16 = 0, 1
SOFTMAX, RELU = 0, 1
MODE_STCA, MODE_POINTWISE, MODE_HYFORMER = 0, 1, 2

_vp = ctypes.c_void_p
_i32 = ctypes.c_int
_i64 = ctypes.c_int64


class StcaConfig(ctypes.Structure):
    _fields_ = [("mode", _i32), ("M", _i32), ("d", _i32), ("H", _i32), ("hidden", _i32),
                ("dtype", _i32), ("score", _i32), ("time_buckets", _i32), ("max_users", _i32),
                ("max_tokens", _i32), ("max_targets", _i32), ("dedup", _i32), ("ln_eps", ctypes.c_float),
                ("kv_fold", _i32)]


class StcaFfn(ctypes.Structure):
    _fields_ = [("W1", _vp), ("W3", _vp), ("W2", _vp), ("gamma", _vp), ("beta", _vp)]


class StcaWeights(ctypes.Structure):
    _fields_ = [("table", _vp), ("n_items", _i64), ("dt_table", _vp),
                ("hist", StcaFfn * MAX_LAYERS), ("WQ", _vp * MAX_LAYERS), ("WK", _vp * MAX_LAYERS),
                ("WV", _vp * MAX_LAYERS), ("WO", _vp * MAX_LAYERS), ("tgt", StcaFfn),
                ("WC", _vp * MAX_LAYERS), ("fuse", StcaFfn * MAX_LAYERS), ("WZ", _vp), ("zffn", StcaFfn)]


class HyfSeqWeights(ctypes.Structure):
    _fields_ = [("ffn", StcaFfn), ("WQ", _vp), ("WK", _vp), ("WV", _vp), ("WO", _vp)]


class HyfBlockWeights(ctypes.Structure):
    _fields_ = [("seq", HyfSeqWeights * 2), ("tok", StcaFfn * MAX_QUERY_TOKENS)]


class HyfWeights(ctypes.Structure):
    _fields_ = [("table", _vp), ("n_items", _i64), ("blocks", _i32),
                ("blk", HyfBlockWeights * MAX_LAYERS)]


class StcaError(RuntimeError):
    def __init__(self, code, what=""):
        self.code = code
        super().__init__(f"{what}: libstca status {code} ({strerror(code)})")


_LIB = None

# (name, restype, argtypes)
_SIGS = [
    ("stca_create", _i32, [ctypes.POINTER(StcaConfig), ctypes.POINTER(_vp)]),
    ("stca_destroy", None, [_vp]),
    ("stca_pin_weights", _i32, [_vp, _vp, _vp]),
    ("stca_unpin_weights", None, [_vp]),
    ("stca_forward", _i32, [_vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, ctypes.POINTER(StcaWeights), _vp, _vp,
                            _vp]),
    ("stca_forward_host", _i32, [_vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, ctypes.POINTER(StcaWeights), _vp,
                                 _vp]),
    ("stca_host_fence", _i32, [_vp, _vp]),
    ("stca_lsplit_begin", _i32, [_vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, ctypes.POINTER(StcaWeights), _vp]),
    ("stca_lsplit_partial", _i32, [_vp, _i32, _vp, _vp, _vp]),
    ("stca_lsplit_merge", _i32, [_vp, _i32, _i32, _vp, _vp, _vp, _vp]),
    ("stca_pointwise_forward", _i32, [_vp, _vp, _vp, _vp, _vp, _i64, _i32, _i32, _vp, _vp]),
    ("stca_pointwise_forward_noalloc", _i32, [_vp, _vp, _vp, _vp, _i64, _i32, _i32, _vp, _vp, _vp]),
    ("stca_attention_train_forward", _i32, [_vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32, _vp, _vp, _vp,
                                            _vp, _vp, _vp]),
    ("stca_attention_backward", _i32, [_vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32, _vp, _vp, _vp, _vp,
                                       _vp, _vp, _vp, _vp]),
    ("hyformer_forward", _i32, [_vp, _vp, _vp, _i32, _vp, _vp, _i32, _vp, _i32, _i32, ctypes.POINTER(HyfWeights),
                                _vp, _vp]),
    ("stca_sync_status", _i32, [_vp]),
    ("stca_stream_wait", _i32, [_vp, _i32]),
    ("stca_k_wait_selftest", _i32, [_vp, _vp]),
    ("stca_profile_enable", _i32, [_vp, _i32]),
    ("stca_profile_stages", _i32, [_vp, ctypes.c_uint32]),
    ("stca_profile_read", _i32, [_vp, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_int64)]),
    ("stca_launch_count", ctypes.c_uint64, []),
    ("stca_strerror", ctypes.c_char_p, [_i32]),
    ("stca_k_offsets", _i32, [_vp, _i32, _vp, _i32, _vp, _vp]),
    ("stca_k_pack_weight", _i32, [_vp, _i32, _i32, _vp, _i32, _i32, _vp]),
    ("stca_k_gemm_resident", _i32, [_i32, _i32, _vp, _vp, _vp, _vp, _vp, _i64, _i32, _i32, _vp, _i32, _vp, _i32, _vp,
                                    _vp, _vp, _vp]),
    ("stca_k_ffn_fused", _i32, [_vp, _vp, _vp, _vp, _i64, _i32, _i32, _i32, _vp, _vp, _vp, ctypes.c_float, _vp,
                          _i32, _vp, _vp, _vp]),
    ("stca_k_gemm_query", _i32, [_vp, _i64, _i32, _i32, _i32, _i32, _vp, _i32, _i32, _vp, _i64, _vp, _i64, _vp,
                                 _vp]),
    ("stca_k_gemm_rowwise", _i32, [_i32, _vp, _i32, _i32, _vp, _i32, _vp, _vp, ctypes.c_float, _vp, _i32, _vp, _vp]),
    ("stca_k_attention", _i32, [_i32, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32, _vp, _vp, _vp, _vp,
                                _vp]),
    ("stca_k_attention_rows", _i32, [_i32, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32,
                                     _vp, _vp, _vp, _vp, _vp]),
    ("stca_k_gemm_wgrad_workspace_bytes", ctypes.c_size_t, [_i32, _i32, _i32]),
    ("stca_k_gemm_wgrad", _i32, [_vp, _i64, _vp, _i64, _i32, _i32, _i32, _vp, _i64, _i32, _i32, _vp, ctypes.c_size_t,
                                 _vp, _vp]),
    ("stca_k_layer_norm_bwd_workspace_bytes", ctypes.c_size_t, [_i32, _i32]),
    ("stca_k_layer_norm_bwd", _i32, [_vp, _vp, _i32, _i32, _i32, _vp, _vp, ctypes.c_float, _vp, _vp, _vp, _vp, _i32,
                                     _vp, ctypes.c_size_t, _vp]),
    ("stca_k_layer_norm", _i32, [_vp, _i64, _i32, _i32, _i32, _vp, _vp, ctypes.c_float, _vp, _i64, _i32, _vp]),
    ("stca_k_f32_to_bf16", _i32, [_vp, _i64, _i32, _i32, _vp, _i64, _vp]),
    ("stca_k_swiglu_bwd", _i32, [_vp, _vp, _i32, _i32, _i32, _vp, _vp, _vp]),
    ("stca_k_table_rows_bwd", _i32, [_vp, _i32, _i32, _vp, _vp, _i64, _vp, _vp, _vp, _vp]),
    ("stca_k_dedup_workspace_bytes", ctypes.c_size_t, [_i32]),
    ("stca_k_dedup", _i32, [_vp, _vp, _i32, _vp, ctypes.c_size_t, _vp, _vp, _vp, _vp, _vp]),
    ("stca_k_compact_user_rows", _i32, [_vp, _i32, _vp, _vp, _vp, _vp, _vp]),
]

EXPORTED = [s[0] for s in _SIGS]


def lib():
    """The loaded libstca (built in-tree by ``target_attention_b200.build``)."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libstca.so is not built ({LIB_PATH}); run "
                               "`python -m target_attention_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, res, args in _SIGS:
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _LIB = L
    return _LIB


def strerror(code: int) -> str:
    try:
        return lib().stca_strerror(code).decode()
    except RuntimeError:
        return "?"


def ptr(t):
    """Device (or host) address of a tensor, or None."""
    return None if t is None else t.data_ptr()


def stream_ptr(stream=None):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def check(rc, what=""):
    if rc != OK:
        raise StcaError(rc, what)
    return rc


# --------------------------------------------------------------------------- handles


def stca_create(cfg: StcaConfig):
    h = _vp()
    check(lib().stca_create(ctypes.byref(cfg), ctypes.byref(h)), "stca_create")
    return h


def stca_destroy(h):
    lib().stca_destroy(h)


def stca_pin_weights(h, weights, stream=None) -> int:
    """weights: the StcaWeights / HyfWeights object later passed to the forward calls."""
    return lib().stca_pin_weights(h, ctypes.byref(weights), stream_ptr(stream))


def stca_unpin_weights(h):
    lib().stca_unpin_weights(h)


def stca_sync_status(h) -> int:
    return lib().stca_sync_status(h)


STAGES = ["setup", "gather_ffn", "ffn_out", "kv", "attention", "merge", "query", "pointwise", "boost", "dedup"]


def stca_profile_enable(h, enable=True) -> int:
    return lib().stca_profile_enable(h, 1 if enable else 0)


def stca_stream_wait(stream=None, timeout_ms=0) -> int:
    """Waits at most timeout_ms for the work enqueued on the stream (OK or ERR_TIMEOUT)."""
    return lib().stca_stream_wait(stream_ptr(stream), timeout_ms)


def stca_k_wait_selftest(err, stream=None) -> int:
    return lib().stca_k_wait_selftest(ptr(err), stream_ptr(stream))


def stca_profile_stages(h, names) -> int:
    """Record only the named stages (an empty list stops recording)."""
    mask = 0
    for n in names:
        mask |= 1 << STAGES.index(n)
    return lib().stca_profile_stages(h, mask)


def stca_profile_read(h):
    """{stage: (total_ms, calls)} for the intervals recorded since enabling."""
    n = len(STAGES)
    ms = (ctypes.c_double * n)()
    calls = (ctypes.c_int64 * n)()
    check(lib().stca_profile_read(h, ms, calls), "stca_profile_read")
    return {STAGES[i]: (ms[i], calls[i]) for i in range(n)}


def stca_launch_count() -> int:
    return lib().stca_launch_count()


# --------------------------------------------------------------------------- forwards


def stca_forward(h, ids, lengths, dt, x_t, tpu, B, n_tok, t_tot, weights: StcaWeights, z_out, o_out=None,
                 stream=None) -> int:
    return lib().stca_forward(h, ptr(ids), ptr(lengths), ptr(dt), ptr(x_t), ptr(tpu), B, n_tok, t_tot,
                              ctypes.byref(weights), ptr(z_out), ptr(o_out), stream_ptr(stream))


def stca_forward_host(h, ids, lengths, dt, x_t, tpu, B, n_tok, t_tot, weights: StcaWeights, z_out,
                      stream=None) -> int:
    return lib().stca_forward_host(h, ptr(ids), ptr(lengths), ptr(dt), ptr(x_t), ptr(tpu), B, n_tok, t_tot,
                                   ctypes.byref(weights), ptr(z_out), stream_ptr(stream))


def stca_host_fence(h, stream=None) -> int:
    return lib().stca_host_fence(h, stream_ptr(stream))


def stca_lsplit_begin(h, ids, lengths, dt, x_t, tpu, B, n_tok, t_tot, weights: StcaWeights, stream=None) -> int:
    return lib().stca_lsplit_begin(h, ptr(ids), ptr(lengths), ptr(dt), ptr(x_t), ptr(tpu), B, n_tok, t_tot,
                                   ctypes.byref(weights), stream_ptr(stream))


def stca_lsplit_partial(h, layer, acc, ml, stream=None) -> int:
    return lib().stca_lsplit_partial(h, layer, ptr(acc), ptr(ml), stream_ptr(stream))


def stca_lsplit_merge(h, layer, ranks, all_acc, all_ml, z_out, stream=None) -> int:
    return lib().stca_lsplit_merge(h, layer, ranks, ptr(all_acc), ptr(all_ml), ptr(z_out), stream_ptr(stream))


def stca_pointwise_forward(h, ids, lengths, q, table, n_items, B, n_tok, out, stream=None) -> int:
    return lib().stca_pointwise_forward(h, ptr(ids), ptr(lengths), ptr(q), ptr(table), n_items, B, n_tok, ptr(out),
                                        stream_ptr(stream))


def stca_pointwise_forward_noalloc(ids, lengths, q, table, n_items, B, n_tok, out, err=None, stream=None) -> int:
    """Pointwise ReLU TA without a handle or any device allocation (scratch in the library)."""
    return lib().stca_pointwise_forward_noalloc(ptr(ids), ptr(lengths), ptr(q), ptr(table), n_items, B, n_tok,
                                                ptr(out), ptr(err), stream_ptr(stream))


def stca_k_ffn_fused(ids, dt, table, dt_table, n_items, M, layers, hidden, W13p, W2p, gammas, eps, Y, layer_stride,
                     stats, err=None, stream=None) -> int:
    """Fused history FFN (d = 256); gammas: list of per-layer device tensors."""
    arr = (ctypes.c_void_p * len(gammas))(*[g.data_ptr() for g in gammas])
    return lib().stca_k_ffn_fused(ptr(ids), ptr(dt), ptr(table), ptr(dt_table), n_items, M, layers, hidden, ptr(W13p),
                                  ptr(W2p), arr, eps, ptr(Y), layer_stride, ptr(stats), ptr(err), stream_ptr(stream))


def stca_attention_train_forward(Q, KV, hoff, toff, B, T, d, H, splits, score, part_acc, part_ml, out, lse,
                                 err=None, stream=None) -> int:
    """Training forward of the attention step: out and (softmax) lse [T, H]."""
    return lib().stca_attention_train_forward(ptr(Q), ptr(KV), ptr(hoff), ptr(toff), B, T, d, H, splits, score,
                                              ptr(part_acc), ptr(part_ml), ptr(out), ptr(lse), ptr(err),
                                              stream_ptr(stream))


def stca_attention_backward(Q, KV, hoff, toff, B, T, d, H, splits, score, out, lse, dout, dQ, dKV, part_dq=None,
                            stream=None, dKV16=None) -> int:
    """Backward of the attention step: dQ [T, d] and dKV [N, H, 2 d_h] (fp32; or bf16 into
    dKV16 when given, dKV then holding only partial sums)."""
    return lib().stca_attention_backward(ptr(Q), ptr(KV), ptr(hoff), ptr(toff), B, T, d, H, splits, score, ptr(out),
                                         ptr(lse), ptr(dout), ptr(dQ), ptr(dKV), ptr(part_dq), ptr(dKV16),
                                         stream_ptr(stream))


def hyformer_forward(h, ids_feed, len_feed, n_feed, ids_search, len_search, n_search, q0, B, n_query,
                     weights: HyfWeights, out, stream=None) -> int:
    return lib().hyformer_forward(h, ptr(ids_feed), ptr(len_feed), n_feed, ptr(ids_search), ptr(len_search),
                                  n_search, ptr(q0), B, n_query, ctypes.byref(weights), ptr(out),
                                  stream_ptr(stream))


# --------------------------------------------------------------------------- kernel-level


def stca_k_offsets(lengths, B, offsets, expected, err, stream=None) -> int:
    return lib().stca_k_offsets(ptr(lengths), B, ptr(offsets), expected, ptr(err), stream_ptr(stream))


def stca_k_pack_weight(W, K, N, dst, mode, row_offset, stream=None) -> int:
    return lib().stca_k_pack_weight(ptr(W), K, N, ptr(dst), mode, row_offset, stream_ptr(stream))


def stca_k_gemm_resident(amode, epi, A, ids, dt, table, dt_table, n_items, M, K, Wp, Nout, C, ldc, err,
                         stream=None, x_out=None, p_out=None) -> int:
    return lib().stca_k_gemm_resident(amode, epi, ptr(A), ptr(ids), ptr(dt), ptr(table), ptr(dt_table), n_items, M,
                                      K, ptr(Wp), Nout, ptr(C), ldc, ptr(x_out), ptr(p_out), ptr(err),
                                      stream_ptr(stream))


def stca_k_gemm_query(A, lda, M, K, ksplit, kshift, Wp, N, dual, R, ldr, C, ldc, err, stream=None) -> int:
    return lib().stca_k_gemm_query(ptr(A), lda, M, K, ksplit, kshift, ptr(Wp), N, int(dual), ptr(R), ldr, ptr(C),
                                   ldc, ptr(err), stream_ptr(stream))


def stca_k_gemm_rowwise(epi, A, M, K, Wp, N, gamma, beta, eps, C, ldc, err, stream=None) -> int:
    return lib().stca_k_gemm_rowwise(epi, ptr(A), M, K, ptr(Wp), N, ptr(gamma), ptr(beta), eps, ptr(C), ldc,
                                     ptr(err), stream_ptr(stream))


def stca_k_attention(kv_bf16, Q, KV, hoff, toff, B, T, d, H, splits, score, part_acc, part_ml, out, err,
                     stream=None) -> int:
    return lib().stca_k_attention(kv_bf16, ptr(Q), ptr(KV), ptr(hoff), ptr(toff), B, T, d, H, splits, score,
                                  ptr(part_acc), ptr(part_ml), ptr(out), ptr(err), stream_ptr(stream))


def stca_k_attention_rows(kv_bf16, Q, KV, hoff, toff, kv_rows, kv_len, kv_mult, B, T, d, H, splits, score, part_acc,
                          part_ml, out, err, stream=None) -> int:
    return lib().stca_k_attention_rows(kv_bf16, ptr(Q), ptr(KV), ptr(hoff), ptr(toff), ptr(kv_rows), ptr(kv_len),
                                       ptr(kv_mult), B, T, d, H, splits, score, ptr(part_acc), ptr(part_ml), ptr(out),
                                       ptr(err), stream_ptr(stream))


def stca_k_gemm_wgrad_workspace_bytes(M, K, N) -> int:
    return lib().stca_k_gemm_wgrad_workspace_bytes(M, K, N)


def stca_k_gemm_wgrad(A, lda, G, ldg, M, K, N, C, ldc, accumulate, ws, ws_bytes, stream=None, impl=0,
                      err=None) -> int:
    return lib().stca_k_gemm_wgrad(ptr(A), lda, ptr(G), ldg, M, K, N, ptr(C), ldc, accumulate, impl, ptr(ws),
                                   ws_bytes, ptr(err), stream_ptr(stream))


def stca_k_layer_norm_bwd_workspace_bytes(M, d) -> int:
    return lib().stca_k_layer_norm_bwd_workspace_bytes(M, d)


def stca_k_layer_norm_bwd(y, dxt, M, d, gamma, beta, eps, dy, xt, dgamma, dbeta, accumulate, ws, ws_bytes,
                          stream=None, fp32=0) -> int:
    return lib().stca_k_layer_norm_bwd(ptr(y), ptr(dxt), M, d, fp32, ptr(gamma), ptr(beta), eps, ptr(dy), ptr(xt),
                                       ptr(dgamma), ptr(dbeta), accumulate, ptr(ws), ws_bytes, stream_ptr(stream))


def stca_k_layer_norm(x, ldx, x_fp32, M, d, gamma, beta, eps, y, ldy, y_fp32, stream=None) -> int:
    return lib().stca_k_layer_norm(ptr(x), ldx, x_fp32, M, d, ptr(gamma), ptr(beta), eps, ptr(y), ldy, y_fp32,
                                   stream_ptr(stream))


def stca_k_f32_to_bf16(src, lds, rows, cols, dst, ldd, stream=None) -> int:
    return lib().stca_k_f32_to_bf16(ptr(src), lds, rows, cols, ptr(dst), ldd, stream_ptr(stream))


def stca_k_swiglu_bwd(P, dA, M, h, dP, a_out, stream=None, fp32=0) -> int:
    return lib().stca_k_swiglu_bwd(ptr(P), ptr(dA), M, h, fp32, ptr(dP), ptr(a_out), stream_ptr(stream))


def stca_k_table_rows_bwd(dX, M, d, ids, dt, n_items, dtable, ddt_table, err, stream=None) -> int:
    return lib().stca_k_table_rows_bwd(ptr(dX), M, d, ptr(ids), ptr(dt), n_items, ptr(dtable), ptr(ddt_table),
                                       ptr(err), stream_ptr(stream))


def stca_k_dedup_workspace_bytes(n) -> int:
    return lib().stca_k_dedup_workspace_bytes(n)


def stca_k_dedup(ids, dt, n, ws, uniq_idx, uniq_token, count, err, stream=None) -> int:
    return lib().stca_k_dedup(ptr(ids), ptr(dt), n, ptr(ws), ws.numel() * ws.element_size(), ptr(uniq_idx),
                              ptr(uniq_token), ptr(count), ptr(err), stream_ptr(stream))


def stca_k_compact_user_rows(hoff, B, rows, out_rows, out_mult, out_len, stream=None) -> int:
    return lib().stca_k_compact_user_rows(ptr(hoff), B, ptr(rows), ptr(out_rows), ptr(out_mult), ptr(out_len),
                                          stream_ptr(stream))
