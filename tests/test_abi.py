"""C-ABI checks that need no GPU: the library loads, exports every function the headers
declare, and rejects bad arguments on the host before touching CUDA."""
import ctypes
import os
import re

import pytest

import target_attention_b200 as tab
from target_attention_b200 import binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = set()
    for hdr in ("stca.h", "stca_kernels.h"):
        text = open(os.path.join(ROOT, "include", hdr)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"^\s*(?:const\s+)?\w+\s*\*?\s*(\w+)\s*\(", text, flags=re.M):
            names.add(m.group(1))
    return names


def test_library_exports_every_declared_function():
    L = tab.lib()
    declared = _declared_functions()
    assert {"stca_create", "stca_forward", "stca_pointwise_forward", "hyformer_forward"} <= declared
    missing = [n for n in declared if not hasattr(L, n)]
    assert not missing, missing
    assert declared == set(B.EXPORTED), declared ^ set(B.EXPORTED)


def test_struct_layouts_match_c():
    # sizes computed by the C compiler from include/stca.h
    assert ctypes.sizeof(B.StcaConfig) == 56
    assert ctypes.sizeof(B.StcaWeights) == 1072
    assert ctypes.sizeof(B.HyfWeights) == 21656


def test_strerror_covers_all_codes():
    for c in range(8):
        assert B.strerror(c) not in ("?", "unknown status")
    assert B.strerror(99) == "unknown status"


def _cfg(**kw):
    base = dict(mode=B.MODE_STCA, M=2, d=256, H=4, hidden=512, dtype=B.BF16, score=B.SOFTMAX, time_buckets=0,
                max_users=4, max_tokens=100, max_targets=8, dedup=0, ln_eps=1e-5)
    base.update(kw)
    return B.StcaConfig(**base)


@pytest.mark.parametrize("kw, code", [
    (dict(M=0), B.ERR_INVALID_ARG),
    (dict(M=9), B.ERR_INVALID_ARG),
    (dict(d=384, H=6), B.ERR_UNSUPPORTED),        # bf16 needs d in {256, 512}
    (dict(H=8), B.ERR_UNSUPPORTED),               # d_h = 32 with bf16
    (dict(hidden=200), B.ERR_UNSUPPORTED),        # hidden % 128
    (dict(time_buckets=8), B.ERR_UNSUPPORTED),
    (dict(dtype=7), B.ERR_INVALID_ARG),
    (dict(score=3), B.ERR_INVALID_ARG),
    (dict(max_tokens=-1), B.ERR_INVALID_ARG),
    (dict(mode=B.MODE_POINTWISE, d=256), B.ERR_UNSUPPORTED),
    (dict(mode=B.MODE_HYFORMER, d=256), B.ERR_UNSUPPORTED),
    (dict(mode=5), B.ERR_INVALID_ARG),
    (dict(dtype=B.FP32, d=96, H=2), B.ERR_UNSUPPORTED),   # d_h = 48
    (dict(dtype=B.FP32, d=64, H=2, dedup=1), B.ERR_UNSUPPORTED),
    (dict(dtype=B.FP32, d=64, H=2, dedup=2), B.ERR_UNSUPPORTED),
    (dict(dedup=3), B.ERR_INVALID_ARG),
    (dict(kv_fold=2), B.ERR_INVALID_ARG),
    (dict(kv_fold=1, d=512, H=8, hidden=1024), B.ERR_UNSUPPORTED),   # the fold needs d = 256
    (dict(kv_fold=1, dtype=B.FP32, d=64, H=2, hidden=128), B.ERR_UNSUPPORTED),
    (dict(dedup=-1), B.ERR_INVALID_ARG),
])
def test_create_rejects_bad_configs(kw, code):
    h = ctypes.c_void_p()
    assert tab.lib().stca_create(ctypes.byref(_cfg(**kw)), ctypes.byref(h)) == code
    assert h.value is None


def test_null_arguments_rejected_on_host():
    L = tab.lib()
    assert L.stca_create(None, None) == B.ERR_INVALID_ARG
    h = ctypes.c_void_p()
    assert L.stca_create(None, ctypes.byref(h)) == B.ERR_INVALID_ARG
    w = B.StcaWeights()
    assert L.stca_forward(None, None, None, None, None, None, 1, 1, 1, ctypes.byref(w), None, None, None) \
        == B.ERR_INVALID_ARG
    assert L.stca_pointwise_forward(None, None, None, None, None, 1, 1, 1, None, None) == B.ERR_INVALID_ARG
    # rows move by 16-byte-aligned copies: q or table off a 16-byte boundary is refused first
    assert L.stca_pointwise_forward_noalloc(None, 16, 24, 16, 100, 1, 0, 16, None, None) == B.ERR_INVALID_ARG
    assert L.stca_pointwise_forward_noalloc(None, 16, 16, 40, 100, 1, 0, 16, None, None) == B.ERR_INVALID_ARG
    assert L.stca_sync_status(None) == B.ERR_INVALID_ARG
    assert L.stca_pin_weights(None, None, None) == B.ERR_INVALID_ARG
    assert L.stca_lsplit_begin(None, None, None, None, None, None, 1, 1, 1, ctypes.byref(w), None) \
        == B.ERR_INVALID_ARG
    assert L.stca_lsplit_partial(None, 0, None, None, None) == B.ERR_INVALID_ARG
    assert L.stca_lsplit_merge(None, 0, 2, None, None, None, None) == B.ERR_INVALID_ARG
    assert L.stca_k_wait_selftest(None, None) == B.ERR_INVALID_ARG
    assert L.stca_stream_wait(None, -1) == B.ERR_INVALID_ARG
    assert L.stca_host_fence(None, None) == B.ERR_INVALID_ARG
    L.stca_unpin_weights(None)
    L.stca_destroy(None)
    # kernel-level entry points validate before launching
    assert L.stca_k_attention(1, None, None, None, None, 1, 1, 256, 3, 1, 0, None, None, None, None, None) \
        == B.ERR_INVALID_ARG
    assert L.stca_k_attention_rows(1, 16, 16, 16, 16, None, 16, None, 1, 1, 64, 1, 1, 0, 16, 16, 16, None, None) \
        == B.ERR_INVALID_ARG                          # key lengths or weights without key rows
    assert L.stca_k_attention_rows(0, 16, 16, 16, 16, 16, None, 16, 1, 1, 64, 1, 1, 0, 16, 16, 16, None, None) \
        == B.ERR_UNSUPPORTED                          # key weights with fp32 K/V
    assert L.stca_k_pack_weight(None, 4, 4, None, 0, 0, None) == B.ERR_INVALID_ARG
    assert L.stca_k_pack_weight(16, 64, 100, 16, 3, 0, None) == B.ERR_INVALID_ARG   # mode 3 needs N % 64
    assert L.stca_k_pack_weight(16, 64, 64, 16, 3, 32, None) == B.ERR_INVALID_ARG   # ... and the K or V half
    assert L.stca_k_pack_weight(16, 64, 64, 16, 5, 0, None) == B.ERR_INVALID_ARG
    # training entries: shapes the kernels do not take, workspace too small, missing buffers
    assert L.stca_k_gemm_wgrad(16, 128, 16, 128, 100, 96, 128, 16, 128, 0, 0, 16, 1 << 30, None, None) == \
        B.ERR_UNSUPPORTED
    for impl in (0, 1):
        assert L.stca_k_gemm_wgrad(16, 128, 16, 128, 100, 128, 128, 16, 128, 0, impl, 16, 16, None, None) == \
            B.ERR_CAPACITY
    assert L.stca_k_gemm_wgrad(16, 120, 16, 128, 100, 128, 128, 16, 128, 0, 0, 16, 1 << 30, None, None) == \
        B.ERR_INVALID_ARG
    assert L.stca_k_gemm_wgrad(None, 128, 16, 128, 100, 128, 128, 16, 128, 0, 0, 16, 1 << 30, None, None) == \
        B.ERR_INVALID_ARG
    assert L.stca_k_gemm_wgrad(16, 128, 16, 128, 100, 128, 128, 16, 128, 0, 3, 16, 1 << 30, None, None) == \
        B.ERR_INVALID_ARG
    assert L.stca_k_layer_norm_bwd(16, 16, 10, 384, 0, 16, None, 1e-5, 16, None, 16, 16, 0, 16, 1 << 20, None) \
        == B.ERR_UNSUPPORTED
    assert L.stca_k_layer_norm_bwd(16, 16, 10, 256, 0, 16, None, 1e-5, 16, None, 16, 16, 0, 16, 4, None) \
        == B.ERR_CAPACITY
    assert L.stca_k_swiglu_bwd(16, 16, 10, 12, 0, 16, None, None) == B.ERR_UNSUPPORTED        # h % 8
    assert L.stca_k_swiglu_bwd(16, 16, 10, 16, 0, 24, None, None) == B.ERR_INVALID_ARG        # alignment
    assert L.stca_k_table_rows_bwd(16, 10, 12, 16, None, 100, 16, None, None, None) == B.ERR_INVALID_ARG
    assert L.stca_k_layer_norm(16, 256, 1, 10, 256, 16, None, 1e-5, 16, 256, 0, None) == B.ERR_UNSUPPORTED  # fp32 -> bf16
    assert L.stca_k_layer_norm(16, 100, 1, 10, 256, 16, None, 1e-5, 16, 256, 1, None) == B.ERR_INVALID_ARG  # ldx < d
    assert L.stca_k_f32_to_bf16(16, 8, 4, 16, 16, 16, None) == B.ERR_INVALID_ARG                           # lds < cols
    assert L.stca_k_table_rows_bwd(16, 10, 256, None, None, 100, 16, None, None, None) == B.ERR_INVALID_ARG
    assert L.stca_k_gemm_resident(1, 1, None, None, None, None, None, 0, 5, 256, None, 128, None, 128, None, None,
                                  None, None) == B.ERR_INVALID_ARG
    # x_out only with the gather, p_out only with the SwiGLU epilogue
    assert L.stca_k_gemm_resident(0, 0, 16, None, None, None, None, 0, 5, 256, 16, 256, 16, 256, 16, None,
                                  None, None) == B.ERR_INVALID_ARG
    assert L.stca_k_gemm_resident(0, 0, 16, None, None, None, None, 0, 5, 256, 16, 256, 16, 256, None, 16,
                                  None, None) == B.ERR_INVALID_ARG
    assert L.stca_k_attention(1, 16, 16, 16, 16, 1, 1, 256, 4, 33, 0, 16, 16, 16, None, None) == B.ERR_INVALID_ARG
    # target-side GEMM: missing operands, then shapes the tensor-core kernel does not take
    assert L.stca_k_gemm_query(None, 64, 1, 64, 64, 0, None, 32, 0, None, 0, None, 32, None, None) \
        == B.ERR_INVALID_ARG
    assert L.stca_k_gemm_query(16, 100, 1, 100, 100, 0, 16, 32, 0, None, 0, 16, 32, None, None) \
        == B.ERR_UNSUPPORTED                          # K % 64
    assert L.stca_k_gemm_query(16, 64, 1, 64, 64, 0, 16, 64, 1, None, 0, 16, 64, None, None) \
        == B.ERR_UNSUPPORTED                          # dual needs N % 128
    assert L.stca_k_gemm_rowwise(5, None, 0, 64, None, 256, None, None, 1e-5, None, 256, None, None) \
        == B.ERR_INVALID_ARG


def test_training_entries_reject_bad_arguments_on_host():
    L = tab.lib()
    f, b = L.stca_attention_train_forward, L.stca_attention_backward
    # splits outside 1..32, a bad score, a negative count, missing buffers
    assert f(16, 16, 16, 16, 1, 1, 256, 4, 0, 0, None, None, 16, 16, None, None) == B.ERR_INVALID_ARG
    assert f(16, 16, 16, 16, 1, 1, 256, 4, 33, 0, 16, 16, 16, 16, None, None) == B.ERR_INVALID_ARG
    assert f(16, 16, 16, 16, 1, 1, 256, 4, 1, 2, None, None, 16, 16, None, None) == B.ERR_INVALID_ARG
    assert f(16, 16, 16, 16, -1, 1, 256, 4, 1, 0, None, None, 16, 16, None, None) == B.ERR_INVALID_ARG
    assert f(16, 16, 16, 16, 1, 1, 256, 4, 1, 0, None, None, 16, None, None, None) == B.ERR_INVALID_ARG  # lse
    assert f(16, 16, 16, 16, 1, 1, 256, 4, 2, 0, None, None, 16, 16, None, None) == B.ERR_INVALID_ARG  # scratch
    assert f(16, 16, 16, 16, 1, 1, 256, 8, 1, 0, None, None, 16, 16, None, None) == B.ERR_UNSUPPORTED  # d_h 32
    assert b(16, 16, 16, 16, 1, 1, 256, 4, 1, 0, 16, 16, 16, 16, None, None, None, None) == B.ERR_INVALID_ARG  # dKV
    assert b(16, 16, 16, 16, 1, 1, 256, 4, 2, 0, 16, 16, 16, 16, 16, None, None, None) == B.ERR_INVALID_ARG  # part_dq
    assert b(16, 16, 16, 16, 1, 1, 256, 4, 1, 0, None, None, 16, 16, 16, None, None, None) == B.ERR_INVALID_ARG  # out
    assert b(16, 16, 16, 16, 1, 1, 512, 4, 1, 0, 16, 16, 16, 16, 16, None, None, None) == B.ERR_UNSUPPORTED  # d_h 128
    assert b(16, 16, 16, 16, 1, 1, 256, 4, 1, 0, 16, 16, 16, 16, 16, None, 18, None) == B.ERR_INVALID_ARG  # bf16 out


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(B, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(B, "_LIB", None)
    with pytest.raises(RuntimeError, match="not built"):
        B.lib()
