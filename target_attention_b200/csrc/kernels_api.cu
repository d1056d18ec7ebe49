// Kernel-level C entry points (include/stca_kernels.h): thin wrappers over the launchers.
#include <cstring>

#include "../../include/stca_kernels.h"
#include "common.cuh"
#include "internal.h"

using namespace stca;

namespace {

// One CTA waits on an mbarrier whose phase never completes: the bounded wait gives up and
// the kernel records the timeout and returns (the pattern of every pipelined kernel).
__global__ void wait_selftest_kernel(int32_t* err) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0 && !mbar_wait(&bar, 0)) set_error(err, STCA_ERR_TIMEOUT);
  __syncthreads();
}

}  // namespace

extern "C" {

int stca_k_wait_selftest(int32_t* err, void* stream) {
  if (!err) return STCA_ERR_INVALID_ARG;
  wait_selftest_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(err);
  note_launch();
  return cudaGetLastError() == cudaSuccess ? 0 : STCA_ERR_CUDA;
}


int stca_k_offsets(const int32_t* lengths, int B, int32_t* offsets, int expected, int32_t* err, void* stream) {
  if (B < 0 || !offsets || (B > 0 && !lengths)) return STCA_ERR_INVALID_ARG;
  return exclusive_offsets(lengths, B, offsets, expected, err, reinterpret_cast<cudaStream_t>(stream));
}

int stca_k_pack_weight(const void* W, int K, int N, void* dst, int mode, int row_offset, void* stream) {
  if (!W || !dst || mode < 0 || mode > 4) return STCA_ERR_INVALID_ARG;
  if (mode >= 3) return place_cols(W, K, N, dst, mode, row_offset, reinterpret_cast<cudaStream_t>(stream));
  return tc_pack_weight(W, K, N, dst, mode, row_offset, reinterpret_cast<cudaStream_t>(stream));
}

size_t stca_k_gemm_wgrad_workspace_bytes(int M, int K, int N) { return gemm_wgrad_workspace_bytes(M, K, N); }

int stca_k_gemm_wgrad(const void* A, int64_t lda, const void* G, int64_t ldg, int M, int K, int N, float* C,
                      int64_t ldc, int accumulate, int impl, void* ws, size_t ws_bytes, int32_t* err, void* stream) {
  if (M < 0 || (M > 0 && (!A || !G || !ws)) || !C) return STCA_ERR_INVALID_ARG;
  return gemm_wgrad(A, lda, G, ldg, M, K, N, C, ldc, accumulate, impl, ws, ws_bytes, err,
                    reinterpret_cast<cudaStream_t>(stream));
}

size_t stca_k_layer_norm_bwd_workspace_bytes(int M, int d) { return M < 0 ? 0 : layer_norm_bwd_workspace_bytes(M, d); }

int stca_k_layer_norm_bwd(const void* y, const void* dxt, int M, int d, int fp32, const float* gamma,
                          const float* beta, float eps, void* dy, void* xt, float* dgamma, float* dbeta,
                          int accumulate, void* ws, size_t ws_bytes, void* stream) {
  return layer_norm_bwd(y, dxt, M, d, fp32, gamma, beta, eps, dy, xt, dgamma, dbeta, accumulate, ws, ws_bytes,
                        reinterpret_cast<cudaStream_t>(stream));
}

int stca_k_layer_norm(const void* x, int64_t ldx, int x_fp32, int M, int d, const float* gamma, const float* beta,
                      float eps, void* y, int64_t ldy, int y_fp32, void* stream) {
  return layer_norm_fwd(x, ldx, x_fp32, M, d, gamma, beta, eps, y, ldy, y_fp32, reinterpret_cast<cudaStream_t>(stream));
}

int stca_k_swiglu_bwd(const void* P, const void* dA, int M, int h, int fp32, void* dP, void* a_out, void* stream) {
  return swiglu_bwd(P, dA, M, h, fp32, dP, a_out, reinterpret_cast<cudaStream_t>(stream));
}

int stca_k_f32_to_bf16(const float* src, int64_t lds, int rows, int cols, void* dst, int64_t ldd, void* stream) {
  return f32_to_bf16(src, lds, rows, cols, dst, ldd, reinterpret_cast<cudaStream_t>(stream));
}

int stca_k_table_rows_bwd(const void* dX, int M, int d, const int32_t* ids, const int32_t* dt, int64_t n_items,
                          float* dtable, float* ddt_table, int32_t* err, void* stream) {
  return table_rows_bwd(dX, M, d, ids, dt, n_items, dtable, ddt_table, err, reinterpret_cast<cudaStream_t>(stream));
}

int stca_k_gemm_resident(int amode, int epi, const void* A, const int32_t* ids, const int32_t* dt, const void* table,
                         const void* dt_table, int64_t n_items, int M, int K, const void* Wp, int Nout, void* C,
                         int ldc, void* x_out, void* p_out, int32_t* err, void* stream) {
  if (M < 0 || !Wp || (M > 0 && !C)) return STCA_ERR_INVALID_ARG;
  if (x_out && amode != A_GATHER) return STCA_ERR_INVALID_ARG;
  if (p_out && epi != EPI_SWIGLU) return STCA_ERR_INVALID_ARG;
  if (epi != EPI_PLAIN && epi != EPI_SWIGLU) return STCA_ERR_INVALID_ARG;
  GatherSrc g;
  memset(&g, 0, sizeof(g));
  if (amode == A_GATHER) {
    if (M > 0 && (!ids || !table || n_items <= 0)) return STCA_ERR_INVALID_ARG;
    g.ids = ids;
    g.dt = dt_table ? dt : nullptr;
    g.table = table;
    g.dt_table = dt ? dt_table : nullptr;
    g.n_items = n_items;
  } else if (amode != A_TMA || (M > 0 && !A)) {
    return STCA_ERR_INVALID_ARG;
  }
  return tc_gemm_resident(amode, epi, A, g, M, K, Wp, Nout, C, ldc, err, reinterpret_cast<cudaStream_t>(stream),
                          nullptr, x_out, nullptr, 0, p_out);
}

int stca_k_ffn_fused(const int32_t* ids, const int32_t* dt, const void* table, const void* dt_table, int64_t n_items,
                     int M, int layers, int hidden, const void* W13p, const void* W2p, const float* const* gammas,
                     float eps, void* Y, int layer_stride, float* stats, int32_t* err, void* stream) {
  if (M < 0 || (M > 0 && (!ids || !table || n_items <= 0 || !gammas))) return STCA_ERR_INVALID_ARG;
  GatherSrc g;
  memset(&g, 0, sizeof(g));
  g.ids = ids;
  g.dt = dt_table ? dt : nullptr;
  g.table = table;
  g.dt_table = dt ? dt_table : nullptr;
  g.n_items = n_items;
  return tc_ffn_fused(g, M, nullptr, layers, hidden, W13p, W2p, gammas, eps, Y, layer_stride, stats, err,
                      reinterpret_cast<cudaStream_t>(stream));
}

int stca_k_gemm_query(const float* A, int64_t lda, int M, int K, int ksplit, int kshift, const void* Wp, int N,
                      int dual, const float* R, int64_t ldr, float* C, int64_t ldc, int32_t* err, void* stream) {
  if (M < 0 || K <= 0 || N <= 0 || !Wp || (M > 0 && (!A || !C)) || ksplit < 0 || kshift < 0 ||
      (dual != 0 && dual != 1))
    return STCA_ERR_INVALID_ARG;
  SimtGemmArgs<float, bf16> a;
  memset(&a, 0, sizeof(a));
  a.M = M;
  a.N = N;
  a.K = K;
  a.A = A;
  a.lda = lda;
  a.ksplit = ksplit < K ? ksplit : K;
  a.kshift = ksplit < K ? kshift : 0;
  a.B = reinterpret_cast<const bf16*>(Wp);
  a.B2 = dual ? reinterpret_cast<const bf16*>(Wp) : nullptr;
  a.C = C;
  a.ldc = ldc;
  a.R = R;
  a.ldr = ldr;
  a.batch = 1;
  a.err = err;
  return tc_query_gemm(a, Wp, reinterpret_cast<cudaStream_t>(stream));
}

int stca_k_gemm_rowwise(int epi, const void* A, int M, int K, const void* Wp, int N, const float* gamma,
                        const float* beta, float eps, void* C, int ldc, int32_t* err, void* stream) {
  if (M < 0 || (M > 0 && (!A || !C)) || !Wp) return STCA_ERR_INVALID_ARG;
  if (epi != EPI_PLAIN && epi != EPI_LN) return STCA_ERR_INVALID_ARG;
  return tc_gemm_rowwise(epi, A, M, K, Wp, N, gamma, beta, eps, C, ldc, err, reinterpret_cast<cudaStream_t>(stream));
}

int stca_k_attention_rows(int kv_bf16, const float* Q, const void* KV, const int32_t* hoff, const int32_t* toff,
                          const int32_t* kv_rows, const int32_t* kv_len, const int32_t* kv_mult, int B, int T, int d,
                          int H, int splits, int score, float* part_acc, float* part_ml, float* out, int32_t* err,
                          void* stream) {
  if (B < 0 || T < 0 || d <= 0 || H <= 0 || d % H != 0 || splits < 1 || splits > 32 || (score != 0 && score != 1))
    return STCA_ERR_INVALID_ARG;
  if (B > 0 && T > 0 && (!Q || !KV || !hoff || !toff || !part_acc || !part_ml || !out)) return STCA_ERR_INVALID_ARG;
  if (!kv_rows && (kv_len || kv_mult)) return STCA_ERR_INVALID_ARG;
  if (!kv_bf16 && (kv_len || kv_mult)) return STCA_ERR_UNSUPPORTED;
  AttnArgs a;
  a.Q = Q;
  a.KV = KV;
  a.hoff = hoff;
  a.toff = toff;
  a.kv_rows = kv_rows;
  a.kv_len = kv_len;
  a.kv_mult = kv_mult;
  a.B = B;
  a.T = T;
  a.d = d;
  a.H = H;
  a.splits = splits;
  a.score = score;
  a.part_acc = part_acc;
  a.part_ml = part_ml;
  a.out = out;
  a.err = err;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int rc = kv_bf16 ? attention_bf16(a, s) : attention_f32(a, s);
  if (rc != STCA_OK) return rc;
  return attention_needs_merge(a, kv_bf16 != 0) ? attention_merge(a, s) : STCA_OK;
}

int stca_k_attention(int kv_bf16, const float* Q, const void* KV, const int32_t* hoff, const int32_t* toff, int B,
                     int T, int d, int H, int splits, int score, float* part_acc, float* part_ml, float* out,
                     int32_t* err, void* stream) {
  return stca_k_attention_rows(kv_bf16, Q, KV, hoff, toff, nullptr, nullptr, nullptr, B, T, d, H, splits, score,
                               part_acc, part_ml, out, err, stream);
}

size_t stca_k_dedup_workspace_bytes(int n) { return n < 0 ? 0 : dedup_workspace_bytes(n); }

int stca_k_dedup(const int32_t* ids, const int32_t* dt, int n, void* ws, size_t ws_bytes, int32_t* uniq_idx,
                 int32_t* uniq_token, int32_t* count, int32_t* err, void* stream) {
  if (n < 0 || !count || (n > 0 && (!ids || !ws || !uniq_idx || !uniq_token))) return STCA_ERR_INVALID_ARG;
  return dedup_fused(ids, dt, n, ws, ws_bytes, uniq_idx, uniq_token, count, nullptr, 0, nullptr, nullptr, nullptr,
                     err, reinterpret_cast<cudaStream_t>(stream));
}

int stca_k_compact_user_rows(const int32_t* hoff, int B, const int32_t* rows, int32_t* out_rows, int32_t* out_mult,
                             int32_t* out_len, void* stream) {
  if (B < 0 || (B > 0 && (!hoff || !rows || !out_rows || !out_mult || !out_len))) return STCA_ERR_INVALID_ARG;
  return compact_user_rows(hoff, B, rows, out_rows, out_mult, out_len, reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"
