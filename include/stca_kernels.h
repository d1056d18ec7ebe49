/*
 * stca_kernels.h - kernel-level entry points of libstca.  Each runs one step of the
 * forward passes declared in stca.h, on caller-provided device buffers, so that a step
 * can be checked on its own.  The same conventions hold (row-major, device pointers,
 * asynchronous on `stream`, int status, device-detected errors recorded in `err`, a
 * device int32 the caller zeroes and reads).  Nothing here allocates.
 */
#ifndef STCA_KERNELS_H
#define STCA_KERNELS_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Ragged layout ([notes] problem statement: one history of length L_u per user; RLB:
 * targets grouped per user).  offsets[0] = 0, offsets[i+1] = offsets[i] + lengths[i]
 * ([B+1] int32), every entry clamped to min(prefix sum, expected) with negative lengths
 * counted as 0, so offsets[B] <= expected always holds and no later kernel that trusts
 * the offsets leaves buffers sized by `expected`; records STCA_ERR_BAD_LENGTHS in err
 * for a negative length or a total different from `expected`. */
int stca_k_offsets(const int32_t* lengths, int B, int32_t* offsets, int expected, int32_t* err, void* stream);

/* Packs a bf16 weight W [K, N] (row-major, y = x W) into the K-major operand layout of
 * the tensor-core GEMMs: mode 0 writes column n to row row_offset + n of dst [rows, K];
 * modes 1 / 2 write W1 / W3 of a SwiGLU into the gate / up halves of 256-row groups
 * (row (n/128)*256 + n%128, plus 128 for mode 2).  Modes 3 and 4 place W's columns into a
 * [K, 2N] matrix WITHOUT transposing, which is the operand layout of the backward GEMMs
 * (dx = dy W^T takes W itself as its K-major operand): mode 3 puts column n at column
 * 128 (n / 64) + row_offset + n % 64 (row_offset 0 for W_K, 64 for W_V: the head-
 * interleaved [K_h | V_h] columns of the K/V rows, d_h = 64, N % 64 == 0), mode 4 at
 * column row_offset + n (row_offset 0 or N: [W1 | W3] side by side). */
int stca_k_pack_weight(const void* W, int K, int N, void* dst, int mode, int row_offset, void* stream);

/* Tensor-core GEMM with A resident in shared memory (K = 256 or 512), bf16 in, fp32
 * accumulate, bf16 out C [M, ldc]:
 *   amode 0: A dense [M, K];  amode 1: A row r = table[ids[r]] (+ dt_table[b(dt[r])]),
 *   b(x) = min(15, floor(log2(x + 1))): the fused embedding gather ([wechat] §1.1
 *   "lookup while computing"; time feature of [review] §四).
 *   epi 0: C = A Wp^T (Wp packed mode 0, [Nout, K], Nout % 256 == 0)
 *   epi 1: C = SiLU(A W1) * (A W3) (Wp packed modes 1+2, [2 Nout, K], Nout % 128 == 0).
 * An id outside [0, n_items) reads as a zero row and records STCA_ERR_ID_OUT_OF_RANGE.
 * x_out (amode 1 only, else STCA_ERR_INVALID_ARG; may be null): bf16 [M, K], 16-byte
 * aligned, receives the gathered A rows exactly as the MMAs consumed them, so that later
 * GEMMs over the same rows can take them as a dense amode-0 operand.  p_out (epi 1 only,
 * else STCA_ERR_INVALID_ARG; may be null): bf16 [M, 2 Nout], 16-byte aligned, receives the
 * pre-activations [A W1 | A W3] rounded from the same fp32 accumulators (the training
 * backward's SwiGLU derivative needs them). */
int stca_k_gemm_resident(int amode, int epi, const void* A, const int32_t* ids, const int32_t* dt, const void* table,
                         const void* dt_table, int64_t n_items, int M, int K, const void* Wp, int Nout, void* C,
                         int ldc, void* x_out, void* p_out, int32_t* err, void* stream);

/* Fused history FFN of `layers` layers for d = 256 ([notes] STCA: X~_l = LN_l(SwiGLU_l(X))
 * from the original X; [wechat] §1.1 lookup while computing).  Rows r < M of X are
 * gathered as in stca_k_gemm_resident amode 1 (K = 256); the SwiGLU hidden activations of
 * every layer stay on chip.  W13p: all layers' W1|W3 packed (modes 1 + 2) back to back,
 * [layers 2 hidden, 256]; W2p: all layers' W2 packed (mode 0) back to back, [layers 256,
 * hidden]; hidden % 128 == 0.  gammas: host array of `layers` device pointers (LayerNorm
 * gamma [256] fp32 per layer).  Writes, per layer l and row r, y'[l layer_stride + r] =
 * (A_l W2_l) * gamma_l (bf16 [256]) and stats[l layer_stride + r] = (mean, rstd) of A_l W2_l
 * (float2), so that LN_l = rstd (y' - mean gamma) + beta.  layer_stride >= M, a multiple of
 * 256; Y 16-byte aligned. */
int stca_k_ffn_fused(const int32_t* ids, const int32_t* dt, const void* table, const void* dt_table, int64_t n_items,
                     int M, int layers, int hidden, const void* W13p, const void* W2p, const float* const* gammas,
                     float eps, void* Y, int layer_stride, float* stats, int32_t* err, void* stream);

/* Target-side tensor-core GEMM ([review] §三 fusion formula; [notes] STCA query update):
 * fp32 activations A (each split into two bf16 terms, so products keep fp32 accuracy),
 * packed bf16 weights, fp32 result C [M, ldc]:
 *   dual 0: C = A W (+ R),  Wp = stca_k_pack_weight mode 0 of W [K, N] ([N, K]);
 *   dual 1: C = SiLU(A W1) * (A W3) (+ R), Wp = modes 1 + 2 of W1, W3 ([2N, K]).
 * Logical column k of A is read at k (k < ksplit) or k + kshift (two concatenated blocks).
 * Needs K % 64 == 0, ksplit % 64 == 0 when ksplit < K, N % 32 == 0 (N % 128 == 0 when dual),
 * A, C, R 16-byte aligned with lda, ldc, ldr % 4 == 0, else STCA_ERR_UNSUPPORTED.  R may be
 * null. */
int stca_k_gemm_query(const float* A, int64_t lda, int M, int K, int ksplit, int kshift, const void* Wp, int N,
                      int dual, const float* R, int64_t ldr, float* C, int64_t ldc, int32_t* err, void* stream);

/* Tensor-core GEMM with A streamed (K % 64 == 0) and the full output row (N = 256 or
 * 512) in tensor memory: epi 0 plain, epi 2 LayerNorm(gamma, beta, eps) of each row
 * ([notes] STCA: X~ = LN(SwiGLU(X))).  C [M, ldc] bf16. */
int stca_k_gemm_rowwise(int epi, const void* A, int M, int K, const void* Wp, int N, const float* gamma,
                        const float* beta, float eps, void* C, int ldc, int32_t* err, void* stream);

/* Split-L cross attention plus merge ([review] 核心公式; [wechat] §1.1 local attention,
 * then merge; §1.2 ReLU scores).  Q [T, d] fp32 projected queries.  KV bf16 when kv_bf16:
 * [N, H, 2 d_h], row n holding [K_h | V_h] of head h in columns [2 h d_h, 2 (h+1) d_h) (the
 * layout the library's K/V GEMM writes); else fp32 [N, 2d] (K in columns [0, d), V in
 * [d, 2d)).  hoff/toff [B+1] offsets of
 * the users' keys and queries.  score 0 softmax, 1 relu.  1 <= splits <= 32 slices of each
 * user's keys (else STCA_ERR_INVALID_ARG).  part_acc [splits, T, d] and part_ml
 * [splits, T, H, 2] float32 scratch; out [T, d] float32. */
int stca_k_attention(int kv_bf16, const float* Q, const void* KV, const int32_t* hoff, const int32_t* toff, int B,
                     int T, int d, int H, int splits, int score, float* part_acc, float* part_ml, float* out,
                     int32_t* err, void* stream);

/* The same attention over gathered, weighted keys (the form the library runs with
 * per-user compaction, [hyformer] §3.8.1 pooling of repeated keys): user u's keys are the
 * entries n = hoff[u] .. hoff[u] + len_u - 1 of kv_rows, len_u = kv_len[u] (NULL:
 * hoff[u+1] - hoff[u]); entry n is K/V row kv_rows[n] of KV and weighs kv_mult[n] tokens
 * (NULL: 1), which equals repeating that key kv_mult[n] times.  kv_rows [hoff[B]] int32
 * (required, each in [0, rows of KV): the caller's promise, not checked), kv_len [B],
 * kv_mult [hoff[B]] int32 (>= 1), device memory.  bf16 K/V only (kv_bf16 = 0 returns
 * STCA_ERR_UNSUPPORTED when kv_len or kv_mult is given); other arguments as above. */
int stca_k_attention_rows(int kv_bf16, const float* Q, const void* KV, const int32_t* hoff, const int32_t* toff,
                          const int32_t* kv_rows, const int32_t* kv_len, const int32_t* kv_mult, int B, int T, int d,
                          int H, int splits, int score, float* part_acc, float* part_ml, float* out, int32_t* err,
                          void* stream);

/* ---- training: the backward of one layer's history side ([notes] STCA: Xt = LN(SwiGLU(X)),
 * K, V = Xt W_K, Xt W_V; the pages train at about 2K-long histories).  The plain GEMMs of
 * the backward (dXt = dKV [W_K | W_V]^T, dA = dy W2^T, dX = dP [W1 | W3]^T) run on
 * stca_k_gemm_resident / stca_k_gemm_rowwise with the weights placed by pack modes 3 / 4
 * or taken as they are; the entries below are the rest. */

/* Weight gradient C [K, N] = A^T G (accumulate: C += A^T G) over M tokens: A [M, lda] and
 * G [M, ldg] bf16 row-major (features K and N of each token), C [K, ldc] fp32.  K and N
 * multiples of 128, lda and ldg multiples of 8, ldc of 4, pointers 16-byte aligned (else
 * STCA_ERR_UNSUPPORTED / STCA_ERR_INVALID_ARG).  ws: device scratch of at least
 * stca_k_gemm_wgrad_workspace_bytes(M, K, N) bytes (else STCA_ERR_CAPACITY): the token
 * slices' partial tiles, added in a fixed order, so the result is the same every run.
 * impl: 0 the tcgen05 kernel (both operands read MN-major from their token-major rows by
 * TMA), 1 the mma.sync kernel; other values STCA_ERR_INVALID_ARG.  err (device, may be
 * NULL) receives STCA_ERR_TIMEOUT if a bounded wait of the tcgen05 kernel ran out. */
size_t stca_k_gemm_wgrad_workspace_bytes(int M, int K, int N);
int stca_k_gemm_wgrad(const void* A, int64_t lda, const void* G, int64_t ldg, int M, int K, int N, float* C,
                      int64_t ldc, int accumulate, int impl, void* ws, size_t ws_bytes, int32_t* err, void* stream);

/* LayerNorm backward over rows of d = 256 or 512 (biased variance, eps): y [M, d] the
 * LayerNorm's input, dxt [M, d] the gradient of its output (bf16, or fp32 when fp32 != 0:
 * the target side keeps fp32 rows), gamma (beta may be NULL) [d] fp32.  Writes dy [M, d]
 * and, when xt is not NULL, the output xt = LN(y) [M, d] in the same type (for the K/V
 * weight gradients); dgamma, dbeta [d] fp32 are set (accumulate: added to).  Rows dense.
 * ws: at least stca_k_layer_norm_bwd_workspace_bytes(M, d) bytes. */
size_t stca_k_layer_norm_bwd_workspace_bytes(int M, int d);
int stca_k_layer_norm_bwd(const void* y, const void* dxt, int M, int d, int fp32, const float* gamma,
                          const float* beta, float eps, void* dy, void* xt, float* dgamma, float* dbeta,
                          int accumulate, void* ws, size_t ws_bytes, void* stream);

/* LayerNorm forward (biased variance, eps) of rows x [M, ldx] -> y [M, ldy], d = 256 or
 * 512, both bf16 or both fp32 (x_fp32 = y_fp32; else STCA_ERR_UNSUPPORTED): the training
 * step recomputes the forward's LayerNorm outputs with it. */
int stca_k_layer_norm(const void* x, int64_t ldx, int x_fp32, int M, int d, const float* gamma, const float* beta,
                      float eps, void* y, int64_t ldy, int y_fp32, void* stream);

/* dst [rows, ldd] bf16 = src [rows, lds] fp32 rounded to nearest even (operands of the
 * weight-gradient GEMM from the target side's fp32 rows). */
int stca_k_f32_to_bf16(const float* src, int64_t lds, int rows, int cols, void* dst, int64_t ldd, void* stream);

/* SwiGLU backward: A = SiLU(P1) * P3 with P = [P1 | P3] [M, 2h] (x W1 and x W3 side by side)
 * and dA [M, h], bf16 (fp32 when fp32 != 0).  Writes dP = [dP1 | dP3] [M, 2h] with
 * dP1 = dA P3 SiLU'(P1), dP3 = dA SiLU(P1), and A [M, h] into a_out when not NULL, in the
 * same type.  h % 8 == 0; bf16 pointers 16-byte aligned. */
int stca_k_swiglu_bwd(const void* P, const void* dA, int M, int h, int fp32, void* dP, void* a_out, void* stream);

/* The lookup's backward: dtable[ids[n]] += dX[n] for n < M (dX [M, d] bf16, dtable
 * [n_items, d] fp32) and, with dt and ddt_table, ddt_table[b(dt[n])] += dX[n] ([16, d] fp32,
 * b as in stca_k_gemm_resident).  d % 8 == 0 (at most 768 with dt), dX and dtable 16-byte
 * aligned.  fp32 atomic adds: the order of the additions into a row varies between runs.
 * An id outside [0, n_items) is skipped and records STCA_ERR_ID_OUT_OF_RANGE in err. */
int stca_k_table_rows_bwd(const void* dX, int M, int d, const int32_t* ids, const int32_t* dt, int64_t n_items,
                          float* dtable, float* ddt_table, int32_t* err, void* stream);

/* Distinct history keys (HyFormer page §3.8.1, GPU pooling): key(n) = (ids[n], bucket(dt[n]))
 * (bucket 0 when dt is NULL).  Writes uniq_idx[n] in [0, *count) with equal keys mapped to
 * the same index and distinct keys to distinct indices, and uniq_token[u] = a token whose
 * key is u.  The numbering order is unspecified.  ws: caller scratch of at least
 * stca_k_dedup_workspace_bytes(n) bytes; count: device int32. */
size_t stca_k_dedup_workspace_bytes(int n);
int stca_k_dedup(const int32_t* ids, const int32_t* dt, int n, void* ws, size_t ws_bytes, int32_t* uniq_idx,
                 int32_t* uniq_token, int32_t* count, int32_t* err, void* stream);

/* Per-user compaction of K/V rows (keys of one user with the same row have equal scores, so
 * attention may weigh one entry by the number of its tokens).  User u owns tokens
 * hoff[u] .. hoff[u+1]-1 ([B+1] device offsets) with K/V rows rows[n]; on return
 * out_rows[hoff[u] + i] (i < out_len[u]) are the user's distinct rows in order of first
 * token and out_mult[hoff[u] + i] their token counts.  A user with 16384 or more tokens
 * keeps one entry per token (count 1).  out_rows / out_mult: [hoff[B]] int32, out_len: [B]
 * int32, device memory, not aliasing the inputs. */
int stca_k_compact_user_rows(const int32_t* hoff, int B, const int32_t* rows, int32_t* out_rows, int32_t* out_mult,
                             int32_t* out_len, void* stream);

/* Self-test of the bounded waits every pipelined kernel uses: one CTA waits on a barrier
 * that nothing completes, gives up after the library's wait limit (about 2 s), records
 * STCA_ERR_TIMEOUT in *err (device int32) and exits normally, leaving the context usable.
 * Asynchronous on `stream`. */
int stca_k_wait_selftest(int32_t* err, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* STCA_KERNELS_H */
