// Host-side launchers shared between the library's translation units.
#pragma once

#include <cstring>
#include <utility>

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace stca {

// Counts one kernel launch of this library (read with stca_launch_count()).
void note_launch();

// Rows of A read straight from an embedding table by item id ("lookup while
// computing"): row r of A is table[ids[r]] (+ dt_table[bucket(dt[r])]).
struct GatherSrc {
  const int32_t* ids;
  const int32_t* dt;      // may be null
  const int32_t* rows;    // row r reads token rows[r] (distinct-row form), or null: token r
  const void* table;      // [n_items, K] (bf16 or fp32, the kernel's type)
  const void* dt_table;   // [16, K] or null
  int64_t n_items;
};

enum AMode { A_TMA = 0, A_GATHER = 1 };
enum Epi { EPI_PLAIN = 0, EPI_SWIGLU = 1, EPI_LN = 2, EPI_LNSTAT = 3, EPI_LNFOLD = 4 };

// LayerNorm folded into the GEMM that follows it.  With s = (mean_r, rstd_r) of row r of y
// and y' = y * gamma (per column), LN(y) W = rstd_r (y' W - mean_r c) + b with
// c = gamma^T W and b = beta^T W, so the LN GEMM only has to write y' and the row moments
// (EPI_LNSTAT) and the next GEMM applies the row scale and shift in its epilogue
// (EPI_LNFOLD).  stats: [rows][2] fp32; cvec, bvec: [N] fp32 for the N output columns.
struct EpiFold {
  const float* stats;
  const float* cvec;
  const float* bvec;
  // EPI_SWIGLU only: when set, bf16 [M, 2 Nout] receiving the pre-activations [A W1 | A W3]
  // (rounded from the same fp32 accumulators), which the training backward needs
  void* p_out;
};
// c and b of the fold for W = [WK | WV] ([d, d] bf16 each, row-major): out [2][2d] fp32,
// in the K/V GEMM's output column order: head-interleaved [K_h | V_h] per head of width dh
// (the order pack mode 3 gives), or K then V when dh == 0.
int fold_consts(const float* gamma, const float* beta, const void* WK, const void* WV, int d, int dh, float* out,
                cudaStream_t s);

// ---------------------------------------------------------------- tcgen05 GEMMs (bf16)

// Packs a [K, N] row-major bf16 weight into the K-major [rows, K] operand layout.
// mode 0: dst row (row_offset + n)        <- column n
// mode 1: SwiGLU gate half:  dst row (n/128)*256 + n%128       <- column n of W1
// mode 2: SwiGLU up half:    dst row (n/128)*256 + 128 + n%128 <- column n of W3
// mode 3: head-interleaved:  dst row (n/group)*2*group + row_offset + n%group <- column n
// modes 4, 5: block-diagonal folds of a [d, d] projection per head of width group (the
//   W_K / W_V fold into the queries): mode 4 writes W[k][n] to dst[(n/group) K + k][n] of
//   dst [H K, N]; mode 5 to dst[n][(n/group) K + k] of dst [N, H K]; the rest of dst stays
//   as it was (zero it once)
int tc_pack_weight(const void* W, int K, int N, void* dst, int mode, int row_offset, cudaStream_t s);

// The same packing for many matrices with one launch per PACK_MAX_JOBS jobs.
struct PackJob {
  const void* W;  // [K, N] bf16
  void* dst;
  int K, N, mode, row_offset;
  // mode 3 (head-interleaved K|V): column n goes to row (n / group) * 2 group + row_offset
  // + n % group, so that W_K (row_offset 0) and W_V (row_offset group) of head n / group
  // make one 2 group-row block and the GEMM output row holds [K_h | V_h] per head
  int group;
};
constexpr int PACK_MAX_JOBS = 48;
int tc_pack_weights(const PackJob* jobs, int n, cudaStream_t s);

// C[M, Nout] (bf16, row stride ldc) from A (resident in shared memory, K in {256, 512}):
//   amode A_TMA: A is a dense bf16 [M, K] matrix; A_GATHER: rows gathered via `g`.
//   epi EPI_PLAIN:  C = A Wp^T, Wp packed [N, K], N a multiple of 256, Nout = N
//   epi EPI_SWIGLU: Wp packed gate/up interleaved [2*Nout, K], C = SiLU(A W1) * (A W3)
// M_dev, when not null, is a device int holding the number of rows actually present
// (<= M); M then only sizes the tensor maps and buffers.  x_out (A_GATHER only, may be
// null): bf16 [M, K] receiving the gathered A rows (E[id] + T[bucket]) as the MMAs used them.
// p_out (EPI_SWIGLU only, may be null): bf16 [M, 2 Nout] receiving [A W1 | A W3].
// max_pairs > 0 caps the persistent grid at that many CTA pairs (leaving SMs to kernels that
// run beside it on another stream).
int tc_gemm_resident(int amode, int epi, const void* A, GatherSrc g, int M, int K, const void* Wp,
                     int Nout, void* C, int ldc, int32_t* err, cudaStream_t s, const int32_t* M_dev = nullptr,
                     void* x_out = nullptr, const EpiFold* fold = nullptr, int max_pairs = 0,
                     void* p_out = nullptr);

// C[M, N] (bf16) = epi(A Wp^T), A dense bf16 [M, K] streamed (K a multiple of 64),
// N in {256, 512}; epi EPI_LN applies LayerNorm (gamma, beta, eps) over the full row.
// lda: row stride of A in elements (0: K).  epi EPI_LNSTAT writes C = (A Wp^T) * gamma and
// the row moments (mean, rstd) to stats [M][2].
int tc_gemm_rowwise(int epi, const void* A, int M, int K, const void* Wp, int N, const float* gamma,
                    const float* beta, float eps, void* C, int ldc, int32_t* err, cudaStream_t s,
                    const int32_t* M_dev = nullptr, int lda = 0, float* stats = nullptr);

// 2-D bf16 tensor map over a [rows, cols] row-major matrix (row stride ld elements),
// box = 64 columns x box_rows rows, 128-byte swizzle, zero fill outside the matrix.
bool make_tmap(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint64_t ld, uint32_t box_rows);
// fp32 [rows, cols] (row stride ld elements), box 32 x 32, 128-byte swizzle: tile stores.
bool make_tmap_f32_out(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint64_t ld);
// bf16 [rows, cols] (row stride ld elements), box 32 x 32, 64-byte swizzle: the epilogue's
// staged tile stores.
bool make_tmap_out(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint64_t ld);
// Fused history FFN of every layer for d = 256 (tc_ffn.cu): rows gathered via g (M rows, or
// *M_dev when given), W13p = all layers' packed W1|W3 [layers 2 hidden, 256], W2p = all
// layers' packed W2 [layers 256, hidden]; writes y'_l = (A_l W2_l) * gamma_l as bf16 rows
// l * layer_stride + r of Y [layers layer_stride, 256] and the row moments (mean, rstd) to
// stats [layers layer_stride] float2.  layer_stride >= M, a multiple of 256.
int tc_ffn_fused(const GatherSrc& g, int M, const int32_t* M_dev, int layers, int hidden, const void* W13p,
                 const void* W2p, const float* const* gammas, float eps, void* Y, int layer_stride, float* stats,
                 int32_t* err, cudaStream_t s, int max_pairs = 0);

// ---------------------------------------------------------------- SIMT fp32 GEMMs

constexpr int MAX_BATCH_PTRS = 64;

template <typename TA, typename TB>
struct SimtGemmArgs {
  int M, N, K;
  // A: logical row r lives at physical row ra = remap(r, a_grp, a_gstride, a_goff) with
  // remap(r, g, s, o) = g ? (r / g) * s + o + r % g : r; column k at
  // A[ra*lda + (k < ksplit ? k : k + kshift)].  When gather.ids != null, row r is
  // table[ids[r]*K + k] (+ dt_table[bucket(dt[r])*K + k]) instead.
  const TA* A;
  int64_t lda;
  int ksplit, kshift;
  int a_grp, a_gstride, a_goff;
  GatherSrc gather;
  const TB* B;   // [K, N] row-major (ldb = N)
  const TB* B2;  // second operand for the SwiGLU form SiLU(A B) * (A B2), or null
  // per-batch operands (batch z uses Bz[z] / B2z[z] when Bz[0] != null)
  const TB* Bz[MAX_BATCH_PTRS];
  const TB* B2z[MAX_BATCH_PTRS];
  float* C;      // logical row r at physical row remap(r, c_grp, c_gstride, c_goff)
  int64_t ldc;
  int c_grp, c_gstride, c_goff;
  const float* R;  // residual added to the result, row m at R[m*ldr], or null
  int64_t ldr;
  // batch (grid z): element offsets of A, C and R per batch; B per batch via bsB or Bz
  int64_t bsA, bsB, bsC, bsR;
  int batch;
  int32_t* err;
};

template <typename TA, typename TB>
int simt_gemm(const SimtGemmArgs<TA, TB>& a, cudaStream_t s);

// Tensor-core (mma.sync) form of simt_gemm<float, bf16> with fp32-accurate products
// (activations split into two bf16 terms); used by simt_gemm when the shapes allow.
bool query_gemm_supported(const SimtGemmArgs<float, __nv_bfloat16>& a);
int query_gemm(const SimtGemmArgs<float, __nv_bfloat16>& a, cudaStream_t s);

// tcgen05 form of simt_gemm<float, bf16> (same fp32-accurate split products) without
// gather, K % 64 == 0, ksplit % 64 == 0 (when < K), N % 32 == 0 (N % 128 == 0 with B2),
// 16-byte aligned A, C, R with row strides % 4 == 0.  Wp holds B (and B2) packed K-major:
// tc_pack_weight mode 0 [N, K], or modes 1 + 2 [2N, K] for the SwiGLU pair; with batch > 1
// the batches' packed matrices follow one another (and a.B / a.Bz are not read).
bool tc_query_supported(const SimtGemmArgs<float, __nv_bfloat16>& a);
int tc_query_gemm(const SimtGemmArgs<float, __nv_bfloat16>& a, const void* Wp, cudaStream_t s);

// y = LayerNorm(x) row-wise over d columns, fp32; x and y may alias.
int layer_norm_f32(const float* x, int64_t ldx, float* y, int64_t ldy, int rows, int d, const float* gamma,
                   const float* beta, float eps, cudaStream_t s);

// ---------------------------------------------------------------- attention

struct AttnArgs {
  const float* Q;       // [T, d] fp32 (projected queries)
  // bf16: [N, H, 2 d_h], row n holds [K_h | V_h] of head h in columns [2 h d_h, 2 (h+1) d_h)
  // (one contiguous 256-byte segment per key and head); fp32: [N, 2d], K in columns
  // [0, d), V in [d, 2d)
  const void* KV;
  const int32_t* hoff;  // [B+1] history offsets
  const int32_t* toff;  // [B+1] target offsets
  const int32_t* kv_rows;  // K/V row of history token n (distinct-row form), or null: row n
  // per-user compacted keys (with kv_rows): user u has kv_len[u] entries from hoff[u], entry
  // n standing for kv_mult[n] tokens with the same K/V row; null: one entry per token
  const int32_t* kv_len;
  const int32_t* kv_mult;
  int B, T, d, H, splits;
  int score;            // 0 softmax, 1 relu
  float* part_acc;      // [splits, T, d]
  float* part_ml;       // [splits, T, H, 2]
  float* out;           // [T, d]
  int32_t* err;
  // attention: write the slice states (part_acc, part_ml) even when splits == 1
  int partial_out = 0;
  // merge: when set, combine the slices into ONE state instead of the output: out gets
  // the unnormalised acc and ml_out [T, H, 2] the (max, sum) of the softmax
  float* ml_out = nullptr;
  // softmax, when set: lse_out [T, H] = log sum_j exp(s_j) over all of the user's keys
  // (natural log; -inf for an empty history), written with the normalised output (bf16
  // kernel with one slice, or the merge) for the backward pass
  float* lse_out = nullptr;
};
int attention_bf16(const AttnArgs& a, cudaStream_t s);
// Attention with W_K / W_V folded into the queries (d = 256, d_h = 64): scores of the
// folded queries Qf [T H, d] (row t H + h = Q_{t,h} W_K,h^T) against the history rows
// y' = y * gamma with their LayerNorm moments, and r = sum_j a_j x~_j per (target, head)
// into out [T H, d] (one slice), or unnormalised states [splits, T H, d] + (max, sum)
// [splits, T H, 2] for attention_merge with T' = T H, H' = 1.
struct FoldArgs {
  const float* Qf;
  const void* Y;           // [U, d] bf16 history rows y'
  const float* stats;      // [U, 2] (mean, rstd)
  const float* gamma;      // [d]
  const float* beta;       // [d]
  const int32_t* hoff;
  const int32_t* toff;
  const int32_t* kv_rows;  // as in AttnArgs
  const int32_t* kv_len;
  const int32_t* kv_mult;
  int B, T, d, H, splits, score;
  float* part_acc;
  float* part_ml;
  float* out;
  int partial_out = 0;
  int32_t* err;
};
int attention_fold_bf16(const FoldArgs& a, cudaStream_t s);
// Backward of the bf16 attention (per-token K/V rows, d_h = 64); see stca_attention_backward.
int attention_bwd_bf16(const float* Q, const void* KV, const int32_t* hoff, const int32_t* toff, int B, int T, int d,
                       int H, int splits, int score, const float* O, const float* lse, const float* dO, float* dQ,
                       float* dKV, float* part_dq, void* dKV16, cudaStream_t s);
int attention_f32(const AttnArgs& a, cudaStream_t s);
// combines the slices; not needed after attention_bf16 with splits == 1, which writes out
int attention_merge(const AttnArgs& a, cudaStream_t s);
inline bool attention_needs_merge(const AttnArgs& a, bool kv_bf16) {
  return !(kv_bf16 && a.splits == 1 && !a.partial_out);
}
// Launches kern as a programmatic dependent of the previous kernel on stream s (its CTAs
// may start while that kernel drains).  Every kernel launched this way calls griddep_wait()
// before it reads or writes any data.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_dep(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              Args&&... args) {
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}
// streaming multiprocessors of the current device
int sm_count();

// ---------------------------------------------------------------- small kernels

// offsets[0] = 0, offsets[i+1] = offsets[i] + lengths[i], each clamped to `expected`
// (negative lengths count as 0); checks lengths >= 0 and the total against `expected`
// (records STCA_ERR_BAD_LENGTHS otherwise).
int exclusive_offsets(const int32_t* lengths, int B, int32_t* offsets, int expected, int32_t* err,
                      cudaStream_t s);
// dst[r, col0 + c] = float(src[r, c]) for c < d (src bf16 or fp32 by `src_bf16`).
int copy_rows_to_f32(const void* src, int src_bf16, int rows, int d, float* dst, int64_t ldd, int col0,
                     cudaStream_t s);

// ---------------------------------------------------------------- distinct history rows

// Table slots and workspace bytes for up to max_tokens rows.
size_t dedup_table_slots(int max_tokens);
size_t dedup_workspace_bytes(int max_tokens);
// Distinct keys (id, time bucket) of n history tokens: uniq_idx[n] in [0, *count),
// uniq_token[u] = one token with key u.  All on the stream.
int dedup_rows(const int32_t* ids, const int32_t* dt, int n, void* ws, size_t ws_bytes, int32_t* uniq_idx,
               int32_t* uniq_token, int32_t* count, int32_t* err, cudaStream_t s);
// Per user u (tokens hoff[u] .. hoff[u+1]-1 with K/V rows rows[n]): the distinct rows of
// the user in order of first token, out_rows[hoff[u] + i], with their token counts
// out_mult[hoff[u] + i], i < out_len[u].  A user of 16384 or more tokens keeps one entry
// per token (multiplicity 1).
// dedup_rows and (when hoff != null) compact_user_rows in one cooperative launch.
int dedup_fused(const int32_t* ids, const int32_t* dt, int n, void* ws, size_t ws_bytes, int32_t* uniq_idx,
                int32_t* uniq_token, int32_t* count, const int32_t* hoff, int B, int32_t* c_rows, int32_t* c_mult,
                int32_t* c_len, int32_t* err, cudaStream_t s);
int compact_user_rows(const int32_t* hoff, int B, const int32_t* rows, int32_t* out_rows, int32_t* out_mult,
                      int32_t* out_len, cudaStream_t s);

// ---------------------------------------------------------------- training: history side
// C [K, N] (+)= A^T G over M tokens (A [M, K], G [M, N] bf16, C fp32); K, N % 128 == 0;
// ws: gemm_wgrad_workspace_bytes(M, K, N) bytes (per-slice partial tiles).  impl: 0 the
// tcgen05 kernel (tc_wgrad.cu), 1 the mma.sync kernel; err: timeouts (may be null).
size_t gemm_wgrad_workspace_bytes(int M, int K, int N);
int gemm_wgrad(const void* A, int64_t lda, const void* G, int64_t ldg, int M, int K, int N, float* C, int64_t ldc,
               int accumulate, int impl, void* ws, size_t ws_bytes, int32_t* err, cudaStream_t s);
// the tcgen05 kernel alone: per-slice partial tiles part [splits, K, N]
int tc_wgrad_splits(int M, int K, int N);
int tc_wgrad_partials(const void* A, int64_t lda, const void* G, int64_t ldg, int M, int K, int N, int splits,
                      float* part, int32_t* err, cudaStream_t s);
size_t layer_norm_bwd_workspace_bytes(int M, int d);
int layer_norm_bwd(const void* y, const void* dxt, int M, int d, int fp32, const float* gamma, const float* beta,
                   float eps, void* dy, void* xt, float* dgamma, float* dbeta, int accumulate, void* ws,
                   size_t ws_bytes, cudaStream_t s);
int swiglu_bwd(const void* P, const void* dA, int M, int h, int fp32, void* dP, void* a_out, cudaStream_t s);
int layer_norm_fwd(const void* x, int64_t ldx, int x_fp32, int M, int d, const float* gamma, const float* beta,
                   float eps, void* y, int64_t ldy, int y_fp32, cudaStream_t s);
int f32_to_bf16(const float* src, int64_t lds, int rows, int cols, void* dst, int64_t ldd, cudaStream_t s);
int table_rows_bwd(const void* dX, int M, int d, const int32_t* ids, const int32_t* dt, int64_t n_items,
                   float* dtable, float* ddt_table, int32_t* err, cudaStream_t s);
int place_cols(const void* W, int K, int N, void* dst, int mode, int off, cudaStream_t s);

// ---------------------------------------------------------------- pointwise ReLU TA

int pointwise_relu_ta(const int32_t* ids, const int32_t* offsets, const void* q, const void* table,
                      int64_t n_items, int B, int D, int splits, float* partials, float* out, int32_t* err,
                      cudaStream_t s);

// ---------------------------------------------------------------- query boosting

// mixed[b, h, t*sub + j] = Q[b, t, h*sub + j], sub = d / T
int token_mix(const float* Q, int B, int T, int d, float* mixed, cudaStream_t s);
// out[i] = i * step for i in [0, n)
int fill_arange(int32_t* out, int n, int step, cudaStream_t s);

}  // namespace stca
