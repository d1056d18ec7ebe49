/*
 * stca.h - C ABI of libstca: forward pass of stacked target-to-history cross
 * attention (STCA) and two related target-attention forms, on one NVIDIA B200.
 *
 * Sources for what is computed (page title, section / equation):
 *   [notes]   "超长序列建模 —— STCA 精读笔记" (wln20.github.io): problem statement,
 *             sections "STCA" and "Request Level Batching（RLB）".
 *   [review]  "Make It Long, Keep It Fast" paper review (xllm-io.github.io):
 *             §三 核心公式 and the architecture tree; §四 table (SwiGLU FFN, time gap).
 *   [wechat]  "视频号推荐超长序列技术演进" (dingyadong.top): §1.1 distributed TA
 *             (local attention, then merge) and the low-memory TA operator (lookup
 *             fused with attention); §1.2 element-wise ReLU scores.
 *   [hyformer] "HyFormer：重新审视序列建模和特征交互在 CTR 预测中的作用"
 *             (gitcode.csdn.net): §3.4-3.7, eq (7)-(16).
 *
 * Conventions for every entry point:
 *   - All tensors are row-major and dense.  Weight matrices are [in, out] and act as
 *     y = x W ([review] 核心公式 writes q W_Q and X~ W_K).  Head h of a d-wide
 *     projection is columns [h*d/H, (h+1)*d/H).
 *   - "dtype" tensors are float32 for STCA_FP32 and bfloat16 for STCA_BF16.  LayerNorm
 *     gamma/beta are always float32.  Outputs are always float32.
 *   - Pointers are DEVICE pointers unless the entry point's name ends in _host.  The
 *     caller owns every buffer; the library never frees or keeps them past the call.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default stream) and
 *     is asynchronous.  Argument errors are detected on the host before anything is
 *     launched and returned synchronously.  Errors the GPU detects (an item id outside
 *     [0, n_items), lengths that do not add up, a bounded wait that ran out) are
 *     recorded in the handle's device error word; the kernels never trap and keep
 *     going, and outputs are then undefined.  stca_sync_status() reads and clears it.
 *     Lengths that add up to more than n_tok (targets_per_user to more than t_tot) are
 *     cut at the declared total: the ragged offsets are clamped to it, so no kernel
 *     reads or writes past the buffers that n_tok and t_tot describe.
 *   - A handle is not thread-safe; use one handle per host thread or serialise calls.
 */
#ifndef STCA_H
#define STCA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define STCA_MAX_LAYERS 8
#define STCA_MAX_QUERY_TOKENS 64

enum stca_status {
  STCA_OK = 0,
  STCA_ERR_INVALID_ARG = 1,      /* null pointer, bad size, inconsistent counts */
  STCA_ERR_UNSUPPORTED = 2,      /* configuration outside what the kernels implement */
  STCA_ERR_CAPACITY = 3,         /* a size above the handle's max_* limits */
  STCA_ERR_CUDA = 4,             /* a CUDA runtime/driver call failed */
  STCA_ERR_ID_OUT_OF_RANGE = 5,  /* device: an item id outside [0, n_items) (row read as 0) */
  STCA_ERR_TIMEOUT = 6,          /* device: a bounded wait ran out */
  STCA_ERR_BAD_LENGTHS = 7       /* device: negative lengths or a sum != n_tok / t_tot */
};

enum stca_dtype { STCA_FP32 = 0, STCA_BF16 = 1 };
/* Which entry point a handle serves; stca_create sizes the workspace for it. */
enum stca_mode { STCA_MODE_STCA = 0, STCA_MODE_POINTWISE = 1, STCA_MODE_HYFORMER = 2 };
enum stca_score { STCA_SOFTMAX = 0, STCA_RELU = 1 };

/* Model shape and capacity.  mode: enum stca_mode.  M layers (or HyFormer blocks), model
 * width d, H heads (d_h = d/H, which must be 32, 64 or 128 for STCA_FP32 and 64 for
 * STCA_BF16 in this build), SwiGLU hidden width `hidden`.
 * time_buckets: 0, or 16 for the time-difference feature of [review] §四.
 * max_users / max_tokens / max_targets bound B, n_tok and t_tot of every later call;
 * stca_create sizes all device workspace from them, and later calls allocate nothing.
 * dedup follows the HyFormer page §3.8.1 (GPU pooling: few ids of a long sequence are
 * distinct): X~, K and V of a history token depend only on its item id and time bucket,
 * so they are computed once per distinct key and every token reads its key's K/V row.
 * Tokens of one user with the same key also have equal scores, so a softmax (or ReLU)
 * over them equals one over the user's distinct keys with each weight multiplied by the
 * key's token count (dedup = 2). */
typedef struct {
  int mode;         /* enum stca_mode */
  int M, d, H, hidden;
  int dtype;        /* enum stca_dtype */
  int score;        /* enum stca_score */
  int time_buckets; /* 0 or 16 */
  int max_users, max_tokens, max_targets;
  int dedup;        /* STCA_BF16 only.  1: run the per-token history GEMMs once per distinct
                       (id, time bucket) key of the call; results are bit-identical to 0.
                       2: also attend once per distinct key of each user, weighting the key
                       by the number of its tokens; the same result up to summation order */
  float ln_eps;     /* LayerNorm epsilon (biased variance) */
  int kv_fold;      /* 1: fold W_K and W_V into the queries ([review] 核心公式 by associativity:
                       s = (q W_Q,h W_K,h^T) . x~, o_h = (sum a x~) W_V,h), so that no K/V row is
                       ever computed; attention reads the d-wide history rows and their
                       LayerNorm moments.  STCA_BF16 STCA handles with d = 256, d / H = 64
                       only (else STCA_ERR_UNSUPPORTED), not with the sequence-parallel
                       phases.  0: project K/V per history row (default) */
} stca_config;

/* One SwiGLU FFN, SwiGLU(x) = (SiLU(x W1) * (x W3)) W2 (the "dimension-preserving"
 * SwiGLU FFN of [review] §四), optionally followed by LayerNorm.
 * W1, W3: [d, hidden] dtype;  W2: [hidden, d] dtype;  gamma, beta: [d] float32 or NULL
 * where the block has no LayerNorm. */
typedef struct {
  const void* W1;
  const void* W3;
  const void* W2;
  const float* gamma;
  const float* beta;
} stca_ffn;

/* STCA weights ([notes] STCA, [review] 核心公式).  Layer index i = 0..M-1.
 *   table    E [n_items, d] dtype              item embedding table
 *   dt_table T [16, d] dtype or NULL           time-difference bucket embeddings
 *   hist[i]  history SwiGLU + LN of layer i (X~^(i) from the ORIGINAL X)
 *   WQ/WK/WV/WO[i] [d, d] dtype
 *   tgt      target-side SwiGLU + LN of layer 1 (q^(1) = LN(SwiGLU(x_t)))
 *   WC[i]    for i = 1..M-1: [(i+1) d, d] dtype, fusion input of layer i+1
 *            (rows [0, i*d) multiply o^(1..i), rows [i*d, (i+1)d) multiply x_t)
 *   fuse[i]  for i = 1..M-1: SwiGLU + LN of the fusion into q^(i+1)
 *   WZ       [(M+1) d, d] dtype;  zffn: SwiGLU without LN, z = SwiGLU_Z([o|x_t] WZ) */
typedef struct {
  const void* table;
  int64_t n_items;
  const void* dt_table;
  stca_ffn hist[STCA_MAX_LAYERS];
  const void* WQ[STCA_MAX_LAYERS];
  const void* WK[STCA_MAX_LAYERS];
  const void* WV[STCA_MAX_LAYERS];
  const void* WO[STCA_MAX_LAYERS];
  stca_ffn tgt;
  const void* WC[STCA_MAX_LAYERS];
  stca_ffn fuse[STCA_MAX_LAYERS];
  const void* WZ;
  stca_ffn zffn;
} stca_weights;

typedef struct stca_handle stca_handle;

/* Validates the configuration and allocates every device buffer later calls need
 * (workspace, error word).  Returns STCA_ERR_UNSUPPORTED for shapes the kernels do not
 * implement (bf16: d in {256, 512} with d_h = 64 and hidden a multiple of 128 up to
 * 1024; fp32: d_h = 32, d <= 1024), STCA_ERR_CUDA if allocation fails.  On error *out
 * is set to NULL and nothing is leaked. */
int stca_create(const stca_config* cfg, stca_handle** out);

/* STCA forward for B users and their targets (Request-Level Batching, [notes] RLB:
 * each user's per-layer K/V is computed once and serves all of that user's targets).
 *   hist_ids         [n_tok] int32   item ids of all histories, user after user
 *   hist_lengths     [B] int32       L_u >= 0; sum = n_tok
 *   hist_dt          [n_tok] int32   time differences >= 0 (seconds), or NULL when the
 *                                    handle has time_buckets == 0 (must be non-NULL
 *                                    otherwise)
 *   target_emb       [t_tot, d] dtype  x_t of every target, user after user
 *   targets_per_user [B] int32       m_u >= 0; sum = t_tot
 *   z_out            [t_tot, d] float32  z of every target
 *   o_out            [M, t_tot, d] float32 per-layer o^(i), or NULL
 * A user with L_u = 0 gets o_h = 0 in every head.  Device-side checks: ids in range,
 * lengths non-negative and summing to n_tok / t_tot. */
int stca_forward(stca_handle* h, const int32_t* hist_ids, const int32_t* hist_lengths,
                 const int32_t* hist_dt, const void* target_emb, const int32_t* targets_per_user,
                 int B, int n_tok, int t_tot, const stca_weights* w, float* z_out, float* o_out,
                 void* stream);

/* stca_forward with the per-request inputs and the output in HOST memory (pinned memory
 * makes the copies asynchronous): the library copies the inputs into one of two staging
 * slots of its workspace on an internal copy stream, runs the forward on `stream` once
 * they have landed into one of two output slots, and copies z back to z_out_host on a
 * second internal stream.  So one call's input copies and the previous call's read-back
 * both overlap the forward in between.  Weights and the table stay device pointers.
 * Returns after enqueueing.  Once `stream` has been synchronised the inputs have been
 * read (keep the host inputs unchanged until then); z_out_host holds the result once
 * stca_host_fence(h, stream) has been called after this call and `stream` synchronised,
 * or once stca_sync_status(h) has returned (or the device has been synchronised). */
int stca_forward_host(stca_handle* h, const int32_t* hist_ids_host, const int32_t* hist_lengths_host,
                      const int32_t* hist_dt_host, const void* target_emb_host,
                      const int32_t* targets_per_user_host, int B, int n_tok, int t_tot,
                      const stca_weights* w, float* z_out_host, void* stream);

/* Makes `stream` wait until the z read-backs of every stca_forward_host call enqueued on
 * the handle so far have landed in host memory (nothing to wait for before the first
 * call).  Enqueues a wait and returns; STCA_ERR_CUDA if that fails. */
int stca_host_fence(stca_handle* h, void* stream);

/* Sequence-parallel (L-split) forward, in phases, for histories split across R ranks (one
 * GPU each).  Attention over a history is a merge of attention over its slices: each slice
 * keeps its running max m, sum l and weighted sum acc of V, and the slices combine exactly
 * ([wechat] §1.1, local attention then merge).  Every rank calls, on its own handle:
 *
 *   stca_lsplit_begin   with ITS slice of every user's history (hist_lengths = the slice
 *                       lengths, zeros allowed; ids/dt of the slices back to back) and ALL
 *                       of the users' targets (the same on every rank);
 *   for layer i = 0 .. M-1:
 *     stca_lsplit_partial(i, acc, ml)   this rank's attention state of layer i:
 *                       acc [t_tot, d] fp32, unnormalised sum of weights x V per head
 *                       ml  [t_tot, H, 2] fp32, (max in log2 units, sum of weights) per
 *                       target and head (softmax; not written for the ReLU score)
 *     the caller gathers acc and ml of all ranks in rank order: all_acc [R, t_tot, d],
 *                       all_ml [R, t_tot, H, 2] (e.g. an NCCL all-gather on `stream`)
 *     stca_lsplit_merge(i, R, all_acc, all_ml, z_out)   merges the R states into o^(i),
 *                       then q^(i+1), and after the last layer z [t_tot, d] into z_out
 *
 * Everything but the attention is computed on every rank (the target side is small).
 * The phases must come in this order; another order returns STCA_ERR_INVALID_ARG, and a
 * stca_forward on the handle closes an open sequence-parallel forward.  The device
 * pointers given to stca_lsplit_begin (ids, dt, lengths, target rows, weights) must stay
 * valid until the last merge.  1 <= R <= 32. */
int stca_lsplit_begin(stca_handle* h, const int32_t* hist_ids, const int32_t* hist_lengths,
                      const int32_t* hist_dt, const void* target_emb, const int32_t* targets_per_user,
                      int B, int n_tok, int t_tot, const stca_weights* w, void* stream);
int stca_lsplit_partial(stca_handle* h, int layer, float* acc, float* ml, void* stream);
int stca_lsplit_merge(stca_handle* h, int layer, int ranks, const float* all_acc, const float* all_ml,
                      float* z_out, void* stream);

/* Pointwise ReLU target attention with fused lookup ([wechat] §1.1 low-memory TA
 * operator, §1.2 ReLU scores): for each sample b,
 *   out[b] = sum_{j < L_b} relu(q_b . e_j / sqrt(D)) e_j,   e_j = table[ids_b[j]]
 * Keys and values are the looked-up rows themselves; the gathered [B, L, D] matrix is
 * never written.  Handle: dtype STCA_BF16, d = D = 128 (the only width in this build),
 * max_users >= B, max_tokens >= n_tok.
 *   ids [n_tok] int32, lengths [B] int32, q [B, D] bf16, table [n_items, D] bf16,
 *   out [B, D] float32.  q and table start on 16-byte boundaries (rows are moved by
 *   16-byte copies), else STCA_ERR_INVALID_ARG with nothing launched. */
int stca_pointwise_forward(stca_handle* h, const int32_t* ids, const int32_t* lengths, const void* q,
                           const void* table, int64_t n_items, int B, int n_tok, float* out,
                           void* stream);

/* Largest batch the allocation-free variant below accepts. */
#define STCA_NOALLOC_MAX_USERS 2048

/* stca_pointwise_forward without a handle and without any device allocation.  The pages
 * have no counterpart to this entry point; it exists for callers that cannot call
 * cudaMalloc (a plugin inside a host runtime that owns all device memory, or a request
 * path where an allocation, which may synchronise the device, is not allowed).
 * Same arguments and result as stca_pointwise_forward (D = 128, bf16 q and table,
 * float32 out), plus err_out: a caller-owned device int32 that receives the first error
 * the GPU detects (an id out of range, lengths not adding up to n_tok) if it was 0, or
 * NULL.  Scratch lives in a fixed array of about 4.2 MB in the library's device image,
 * which every GPU that loads the library holds until the process exits; B above
 * STCA_NOALLOC_MAX_USERS returns STCA_ERR_CAPACITY.  The first call on a device, and the
 * first one after a cudaDeviceReset there, looks up that array's device address (make
 * that call before any stream capture).  All
 * calls share the array: calls that overlap on the GPU (different streams, or different
 * host threads on the same device) race and give undefined results; calls serialised
 * on one stream are safe. */
int stca_pointwise_forward_noalloc(const int32_t* ids, const int32_t* lengths, const void* q, const void* table,
                                   int64_t n_items, int B, int n_tok, float* out, int32_t* err_out, void* stream);

/* Multi-query multi-sequence decode ([hyformer] §3.4-3.7).  Two sequences per user
 * (s = 0 "feed", s = 1 "search"), each with n_query query tokens.  Per block l and
 * sequence s: H = SwiGLU_{l,s}(X_s) (eq 7), K,V = H W_K, H W_V (eq 8), decoded queries
 * = multi-head CrossAttn(Q_s W_Q, K, V) W_O (eq 9/16).  Then Q = [Q^_0; Q^_1]
 * (T = 2 n_query tokens, eq 10), token mixing (eq 11-13), a per-token SwiGLU per token
 * index (eq 14) and the residual Q + Q~ (eq 15) give the next block's queries.
 * Handle: dtype STCA_BF16, d = 512, H = 8, hidden = 1024 in this build; M = number of
 * blocks; max_users >= B; max_tokens >= max(n_feed, n_search); max_targets >=
 * B * 2 * n_query.  T must divide d. */
typedef struct {
  stca_ffn ffn; /* W1, W3, W2 only (no LayerNorm, eq 7) */
  const void* WQ;
  const void* WK;
  const void* WV;
  const void* WO;
} hyf_seq_weights;

typedef struct {
  hyf_seq_weights seq[2];
  stca_ffn tok[STCA_MAX_QUERY_TOKENS]; /* per-token SwiGLU, token index 0..T-1 */
} hyf_block_weights;

typedef struct {
  const void* table;
  int64_t n_items;
  int blocks;
  hyf_block_weights blk[STCA_MAX_LAYERS];
} hyf_weights;

/*   ids_feed [n_feed] int32, len_feed [B] int32, ids_search [n_search], len_search [B],
 *   q0 [B, 2*n_query, d] bf16 (rows 0..n_query-1 query sequence 0), out [B, 2*n_query, d]
 *   float32. */
int hyformer_forward(stca_handle* h, const int32_t* ids_feed, const int32_t* len_feed, int n_feed,
                     const int32_t* ids_search, const int32_t* len_search, int n_search,
                     const void* q0, int B, int n_query, const hyf_weights* w, float* out,
                     void* stream);

/* Per-stage device timing for measurement: when enabled, each stage's launches are
 * bracketed by CUDA events on the call's stream.  Stages: */
enum stca_stage {
  STCA_STAGE_SETUP = 0,      /* offsets, weight packing, input conversion */
  STCA_STAGE_GATHER_FFN = 1, /* fused gather + X [W1|W3] + SwiGLU (tensor cores) */
  STCA_STAGE_FFN_OUT = 2,    /* A W2 (+ LayerNorm) (tensor cores) */
  STCA_STAGE_KV = 3,         /* X~ [W_K|W_V] (tensor cores) */
  STCA_STAGE_ATTENTION = 4,  /* split-L attention */
  STCA_STAGE_MERGE = 5,      /* merge of the splits */
  STCA_STAGE_QUERY = 6,      /* target side: SwiGLU/LN, W_Q, W_O, W_C, W_Z */
  STCA_STAGE_POINTWISE = 7,  /* fused pointwise ReLU target attention */
  STCA_STAGE_BOOST = 8,      /* token mix + per-token SwiGLU + residual */
  STCA_STAGE_DEDUP = 9,      /* distinct history keys (when the handle has dedup = 1) */
  STCA_N_STAGES = 10
};

/* enable = 1 starts recording every stage (totals reset), 0 stops it. */
int stca_profile_enable(stca_handle* h, int enable);

/* Records only the stages whose bit (1 << stage) is set in stage_mask (totals reset; 0
 * stops).  Each recorded stage costs its stream two event records per stage call, about a
 * microsecond each on the device, so a measurement of the whole forward records only the
 * stage it needs. */
int stca_profile_stages(stca_handle* h, uint32_t stage_mask);

/* Waits for the recorded work, then writes per stage the summed device milliseconds
 * and the number of recorded stage intervals (arrays of STCA_N_STAGES entries). */
int stca_profile_read(stca_handle* h, double* total_ms, int64_t* calls);

/* Kernel launches this library has issued since it was loaded (all handles). */
uint64_t stca_launch_count(void);

/* Synchronises the stream of the handle's last call and the host entry's read-back
 * stream, then returns and clears the device error word (STCA_OK if no error was
 * recorded), or STCA_ERR_CUDA. */
int stca_sync_status(stca_handle* h);

/* Host watchdog: waits at most timeout_ms for the work enqueued so far on `stream` (a
 * cudaStream_t; NULL = legacy default stream), polling an event.  STCA_OK when it has
 * finished, STCA_ERR_TIMEOUT when the deadline passed first (the work keeps running and
 * may be waited for again), STCA_ERR_CUDA on a CUDA error.  Never blocks past the deadline. */
int stca_stream_wait(void* stream, int timeout_ms);

/* Static description of a status code. */
const char* stca_strerror(int code);

/* Weight conversion done once (no counterpart on the pages: a load-time layout step, as a
 * serving system prepares constant weights when it loads a model).  Every bf16 forward
 * call converts the weights it is given into the tensor cores' K-major operand layout in
 * handle workspace.  stca_pin_weights does that now, on `stream`, for `weights` (a
 * `const stca_weights*` for STCA handles, a `const hyf_weights*` for HyFormer handles; for
 * the latter also the per-token FFNs of every query token slot whose three matrices are
 * set, up to max_targets / max_users tokens) and records the struct's address and
 * contents: later calls given the same struct skip the conversion.  Between pin and
 * unpin (or destroy) the weight arrays must not change.  Pinning other weights replaces
 * the pin.  Errors: STCA_ERR_INVALID_ARG (null or incomplete weights, pointwise handle),
 * STCA_ERR_UNSUPPORTED (fp32 handle), STCA_ERR_CUDA. */
int stca_pin_weights(stca_handle* h, const void* weights, void* stream);

/* Forgets the pin; later calls convert the weights they are given again. */
void stca_unpin_weights(stca_handle* h);

/* Frees the handle's device memory.  NULL is a no-op. */
void stca_destroy(stca_handle* h);

/* ---------------------------------------------------------------------------------
 * Training: the attention step's forward with its softmax statistics, and its backward.
 * The pages train on ~2K-item histories and serve 10K ([notes] "短序列训练，长序列推理";
 * [review] architecture branch (C) "Extrapolation Aware Training").  Handle-free: the
 * caller passes every buffer (device pointers, caller-owned) and any scratch.  One K/V
 * row per history token (no distinct-key compaction), bf16 K/V, d_h = d / H = 64 (else
 * STCA_ERR_UNSUPPORTED); 1 <= splits <= 32 slices of each user's keys (else
 * STCA_ERR_INVALID_ARG).  Layouts:
 *   Q, out, dout, dQ   [T, d] float32, row t = target t (targets grouped by user, toff)
 *   KV                 [N, H, 2 d_h] bf16: row n = history token n (users by hoff), head
 *                      h's K in columns [2 h d_h, 2 h d_h + d_h) and V in the next d_h
 *   dKV                [N, H, 2 d_h] float32 in the same layout ([dK_h | dV_h])
 *   lse                [T, H] float32: log sum_j exp(q_h . k_j / sqrt(d_h)) over the
 *                      user's keys (natural log; -inf for an empty history)
 *   hoff, toff         [B + 1] int32 offsets of the users' keys and targets, trusted as
 *                      given: rows hoff[0] .. hoff[B] - 1 of KV / dKV and toff[0] ..
 *                      toff[B] - 1 of the [T, d] arrays must exist
 * Scores: 0 softmax, 1 relu (the unnormalised ReLU form keeps no lse; lse may be NULL).
 * ---------------------------------------------------------------------------------- */

/* out[t, head h] = attention of query h of target t over its user's keys ([review] 核心公式;
 * [wechat] §1.2 for relu), plus lse (softmax).  part_acc [splits, T, d] and part_ml
 * [splits, T, H, 2] float32 scratch (unused, may be NULL, when splits == 1). */
int stca_attention_train_forward(const float* Q, const void* KV, const int32_t* hoff, const int32_t* toff, int B,
                                 int T, int d, int H, int splits, int score, float* part_acc, float* part_ml,
                                 float* out, float* lse, int32_t* err, void* stream);

/* Gradients of sum_t dout[t] . out[t] with respect to Q and K/V, given the forward's out
 * and lse:
 *   softmax: p = exp(s - lse), D_t = dout_t . out_t, ds = p (dout_t . v_j - D_t)
 *   relu:    p = relu(s),                            ds = (dout_t . v_j) [s > 0]
 *   dV_j = sum_t p_tj dout_t, dK_j = sum_t ds_tj q_t / sqrt(d_h), dQ_t = sum_j ds_tj k_j / sqrt(d_h)
 * with s = q . k / sqrt(d_h) per head; a key's gradient sums over all of its user's
 * targets, and a key with no target of its user gets 0.  part_dq [splits, T, d] float32
 * scratch for splits > 1 (may be NULL when splits == 1).  dkv_bf16 (may be NULL): when
 * given, the K/V gradients are written there as bf16 [N, H, 2 d_h] (rounded to nearest
 * even from the same fp32 sums) and dKV only holds the fp32 partial sums of users with
 * more than 16 targets; 16-byte aligned.  Deterministic: no atomics. */
int stca_attention_backward(const float* Q, const void* KV, const int32_t* hoff, const int32_t* toff, int B, int T,
                            int d, int H, int splits, int score, const float* out, const float* lse,
                            const float* dout, float* dQ, float* dKV, float* part_dq, void* dkv_bf16, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* STCA_H */
