// C ABI of libstca: argument checks, the workspace, and the launch sequence of each
// forward pass.  Every step of the path runs in this library's kernels; PyTorch (or any
// other caller) only provides device memory and the stream.
#include <atomic>
#include <chrono>
#include <cstdio>
#include <cstring>
#include <new>
#include <thread>
#include <vector>

#include "common.cuh"
#include "internal.h"

using namespace stca;

namespace {

constexpr int MAX_SPLITS = 16;
// Distinct keys of calls up to this many tokens are found in one cooperative launch
// (dedup_fused): at short histories the separate launches cost more than the work (config
// 2, 87K tokens: 47 -> 41 us per call), while at 2.56M tokens the fused kernel's one block
// per SM gives the atomic inserts half the occupancy of the separate kernels (102 -> 121 us).
constexpr int FUSED_DEDUP_MAX_TOKENS = 1 << 18;

}  // namespace

struct stca_handle {
  stca_config cfg;
  int device = 0;
  cudaStream_t last_stream = nullptr;
  std::vector<void*> allocs;
  int32_t* err = nullptr;
  int32_t *hoff = nullptr, *toff = nullptr, *hoff2 = nullptr;
  // history side
  // history weights in tensor-core operand order, per slot (sequence sq, layer l) at
  // sq * M + l: all slots' W1|W3 [2h, d] back to back (so one GEMM covers the M layers of
  // a sequence), then all W2 [d, h], then all W_K|W_V [2d, d]
  void* wpack = nullptr;
  int wslots = 0;
  // LayerNorm folded into the K/V GEMM: per slot c = gamma^T [WK|WV] and b = beta^T [WK|WV]
  // ([2][2d] fp32), and the row moments of the current layer ([N][2] fp32)
  float *fold = nullptr, *rowstats = nullptr;
  void *hidden = nullptr, *xt = nullptr, *kv = nullptr;
  // target-side weights packed K-major for the tensor cores (bf16 STCA), element offsets
  void* qpack = nullptr;
  struct QLayout {
    // STCA
    size_t tgt13, tgt2, wq[STCA_MAX_LAYERS], wo[STCA_MAX_LAYERS], wc[STCA_MAX_LAYERS], fuse13[STCA_MAX_LAYERS],
        fuse2[STCA_MAX_LAYERS], wz, z13, z2;
    // W_K / W_V folded into the queries (kv_fold): block-diagonal [H d, d] (q~ = Q Kfold^T
    // per head) and [d, H d] (o = r Vfold^T), zero outside the diagonal blocks
    size_t kfold[STCA_MAX_LAYERS], vfold[STCA_MAX_LAYERS], fold_begin, fold_end;
    // decode blocks: W_Q / W_O per block and sequence, the per-token FFNs of a block back to
    // back (tok_cap tokens at most)
    size_t hwq[2 * STCA_MAX_LAYERS], hwo[2 * STCA_MAX_LAYERS], htok13[STCA_MAX_LAYERS], htok2[STCA_MAX_LAYERS];
    int tok_cap;
    size_t total;
  } ql{};
  // query side
  float *cat = nullptr, *qbuf = nullptr, *qproj = nullptr, *attn = nullptr, *tmp_h = nullptr, *tmp_d = nullptr;
  float *part_acc = nullptr, *part_ml = nullptr;
  float* qfold = nullptr;  // kv_fold: folded queries [T H, d], then the weighted rows r
  float *hq = nullptr, *hqhat = nullptr, *hmix = nullptr;
  // distinct history rows
  void* dedup_ws = nullptr;
  size_t dedup_ws_bytes = 0;
  int32_t *uniq_idx = nullptr, *uniq_token = nullptr, *uniq_count = nullptr;
  // per-user compacted K/V rows with multiplicities (dedup = 2), per history sequence
  int32_t *c_rows = nullptr, *c_mult = nullptr, *c_len = nullptr;
  // weights converted once by stca_pin_weights (address, a copy of the struct, and the
  // number of decode query tokens whose FFNs were converted)
  const void* pinned = nullptr;
  std::vector<uint8_t> pinned_copy;
  int pinned_tokens = 0;
  // staging for the host-buffer entry point: two input slots and two output slots, so the
  // copies of one call's inputs (on copy_stream) and the read-back of its z (on back_stream)
  // overlap the neighbouring calls' forwards
  int32_t *in_ids[2] = {}, *in_len[2] = {}, *in_dt[2] = {}, *in_tpu[2] = {};
  void* in_xt[2] = {};
  float* out_z[2] = {};
  cudaStream_t copy_stream = nullptr, back_stream = nullptr;
  // the fused-FFN path's K/V GEMMs of layers >= 1 run on side_stream beside layer 0's
  // attention and target side; kv_done[l] marks layer l's K/V rows ready
  cudaStream_t side_stream = nullptr;
  cudaEvent_t ffn_done = nullptr, kv_done[STCA_MAX_LAYERS] = {};
  cudaEvent_t in_ready[2] = {}, in_free[2] = {};  // slot copied / slot read by its forward
  cudaEvent_t z_ready[2] = {}, z_free[2] = {};    // slot written by its forward / slot read back
  bool in_used[2] = {false, false}, z_used[2] = {false, false};
  int in_slot = 0, z_last = -1;  // z_last: slot of the latest read-back, -1 before the first
  // one STCA forward between its phases (set by its first phase)
  struct Fwd {
    int B = 0, n_tok = 0, t_tot = 0, splits = 1, fold_splits = 1;
    bool kv_ahead = false;  // the K/V GEMMs of layers >= 1 were issued on the side stream
    const stca_weights* w = nullptr;
    GatherSrc g{};
    const int32_t *M_dev = nullptr, *kv_rows = nullptr, *kv_len = nullptr, *kv_mult = nullptr;
    int next_layer = -1;  // sequence-parallel forward: next layer to run, -1 when none is open
    bool partial_done = false;
  } fwd;
  // per-stage timing: bit s set = stage s's launches are bracketed by events
  uint32_t prof = 0;
  struct Rec {
    int stage;
    cudaEvent_t a, b;
  };
  std::vector<Rec> recs;
  std::vector<cudaEvent_t> spare;
};

namespace stca {
static std::atomic<uint64_t> g_launches{0};
void note_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }
}  // namespace stca

namespace {

#define CK(x)                      \
  do {                             \
    const int _rc = (x);           \
    if (_rc != STCA_OK) return _rc; \
  } while (0)

cudaEvent_t take_event(stca_handle* h) {
  if (!h->spare.empty()) {
    cudaEvent_t e = h->spare.back();
    h->spare.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

// Brackets one stage's launches with events when the handle records timings.
struct Prof {
  stca_handle* h;
  int stage;
  cudaStream_t s;
  cudaEvent_t a = nullptr;
  Prof(stca_handle* h_, int stage_, cudaStream_t s_) : h(h_), stage(stage_), s(s_) {
    if ((h->prof >> stage) & 1u) {
      a = take_event(h);
      cudaEventRecord(a, s);
    }
  }
  ~Prof() {
    if (a) {
      cudaEvent_t b = take_event(h);
      cudaEventRecord(b, s);
      h->recs.push_back({stage, a, b});
    }
  }
};

#define STAGE(h, st, s, expr)       \
  do {                              \
    Prof _prof((h), (st), (s));     \
    CK(expr);                       \
  } while (0)

void recycle_events(stca_handle* h) {
  for (auto& r : h->recs) {
    h->spare.push_back(r.a);
    h->spare.push_back(r.b);
  }
  h->recs.clear();
}

template <typename T>
bool dalloc(stca_handle* h, T** p, size_t bytes) {
  void* q = nullptr;
  if (bytes == 0) bytes = 16;
  if (cudaMalloc(&q, bytes) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  h->allocs.push_back(q);
  *p = reinterpret_cast<T*>(q);
  return true;
}

void free_all(stca_handle* h) {
  for (void* p : h->allocs) cudaFree(p);
  h->allocs.clear();
}

int choose_splits(int64_t n_tok, int B, int per_split) {
  if (B <= 0) return 1;
  const int64_t avg = n_tok / B;
  int64_t s = (avg + per_split - 1) / per_split;
  if (s < 1) s = 1;
  if (s > MAX_SPLITS) s = MAX_SPLITS;
  return int(s);
}

// L-slices per user for the attention: about enough (user, head, slice) CTAs to fill one
// wave of the GPU (ctas_per_sm resident CTAs per SM), never so many that a slice averages
// fewer than min_keys keys.  Every extra slice costs a merge launch and a round trip of the
// slice states, which on short, latency-bound steps outweighs the idle SMs of a partly
// filled wave (config 2, 64 users x 4 heads: one slice 0.042 ms of attention and no merge,
// against 0.050 + 0.017 ms with two).
int attention_splits(int64_t n_tok, int B, int H, int min_keys, int ctas_per_sm = 2) {
  if (B <= 0 || H <= 0) return 1;
  const int64_t ctas = int64_t(B) * H;
  const int64_t slots = int64_t(ctas_per_sm) * sm_count();
  const int64_t want = (slots + ctas / 2) / ctas;  // the nearest whole number of slices
  const int64_t cap = choose_splits(n_tok, B, min_keys);
  const int64_t s = want < cap ? want : cap;
  return int(s < 1 ? 1 : s);
}

int esize(const stca_config& c) { return c.dtype == STCA_BF16 ? 2 : 4; }

int validate_config(const stca_config& c) {
  if (c.M < 1 || c.M > STCA_MAX_LAYERS || c.d <= 0 || c.H <= 0 || c.max_users < 0 || c.max_tokens < 0 ||
      c.max_targets < 0 || !(c.ln_eps >= 0.f))
    return STCA_ERR_INVALID_ARG;
  if (c.dtype != STCA_FP32 && c.dtype != STCA_BF16) return STCA_ERR_INVALID_ARG;
  if (c.score != STCA_SOFTMAX && c.score != STCA_RELU) return STCA_ERR_INVALID_ARG;
  if (c.time_buckets != 0 && c.time_buckets != 16) return STCA_ERR_UNSUPPORTED;
  if (c.dedup < 0 || c.dedup > 2) return STCA_ERR_INVALID_ARG;
  if (c.kv_fold != 0 && c.kv_fold != 1) return STCA_ERR_INVALID_ARG;
  if (c.kv_fold && (c.mode != STCA_MODE_STCA || c.dtype != STCA_BF16 || c.d != 256 || c.H <= 0 || c.d % c.H != 0 ||
                    c.d / c.H != 64))
    return STCA_ERR_UNSUPPORTED;
  if (c.mode == STCA_MODE_POINTWISE) {
    if (c.dtype != STCA_BF16 || c.d != 128 || c.dedup) return STCA_ERR_UNSUPPORTED;
    return STCA_OK;
  }
  if (c.dedup && c.dtype != STCA_BF16) return STCA_ERR_UNSUPPORTED;
  if (c.hidden <= 0 || c.d % c.H != 0) return STCA_ERR_INVALID_ARG;
  const int dh = c.d / c.H;
  if (c.mode == STCA_MODE_HYFORMER) {
    if (c.dtype != STCA_BF16 || c.score != STCA_SOFTMAX || c.d != 512 || dh != 64 || c.hidden % 128 != 0)
      return STCA_ERR_UNSUPPORTED;
    return STCA_OK;
  }
  if (c.mode != STCA_MODE_STCA) return STCA_ERR_INVALID_ARG;
  if (c.dtype == STCA_BF16) {
    if ((c.d != 256 && c.d != 512) || dh != 64 || c.hidden % 128 != 0) return STCA_ERR_UNSUPPORTED;
  } else {
    if ((dh != 32 && dh != 64 && dh != 128) || c.d > 1024) return STCA_ERR_UNSUPPORTED;
  }
  return STCA_OK;
}

// Element offsets of every target-side weight in the packed buffer.
stca_handle::QLayout q_layout(const stca_config& c) {
  stca_handle::QLayout q{};
  const size_t d = size_t(c.d), hd = size_t(c.hidden);
  size_t at = 0;
  auto take = [&](size_t n) {
    const size_t o = at;
    at += (n + 63) / 64 * 64;  // keep every matrix 128-byte aligned
    return o;
  };
  q.tgt13 = take(2 * hd * d);
  q.tgt2 = take(d * hd);
  for (int i = 0; i < c.M; ++i) {
    q.wq[i] = take(d * d);
    q.wo[i] = take(d * d);
    if (i > 0) {
      q.wc[i] = take(d * (i + 1) * d);
      q.fuse13[i] = take(2 * hd * d);
      q.fuse2[i] = take(d * hd);
    }
  }
  q.wz = take(d * (c.M + 1) * d);
  q.z13 = take(2 * hd * d);
  q.z2 = take(d * hd);
  q.fold_begin = at;
  if (c.kv_fold) {
    const size_t H = size_t(c.H);
    for (int i = 0; i < c.M; ++i) {
      q.kfold[i] = take(H * d * d);
      q.vfold[i] = take(d * H * d);
    }
  }
  q.fold_end = at;
  q.total = at;
  return q;
}

stca_handle::QLayout hq_layout(const stca_config& c) {
  stca_handle::QLayout q{};
  const size_t d = size_t(c.d), hd = size_t(c.hidden);
  // query tokens per user that the workspace was sized for (max_targets = users x tokens)
  int cap = c.max_users > 0 ? c.max_targets / c.max_users : 0;
  q.tok_cap = cap < STCA_MAX_QUERY_TOKENS ? cap : STCA_MAX_QUERY_TOKENS;
  size_t at = 0;
  auto take = [&](size_t n) {
    const size_t o = at;
    at += (n + 63) / 64 * 64;
    return o;
  };
  for (int l = 0; l < c.M; ++l) {
    for (int sq = 0; sq < 2; ++sq) {
      q.hwq[2 * l + sq] = take(d * d);
      q.hwo[2 * l + sq] = take(d * d);
    }
    q.htok13[l] = take(size_t(q.tok_cap) * 2 * hd * d);
    q.htok2[l] = take(size_t(q.tok_cap) * d * hd);
  }
  q.total = at;
  return q;
}

// bf16 STCA with d = 256: the history FFN of every layer runs in one fused kernel that
// keeps the SwiGLU hidden activations on chip (tc_ffn_fused); its per-layer outputs sit
// layer_stride rows apart.
bool fused_ffn(const stca_config& c) {
  return c.mode == STCA_MODE_STCA && c.dtype == STCA_BF16 && c.d == 256 && c.hidden % 128 == 0;
}
size_t ffn_layer_stride(const stca_config& c) { return (size_t(c.max_tokens) + 255) / 256 * 256; }

int allocate(stca_handle* h) {
  const stca_config& c = h->cfg;
  const size_t U = size_t(c.max_users) + 1, N = size_t(c.max_tokens), T = size_t(c.max_targets);
  const size_t d = size_t(c.d), hd = size_t(c.hidden);
  bool ok = dalloc(h, &h->err, 4) && dalloc(h, &h->hoff, U * 4) && dalloc(h, &h->toff, U * 4);
  if (!ok) return STCA_ERR_CUDA;
  if (c.mode == STCA_MODE_POINTWISE) {
    ok = dalloc(h, &h->part_acc, size_t(MAX_SPLITS) * c.max_users * d * 4);
    return ok ? STCA_OK : STCA_ERR_CUDA;
  }
  const size_t E = esize(c);
  const int nseq = c.mode == STCA_MODE_HYFORMER ? 2 : 1;
  if (c.dtype == STCA_BF16) {
    h->wslots = c.M * nseq;
    ok = ok && dalloc(h, &h->wpack, size_t(h->wslots) * (2 * hd * d + d * hd + 2 * d * d) * 2);
  }
  const bool fused = fused_ffn(c);
  // rows of the LN GEMM outputs and their moments: every layer's with the fused FFN
  const size_t xt_rows = fused ? size_t(c.M) * ffn_layer_stride(c) : N;
  if (c.dtype == STCA_BF16)
    ok = ok && dalloc(h, &h->fold, size_t(h->wslots) * 4 * d * 4) && dalloc(h, &h->rowstats, xt_rows * 2 * 4);
  // bf16: the hidden activations of all M layers of every sequence ([N, M h] per sequence),
  // not needed when the fused FFN keeps them on chip
  const size_t hid_elems = fused ? 0 : c.dtype == STCA_BF16 ? nseq * N * size_t(c.M) * hd : N * hd;
  // K/V rows: one buffer per layer on the fused-FFN path (its layers' K/V GEMMs run ahead)
  const size_t kv_layers = (fused && !c.kv_fold) ? size_t(c.M) : 1;
  ok = ok && dalloc(h, &h->hidden, hid_elems * E) && dalloc(h, &h->xt, xt_rows * d * E) &&
       dalloc(h, &h->kv, kv_layers * N * 2 * d * E);
  ok = ok && dalloc(h, &h->qproj, T * d * 4) && dalloc(h, &h->attn, T * d * 4) && dalloc(h, &h->tmp_h, T * hd * 4) &&
       dalloc(h, &h->tmp_d, T * d * 4);
  // the folded attention keeps a d-wide state per (target, head)
  const size_t acc_rows = c.kv_fold ? T * size_t(c.H) : T;
  ok = ok && dalloc(h, &h->part_acc, size_t(MAX_SPLITS) * acc_rows * d * 4) &&
       dalloc(h, &h->part_ml, size_t(MAX_SPLITS) * T * c.H * 2 * 4);
  if (c.kv_fold) ok = ok && dalloc(h, &h->qfold, T * size_t(c.H) * d * 4);
  if (c.dedup) {
    // one map per history sequence (the decode variant keeps both of its sequences' maps)
    h->dedup_ws_bytes = dedup_workspace_bytes(c.max_tokens);
    ok = ok && dalloc(h, &h->dedup_ws, h->dedup_ws_bytes) && dalloc(h, &h->uniq_idx, nseq * N * 4) &&
         dalloc(h, &h->uniq_token, nseq * N * 4) && dalloc(h, &h->uniq_count, 16);
    if (c.dedup == 2)
      ok = ok && dalloc(h, &h->c_rows, nseq * N * 4) && dalloc(h, &h->c_mult, nseq * N * 4) &&
           dalloc(h, &h->c_len, nseq * U * 4);
  }
  if (c.mode == STCA_MODE_STCA) {
    ok = ok && dalloc(h, &h->cat, T * (c.M + 1) * d * 4) && dalloc(h, &h->qbuf, T * d * 4);
    for (int b = 0; b < 2; ++b) {
      ok = ok && dalloc(h, &h->in_ids[b], N * 4) && dalloc(h, &h->in_len[b], U * 4) &&
           dalloc(h, &h->in_tpu[b], U * 4) && dalloc(h, &h->in_xt[b], T * d * E);
      if (c.time_buckets) ok = ok && dalloc(h, &h->in_dt[b], N * 4);
    }
    ok = ok && dalloc(h, &h->out_z[0], T * d * 4) && dalloc(h, &h->out_z[1], T * d * 4);
    if (c.dtype == STCA_BF16) {
      h->ql = q_layout(c);
      ok = ok && dalloc(h, &h->qpack, h->ql.total * 2);
      // the fold matrices are block-diagonal: zero once, packing writes the blocks only
      if (ok && h->ql.fold_end > h->ql.fold_begin)
        ok = cudaMemset(reinterpret_cast<bf16*>(h->qpack) + h->ql.fold_begin, 0,
                        (h->ql.fold_end - h->ql.fold_begin) * 2) == cudaSuccess;
    }
  } else {
    ok = ok && dalloc(h, &h->hoff2, U * 4) && dalloc(h, &h->hq, T * d * 4) && dalloc(h, &h->hqhat, T * d * 4) &&
         dalloc(h, &h->hmix, T * d * 4);
    h->ql = hq_layout(c);
    ok = ok && dalloc(h, &h->qpack, h->ql.total * 2);
  }
  return ok ? STCA_OK : STCA_ERR_CUDA;
}

template <typename TB>
SimtGemmArgs<float, TB> gemm_args(int M, int N, int K, const float* A, int64_t lda, const void* B, float* C,
                                  int64_t ldc, int32_t* err) {
  SimtGemmArgs<float, TB> a;
  memset(&a, 0, sizeof(a));
  a.M = M;
  a.N = N;
  a.K = K;
  a.A = A;
  a.lda = lda;
  a.ksplit = K;
  a.B = reinterpret_cast<const TB*>(B);
  a.C = C;
  a.ldc = ldc;
  a.batch = 1;
  a.err = err;
  return a;
}

// Target-side GEMM: tcgen05 with the packed weights Wp when given and the shape allows,
// else the generic kernels (fp32 weights, per-batch weights).
int qgemm(const SimtGemmArgs<float, float>& a, const bf16*, cudaStream_t s) { return simt_gemm(a, s); }
int qgemm(const SimtGemmArgs<float, bf16>& a, const bf16* Wp, cudaStream_t s) {
  if (Wp && tc_query_supported(a)) return tc_query_gemm(a, Wp, s);
  return simt_gemm(a, s);
}

const bf16* qp(const stca_handle* h, size_t off) {
  return h->qpack ? reinterpret_cast<const bf16*>(h->qpack) + off : nullptr;
}

// out[rows, d] = SwiGLU(A) (then LayerNorm when ffn.gamma != null); A [rows, K=d] fp32.
// p13 / p2: the FFN's packed W1|W3 and W2 (or null).
template <typename TB>
int query_ffn(stca_handle* h, const float* A, int64_t lda, int rows, const stca_ffn& f, float* out, int64_t ldo,
              cudaStream_t s, const bf16* p13 = nullptr, const bf16* p2 = nullptr) {
  const int d = h->cfg.d, hd = h->cfg.hidden;
  auto g = gemm_args<TB>(rows, hd, d, A, lda, f.W1, h->tmp_h, hd, h->err);
  g.B2 = reinterpret_cast<const TB*>(f.W3);
  CK(qgemm(g, p13, s));
  auto g2 = gemm_args<TB>(rows, d, hd, h->tmp_h, hd, f.W2, out, ldo, h->err);
  CK(qgemm(g2, p2, s));
  if (f.gamma) CK(layer_norm_f32(out, ldo, out, ldo, rows, d, f.gamma, f.beta, h->cfg.ln_eps, s));
  return STCA_OK;
}

bool ffn_ok(const stca_ffn& f, bool ln) { return f.W1 && f.W3 && f.W2 && (!ln || (f.gamma && f.beta)); }

int check_weights(const stca_config& c, const stca_weights* w) {
  if (!w || !w->table || w->n_items <= 0) return STCA_ERR_INVALID_ARG;
  if (c.time_buckets && !w->dt_table) return STCA_ERR_INVALID_ARG;
  if (!ffn_ok(w->tgt, true) || !w->WZ || !ffn_ok(w->zffn, false)) return STCA_ERR_INVALID_ARG;
  for (int i = 0; i < c.M; ++i) {
    if (!ffn_ok(w->hist[i], true) || !w->WQ[i] || !w->WK[i] || !w->WV[i] || !w->WO[i]) return STCA_ERR_INVALID_ARG;
    if (i > 0 && (!w->WC[i] || !ffn_ok(w->fuse[i], true))) return STCA_ERR_INVALID_ARG;
  }
  return STCA_OK;
}

// Packing jobs (K-major operand order, bf16) for one SwiGLU FFN: W1|W3 interleaved into
// p13 [2 hd, d], W2 into p2 [d, hd].
void ffn_jobs(const stca_ffn& f, int d, int hd, bf16* p13, bf16* p2, std::vector<PackJob>& jobs) {
  jobs.push_back({f.W1, p13, d, hd, 1, 0});
  jobs.push_back({f.W3, p13, d, hd, 2, 0});
  jobs.push_back({f.W2, p2, hd, d, 0, 0});
}

// True when `w` is the weight struct stca_pin_weights converted (same address and contents).
bool is_pinned(const stca_handle* h, const void* w, size_t bytes) {
  return h->pinned && h->pinned == w && h->pinned_copy.size() == bytes &&
         memcmp(h->pinned_copy.data(), w, bytes) == 0;
}

// Packed history operands of slot sq * M + l.
bf16* wp13(const stca_handle* h, int slot) {
  const size_t d = size_t(h->cfg.d), hd = size_t(h->cfg.hidden);
  return reinterpret_cast<bf16*>(h->wpack) + size_t(slot) * 2 * hd * d;
}
bf16* wp2(const stca_handle* h, int slot) {
  const size_t d = size_t(h->cfg.d), hd = size_t(h->cfg.hidden);
  return wp13(h, h->wslots) + size_t(slot) * d * hd;
}
bf16* wp3(const stca_handle* h, int slot) {
  const size_t d = size_t(h->cfg.d), hd = size_t(h->cfg.hidden);
  return reinterpret_cast<bf16*>(h->wpack) + size_t(h->wslots) * (2 * hd * d + d * hd) + size_t(slot) * 2 * d * d;
}

// One history layer: the FFN, then W_K and W_V interleaved by head into [2 d, d] (rows
// [2 h d_h, 2 h d_h + d_h) are head h of W_K, the next d_h rows head h of W_V), so that the
// K/V GEMM writes each history row as [K_1 | V_1 | K_2 | V_2 | ...] and attention reads one
// contiguous 2 d_h-element segment per (key, head).
void layer_jobs(stca_handle* h, int slot, const stca_ffn& f, const void* WK, const void* WV,
                std::vector<PackJob>& jobs) {
  const int d = h->cfg.d, hd = h->cfg.hidden, dh = d / h->cfg.H;
  ffn_jobs(f, d, hd, wp13(h, slot), wp2(h, slot), jobs);
  jobs.push_back({WK, wp3(h, slot), d, d, 3, 0, dh});
  jobs.push_back({WV, wp3(h, slot), d, d, 3, dh, dh});
}

// The target-side weights of a bf16 STCA call.
void query_jobs(stca_handle* h, const stca_weights* w, std::vector<PackJob>& jobs) {
  const int d = h->cfg.d, hd = h->cfg.hidden, M = h->cfg.M;
  bf16* q = reinterpret_cast<bf16*>(h->qpack);
  const stca_handle::QLayout& L = h->ql;
  ffn_jobs(w->tgt, d, hd, q + L.tgt13, q + L.tgt2, jobs);
  for (int i = 0; i < M; ++i) {
    jobs.push_back({w->WQ[i], q + L.wq[i], d, d, 0, 0});
    jobs.push_back({w->WO[i], q + L.wo[i], d, d, 0, 0});
    if (i > 0) {
      jobs.push_back({w->WC[i], q + L.wc[i], (i + 1) * d, d, 0, 0});
      ffn_jobs(w->fuse[i], d, hd, q + L.fuse13[i], q + L.fuse2[i], jobs);
    }
  }
  jobs.push_back({w->WZ, q + L.wz, (M + 1) * d, d, 0, 0});
  ffn_jobs(w->zffn, d, hd, q + L.z13, q + L.z2, jobs);
  if (h->cfg.kv_fold) {
    const int dh = d / h->cfg.H;
    for (int i = 0; i < M; ++i) {
      jobs.push_back({w->WK[i], q + L.kfold[i], d, d, 4, 0, dh});
      jobs.push_back({w->WV[i], q + L.vfold[i], d, d, 5, 0, dh});
    }
  }
}

// Every tensor-core operand of a bf16 STCA call.
void stca_jobs(stca_handle* h, const stca_weights* w, std::vector<PackJob>& jobs) {
  for (int i = 0; i < h->cfg.M; ++i) layer_jobs(h, i, w->hist[i], w->WK[i], w->WV[i], jobs);
  if (h->qpack) query_jobs(h, w, jobs);
}

// The fold constants of every history layer's LayerNorm (see EpiFold).
int stca_folds(stca_handle* h, const stca_weights* w, cudaStream_t s) {
  const int d = h->cfg.d;
  for (int i = 0; i < h->cfg.M; ++i)
    CK(fold_consts(w->hist[i].gamma, w->hist[i].beta, w->WK[i], w->WV[i], d, d / h->cfg.H,
                   h->fold + size_t(i) * 4 * d, s));
  return STCA_OK;
}

// The decode blocks' operands: per block and sequence the history FFN, W_K|W_V, W_Q and
// W_O; then the per-token FFNs of query tokens 0 .. tokens-1 of every block.
void hyf_jobs(stca_handle* h, const hyf_weights* w, int tokens, std::vector<PackJob>& jobs) {
  const int d = h->cfg.d, hd = h->cfg.hidden;
  const stca_handle::QLayout& L = h->ql;
  bf16* q = reinterpret_cast<bf16*>(h->qpack);
  for (int l = 0; l < h->cfg.M; ++l)
    for (int sq = 0; sq < 2; ++sq) {
      const hyf_seq_weights& f = w->blk[l].seq[sq];
      layer_jobs(h, sq * h->cfg.M + l, f.ffn, f.WK, f.WV, jobs);
      jobs.push_back({f.WQ, q + L.hwq[2 * l + sq], d, d, 0, 0});
      jobs.push_back({f.WO, q + L.hwo[2 * l + sq], d, d, 0, 0});
    }
  for (int l = 0; l < h->cfg.M; ++l)
    for (int t = 0; t < tokens; ++t)
      ffn_jobs(w->blk[l].tok[t], d, hd, q + L.htok13[l] + size_t(t) * 2 * hd * d, q + L.htok2[l] + size_t(t) * d * hd,
               jobs);
}

// SwiGLU hidden activations of all M layers of history sequence sq in one launch: the X
// rows are gathered once (E[id] + T[bucket]) and multiplied by the M layers' W1|W3 packed
// back to back (N = M 2h); layer l's hidden lands in columns [l h, (l+1) h) of the
// sequence's [n_tok, M h] buffer.  Every layer reads the ORIGINAL X, so this is exact.
int history_hidden_bf16(stca_handle* h, int sq, const GatherSrc& g, int n_tok, cudaStream_t s,
                        const int32_t* M_dev) {
  const int d = h->cfg.d, hd = h->cfg.hidden, M = h->cfg.M;
  bf16* hid = reinterpret_cast<bf16*>(h->hidden) + size_t(sq) * size_t(h->cfg.max_tokens) * M * hd;
  STAGE(h, STCA_STAGE_GATHER_FFN, s,
        tc_gemm_resident(A_GATHER, EPI_SWIGLU, nullptr, g, n_tok, d, wp13(h, sq * M), M * hd, hid, M * hd, h->err, s,
                         M_dev));
  return STCA_OK;
}

// X~ = LN(A W2) and [K | V] = X~ [W_K | W_V] of layer l of sequence sq (bf16 tensor cores).
int history_kv_bf16(stca_handle* h, int sq, int l, int n_tok, const float* gamma, const float* beta, cudaStream_t s,
                    const int32_t* M_dev) {
  const int d = h->cfg.d, hd = h->cfg.hidden, M = h->cfg.M;
  const int slot = sq * M + l;
  const bf16* hid = reinterpret_cast<const bf16*>(h->hidden) + size_t(sq) * size_t(h->cfg.max_tokens) * M * hd +
                    size_t(l) * hd;
  GatherSrc none;
  memset(&none, 0, sizeof(none));
  if (!gamma) {  // no LayerNorm (decode blocks): X~ = A W2
    STAGE(h, STCA_STAGE_FFN_OUT, s,
          tc_gemm_rowwise(EPI_PLAIN, hid, n_tok, hd, wp2(h, slot), d, nullptr, nullptr, h->cfg.ln_eps, h->xt, d,
                          h->err, s, M_dev, M * hd));
    STAGE(h, STCA_STAGE_KV, s,
          tc_gemm_resident(A_TMA, EPI_PLAIN, h->xt, none, n_tok, d, wp3(h, slot), 2 * d, h->kv, 2 * d, h->err, s,
                           M_dev));
    return STCA_OK;
  }
  // X~ = LN(A W2) folded into the K/V GEMM: the LN GEMM writes (A W2) * gamma and the row
  // moments, the K/V GEMM applies rstd (acc - mean c) + b per row and column
  STAGE(h, STCA_STAGE_FFN_OUT, s,
        tc_gemm_rowwise(EPI_LNSTAT, hid, n_tok, hd, wp2(h, slot), d, gamma, beta, h->cfg.ln_eps, h->xt, d, h->err,
                        s, M_dev, M * hd, h->rowstats));
  const EpiFold fold{h->rowstats, h->fold + size_t(slot) * 4 * d, h->fold + size_t(slot) * 4 * d + 2 * d};
  STAGE(h, STCA_STAGE_KV, s,
        tc_gemm_resident(A_TMA, EPI_LNFOLD, h->xt, none, n_tok, d, wp3(h, slot), 2 * d, h->kv, 2 * d, h->err, s,
                         M_dev, nullptr, &fold));
  return STCA_OK;
}

// K/V rows of layer l: their own buffer on the fused-FFN path, else the one shared buffer.
void* kv_ptr(const stca_handle* h, int l) {
  const stca_config& c = h->cfg;
  if (!fused_ffn(c) || c.kv_fold) return h->kv;
  return reinterpret_cast<bf16*>(h->kv) + size_t(l) * size_t(c.max_tokens) * 2 * c.d;
}

bool make_side_stream(stca_handle* h) {
  if (h->side_stream) return true;
  bool ok = cudaStreamCreateWithFlags(&h->side_stream, cudaStreamNonBlocking) == cudaSuccess &&
            cudaEventCreateWithFlags(&h->ffn_done, cudaEventDisableTiming) == cudaSuccess;
  for (int l = 0; l < STCA_MAX_LAYERS && ok; ++l)
    ok = cudaEventCreateWithFlags(&h->kv_done[l], cudaEventDisableTiming) == cudaSuccess;
  return ok;
}

// d = 256: y'_l = (A_l W2_l) * gamma_l and the row moments of every layer in one fused
// launch (the hidden activations A_l stay on chip).
int history_ffn_fused(stca_handle* h, const GatherSrc& g, int n_tok, const stca_weights* w, cudaStream_t s,
                      const int32_t* M_dev, int max_pairs = 0) {
  const stca_config& c = h->cfg;
  const float* gammas[STCA_MAX_LAYERS] = {};
  for (int l = 0; l < c.M; ++l) gammas[l] = w->hist[l].gamma;
  STAGE(h, STCA_STAGE_GATHER_FFN, s,
        tc_ffn_fused(g, n_tok, M_dev, c.M, c.hidden, wp13(h, 0), wp2(h, 0), gammas, c.ln_eps, h->xt,
                     int(ffn_layer_stride(c)), h->rowstats, h->err, s, max_pairs));
  return STCA_OK;
}

// [K | V] of layer l from the fused FFN's outputs, with the LayerNorm folded in.
int history_kv_fused(stca_handle* h, int l, int n_tok, cudaStream_t s, const int32_t* M_dev, int max_pairs = 0) {
  const int d = h->cfg.d;
  const size_t stride = ffn_layer_stride(h->cfg);
  GatherSrc none;
  memset(&none, 0, sizeof(none));
  const bf16* y = reinterpret_cast<const bf16*>(h->xt) + size_t(l) * stride * d;
  const EpiFold fold{h->rowstats + size_t(l) * stride * 2, h->fold + size_t(l) * 4 * d,
                     h->fold + size_t(l) * 4 * d + 2 * d};
  STAGE(h, STCA_STAGE_KV, s,
        tc_gemm_resident(A_TMA, EPI_LNFOLD, y, none, n_tok, d, wp3(h, l), 2 * d, kv_ptr(h, l), 2 * d, h->err, s,
                         M_dev, nullptr, &fold, max_pairs));
  return STCA_OK;
}

// SM pairs the history-side GEMMs on the side stream may use: the rest stay free for the
// latency-bound target-side and attention kernels running beside them.
constexpr int KV_AHEAD_PAIRS = 64;

// K/V of every history token for one layer: fp32 SIMT path.
int history_f32(stca_handle* h, const GatherSrc& g, int n_tok, const stca_ffn& f, const void* WK, const void* WV,
                cudaStream_t s) {
  const int d = h->cfg.d, hd = h->cfg.hidden;
  float* hid = reinterpret_cast<float*>(h->hidden);
  float* xt = reinterpret_cast<float*>(h->xt);
  float* kv = reinterpret_cast<float*>(h->kv);
  auto a = gemm_args<float>(n_tok, hd, d, nullptr, d, f.W1, hid, hd, h->err);
  a.B2 = reinterpret_cast<const float*>(f.W3);
  a.gather = g;
  STAGE(h, STCA_STAGE_GATHER_FFN, s, simt_gemm(a, s));
  {
    Prof p(h, STCA_STAGE_FFN_OUT, s);
    CK(simt_gemm(gemm_args<float>(n_tok, d, hd, hid, hd, f.W2, xt, d, h->err), s));
    CK(layer_norm_f32(xt, d, xt, d, n_tok, d, f.gamma, f.beta, h->cfg.ln_eps, s));
  }
  {
    Prof p(h, STCA_STAGE_KV, s);
    CK(simt_gemm(gemm_args<float>(n_tok, d, d, xt, d, WK, kv, 2 * d, h->err), s));
    CK(simt_gemm(gemm_args<float>(n_tok, d, d, xt, d, WV, kv + d, 2 * d, h->err), s));
  }
  return STCA_OK;
}

int run_attention(stca_handle* h, const float* Q, const int32_t* hoff, const int32_t* toff, int B, int T,
                  int splits, int score, cudaStream_t s, const int32_t* kv_rows, const int32_t* kv_len = nullptr,
                  const int32_t* kv_mult = nullptr, const void* kv = nullptr) {
  AttnArgs a;
  a.Q = Q;
  a.KV = kv ? kv : h->kv;
  a.hoff = hoff;
  a.toff = toff;
  a.kv_rows = kv_rows;
  a.kv_len = kv_len;
  a.kv_mult = kv_mult;
  a.B = B;
  a.T = T;
  a.d = h->cfg.d;
  a.H = h->cfg.H;
  a.splits = splits;
  a.score = score;
  a.part_acc = h->part_acc;
  a.part_ml = h->part_ml;
  a.out = h->attn;
  a.err = h->err;
  const bool bf = h->cfg.dtype == STCA_BF16;
  STAGE(h, STCA_STAGE_ATTENTION, s, bf ? attention_bf16(a, s) : attention_f32(a, s));
  if (attention_needs_merge(a, bf)) STAGE(h, STCA_STAGE_MERGE, s, attention_merge(a, s));
  return STCA_OK;
}

// First phase of an STCA forward: offsets, targets into the concatenation buffer, weights
// converted (unless pinned), q^(1) = LN(SwiGLU_t(x_t)), distinct keys; fills h->fwd.
template <typename TB>
int fwd_begin(stca_handle* h, const int32_t* ids, const int32_t* lens, const int32_t* dt, const void* x_t,
              const int32_t* tpu, int B, int n_tok, int t_tot, const stca_weights* w, cudaStream_t s,
              bool ahead = false) {
  const stca_config& c = h->cfg;
  const int d = c.d, M = c.M;
  const bool bf = c.dtype == STCA_BF16;
  const int64_t ldcat = int64_t(M + 1) * d;
  {
    Prof p(h, STCA_STAGE_SETUP, s);
    CK(exclusive_offsets(lens, B, h->hoff, n_tok, h->err, s));
    CK(exclusive_offsets(tpu, B, h->toff, t_tot, h->err, s));
    CK(copy_rows_to_f32(x_t, bf, t_tot, d, h->cat, ldcat, M * d, s));
    if (bf && !is_pinned(h, w, sizeof(*w))) {
      std::vector<PackJob> jobs;
      stca_jobs(h, w, jobs);
      CK(tc_pack_weights(jobs.data(), int(jobs.size()), s));
      CK(stca_folds(h, w, s));
    }
  }
  // `ahead`: the history side (distinct keys, FFN, every layer's K/V) runs on the side
  // stream from here, beside the target side on the caller's stream
  cudaStream_t hs = s;
  if (ahead) {
    if (cudaEventRecord(h->ffn_done, s) != cudaSuccess || cudaStreamWaitEvent(h->side_stream, h->ffn_done, 0) != cudaSuccess)
      return STCA_ERR_CUDA;
    hs = h->side_stream;
  }
  const stca_handle::QLayout& L = h->ql;
  const float* xcol = h->cat + int64_t(M) * d;
  // q^(1) = LN(SwiGLU_t(x_t))
  STAGE(h, STCA_STAGE_QUERY, s,
        query_ffn<TB>(h, xcol, ldcat, t_tot, w->tgt, h->qbuf, d, s, qp(h, L.tgt13), qp(h, L.tgt2)));
  stca_handle::Fwd& f = h->fwd;
  f = stca_handle::Fwd{};
  f.kv_ahead = ahead;
  f.B = B;
  f.n_tok = n_tok;
  f.t_tot = t_tot;
  f.w = w;
  f.g.ids = ids;
  f.g.dt = c.time_buckets ? dt : nullptr;
  f.g.table = w->table;
  f.g.dt_table = c.time_buckets ? w->dt_table : nullptr;
  f.g.n_items = w->n_items;
  if (c.dedup) {
    // distinct keys of the call and (dedup = 2) each user's compacted rows, one launch
    const bool compact = c.dedup == 2;
    if (n_tok <= FUSED_DEDUP_MAX_TOKENS) {
      STAGE(h, STCA_STAGE_DEDUP, hs,
            dedup_fused(ids, f.g.dt, n_tok, h->dedup_ws, h->dedup_ws_bytes, h->uniq_idx, h->uniq_token,
                        h->uniq_count, compact ? h->hoff : nullptr, B, h->c_rows, h->c_mult, h->c_len, h->err, hs));
    } else {
      STAGE(h, STCA_STAGE_DEDUP, hs,
            dedup_rows(ids, f.g.dt, n_tok, h->dedup_ws, h->dedup_ws_bytes, h->uniq_idx, h->uniq_token,
                       h->uniq_count, h->err, hs));
      if (compact)
        STAGE(h, STCA_STAGE_DEDUP, hs,
              compact_user_rows(h->hoff, B, h->uniq_idx, h->c_rows, h->c_mult, h->c_len, hs));
    }
    f.g.rows = h->uniq_token;
    f.M_dev = h->uniq_count;
    f.kv_rows = h->uniq_idx;
    if (compact) {
      // attention over each user's distinct rows, each weighted by its token count
      f.kv_rows = h->c_rows;
      f.kv_len = h->c_len;
      f.kv_mult = h->c_mult;
    }
  }
  f.splits = attention_splits(n_tok, B, c.H, 1024);
  // the folded attention has one CTA per (user, slice) for all heads: slices of >= 256 keys
  f.fold_splits = attention_splits(n_tok, B, 1, 256, 3);
  return STCA_OK;
}

// Layer i up to the attention: the history side (K/V of every key) and Q^(i) = q^(i) W_Q.
template <typename TB>
int fwd_layer_inputs(stca_handle* h, int i, cudaStream_t s) {
  const stca_config& c = h->cfg;
  const stca_handle::Fwd& f = h->fwd;
  const stca_weights* w = f.w;
  if (c.dtype == STCA_BF16 && fused_ffn(c)) {
    if (f.kv_ahead) {
      // the history side on the side stream: the fused FFN, then every layer's K/V (each
      // depends only on the FFN), each marked by its event; grids capped so that SMs stay
      // free for the target side running beside them
      if (i == 0) {
        CK(history_ffn_fused(h, f.g, f.n_tok, w, h->side_stream, f.M_dev, KV_AHEAD_PAIRS));
        for (int l = 0; l < c.M; ++l) {
          CK(history_kv_fused(h, l, f.n_tok, h->side_stream, f.M_dev, KV_AHEAD_PAIRS));
          if (cudaEventRecord(h->kv_done[l], h->side_stream) != cudaSuccess) return STCA_ERR_CUDA;
        }
      }
    } else {
      if (i == 0) CK(history_ffn_fused(h, f.g, f.n_tok, w, s, f.M_dev));
      if (!c.kv_fold) CK(history_kv_fused(h, i, f.n_tok, s, f.M_dev));  // the fold needs no K/V rows
    }
  } else if (c.dtype == STCA_BF16) {
    if (i == 0) CK(history_hidden_bf16(h, 0, f.g, f.n_tok, s, f.M_dev));
    CK(history_kv_bf16(h, 0, i, f.n_tok, w->hist[i].gamma, w->hist[i].beta, s, f.M_dev));
  } else {
    CK(history_f32(h, f.g, f.n_tok, w->hist[i], w->WK[i], w->WV[i], s));
  }
  STAGE(h, STCA_STAGE_QUERY, s,
        qgemm(gemm_args<TB>(f.t_tot, c.d, c.d, h->qbuf, c.d, w->WQ[i], h->qproj, c.d, h->err), qp(h, h->ql.wq[i]), s));
  if (f.kv_ahead && cudaStreamWaitEvent(s, h->kv_done[i], 0) != cudaSuccess) return STCA_ERR_CUDA;
  if (c.kv_fold) {  // q~_{t,h} = Q_{t,h} W_K,h^T: [T, d] x block-diagonal -> [T, H d]
    const int Hd = c.H * c.d;
    STAGE(h, STCA_STAGE_QUERY, s,
          tc_query_gemm(gemm_args<bf16>(f.t_tot, Hd, c.d, h->qproj, c.d, nullptr, h->qfold, Hd, h->err),
                        qp(h, h->ql.kfold[i]), s));
  }
  return STCA_OK;
}

// Layer i's attention with W_K / W_V folded into the queries: r = sum_j a_j x~_j per (target,
// head) from the history rows y' and their LayerNorm moments, then o_h = r_h W_V,h for all
// heads at once into the heads buffer.
int run_attention_fold(stca_handle* h, int i, cudaStream_t s) {
  const stca_config& c = h->cfg;
  const stca_handle::Fwd& f = h->fwd;
  const size_t stride = ffn_layer_stride(c);
  FoldArgs a;
  a.Qf = h->qfold;
  a.Y = reinterpret_cast<const bf16*>(h->xt) + size_t(i) * stride * c.d;
  a.stats = h->rowstats + size_t(i) * stride * 2;
  a.gamma = f.w->hist[i].gamma;
  a.beta = f.w->hist[i].beta;
  a.hoff = h->hoff;
  a.toff = h->toff;
  a.kv_rows = f.kv_rows;
  a.kv_len = f.kv_len;
  a.kv_mult = f.kv_mult;
  a.B = f.B;
  a.T = f.t_tot;
  a.d = c.d;
  a.H = c.H;
  a.splits = f.fold_splits;
  a.score = c.score;
  a.part_acc = h->part_acc;
  a.part_ml = h->part_ml;
  a.out = h->qfold;  // a CTA reads only its user's query rows before writing them
  a.err = h->err;
  STAGE(h, STCA_STAGE_ATTENTION, s, attention_fold_bf16(a, s));
  if (a.splits > 1) {  // the slices' d-wide states: the merge with one "head" of width d
    AttnArgs m;
    memset(&m, 0, sizeof(m));
    m.T = f.t_tot * c.H;
    m.d = c.d;
    m.H = 1;
    m.splits = a.splits;
    m.score = c.score;
    m.part_acc = h->part_acc;
    m.part_ml = h->part_ml;
    m.out = h->qfold;
    m.err = h->err;
    STAGE(h, STCA_STAGE_MERGE, s, attention_merge(m, s));
  }
  const int Hd = c.H * c.d;
  STAGE(h, STCA_STAGE_QUERY, s,
        tc_query_gemm(gemm_args<bf16>(f.t_tot, c.d, Hd, h->qfold, Hd, nullptr, h->attn, c.d, h->err),
                      qp(h, h->ql.vfold[i]), s));
  return STCA_OK;
}

// Layer i after the attention (heads in h->attn): o^(i) = [o_1 .. o_H] W_O into the
// concatenation buffer, then q^(i+2) = LN(SwiGLU([o^(1) .. o^(i+1) | x_t] W_C)), or after
// the last layer z = SwiGLU_Z([o^(1) .. o^(M) | x_t] W_Z).
template <typename TB>
int fwd_layer_outputs(stca_handle* h, int i, float* z_out, cudaStream_t s) {
  const stca_config& c = h->cfg;
  const stca_handle::Fwd& f = h->fwd;
  const stca_weights* w = f.w;
  const stca_handle::QLayout& L = h->ql;
  const int d = c.d, M = c.M, t_tot = f.t_tot;
  const int64_t ldcat = int64_t(M + 1) * d;
  {
    Prof p(h, STCA_STAGE_QUERY, s);
    CK(qgemm(gemm_args<TB>(t_tot, d, d, h->attn, d, w->WO[i], h->cat + int64_t(i) * d, ldcat, h->err),
             qp(h, L.wo[i]), s));
    if (i + 1 < M) {
      const int K = (i + 2) * d;
      auto a = gemm_args<TB>(t_tot, d, K, h->cat, ldcat, w->WC[i + 1], h->tmp_d, d, h->err);
      a.ksplit = (i + 1) * d;
      a.kshift = (M - (i + 1)) * d;
      CK(qgemm(a, qp(h, L.wc[i + 1]), s));
      CK(query_ffn<TB>(h, h->tmp_d, d, t_tot, w->fuse[i + 1], h->qbuf, d, s, qp(h, L.fuse13[i + 1]),
                       qp(h, L.fuse2[i + 1])));
    }
  }
  if (i + 1 == M) {
    Prof p(h, STCA_STAGE_QUERY, s);
    CK(qgemm(gemm_args<TB>(t_tot, d, int(ldcat), h->cat, ldcat, w->WZ, h->tmp_d, d, h->err), qp(h, L.wz), s));
    CK(query_ffn<TB>(h, h->tmp_d, d, t_tot, w->zffn, z_out, d, s, qp(h, L.z13), qp(h, L.z2)));
  }
  return STCA_OK;
}

template <typename TB>
int run_stca(stca_handle* h, const int32_t* ids, const int32_t* lens, const int32_t* dt, const void* x_t,
             const int32_t* tpu, int B, int n_tok, int t_tot, const stca_weights* w, float* z_out, float* o_out,
             cudaStream_t s) {
  const stca_config& c = h->cfg;
  const int d = c.d, M = c.M;
  const int64_t ldcat = int64_t(M + 1) * d;
  h->fwd.next_layer = -1;  // a whole forward closes any open sequence-parallel one
  const bool ahead = c.dtype == STCA_BF16 && fused_ffn(c) && !c.kv_fold;
  if (ahead && !make_side_stream(h)) return STCA_ERR_CUDA;
  CK(fwd_begin<TB>(h, ids, lens, dt, x_t, tpu, B, n_tok, t_tot, w, s, ahead));
  const stca_handle::Fwd& f = h->fwd;
  for (int i = 0; i < M; ++i) {
    CK(fwd_layer_inputs<TB>(h, i, s));
    if (c.kv_fold) CK(run_attention_fold(h, i, s));
    else CK(run_attention(h, h->qproj, h->hoff, h->toff, B, t_tot, f.splits, c.score, s, f.kv_rows, f.kv_len,
                          f.kv_mult, kv_ptr(h, i)));
    CK(fwd_layer_outputs<TB>(h, i, z_out, s));
  }
  if (o_out && t_tot > 0) {
    for (int i = 0; i < M; ++i)
      if (cudaMemcpy2DAsync(o_out + int64_t(i) * t_tot * d, size_t(d) * 4, h->cat + int64_t(i) * d, size_t(ldcat) * 4,
                            size_t(d) * 4, t_tot, cudaMemcpyDeviceToDevice, s) != cudaSuccess)
        return STCA_ERR_CUDA;
  }
  return STCA_OK;
}

int check_forward_args(stca_handle* h, const int32_t* ids, const int32_t* lens, const int32_t* dt, const void* x_t,
                       const int32_t* tpu, int B, int n_tok, int t_tot, const stca_weights* w, const float* z,
                       bool need_z = true) {
  if (!h) return STCA_ERR_INVALID_ARG;
  const stca_config& c = h->cfg;
  if (c.mode != STCA_MODE_STCA) return STCA_ERR_INVALID_ARG;
  if (B < 0 || n_tok < 0 || t_tot < 0) return STCA_ERR_INVALID_ARG;
  if (B > c.max_users || n_tok > c.max_tokens || t_tot > c.max_targets) return STCA_ERR_CAPACITY;
  if ((B > 0 && (!lens || !tpu)) || (n_tok > 0 && !ids) || (t_tot > 0 && (!x_t || (need_z && !z))))
    return STCA_ERR_INVALID_ARG;
  if (c.time_buckets && n_tok > 0 && !dt) return STCA_ERR_INVALID_ARG;
  return check_weights(c, w);
}

}  // namespace

extern "C" {

const char* stca_strerror(int code) {
  switch (code) {
    case STCA_OK: return "ok";
    case STCA_ERR_INVALID_ARG: return "invalid argument";
    case STCA_ERR_UNSUPPORTED: return "unsupported configuration";
    case STCA_ERR_CAPACITY: return "size exceeds the handle's capacity";
    case STCA_ERR_CUDA: return "CUDA error";
    case STCA_ERR_ID_OUT_OF_RANGE: return "item id out of range";
    case STCA_ERR_TIMEOUT: return "a bounded device wait timed out";
    case STCA_ERR_BAD_LENGTHS: return "lengths negative or inconsistent with the totals";
    default: return "unknown status";
  }
}

int stca_create(const stca_config* cfg, stca_handle** out) {
  if (!out) return STCA_ERR_INVALID_ARG;
  *out = nullptr;
  if (!cfg) return STCA_ERR_INVALID_ARG;
  CK(validate_config(*cfg));
  stca_handle* h = new (std::nothrow) stca_handle();
  if (!h) return STCA_ERR_CUDA;
  h->cfg = *cfg;
  if (cudaGetDevice(&h->device) != cudaSuccess) {
    delete h;
    return STCA_ERR_CUDA;
  }
  const int rc = allocate(h);
  if (rc != STCA_OK || cudaMemset(h->err, 0, 4) != cudaSuccess) {
    free_all(h);
    delete h;
    return rc != STCA_OK ? rc : STCA_ERR_CUDA;
  }
  *out = h;
  return STCA_OK;
}

int stca_pin_weights(stca_handle* h, const void* weights, void* stream) {
  if (!h || !weights || h->cfg.mode == STCA_MODE_POINTWISE) return STCA_ERR_INVALID_ARG;
  if (h->cfg.dtype != STCA_BF16) return STCA_ERR_UNSUPPORTED;
  if (cudaSetDevice(h->device) != cudaSuccess) return STCA_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  h->pinned = nullptr;
  h->pinned_copy.clear();
  std::vector<PackJob> jobs;
  size_t bytes = 0;
  int tokens = 0;
  if (h->cfg.mode == STCA_MODE_STCA) {
    const stca_weights* w = static_cast<const stca_weights*>(weights);
    CK(check_weights(h->cfg, w));
    stca_jobs(h, w, jobs);
    CK(stca_folds(h, w, s));
    bytes = sizeof(*w);
  } else {
    const hyf_weights* w = static_cast<const hyf_weights*>(weights);
    if (w->blocks != h->cfg.M) return STCA_ERR_INVALID_ARG;
    for (int l = 0; l < h->cfg.M; ++l)
      for (int sq = 0; sq < 2; ++sq) {
        const hyf_seq_weights& f = w->blk[l].seq[sq];
        if (!ffn_ok(f.ffn, false) || !f.WQ || !f.WK || !f.WV || !f.WO) return STCA_ERR_INVALID_ARG;
      }
    // the leading query-token slots whose FFNs are set in every block
    while (tokens < h->ql.tok_cap) {
      bool all = true;
      for (int l = 0; l < h->cfg.M; ++l) all = all && ffn_ok(w->blk[l].tok[tokens], false);
      if (!all) break;
      ++tokens;
    }
    hyf_jobs(h, w, tokens, jobs);
    bytes = sizeof(*w);
  }
  CK(tc_pack_weights(jobs.data(), int(jobs.size()), s));
  h->pinned = weights;
  h->pinned_copy.assign(static_cast<const uint8_t*>(weights), static_cast<const uint8_t*>(weights) + bytes);
  h->pinned_tokens = tokens;
  return STCA_OK;
}

void stca_unpin_weights(stca_handle* h) {
  if (!h) return;
  h->pinned = nullptr;
  h->pinned_copy.clear();
  h->pinned_tokens = 0;
}

void stca_destroy(stca_handle* h) {
  if (!h) return;
  cudaSetDevice(h->device);
  if (!h->recs.empty()) cudaDeviceSynchronize();
  recycle_events(h);
  for (cudaEvent_t e : h->spare) cudaEventDestroy(e);
  if (h->copy_stream) {
    cudaStreamSynchronize(h->copy_stream);
    cudaStreamSynchronize(h->back_stream);
    cudaStreamDestroy(h->copy_stream);
    cudaStreamDestroy(h->back_stream);
    for (int b = 0; b < 2; ++b) {
      cudaEventDestroy(h->in_ready[b]);
      cudaEventDestroy(h->in_free[b]);
      cudaEventDestroy(h->z_ready[b]);
      cudaEventDestroy(h->z_free[b]);
    }
  }
  if (h->side_stream) {
    cudaStreamSynchronize(h->side_stream);
    cudaStreamDestroy(h->side_stream);
    cudaEventDestroy(h->ffn_done);
    for (int l = 0; l < STCA_MAX_LAYERS; ++l) cudaEventDestroy(h->kv_done[l]);
  }
  free_all(h);
  delete h;
}

int stca_forward(stca_handle* h, const int32_t* hist_ids, const int32_t* hist_lengths, const int32_t* hist_dt,
                 const void* target_emb, const int32_t* targets_per_user, int B, int n_tok, int t_tot,
                 const stca_weights* w, float* z_out, float* o_out, void* stream) {
  CK(check_forward_args(h, hist_ids, hist_lengths, hist_dt, target_emb, targets_per_user, B, n_tok, t_tot, w, z_out));
  if (cudaSetDevice(h->device) != cudaSuccess) return STCA_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  h->last_stream = s;
  if (B == 0) return STCA_OK;
  return h->cfg.dtype == STCA_BF16
             ? run_stca<bf16>(h, hist_ids, hist_lengths, hist_dt, target_emb, targets_per_user, B, n_tok, t_tot, w,
                              z_out, o_out, s)
             : run_stca<float>(h, hist_ids, hist_lengths, hist_dt, target_emb, targets_per_user, B, n_tok, t_tot, w,
                               z_out, o_out, s);
}

int stca_forward_host(stca_handle* h, const int32_t* ids, const int32_t* lens, const int32_t* dt, const void* x_t,
                      const int32_t* tpu, int B, int n_tok, int t_tot, const stca_weights* w, float* z_host,
                      void* stream) {
  CK(check_forward_args(h, ids, lens, dt, x_t, tpu, B, n_tok, t_tot, w, z_host));
  if (cudaSetDevice(h->device) != cudaSuccess) return STCA_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  h->last_stream = s;
  if (B == 0) return STCA_OK;
  const size_t E = esize(h->cfg);
  const size_t d = size_t(h->cfg.d);
  if (!h->copy_stream) {
    bool made = cudaStreamCreateWithFlags(&h->copy_stream, cudaStreamNonBlocking) == cudaSuccess &&
                cudaStreamCreateWithFlags(&h->back_stream, cudaStreamNonBlocking) == cudaSuccess;
    for (int b = 0; b < 2; ++b)
      made = made && cudaEventCreateWithFlags(&h->in_ready[b], cudaEventDisableTiming) == cudaSuccess &&
             cudaEventCreateWithFlags(&h->in_free[b], cudaEventDisableTiming) == cudaSuccess &&
             cudaEventCreateWithFlags(&h->z_ready[b], cudaEventDisableTiming) == cudaSuccess &&
             cudaEventCreateWithFlags(&h->z_free[b], cudaEventDisableTiming) == cudaSuccess;
    if (!made) return STCA_ERR_CUDA;
  }
  // this call's inputs go to slot b on the copy stream, once the forward that read slot b
  // two calls ago is done; the forward on s waits for them
  const int b = h->in_slot;
  cudaStream_t c = h->copy_stream;
  bool ok = !h->in_used[b] || cudaStreamWaitEvent(c, h->in_free[b], 0) == cudaSuccess;
  ok = ok && cudaMemcpyAsync(h->in_len[b], lens, size_t(B) * 4, cudaMemcpyHostToDevice, c) == cudaSuccess &&
       cudaMemcpyAsync(h->in_tpu[b], tpu, size_t(B) * 4, cudaMemcpyHostToDevice, c) == cudaSuccess;
  if (n_tok > 0) ok = ok && cudaMemcpyAsync(h->in_ids[b], ids, size_t(n_tok) * 4, cudaMemcpyHostToDevice, c) == cudaSuccess;
  if (n_tok > 0 && h->cfg.time_buckets)
    ok = ok && cudaMemcpyAsync(h->in_dt[b], dt, size_t(n_tok) * 4, cudaMemcpyHostToDevice, c) == cudaSuccess;
  if (t_tot > 0)
    ok = ok && cudaMemcpyAsync(h->in_xt[b], x_t, size_t(t_tot) * d * E, cudaMemcpyHostToDevice, c) == cudaSuccess;
  ok = ok && cudaEventRecord(h->in_ready[b], c) == cudaSuccess && cudaStreamWaitEvent(s, h->in_ready[b], 0) == cudaSuccess;
  // the forward writes output slot b once the read-back of the call before last has left it
  ok = ok && (!h->z_used[b] || cudaStreamWaitEvent(s, h->z_free[b], 0) == cudaSuccess);
  if (!ok) return STCA_ERR_CUDA;
  h->in_slot ^= 1;
  const int rc = h->cfg.dtype == STCA_BF16
                     ? run_stca<bf16>(h, h->in_ids[b], h->in_len[b], h->in_dt[b], h->in_xt[b], h->in_tpu[b], B, n_tok,
                                      t_tot, w, h->out_z[b], nullptr, s)
                     : run_stca<float>(h, h->in_ids[b], h->in_len[b], h->in_dt[b], h->in_xt[b], h->in_tpu[b], B,
                                       n_tok, t_tot, w, h->out_z[b], nullptr, s);
  // slot b is free for the call after next once this forward has read it (recorded even
  // when the forward returned early, so that call never waits on a stale event)
  h->in_used[b] = cudaEventRecord(h->in_free[b], s) == cudaSuccess;
  CK(rc);
  // z goes back on back_stream, so the next call's forward does not queue behind the copy
  cudaStream_t r = h->back_stream;
  ok = cudaEventRecord(h->z_ready[b], s) == cudaSuccess && cudaStreamWaitEvent(r, h->z_ready[b], 0) == cudaSuccess;
  if (t_tot > 0)
    ok = ok && cudaMemcpyAsync(z_host, h->out_z[b], size_t(t_tot) * d * 4, cudaMemcpyDeviceToHost, r) == cudaSuccess;
  h->z_used[b] = ok && cudaEventRecord(h->z_free[b], r) == cudaSuccess;
  if (!h->z_used[b]) return STCA_ERR_CUDA;
  h->z_last = b;
  return STCA_OK;
}

int stca_host_fence(stca_handle* h, void* stream) {
  if (!h) return STCA_ERR_INVALID_ARG;
  if (h->z_last < 0) return STCA_OK;
  if (cudaSetDevice(h->device) != cudaSuccess) return STCA_ERR_CUDA;
  // back_stream runs its copies in call order, so the latest one landing means all have
  return cudaStreamWaitEvent(reinterpret_cast<cudaStream_t>(stream), h->z_free[h->z_last], 0) == cudaSuccess
             ? STCA_OK
             : STCA_ERR_CUDA;
}

// ---- sequence-parallel (L-split) forward in phases: every rank holds a slice of each
// user's history and all of the user's targets; per layer the slices' attention states are
// exchanged by the caller and merged here ([wechat] §1.1: local attentions merge exactly).

int stca_lsplit_begin(stca_handle* h, const int32_t* hist_ids, const int32_t* hist_lengths, const int32_t* hist_dt,
                      const void* target_emb, const int32_t* targets_per_user, int B, int n_tok, int t_tot,
                      const stca_weights* w, void* stream) {
  CK(check_forward_args(h, hist_ids, hist_lengths, hist_dt, target_emb, targets_per_user, B, n_tok, t_tot, w,
                        nullptr, false));
  if (h->cfg.kv_fold) return STCA_ERR_UNSUPPORTED;  // the folded attention keeps no slice state API
  if (cudaSetDevice(h->device) != cudaSuccess) return STCA_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  h->last_stream = s;
  h->fwd.next_layer = -1;
  if (B > 0 && t_tot > 0) {
    CK(h->cfg.dtype == STCA_BF16
           ? fwd_begin<bf16>(h, hist_ids, hist_lengths, hist_dt, target_emb, targets_per_user, B, n_tok, t_tot, w, s)
           : fwd_begin<float>(h, hist_ids, hist_lengths, hist_dt, target_emb, targets_per_user, B, n_tok, t_tot, w,
                              s));
  } else {  // no targets: the phases run without work, so every rank still makes every call
    h->fwd = stca_handle::Fwd{};
    h->fwd.w = w;
  }
  h->fwd.next_layer = 0;
  h->fwd.partial_done = false;
  return STCA_OK;
}

int stca_lsplit_partial(stca_handle* h, int layer, float* acc, float* ml, void* stream) {
  if (!h || h->cfg.mode != STCA_MODE_STCA) return STCA_ERR_INVALID_ARG;
  stca_handle::Fwd& f = h->fwd;
  if (f.next_layer < 0 || layer != f.next_layer || f.partial_done) return STCA_ERR_INVALID_ARG;
  if (f.t_tot > 0 && (!acc || (h->cfg.score == 0 && !ml))) return STCA_ERR_INVALID_ARG;
  if (cudaSetDevice(h->device) != cudaSuccess) return STCA_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  h->last_stream = s;
  if (f.t_tot == 0) {
    f.partial_done = true;
    return STCA_OK;
  }
  const bool bf = h->cfg.dtype == STCA_BF16;
  CK(bf ? fwd_layer_inputs<bf16>(h, layer, s) : fwd_layer_inputs<float>(h, layer, s));
  AttnArgs a;
  a.Q = h->qproj;
  a.KV = kv_ptr(h, layer);
  a.hoff = h->hoff;
  a.toff = h->toff;
  a.kv_rows = f.kv_rows;
  a.kv_len = f.kv_len;
  a.kv_mult = f.kv_mult;
  a.B = f.B;
  a.T = f.t_tot;
  a.d = h->cfg.d;
  a.H = h->cfg.H;
  a.splits = f.splits;
  a.score = h->cfg.score;
  a.err = h->err;
  if (bf && f.splits == 1) {  // the one slice's state straight into the caller's buffers
    a.part_acc = acc;
    a.part_ml = ml;
    a.out = nullptr;
    a.partial_out = 1;
    STAGE(h, STCA_STAGE_ATTENTION, s, attention_bf16(a, s));
  } else {  // this rank's slices, combined into one state
    a.part_acc = h->part_acc;
    a.part_ml = h->part_ml;
    a.out = h->attn;
    STAGE(h, STCA_STAGE_ATTENTION, s, bf ? attention_bf16(a, s) : attention_f32(a, s));
    a.out = acc;
    a.ml_out = h->cfg.score == 0 ? ml : nullptr;
    STAGE(h, STCA_STAGE_MERGE, s, attention_merge(a, s));
  }
  f.partial_done = true;
  return STCA_OK;
}

int stca_lsplit_merge(stca_handle* h, int layer, int ranks, const float* all_acc, const float* all_ml, float* z_out,
                      void* stream) {
  if (!h || h->cfg.mode != STCA_MODE_STCA) return STCA_ERR_INVALID_ARG;
  stca_handle::Fwd& f = h->fwd;
  if (f.next_layer < 0 || layer != f.next_layer || !f.partial_done) return STCA_ERR_INVALID_ARG;
  if (ranks < 1 || ranks > 32) return STCA_ERR_INVALID_ARG;
  const bool last = layer + 1 == h->cfg.M;
  if (f.t_tot > 0 && (!all_acc || (h->cfg.score == 0 && !all_ml) || (last && !z_out))) return STCA_ERR_INVALID_ARG;
  if (cudaSetDevice(h->device) != cudaSuccess) return STCA_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  h->last_stream = s;
  if (f.t_tot == 0) {
    f.partial_done = false;
    f.next_layer = last ? -1 : layer + 1;
    return STCA_OK;
  }
  AttnArgs a;
  memset(&a, 0, sizeof(a));
  a.T = f.t_tot;
  a.d = h->cfg.d;
  a.H = h->cfg.H;
  a.splits = ranks;
  a.score = h->cfg.score;
  a.part_acc = const_cast<float*>(all_acc);
  a.part_ml = const_cast<float*>(all_ml);
  a.out = h->attn;
  a.err = h->err;
  STAGE(h, STCA_STAGE_MERGE, s, attention_merge(a, s));
  const bool bf = h->cfg.dtype == STCA_BF16;
  CK(bf ? fwd_layer_outputs<bf16>(h, layer, z_out, s) : fwd_layer_outputs<float>(h, layer, z_out, s));
  f.partial_done = false;
  f.next_layer = last ? -1 : layer + 1;
  return STCA_OK;
}

int stca_pointwise_forward(stca_handle* h, const int32_t* ids, const int32_t* lengths, const void* q, const void* table,
                           int64_t n_items, int B, int n_tok, float* out, void* stream) {
  if (!h || h->cfg.mode != STCA_MODE_POINTWISE) return STCA_ERR_INVALID_ARG;
  if (B < 0 || n_tok < 0 || n_items <= 0) return STCA_ERR_INVALID_ARG;
  if (B > h->cfg.max_users || n_tok > h->cfg.max_tokens) return STCA_ERR_CAPACITY;
  if (B > 0 && (!lengths || !q || !table || !out)) return STCA_ERR_INVALID_ARG;
  if (n_tok > 0 && !ids) return STCA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(table)) & 15) return STCA_ERR_INVALID_ARG;
  if (cudaSetDevice(h->device) != cudaSuccess) return STCA_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  h->last_stream = s;
  if (B == 0) return STCA_OK;
  STAGE(h, STCA_STAGE_SETUP, s, exclusive_offsets(lengths, B, h->hoff, n_tok, h->err, s));
  const int splits = choose_splits(n_tok, B, 2048);
  STAGE(h, STCA_STAGE_POINTWISE, s,
        pointwise_relu_ta(ids, h->hoff, q, table, n_items, B, h->cfg.d, splits, h->part_acc, out, h->err, s));
  return STCA_OK;
}

int hyformer_forward(stca_handle* h, const int32_t* ids_feed, const int32_t* len_feed, int n_feed,
                     const int32_t* ids_search, const int32_t* len_search, int n_search, const void* q0, int B,
                     int n_query, const hyf_weights* w, float* out, void* stream) {
  if (!h || h->cfg.mode != STCA_MODE_HYFORMER || !w) return STCA_ERR_INVALID_ARG;
  const stca_config& c = h->cfg;
  const int d = c.d, hd = c.hidden;
  const int T = 2 * n_query;
  if (B < 0 || n_feed < 0 || n_search < 0 || n_query <= 0 || T > STCA_MAX_QUERY_TOKENS || d % T != 0)
    return STCA_ERR_INVALID_ARG;
  if (w->blocks != c.M || !w->table || w->n_items <= 0) return STCA_ERR_INVALID_ARG;
  if (B > c.max_users || n_feed > c.max_tokens || n_search > c.max_tokens || int64_t(B) * T > c.max_targets)
    return STCA_ERR_CAPACITY;
  if (B > 0 && (!len_feed || !len_search || !q0 || !out)) return STCA_ERR_INVALID_ARG;
  if ((n_feed > 0 && !ids_feed) || (n_search > 0 && !ids_search)) return STCA_ERR_INVALID_ARG;
  for (int l = 0; l < c.M; ++l) {
    for (int sq = 0; sq < 2; ++sq) {
      const hyf_seq_weights& f = w->blk[l].seq[sq];
      if (!ffn_ok(f.ffn, false) || !f.WQ || !f.WK || !f.WV || !f.WO) return STCA_ERR_INVALID_ARG;
    }
    for (int t = 0; t < T; ++t)
      if (!ffn_ok(w->blk[l].tok[t], false)) return STCA_ERR_INVALID_ARG;
  }
  if (cudaSetDevice(h->device) != cudaSuccess) return STCA_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  h->last_stream = s;
  if (B == 0) return STCA_OK;
  const int rows = B * T, rows_s = B * n_query;
  const stca_handle::QLayout& L = h->ql;
  const bool pinned = is_pinned(h, w, sizeof(*w));
  const bool tok_tc = pinned && T <= h->pinned_tokens;  // per-token FFNs converted at pin time
  {
    Prof p(h, STCA_STAGE_SETUP, s);
    CK(exclusive_offsets(len_feed, B, h->hoff, n_feed, h->err, s));
    CK(exclusive_offsets(len_search, B, h->hoff2, n_search, h->err, s));
    CK(fill_arange(h->toff, B + 1, n_query, s));
    CK(copy_rows_to_f32(q0, 1, rows, d, h->hq, d, 0, s));
    if (!pinned) {
      // per call only the per-sequence operands; the per-token FFNs then run on the generic
      // kernels, which read the weights as given
      std::vector<PackJob> jobs;
      hyf_jobs(h, w, 0, jobs);
      CK(tc_pack_weights(jobs.data(), int(jobs.size()), s));
    }
  }
  const int32_t* ids[2] = {ids_feed, ids_search};
  const int32_t* offs[2] = {h->hoff, h->hoff2};
  const int ntok[2] = {n_feed, n_search};
  for (int l = 0; l < c.M; ++l) {
    for (int sq = 0; sq < 2; ++sq) {
      const hyf_seq_weights& f = w->blk[l].seq[sq];
      GatherSrc g;
      memset(&g, 0, sizeof(g));
      g.ids = ids[sq];
      g.table = w->table;
      g.n_items = w->n_items;
      // H = SwiGLU(X_s) (eq 7), K/V = H W_K, H W_V (eq 8)
      const int32_t* M_dev = nullptr;
      const int32_t* kv_rows = nullptr;
      const int32_t *kv_len = nullptr, *kv_mult = nullptr;
      if (c.dedup) {
        const size_t off = size_t(sq) * c.max_tokens;
        const size_t uoff = size_t(sq) * (size_t(c.max_users) + 1);
        if (l == 0) {
          if (ntok[sq] <= FUSED_DEDUP_MAX_TOKENS) {
            STAGE(h, STCA_STAGE_DEDUP, s,
                  dedup_fused(ids[sq], nullptr, ntok[sq], h->dedup_ws, h->dedup_ws_bytes, h->uniq_idx + off,
                              h->uniq_token + off, h->uniq_count + sq, c.dedup == 2 ? offs[sq] : nullptr, B,
                              h->c_rows + off, h->c_mult + off, h->c_len + uoff, h->err, s));
          } else {
            STAGE(h, STCA_STAGE_DEDUP, s,
                  dedup_rows(ids[sq], nullptr, ntok[sq], h->dedup_ws, h->dedup_ws_bytes, h->uniq_idx + off,
                             h->uniq_token + off, h->uniq_count + sq, h->err, s));
            if (c.dedup == 2)
              STAGE(h, STCA_STAGE_DEDUP, s,
                    compact_user_rows(offs[sq], B, h->uniq_idx + off, h->c_rows + off, h->c_mult + off,
                                      h->c_len + uoff, s));
          }
        }
        g.rows = h->uniq_token + off;
        M_dev = h->uniq_count + sq;
        kv_rows = h->uniq_idx + off;
        if (c.dedup == 2) {
          kv_rows = h->c_rows + off;
          kv_len = h->c_len + uoff;
          kv_mult = h->c_mult + off;
        }
      }
      if (l == 0) CK(history_hidden_bf16(h, sq, g, ntok[sq], s, M_dev));
      CK(history_kv_bf16(h, sq, l, ntok[sq], nullptr, nullptr, s, M_dev));
      // queries of sequence sq: rows b*T + sq*n_query + n
      auto qa = gemm_args<bf16>(rows_s, d, d, h->hq, d, f.WQ, h->qproj, d, h->err);
      qa.a_grp = n_query;
      qa.a_gstride = T;
      qa.a_goff = sq * n_query;
      STAGE(h, STCA_STAGE_QUERY, s, qgemm(qa, qp(h, L.hwq[2 * l + sq]), s));
      CK(run_attention(h, h->qproj, offs[sq], h->toff, B, rows_s, attention_splits(ntok[sq], B, h->cfg.H, 1024),
                       STCA_SOFTMAX, s, kv_rows, kv_len, kv_mult));
      auto oa = gemm_args<bf16>(rows_s, d, d, h->attn, d, f.WO, h->hqhat, d, h->err);
      oa.c_grp = n_query;
      oa.c_gstride = T;
      oa.c_goff = sq * n_query;
      STAGE(h, STCA_STAGE_QUERY, s, qgemm(oa, qp(h, L.hwo[2 * l + sq]), s));
    }
    // query boosting: token mix (eq 11-13), per-token SwiGLU (eq 14), residual (eq 15)
    Prof p(h, STCA_STAGE_BOOST, s);
    CK(token_mix(h->hqhat, B, T, d, h->hmix, s));
    auto a1 = gemm_args<bf16>(B, hd, d, h->hmix, int64_t(T) * d, nullptr, h->tmp_h, int64_t(T) * hd, h->err);
    a1.batch = T;
    a1.bsA = d;
    a1.bsC = hd;
    for (int t = 0; t < T; ++t) {
      a1.Bz[t] = reinterpret_cast<const bf16*>(w->blk[l].tok[t].W1);
      a1.B2z[t] = reinterpret_cast<const bf16*>(w->blk[l].tok[t].W3);
    }
    a1.B2 = a1.B2z[0];
    CK(qgemm(a1, tok_tc ? qp(h, L.htok13[l]) : nullptr, s));
    float* dst = (l + 1 == c.M) ? out : h->hq;
    auto a2 = gemm_args<bf16>(B, d, hd, h->tmp_h, int64_t(T) * hd, nullptr, dst, int64_t(T) * d, h->err);
    a2.batch = T;
    a2.bsA = hd;
    a2.bsC = d;
    a2.R = h->hqhat;
    a2.ldr = int64_t(T) * d;
    a2.bsR = d;
    for (int t = 0; t < T; ++t) a2.Bz[t] = reinterpret_cast<const bf16*>(w->blk[l].tok[t].W2);
    CK(qgemm(a2, tok_tc ? qp(h, L.htok2[l]) : nullptr, s));
  }
  return STCA_OK;
}

int stca_profile_stages(stca_handle* h, uint32_t stage_mask) {
  if (!h) return STCA_ERR_INVALID_ARG;
  if (cudaSetDevice(h->device) != cudaSuccess) return STCA_ERR_CUDA;
  if (!h->recs.empty() && cudaDeviceSynchronize() != cudaSuccess) return STCA_ERR_CUDA;
  recycle_events(h);
  h->prof = stage_mask & ((1u << STCA_N_STAGES) - 1u);
  return STCA_OK;
}

int stca_profile_enable(stca_handle* h, int enable) {
  return stca_profile_stages(h, enable ? (1u << STCA_N_STAGES) - 1u : 0u);
}

int stca_profile_read(stca_handle* h, double* total_ms, int64_t* calls) {
  if (!h || !total_ms || !calls) return STCA_ERR_INVALID_ARG;
  if (cudaSetDevice(h->device) != cudaSuccess) return STCA_ERR_CUDA;
  for (int i = 0; i < STCA_N_STAGES; ++i) {
    total_ms[i] = 0.0;
    calls[i] = 0;
  }
  for (auto& r : h->recs) {
    if (cudaEventSynchronize(r.b) != cudaSuccess) return STCA_ERR_CUDA;
    float ms = 0.f;
    if (cudaEventElapsedTime(&ms, r.a, r.b) != cudaSuccess) return STCA_ERR_CUDA;
    total_ms[r.stage] += ms;
    calls[r.stage] += 1;
  }
  return STCA_OK;
}

uint64_t stca_launch_count(void) { return stca::g_launches.load(); }

int stca_stream_wait(void* stream, int timeout_ms) {
  if (timeout_ms < 0) return STCA_ERR_INVALID_ARG;
  cudaEvent_t e = nullptr;
  if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return STCA_ERR_CUDA;
  int rc = STCA_OK;
  if (cudaEventRecord(e, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) {
    rc = STCA_ERR_CUDA;
  } else {
    const auto deadline = std::chrono::steady_clock::now() + std::chrono::milliseconds(timeout_ms);
    while (true) {
      const cudaError_t q = cudaEventQuery(e);
      if (q == cudaSuccess) break;
      if (q != cudaErrorNotReady) {
        rc = STCA_ERR_CUDA;
        break;
      }
      if (std::chrono::steady_clock::now() >= deadline) {
        rc = STCA_ERR_TIMEOUT;
        break;
      }
      std::this_thread::sleep_for(std::chrono::microseconds(200));
    }
  }
  cudaEventDestroy(e);  // released once the recorded work completes
  return rc;
}

int stca_sync_status(stca_handle* h) {
  if (!h) return STCA_ERR_INVALID_ARG;
  if (cudaSetDevice(h->device) != cudaSuccess) return STCA_ERR_CUDA;
  if (cudaStreamSynchronize(h->last_stream) != cudaSuccess) return STCA_ERR_CUDA;
  if (h->back_stream && cudaStreamSynchronize(h->back_stream) != cudaSuccess) return STCA_ERR_CUDA;
  int32_t e = 0;
  if (cudaMemcpy(&e, h->err, 4, cudaMemcpyDeviceToHost) != cudaSuccess) return STCA_ERR_CUDA;
  if (e != 0 && cudaMemset(h->err, 0, 4) != cudaSuccess) return STCA_ERR_CUDA;
  return e;
}

}  // extern "C"
