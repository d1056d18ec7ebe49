// Split-L few-query cross attention with Request-Level Batching.
//
// For one user u, one head h and one slice c of the user's keys, every target of u
// (all m_u queries at once, so each K/V row is read once for all of them: RLB, STCA
// notes "Request Level Batching") produces a local state over the slice:
//   softmax: mx = max_j s_j, l = sum_j 2^(s_j - mx), acc = sum_j 2^(s_j - mx) v_j
//   relu:    acc = sum_j relu(s_j) v_j
// with s_j = q.k_j / sqrt(d_h) (scores kept in log2 units for the softmax form).
// The merge kernel combines the slices (WeChat TA article §1.1: items of a sequence do
// not interact, so local attention results can be merged); with a single slice the bf16
// kernel writes the normalised output itself and no merge runs:
//   softmax: M = max_c mx_c, o = sum_c 2^(mx_c - M) acc_c / sum_c 2^(mx_c - M) l_c
//   relu:    o = sum_c acc_c
// An empty key set gives o = 0.
#include "common.cuh"
#include "internal.h"

namespace stca {

namespace {

constexpr float LOG2E = 1.4426950408889634f;
constexpr float LN2 = 0.6931471805599453f;
constexpr float RESCALE_SLACK = 8.f;  // log2 units a running max may lag the true max

__device__ __forceinline__ void slice_bounds(const AttnArgs& a, int u, int s, int64_t& k0, int& nk, int& t0, int& m) {
  const int h0 = a.hoff[u], h1 = a.hoff[u + 1];
  const int64_t L = a.kv_len ? a.kv_len[u] : h1 - h0;
  k0 = h0 + (L * s) / a.splits;
  const int64_t k1 = h0 + (L * (s + 1)) / a.splits;
  nk = int(k1 - k0);
  t0 = a.toff[u];
  m = a.toff[u + 1] - t0;
}

// ------------------------------------------------------------------------------------
// bf16 K/V, d_h = 64, tensor-core (mma.sync m16n8k16) scores and P V.
//
// A CTA of 8 warps serves one (user, L-slice, head).  The warps form 4 teams of 2; team t
// streams the 32-key tiles t, t+4, ... of the slice through its own ring of KV_STAGES
// shared-memory stages, both warps of the team copying half of each tile.  Within a team
// the two warps split the work of a tile: by queries when the user has more than 16
// targets in the current chunk (warp w takes 16 of the up to 32), else by keys (warp w
// takes keys 16 w .. 16 w + 15 of every tile, all queries).  Each warp keeps its own
// online-softmax state; the states are combined in shared memory at the end.

constexpr int DH = 64;
constexpr int KT = 32;                        // keys per tile
constexpr int TILE_BYTES = KT * DH * 2;       // 4 KB for K (same for V)
constexpr int TEAM_STAGE = 2 * TILE_BYTES;    // K tile | V tile
constexpr int KV_STAGES = 3;                  // tiles in flight per team
constexpr int TEAMS = 4;
constexpr int ATT_THREADS = 2 * 32 * TEAMS;   // 256
constexpr int TEAM_BYTES = KV_STAGES * TEAM_STAGE;   // 24 KB
constexpr int RING_BYTES = TEAMS * TEAM_BYTES;       // 96 KB
// K/V row indices and key multiplicities of a team's tiles, copied two tiles ahead of the
// K/V copies that need them: slots for the tile computed, the tiles in flight and the next
constexpr int IDX_STAGES = KV_STAGES + 2;
static_assert(KV_STAGES == 2 || KV_STAGES == 3, "the index copy schedule below is laid out for 2 or 3 stages");
constexpr int IDX_BYTES = TEAMS * IDX_STAGES * 2 * KT * 4;
constexpr int ATTN_SMEM = RING_BYTES + IDX_BYTES;    // two CTAs per SM

// Named barrier of one team's 64 threads (ids 1..TEAMS; 0 is __syncthreads).
__device__ __forceinline__ void team_sync(int team) {
  asm volatile("bar.sync %0, 64;" ::"r"(team + 1) : "memory");
}

// Row-index side of a tile (compacted or distinct-row keys): thread tt of the team copies
// entry tt % 32 of the tile's K/V rows (tt < 32) or multiplicities (tt >= 32) into the
// tile's index slot; entries past the slice end read as 0 and are never used.
__device__ __forceinline__ void copy_tile_index(int* slot, const int32_t* kv_rows, const int32_t* kv_mult,
                                                int64_t row0, int valid, int tt) {
  const int key = tt & 31;
  const int32_t* src = tt < 32 ? kv_rows : kv_mult;
  if (!src) return;
  cp_async_4(slot + (tt >> 5) * KT + key, src + row0 + (key < valid ? key : 0), key < valid ? 4u : 0u);
}

// Issues this thread's cp.async copies of the K and V slices of head h for a tile: chunk
// tt % 8 of keys tt / 8 + 8 i, i = 0..3 (128-byte key rows, 16-byte chunk c of key k at
// chunk c ^ (k % 8)).  K/V rows are head-interleaved ([K_h | V_h] at column kvcol = 2 h d_h),
// so a key's K and V slices of head h are one contiguous 256-byte segment.  Rows come from
// the tile's index slot, or are row0 + key; keys past the slice end are zero-filled.
__device__ __forceinline__ void load_kv_tile(uint8_t* stage, const int* slot, int64_t row0, int valid,
                                             const bf16* KV, int64_t ld, int kvcol, int tt) {
  uint8_t* sK = stage;
  uint8_t* sV = stage + TILE_BYTES;
  const int ch = tt & 7;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int key = (tt >> 3) + 8 * i;
    const bool ok = key < valid;
    const int64_t row = ok ? (slot ? int64_t(slot[key]) : row0 + key) : 0;
    const bf16* src = KV + row * ld + kvcol + ch * 8;
    const int off = key * 128 + ((ch ^ (key & 7)) << 4);
    cp_async_16(sK + off, src, ok ? 16u : 0u);
    cp_async_16(sV + off, src + DH, ok ? 16u : 0u);
  }
}

// One warp's work on one tile: its 16 queries (A fragments qa, pre-scaled) against the NJ
// groups of 8 keys starting at group j0, then O += P V.  State per row half hr (rows g and
// g + 8 of the warp's 16): running reference point mrow and sum lrow (softmax), O in o.
template <int SCORE, int NJ>
__device__ __forceinline__ void tile_step(uint32_t sK, uint32_t sV, const float* smul, int j0,
                                          const uint32_t (&qa)[4][4], const uint32_t (&qlo)[4][4],
                                          float (&o)[8][4], float (&mrow)[2], float (&lrow)[2], int valid,
                                          int lane) {
  const int tq = lane & 3;
  // S = Q K^T
  float sacc[NJ][4];
#pragma unroll
  for (int jj = 0; jj < NJ; ++jj)
#pragma unroll
    for (int e = 0; e < 4; ++e) sacc[jj][e] = 0.f;
#pragma unroll
  for (int jj = 0; jj < NJ; ++jj) {
    const int key = (j0 + jj) * 8 + (lane & 7);
#pragma unroll
    for (int p = 0; p < 2; ++p) {
      const int ch = 4 * p + (lane >> 3);
      uint32_t kb[4];
      ldsm_x4(sK + key * 128 + ((ch ^ (key & 7)) << 4), kb);
      mma_bf16_16816(sacc[jj], qa[2 * p], kb[0], kb[1]);
      mma_bf16_16816(sacc[jj], qa[2 * p + 1], kb[2], kb[3]);
      if (SCORE == 1) {  // the low bf16 terms of the queries (see the query fragments)
        mma_bf16_16816(sacc[jj], qlo[2 * p], kb[0], kb[1]);
        mma_bf16_16816(sacc[jj], qlo[2 * p + 1], kb[2], kb[3]);
      }
    }
  }
  // keys past the slice end (last tile only)
  if (valid < KT) {
#pragma unroll
    for (int jj = 0; jj < NJ; ++jj)
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if ((j0 + jj) * 8 + 2 * tq + (e & 1) >= valid) sacc[jj][e] = (SCORE == 0) ? -INFINITY : 0.f;
  }
  // scores -> weights
  if (SCORE == 0) {
    // The reference point m of a row moves only when a score exceeds it by more than
    // RESCALE_SLACK (log2 units): weights 2^(s - m) then stay <= 2^RESCALE_SLACK, exact in
    // fp32, and the state is rescaled rarely.  Each thread checks its own scores against m;
    // only when one of the warp's scores is above m + RESCALE_SLACK are the row maxima
    // gathered across the four threads of each row (shuffles) and the rows that moved
    // rescaled.  Numerator and denominator share m, so the quotient is unchanged.
    float mx[2];
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
      mx[hr] = -INFINITY;
#pragma unroll
      for (int jj = 0; jj < NJ; ++jj) mx[hr] = fmaxf(mx[hr], fmaxf(sacc[jj][2 * hr], sacc[jj][2 * hr + 1]));
    }
    if (__any_sync(0xffffffffu, mx[0] > mrow[0] + RESCALE_SLACK || mx[1] > mrow[1] + RESCALE_SLACK)) {
#pragma unroll
      for (int hr = 0; hr < 2; ++hr) {
        float rm = fmaxf(mx[hr], __shfl_xor_sync(0xffffffffu, mx[hr], 1));
        rm = fmaxf(rm, __shfl_xor_sync(0xffffffffu, rm, 2));
        if (rm > mrow[hr] + RESCALE_SLACK) {
          const float corr = exp2_approx(mrow[hr] - rm);  // 0 while m was -inf
          mrow[hr] = rm;
          lrow[hr] *= corr;
#pragma unroll
          for (int nt = 0; nt < 8; ++nt) {
            o[nt][2 * hr] *= corr;
            o[nt][2 * hr + 1] *= corr;
          }
        }
      }
    }
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
      const float muse = (mrow[hr] == -INFINITY) ? 0.f : mrow[hr];
      float sum = 0.f;
#pragma unroll
      for (int jj = 0; jj < NJ; ++jj) {
        float p0 = exp2_approx(sacc[jj][2 * hr] - muse);
        float p1 = exp2_approx(sacc[jj][2 * hr + 1] - muse);
        if (smul) {  // a compacted key weighs as many tokens as it stands for
          const float2 c = *reinterpret_cast<const float2*>(smul + (j0 + jj) * 8 + 2 * tq);
          p0 *= c.x;
          p1 *= c.y;
        }
        sacc[jj][2 * hr] = p0;
        sacc[jj][2 * hr + 1] = p1;
        sum += p0 + p1;
      }
      lrow[hr] += sum;
    }
  } else {
#pragma unroll
    for (int jj = 0; jj < NJ; ++jj) {
      float2 c = make_float2(1.f, 1.f);
      if (smul) c = *reinterpret_cast<const float2*>(smul + (j0 + jj) * 8 + 2 * tq);
      sacc[jj][0] = fmaxf(sacc[jj][0], 0.f) * c.x;
      sacc[jj][1] = fmaxf(sacc[jj][1], 0.f) * c.y;
      sacc[jj][2] = fmaxf(sacc[jj][2], 0.f) * c.x;
      sacc[jj][3] = fmaxf(sacc[jj][3], 0.f) * c.y;
    }
  }
  // O += P V   (P as A fragments straight from the score accumulators)
#pragma unroll
  for (int kb = 0; kb < NJ / 2; ++kb) {
    uint32_t pa[4];
    pa[0] = pack_bf16x2(sacc[2 * kb][0], sacc[2 * kb][1]);
    pa[1] = pack_bf16x2(sacc[2 * kb][2], sacc[2 * kb][3]);
    pa[2] = pack_bf16x2(sacc[2 * kb + 1][0], sacc[2 * kb + 1][1]);
    pa[3] = pack_bf16x2(sacc[2 * kb + 1][2], sacc[2 * kb + 1][3]);
    const int key = (j0 / 2 + kb) * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
    for (int np = 0; np < 4; ++np) {
      const int ch = 2 * np + (lane >> 4);
      uint32_t vb[4];
      ldsm_x4_t(sV + key * 128 + ((ch ^ (key & 7)) << 4), vb);
      mma_bf16_16816(o[2 * np], pa, vb[0], vb[1]);
      mma_bf16_16816(o[2 * np + 1], pa, vb[2], vb[3]);
    }
  }
}

template <int SCORE>
__global__ void __launch_bounds__(ATT_THREADS, SCORE == 1 ? 1 : 2) attn_bf16_kernel(AttnArgs a) {
  griddep_wait();
  griddep_launch();
  extern __shared__ __align__(128) uint8_t smem[];
  const int u = blockIdx.x / a.splits, s = blockIdx.x % a.splits, h = blockIdx.y;
  int64_t k0;
  int nk, t0, m;
  slice_bounds(a, u, s, k0, nk, t0, m);
  if (m <= 0) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, tq = lane & 3;
  const int team = warp >> 1, mem = warp & 1, tt = mem * 32 + lane;
  const int d = a.d;
  const int64_t ld = 2 * int64_t(d);
  const int hcol = h * DH;
  const bf16* KV = reinterpret_cast<const bf16*>(a.KV);
  uint8_t* tbuf = smem + team * TEAM_BYTES;
  int* tidx = a.kv_rows ? reinterpret_cast<int*>(smem + RING_BYTES) + team * IDX_STAGES * 2 * KT : nullptr;
  const float qscale = (SCORE == 0 ? LOG2E : 1.0f) * rsqrtf(float(DH));
  const int n_tiles = (nk + KT - 1) / KT;

  for (int qp = 0; qp < m; qp += 32) {
    const int mq = min(32, m - qp);
    const bool ksplit = mq <= 16;           // the warps of a team split keys, else queries
    const int qr0 = ksplit ? 0 : 16 * mem;  // this warp's first query row in the chunk
    // ---- query fragments (A operand), scaled, bf16.  The ReLU form's output is not
    // normalised, so its score errors do not cancel: there each query value x is carried as
    // bf16(x) + bf16(x - bf16(x)) (qlo, two MMAs per K step), which keeps the scores at fp32
    // accuracy; one bf16 rounding of the queries dominated its error at d = 256.
    uint32_t qa[4][4], qlo[4][4];
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int row = qr0 + g + ((e & 1) ? 8 : 0);
        const int col = kk * 16 + 2 * tq + ((e & 2) ? 8 : 0);
        float x0 = 0.f, x1 = 0.f;
        if (row < mq) {
          const float* qrow = a.Q + int64_t(t0 + qp + row) * d + hcol + col;
          x0 = qrow[0] * qscale;
          x1 = qrow[1] * qscale;
        }
        qa[kk][e] = pack_bf16x2(x0, x1);
        if (SCORE == 1) {
          const float2 hf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&qa[kk][e]));
          qlo[kk][e] = pack_bf16x2(x0 - hf.x, x1 - hf.y);
        } else {
          qlo[kk][e] = 0u;
        }
      }
    float o[8][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) o[nt][e] = 0.f;
    float mrow[2] = {-INFINITY, -INFINITY}, lrow[2] = {0.f, 0.f};

    // ---- stream the team's tiles (local tile j is tile team + TEAMS j): the K/V of
    // KV_STAGES - 1 tiles are in flight while one is computed, and the row indices (with
    // multiplicities) of a tile are copied two tiles before its K/V
    const int n_local = n_tiles > team ? (n_tiles - team + TEAMS - 1) / TEAMS : 0;
    auto tile_of = [&](int j) { return team + TEAMS * j; };
    auto idx_slot = [&](int j) { return tidx ? tidx + (j % IDX_STAGES) * 2 * KT : nullptr; };
    auto copy_idx = [&](int j) {
      if (tidx && j < n_local) {
        const int tl = tile_of(j);
        copy_tile_index(idx_slot(j), a.kv_rows, a.kv_mult, k0 + int64_t(tl) * KT, min(KT, nk - tl * KT), tt);
      }
    };
    // the key multiplicities of a tile arrive as int32 counts; thread tt >= 32 of the team,
    // which copied entry tt - 32, turns it into a float in place once its own copy has
    // landed, and a team barrier orders that before the consumers read the float weights
    auto to_float_mult = [&](int j) {
      if (tidx && a.kv_mult && tt >= 32 && j < n_local) {
        int* e = idx_slot(j) + KT + (tt - 32);
        *reinterpret_cast<float*>(e) = float(*e);
      }
    };
    auto load_kv = [&](int j, int st) {
      if (j < n_local) {
        const int tl = tile_of(j);
        load_kv_tile(tbuf + st * TEAM_STAGE, idx_slot(j), k0 + int64_t(tl) * KT, min(KT, nk - tl * KT), KV, ld,
                     2 * hcol, tt);
      }
    };
    if (tidx) {
      copy_idx(0);
      copy_idx(1);
      cp_async_commit();
      cp_async_wait_all();
      to_float_mult(0);
      to_float_mult(1);
      team_sync(team);
    }
#pragma unroll
    for (int p = 0; p < KV_STAGES - 1; ++p) {
      load_kv(p, p);
      copy_idx(p + 2);  // indices of tiles 0 and 1 came first
      cp_async_commit();
    }
    int stage = 0;
    for (int j = 0; j < n_local; ++j) {
      cp_async_wait<KV_STAGES - 2>();
      // this thread's copies of tile j (and the indices of tile j + KV_STAGES - 1) have
      // landed; after the barrier the team's have, and both warps are done with tile j - 1
      team_sync(team);
      int st = stage + KV_STAGES - 1;
      st = st >= KV_STAGES ? st - KV_STAGES : st;
      load_kv(j + KV_STAGES - 1, st);
      copy_idx(j + KV_STAGES + 1);
      cp_async_commit();
      // tile j + 2's counts: their copy was in the group the wait above completed; the
      // barriers of the next two iterations order this before their use
      to_float_mult(j + 2);
      const uint32_t sK = smem_u32(tbuf + stage * TEAM_STAGE);
      const uint32_t sV = sK + TILE_BYTES;
      const int valid = min(KT, nk - tile_of(j) * KT);
      const float* smul = a.kv_mult ? reinterpret_cast<const float*>(idx_slot(j) + KT) : nullptr;
      if (ksplit) tile_step<SCORE, 2>(sK, sV, smul, 2 * mem, qa, qlo, o, mrow, lrow, valid, lane);
      else tile_step<SCORE, 4>(sK, sV, smul, 0, qa, qlo, o, mrow, lrow, valid, lane);
      stage = stage + 1 == KV_STAGES ? 0 : stage + 1;
    }
    cp_async_wait_all();

    // ---- combine the warps' states through shared memory
    if (SCORE == 0) {
#pragma unroll
      for (int hr = 0; hr < 2; ++hr) {
        lrow[hr] += __shfl_xor_sync(0xffffffffu, lrow[hr], 1);
        lrow[hr] += __shfl_xor_sync(0xffffffffu, lrow[hr], 2);
      }
    }
    __syncthreads();
    float* comb = reinterpret_cast<float*>(smem);  // [8 warps][16 rows][64]
    float* cm = comb + 8 * 16 * DH;                // [8][16]
    float* cl = cm + 8 * 16;                       // [8][16]
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
      const int r = g + 8 * hr;
      float* dst = comb + (warp * 16 + r) * DH;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        dst[nt * 8 + 2 * tq] = o[nt][2 * hr];
        dst[nt * 8 + 2 * tq + 1] = o[nt][2 * hr + 1];
      }
      if (tq == 0) {
        cm[warp * 16 + r] = mrow[hr];
        cl[warp * 16 + r] = lrow[hr];
      }
    }
    __syncthreads();
    {
      // 32 rows x 8 segments of 8 dims; a row's states sit in all 8 warps (key split) or in
      // the 4 warps w with w % 2 == row / 16 (query split)
      const int row = threadIdx.x >> 3, seg = threadIdx.x & 7;
      if (row < mq) {
        const int t = t0 + qp + row;
        const int nsrc = ksplit ? 8 : 4;
        const int lr = ksplit ? row : (row & 15);
        float wgt[8];
        float M = -INFINITY, Lsum = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int w = ksplit ? i : (row >> 4) + 2 * i;
          wgt[i] = 0.f;
          if (i < nsrc) {
            if (SCORE == 0) M = fmaxf(M, cm[w * 16 + lr]);
            else wgt[i] = 1.f;
          }
        }
        if (SCORE == 0) {
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int w = ksplit ? i : (row >> 4) + 2 * i;
            if (i < nsrc) {
              const float mw = cm[w * 16 + lr];
              wgt[i] = (mw == -INFINITY) ? 0.f : exp2f(mw - M);
              Lsum += wgt[i] * cl[w * 16 + lr];
            }
          }
        }
        // one slice: the state is final, so write the normalised output (no merge pass)
        const bool direct = a.splits == 1 && !a.partial_out;
        const float scale = (SCORE == 0 && direct) ? (Lsum > 0.f ? 1.f / Lsum : 0.f) : 1.f;
        float v[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) v[c] = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          if (i < nsrc) {
            const int w = ksplit ? i : (row >> 4) + 2 * i;
            const float* srcp = comb + (w * 16 + lr) * DH + seg * 8;
#pragma unroll
            for (int c = 0; c < 8; ++c) v[c] += wgt[i] * srcp[c];
          }
        }
        float* pacc = (direct ? a.out + int64_t(t) * d : a.part_acc + (int64_t(s) * a.T + t) * d) + hcol + seg * 8;
        reinterpret_cast<float4*>(pacc)[0] = make_float4(v[0] * scale, v[1] * scale, v[2] * scale, v[3] * scale);
        reinterpret_cast<float4*>(pacc)[1] = make_float4(v[4] * scale, v[5] * scale, v[6] * scale, v[7] * scale);
        if (SCORE == 0 && seg == 0 && !direct) {
          float* pml = a.part_ml + ((int64_t(s) * a.T + t) * a.H + h) * 2;
          pml[0] = M;
          pml[1] = Lsum;
        }
        if (SCORE == 0 && seg == 0 && direct && a.lse_out)  // sum_j e^s_j = 2^M Lsum
          a.lse_out[int64_t(t) * a.H + h] = Lsum > 0.f ? (M + log2f(Lsum)) * LN2 : -INFINITY;
      }
    }
    __syncthreads();
  }
}

// ------------------------------------------------------------------------------------
// fp32 K/V (the fp32 configuration), SIMT; lane c holds dims c, c+32, ... of the head.

template <int DPL, int SCORE>
__global__ void __launch_bounds__(128) attn_f32_kernel(AttnArgs a) {
  __shared__ float comb[4][DPL * 32 + 2];
  const int u = blockIdx.x / a.splits, s = blockIdx.x % a.splits, h = blockIdx.y;
  int64_t k0;
  int nk, t0, m;
  slice_bounds(a, u, s, k0, nk, t0, m);
  if (m <= 0) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int d = a.d, dh = DPL * 32;
  const int64_t ld = 2 * int64_t(d);
  const float* KV = reinterpret_cast<const float*>(a.KV);
  const float scale = (SCORE == 0 ? LOG2E : 1.0f) / sqrtf(float(dh));
  for (int ti = 0; ti < m; ++ti) {
    const int t = t0 + ti;
    float q[DPL], acc[DPL];
#pragma unroll
    for (int i = 0; i < DPL; ++i) {
      q[i] = a.Q[int64_t(t) * d + h * dh + lane + 32 * i] * scale;
      acc[i] = 0.f;
    }
    float mx = -INFINITY, l = 0.f;
    for (int j = warp; j < nk; j += 4) {
      const float* krow = KV + (a.kv_rows ? int64_t(a.kv_rows[k0 + j]) : k0 + j) * ld + h * dh;
      float sc = 0.f;
#pragma unroll
      for (int i = 0; i < DPL; ++i) sc += q[i] * krow[lane + 32 * i];
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) sc += __shfl_xor_sync(0xffffffffu, sc, off);
      const float* vrow = krow + d;
      if (SCORE == 0) {
        const float mnew = fmaxf(mx, sc);
        const float corr = exp2f(mx - mnew);
        const float p = exp2f(sc - mnew);
        l = l * corr + p;
#pragma unroll
        for (int i = 0; i < DPL; ++i) acc[i] = acc[i] * corr + p * vrow[lane + 32 * i];
        mx = mnew;
      } else {
        const float p = fmaxf(sc, 0.f);
#pragma unroll
        for (int i = 0; i < DPL; ++i) acc[i] += p * vrow[lane + 32 * i];
      }
    }
#pragma unroll
    for (int i = 0; i < DPL; ++i) comb[warp][lane + 32 * i] = acc[i];
    if (lane == 0) {
      comb[warp][dh] = mx;
      comb[warp][dh + 1] = l;
    }
    __syncthreads();
    if (warp == 0) {
      float M = -INFINITY, wgt[4], Lsum = 0.f;
      if (SCORE == 0) {
#pragma unroll
        for (int w = 0; w < 4; ++w) M = fmaxf(M, comb[w][dh]);
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          wgt[w] = comb[w][dh] == -INFINITY ? 0.f : exp2f(comb[w][dh] - M);
          Lsum += wgt[w] * comb[w][dh + 1];
        }
      } else {
#pragma unroll
        for (int w = 0; w < 4; ++w) wgt[w] = 1.f;
      }
      float* pacc = a.part_acc + (int64_t(s) * a.T + t) * d + h * dh;
#pragma unroll
      for (int i = 0; i < DPL; ++i) {
        float v = 0.f;
#pragma unroll
        for (int w = 0; w < 4; ++w) v += wgt[w] * comb[w][lane + 32 * i];
        pacc[lane + 32 * i] = v;
      }
      if (SCORE == 0 && lane == 0) {
        float* pml = a.part_ml + ((int64_t(s) * a.T + t) * a.H + h) * 2;
        pml[0] = M;
        pml[1] = Lsum;
      }
    }
    __syncthreads();
  }
}

// ------------------------------------------------------------------------------------
// merge of the per-slice states; one warp per (target, head).  Lane s < splits turns
// slice s's running max and sum into its weight once; the column loop then reads every
// slice's accumulator with the weights broadcast by shuffles, four slices in flight.

template <int SCORE>
__global__ void attn_merge_kernel(AttnArgs a) {
  griddep_wait();
  griddep_launch();
  const int64_t wid = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (wid >= int64_t(a.T) * a.H) return;
  const int t = int(wid / a.H), h = int(wid % a.H);
  const int dh = a.d / a.H;
  const int S = a.splits;
  float w = 0.f, inv = 1.f, M = -INFINITY, Lsum = 0.f;
  if (SCORE == 0) {
    float m = -INFINITY, l = 0.f;
    if (lane < S) {
      const float2 ml = *reinterpret_cast<const float2*>(a.part_ml + ((int64_t(lane) * a.T + t) * a.H + h) * 2);
      m = ml.x;
      l = ml.y;
    }
    M = m;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    w = (m == -INFINITY) ? 0.f : exp2f(m - M);
    Lsum = w * l;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) Lsum += __shfl_xor_sync(0xffffffffu, Lsum, o);
    inv = Lsum > 0.f ? 1.f / Lsum : 0.f;
  } else {
    w = 1.f;
  }
  const int64_t slice = int64_t(a.T) * a.d;
  const float* acc = a.part_acc + int64_t(t) * a.d + h * dh;
  for (int c = lane; c < dh; c += 32) {
    float v = 0.f;
    int s = 0;
    for (; s + 4 <= S; s += 4) {
      const float x0 = acc[(s + 0) * slice + c], x1 = acc[(s + 1) * slice + c];
      const float x2 = acc[(s + 2) * slice + c], x3 = acc[(s + 3) * slice + c];
      v += __shfl_sync(0xffffffffu, w, s + 0) * x0;
      v += __shfl_sync(0xffffffffu, w, s + 1) * x1;
      v += __shfl_sync(0xffffffffu, w, s + 2) * x2;
      v += __shfl_sync(0xffffffffu, w, s + 3) * x3;
    }
    for (; s < S; ++s) v += __shfl_sync(0xffffffffu, w, s) * acc[s * slice + c];
    // one combined state (unnormalised, with its max and sum), or the output
    a.out[int64_t(t) * a.d + h * dh + c] = (SCORE == 0 && !a.ml_out) ? v * inv : v;
  }
  if (SCORE == 0 && a.ml_out && lane == 0) {
    float2* ml = reinterpret_cast<float2*>(a.ml_out + (int64_t(t) * a.H + h) * 2);
    *ml = make_float2(M, Lsum);
  }
  if (SCORE == 0 && a.lse_out && !a.ml_out && lane == 0)
    a.lse_out[int64_t(t) * a.H + h] = Lsum > 0.f ? (M + log2f(Lsum)) * LN2 : -INFINITY;
}

}  // namespace

int attention_bf16(const AttnArgs& a, cudaStream_t s) {
  if (a.B == 0 || a.T == 0) return 0;
  if (a.d / a.H != DH || a.d % a.H != 0) return STCA_ERR_UNSUPPORTED;
  dim3 grid(a.B * a.splits, a.H);
  if (a.score == 0) {
    cudaFuncSetAttribute(attn_bf16_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, ATTN_SMEM);
    launch_dep(attn_bf16_kernel<0>, grid, dim3(ATT_THREADS), ATTN_SMEM, s, a); note_launch();
  } else {
    cudaFuncSetAttribute(attn_bf16_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, ATTN_SMEM);
    launch_dep(attn_bf16_kernel<1>, grid, dim3(ATT_THREADS), ATTN_SMEM, s, a); note_launch();
  }
  return cudaGetLastError() == cudaSuccess ? 0 : STCA_ERR_CUDA;
}

int attention_f32(const AttnArgs& a, cudaStream_t s) {
  if (a.B == 0 || a.T == 0) return 0;
  const int dh = a.d / a.H;
  dim3 grid(a.B * a.splits, a.H);
switch (dh) {
    case 32:
      if (a.score == 0) attn_f32_kernel<1, 0><<<grid, 128, 0, s>>>(a);
      else attn_f32_kernel<1, 1><<<grid, 128, 0, s>>>(a);
      break;
    case 64:
      if (a.score == 0) attn_f32_kernel<2, 0><<<grid, 128, 0, s>>>(a);
      else attn_f32_kernel<2, 1><<<grid, 128, 0, s>>>(a);
      break;
    case 128:
      if (a.score == 0) attn_f32_kernel<4, 0><<<grid, 128, 0, s>>>(a);
      else attn_f32_kernel<4, 1><<<grid, 128, 0, s>>>(a);
      break;
    default:
      return STCA_ERR_UNSUPPORTED;
  }
  note_launch();
  return cudaGetLastError() == cudaSuccess ? 0 : STCA_ERR_CUDA;
}

int attention_merge(const AttnArgs& a, cudaStream_t s) {
  if (a.T == 0) return 0;
  if (a.splits < 1 || a.splits > 32) return STCA_ERR_INVALID_ARG;  // one lane per slice
  const int64_t warps = int64_t(a.T) * a.H;
  const int blocks = int((warps * 32 + 255) / 256);
  if (a.score == 0) launch_dep(attn_merge_kernel<0>, dim3(blocks), dim3(256), 0, s, a);
  else launch_dep(attn_merge_kernel<1>, dim3(blocks), dim3(256), 0, s, a);
  note_launch();
  return cudaGetLastError() == cudaSuccess ? 0 : STCA_ERR_CUDA;
}

}  // namespace stca
