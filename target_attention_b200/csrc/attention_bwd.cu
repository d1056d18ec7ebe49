// Backward of the split-L few-query cross attention (training).
//
// The pages train STCA on histories of about 2K items and serve 10K (STCA notes,
// "短序列训练，长序列推理"; review, architecture branch (C) "Extrapolation Aware
// Training"); training needs the gradient of the attention step.  For one user u, one
// head h and one slice of u's keys (one K/V row per history token), with the forward's
// output O and its log-sum-exp lse per (target, head), scores s_tj = c q_t . k_j and
// c = 1/sqrt(d_h):
//   softmax: p_tj = exp(s_tj - lse_t),  D_t = dO_t . O_t,  ds_tj = p_tj (dO_t . v_j - D_t)
//   relu:    p_tj = relu(s_tj),                            ds_tj = (dO_t . v_j) [s_tj > 0]
//   dV_j = sum_t p_tj dO_t,   dK_j = c sum_t ds_tj q_t,   dQ_t = c sum_j ds_tj k_j
// The sums over t run over all of u's targets inside one CTA (the request-level batching
// of the forward: a key's gradient collects every target that attended to it), so dK and
// dV of a key are complete when its slice is done.  The final lse makes each slice's p
// exact on its own (WeChat TA article §1.1: local attention over slices, then a merge),
// so a slice contributes a partial dQ over its keys; the partials are added by a second
// kernel (one slice writes dQ directly).
//
// A CTA of 4 warps serves one (user, slice, head).  Queries go in chunks of 16: Q (scaled
// by c), the scores' query operand (formed as the forward forms it) and dO of the chunk
// sit in shared memory as bf16 tiles.  Each warp streams its own
// 16-key tiles (keys w, w + 4, ... of the slice) through a 3-stage cp.async ring and, with
// the keys as the MMA row dimension (mma.sync m16n8k16, fp32 accumulation):
//   S^T = K Q^T, dP^T = V dO^T   ->  P^T, dS^T in registers
//   dV = P^T dO,  dK = dS^T Q     ->  stored per key (added across query chunks)
//   dQ += dS K                    (dS^T transposed through a small shared tile)
// and the 4 warps' dQ are added in shared memory at the end of a chunk.
#include "common.cuh"
#include "internal.h"

namespace stca {

namespace {

constexpr float B_LOG2E = 1.4426950408889634f;
constexpr int BD = 64;                         // d_h
constexpr int BKT = 16;                        // keys per warp tile
constexpr int BQ = 16;                         // queries per chunk
constexpr int BW = 4;                          // warps per CTA
constexpr int B_THREADS = BW * 32;
constexpr int BSTAGES = 3;                     // key tiles per warp ring
constexpr int BTILE = BKT * BD * 2;            // 2 KB: K or V of one key tile
constexpr int BSTAGE = 2 * BTILE;              // K | V
constexpr int BRING = BW * BSTAGES * BSTAGE;   // 48 KB
constexpr int BQBYTES = BQ * BD * 2;           // one [16 x 64] bf16 chunk of Q or dO
constexpr int BDS = BKT * BQ * 2;              // dS^T staging of one warp: [16 keys][16 queries] bf16
constexpr int OFF_Q = BRING;
constexpr int OFF_DO = OFF_Q + BQBYTES;
constexpr int OFF_DS = OFF_DO + BQBYTES;
constexpr int OFF_D = OFF_DS + BW * BDS;
constexpr int OFF_L = OFF_D + BQ * 4;
constexpr int OFF_Q2 = OFF_L + BQ * 4;          // the scores' own query tile (see the fill below)
constexpr int BWD_SMEM = OFF_Q2 + BQBYTES;
static_assert(BW * BQ * BD * 4 <= BRING, "the dQ combine reuses the ring");

// Byte offset of 16-byte chunk ch (0..7) of row r in a tile of 128-byte rows (64 bf16),
// XOR-swizzled so that the 8 rows an ldmatrix reads fall in different banks.
__device__ __forceinline__ int sw128(int r, int ch) { return r * 128 + ((ch ^ (r & 7)) << 4); }

struct BwdArgs {
  const float* Q;     // [T, d] projected queries (unscaled)
  const bf16* KV;     // [N, H, 2 d_h]: [K_h | V_h] per head
  const int32_t* hoff;
  const int32_t* toff;
  const float* O;     // [T, d] forward output
  const float* lse;   // [T, H] softmax log-sum-exp (natural log)
  const float* dO;    // [T, d]
  float* dQ;          // [T, d]
  float* dKV;         // [N, H, 2 d_h] fp32: [dK_h | dV_h] per head (with dKV16: partial sums only)
  bf16* dKV16;        // [N, H, 2 d_h] bf16 result, or null
  float* part_dq;     // [splits, T, d] when splits > 1
  int B, T, d, H, splits;
};

template <int SCORE>
__global__ void __launch_bounds__(B_THREADS, 4) attn_bwd_kernel(BwdArgs a) {
  griddep_wait();
  griddep_launch();
  extern __shared__ __align__(128) uint8_t smem[];
  const int u = blockIdx.x / a.splits, s = blockIdx.x % a.splits, h = blockIdx.y;
  const int hbeg = a.hoff[u];
  const int64_t L = a.hoff[u + 1] - hbeg;
  const int64_t k0 = hbeg + (L * s) / a.splits;
  const int nk = int(hbeg + (L * (s + 1)) / a.splits - k0);
  const int t0 = a.toff[u], m = a.toff[u + 1] - t0;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, tq = lane & 3;
  const int d = a.d;
  const int64_t ld = 2 * int64_t(d);
  const int qcol = h * BD, kvcol = 2 * h * BD;
  if (m <= 0) {  // no target attends to these keys: zero gradients
    for (int64_t i = threadIdx.x; i < int64_t(nk) * (2 * BD / 4); i += B_THREADS) {
      const int64_t key = k0 + i / (2 * BD / 4);
      if (a.dKV16)
        reinterpret_cast<uint2*>(a.dKV16 + key * ld + kvcol)[i % (2 * BD / 4)] = make_uint2(0u, 0u);
      else
        reinterpret_cast<float4*>(a.dKV + key * ld + kvcol)[i % (2 * BD / 4)] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    return;
  }
  const float c = rsqrtf(float(BD));
  const int n_tiles = (nk + BKT - 1) / BKT;
  const int n_local = n_tiles > warp ? (n_tiles - warp + BW - 1) / BW : 0;
  uint8_t* ring = smem + warp * BSTAGES * BSTAGE;
  const uint32_t sQ = smem_u32(smem + OFF_Q), sO = smem_u32(smem + OFF_DO), sQ2 = smem_u32(smem + OFF_Q2);
  uint8_t* dS_tile = smem + OFF_DS + warp * BDS;
  float* Ds = reinterpret_cast<float*>(smem + OFF_D);
  float* Ls = reinterpret_cast<float*>(smem + OFF_L);

  // copies of local tile j into ring stage st: lane l moves 16-byte chunk l % 16 of the
  // 256-byte [K_h | V_h] segment of keys l / 16 + 2 i (keys past the slice zero-filled)
  auto load_tile = [&](int j, int st) {
    if (j >= n_local) return;
    const int tl = warp + BW * j;
    const int valid = min(BKT, nk - tl * BKT);
    uint8_t* sK = ring + st * BSTAGE;
    const int ch = lane & 15;
    uint8_t* dst0 = sK + (ch < 8 ? 0 : BTILE);
#pragma unroll
    for (int i = 0; i < BKT / 2; ++i) {
      const int key = (lane >> 4) + 2 * i;
      const bool ok = key < valid;
      const bf16* src = a.KV + (k0 + int64_t(tl) * BKT + (ok ? key : 0)) * ld + kvcol + ch * 8;
      cp_async_16(dst0 + sw128(key, ch & 7), src, ok ? 16u : 0u);
    }
  };

  for (int qp = 0; qp < m; qp += BQ) {
    const int mq = min(BQ, m - qp);
    __syncthreads();  // the previous chunk is done with every shared buffer
    // ---- Q and dO of the chunk as bf16 tiles; D = dO . O; lse in log2 units.  The scores
    // are recomputed exactly as the forward formed them, so that the forward's lse
    // normalises these weights (softmax) and the mask [s > 0] is the forward's (ReLU): Q2
    // holds bf16(q c log2e) for the softmax (the forward's query operand), and for the ReLU
    // the low terms bf16(q c - bf16(q c)) that the forward adds to Q = bf16(q c).  dK takes Q.
    const float qs2 = B_LOG2E * c;
    for (int i = threadIdx.x; i < BQ * 8; i += B_THREADS) {
      const int r = i >> 3, ch = i & 7;
      uint4 qv = make_uint4(0, 0, 0, 0), ov = qv, q2 = qv;
      if (r < mq) {
        const int64_t off = int64_t(t0 + qp + r) * d + qcol + ch * 8;
        const float4 q0 = *reinterpret_cast<const float4*>(a.Q + off);
        const float4 q1 = *reinterpret_cast<const float4*>(a.Q + off + 4);
        const float4 o0 = *reinterpret_cast<const float4*>(a.dO + off);
        const float4 o1 = *reinterpret_cast<const float4*>(a.dO + off + 4);
        const float x[8] = {q0.x * c, q0.y * c, q0.z * c, q0.w * c, q1.x * c, q1.y * c, q1.z * c, q1.w * c};
        qv = make_uint4(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]), pack_bf16x2(x[4], x[5]),
                        pack_bf16x2(x[6], x[7]));
        if (SCORE == 0) {
          const float y[8] = {q0.x * qs2, q0.y * qs2, q0.z * qs2, q0.w * qs2,
                              q1.x * qs2, q1.y * qs2, q1.z * qs2, q1.w * qs2};
          q2 = make_uint4(pack_bf16x2(y[0], y[1]), pack_bf16x2(y[2], y[3]), pack_bf16x2(y[4], y[5]),
                          pack_bf16x2(y[6], y[7]));
        } else {
          const uint32_t hw[4] = {qv.x, qv.y, qv.z, qv.w};
          uint32_t lw[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float2 hf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&hw[k]));
            lw[k] = pack_bf16x2(x[2 * k] - hf.x, x[2 * k + 1] - hf.y);
          }
          q2 = make_uint4(lw[0], lw[1], lw[2], lw[3]);
        }
        ov = make_uint4(pack_bf16x2(o0.x, o0.y), pack_bf16x2(o0.z, o0.w), pack_bf16x2(o1.x, o1.y),
                        pack_bf16x2(o1.z, o1.w));
      }
      *reinterpret_cast<uint4*>(smem + OFF_Q + sw128(r, ch)) = qv;
      *reinterpret_cast<uint4*>(smem + OFF_Q2 + sw128(r, ch)) = q2;
      *reinterpret_cast<uint4*>(smem + OFF_DO + sw128(r, ch)) = ov;
    }
    for (int r = warp; r < BQ; r += BW) {
      float dsum = 0.f;
      if (r < mq) {
        const int64_t off = int64_t(t0 + qp + r) * d + qcol;
        // dO rounded to bf16 as the dP^T MMA sees it: with D and dP from the same dO, ds is
        // the softmax Jacobian applied to that dO.  (With fp32 dO here and bf16 dO in dP the
        // rounding error times the values' common offset no longer cancels in dp - D.)
        const float g0 = __bfloat162float(__float2bfloat16_rn(a.dO[off + lane]));
        const float g1 = __bfloat162float(__float2bfloat16_rn(a.dO[off + lane + 32]));
        dsum = g0 * a.O[off + lane] + g1 * a.O[off + lane + 32];
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) dsum += __shfl_xor_sync(0xffffffffu, dsum, o);
      if (lane == 0) {
        Ds[r] = dsum;
        // a query past the chunk gets lse = +inf, so its weights are exactly 0
        Ls[r] = r < mq ? (SCORE == 0 ? a.lse[int64_t(t0 + qp + r) * a.H + h] * B_LOG2E : 0.f) : INFINITY;
      }
    }
    __syncthreads();
    // this lane's four query columns of the C fragments: nt * 8 + 2 tq + e
    float lse2[4], Dq[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int q = (i >> 1) * 8 + 2 * tq + (i & 1);
      lse2[i] = Ls[q];
      Dq[i] = Ds[q];
    }

    float dq[8][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) dq[nt][e] = 0.f;

#pragma unroll
    for (int p = 0; p < BSTAGES - 1; ++p) {
      load_tile(p, p);
      cp_async_commit();
    }
    int st = 0;
    for (int j = 0; j < n_local; ++j) {
      cp_async_wait<BSTAGES - 2>();
      __syncwarp();  // every lane's copies of tile j landed; every lane is done with tile j - 1
      {
        int sn = st + BSTAGES - 1;
        sn = sn >= BSTAGES ? sn - BSTAGES : sn;
        load_tile(j + BSTAGES - 1, sn);
        cp_async_commit();
      }
      const uint32_t sK = smem_u32(ring + st * BSTAGE), sV = sK + BTILE;
      const int tl = warp + BW * j;
      const int valid = min(BKT, nk - tl * BKT);
      // ---- S^T = K Q^T and dP^T = V dO^T  ([16 keys x 16 queries], k = d_h)
      float sT[2][4], dpT[2][4];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) sT[nt][e] = dpT[nt][e] = 0.f;
      const int ar = (lane & 7) + ((lane >> 3) & 1) * 8;  // A: rows (keys) of matrix lane / 8
      const int br = (lane & 7) + (lane >> 4) * 8;        // B: rows (queries) of matrix lane / 8
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        uint32_t ka[4], va[4], qb[4], ob[4];
        ldsm_x4(sK + sw128(ar, 2 * kk + (lane >> 4)), ka);
        ldsm_x4(sV + sw128(ar, 2 * kk + (lane >> 4)), va);
        ldsm_x4(sQ2 + sw128(br, 2 * kk + ((lane >> 3) & 1)), qb);
        ldsm_x4(sO + sw128(br, 2 * kk + ((lane >> 3) & 1)), ob);
        mma_bf16_16816(sT[0], ka, qb[0], qb[1]);
        mma_bf16_16816(sT[1], ka, qb[2], qb[3]);
        if (SCORE == 1) {  // + the high terms: s = K (Q + Q2)
          ldsm_x4(sQ + sw128(br, 2 * kk + ((lane >> 3) & 1)), qb);
          mma_bf16_16816(sT[0], ka, qb[0], qb[1]);
          mma_bf16_16816(sT[1], ka, qb[2], qb[3]);
        }
        mma_bf16_16816(dpT[0], va, ob[0], ob[1]);
        mma_bf16_16816(dpT[1], va, ob[2], ob[3]);
      }
      // ---- P^T and dS^T (C fragments: row key g + 8 (e >> 1), column query 8 nt + 2 tq + (e & 1))
      float pT[2][4], dsT[2][4];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const bool kok = g + (e >> 1) * 8 < valid;
          const int qi = nt * 2 + (e & 1);
          if (SCORE == 0) {
            const float p = kok ? exp2_approx(sT[nt][e] - lse2[qi]) : 0.f;  // scores in log2 units
            pT[nt][e] = p;
            dsT[nt][e] = p * (dpT[nt][e] - Dq[qi]);
          } else {
            const bool pos = kok && sT[nt][e] > 0.f;
            pT[nt][e] = pos ? sT[nt][e] : 0.f;
            dsT[nt][e] = pos ? dpT[nt][e] : 0.f;
          }
        }
      uint32_t pa[4], da[4];  // as A operands (rows keys, k queries)
      pa[0] = pack_bf16x2(pT[0][0], pT[0][1]);
      pa[1] = pack_bf16x2(pT[0][2], pT[0][3]);
      pa[2] = pack_bf16x2(pT[1][0], pT[1][1]);
      pa[3] = pack_bf16x2(pT[1][2], pT[1][3]);
      da[0] = pack_bf16x2(dsT[0][0], dsT[0][1]);
      da[1] = pack_bf16x2(dsT[0][2], dsT[0][3]);
      da[2] = pack_bf16x2(dsT[1][0], dsT[1][1]);
      da[3] = pack_bf16x2(dsT[1][2], dsT[1][3]);
      // dS^T into the warp's staging tile (row = key, 32 bytes = 16 queries)
      *reinterpret_cast<uint32_t*>(dS_tile + g * 32 + (2 * tq) * 2) = da[0];
      *reinterpret_cast<uint32_t*>(dS_tile + (g + 8) * 32 + (2 * tq) * 2) = da[1];
      *reinterpret_cast<uint32_t*>(dS_tile + g * 32 + (8 + 2 * tq) * 2) = da[2];
      *reinterpret_cast<uint32_t*>(dS_tile + (g + 8) * 32 + (8 + 2 * tq) * 2) = da[3];

      // ---- dV = P^T dO and dK = dS^T Q ([16 keys x 64], k = 16 queries): B from the
      // [query][d_h] tiles, transposed by ldmatrix
      const int64_t row0 = k0 + int64_t(tl) * BKT;
      const int vr = (lane & 7) + ((lane >> 3) & 1) * 8;  // rows (queries, or keys below) of matrix lane / 8
#pragma unroll
      for (int which = 0; which < 2; ++which) {  // 0: dK (dS^T Q), 1: dV (P^T dO)
        float acc[8][4];
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[nt][e] = 0.f;
#pragma unroll
        for (int np = 0; np < 4; ++np) {
          uint32_t b[4];
          ldsm_x4_t((which ? sO : sQ) + sw128(vr, 2 * np + (lane >> 4)), b);
          mma_bf16_16816(acc[2 * np], which ? pa : da, b[0], b[1]);
          mma_bf16_16816(acc[2 * np + 1], which ? pa : da, b[2], b[3]);
        }
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) {
          const int key = g + 8 * hr;
          if (key < valid) {
            const int64_t off = (row0 + key) * ld + kvcol + which * BD + 2 * tq;
            float* dst = a.dKV + off;
            // the last query chunk writes the bf16 result when one is asked for; earlier
            // chunks keep fp32 partial sums
            const bool to16 = a.dKV16 && qp + BQ >= m;
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
              float2 v = make_float2(acc[nt][2 * hr], acc[nt][2 * hr + 1]);
              if (qp > 0) {  // later query chunks add to the earlier chunks' sums
                const float2 prev = *reinterpret_cast<const float2*>(dst + nt * 8);
                v.x += prev.x;
                v.y += prev.y;
              }
              if (to16)
                *reinterpret_cast<uint32_t*>(a.dKV16 + off + nt * 8) = pack_bf16x2(v.x, v.y);
              else
                *reinterpret_cast<float2*>(dst + nt * 8) = v;
            }
          }
        }
      }

      // ---- dQ += dS K ([16 queries x 64], k = 16 keys): A = dS from the staging tile
      // (transposed by ldmatrix), B = K [key][d_h] transposed by ldmatrix
      __syncwarp();
      uint32_t dsa[4];
      {
        const int mi = lane >> 3;
        ldsm_x4_t(smem_u32(dS_tile) + ((lane & 7) + (mi >> 1) * 8) * 32 + (mi & 1) * 16, dsa);
      }
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        uint32_t kb[4];
        ldsm_x4_t(sK + sw128(vr, 2 * np + (lane >> 4)), kb);
        mma_bf16_16816(dq[2 * np], dsa, kb[0], kb[1]);
        mma_bf16_16816(dq[2 * np + 1], dsa, kb[2], kb[3]);
      }
      st = st + 1 == BSTAGES ? 0 : st + 1;
    }
    cp_async_wait_all();

    // ---- the 4 warps' dQ added in shared memory (reusing the ring), scaled by c
    __syncthreads();
    float* comb = reinterpret_cast<float*>(smem);  // [BW][16][64]
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int hr = 0; hr < 2; ++hr) {
        float* p = comb + (warp * BQ + g + 8 * hr) * BD + nt * 8 + 2 * tq;
        *reinterpret_cast<float2*>(p) = make_float2(dq[nt][2 * hr], dq[nt][2 * hr + 1]);
      }
    __syncthreads();
    float* dst = a.splits == 1 ? a.dQ : a.part_dq + int64_t(s) * a.T * d;
    for (int i = threadIdx.x; i < BQ * BD; i += B_THREADS) {
      const int r = i / BD, col = i % BD;
      if (r < mq) {
        float v = 0.f;
#pragma unroll
        for (int w = 0; w < BW; ++w) v += comb[(w * BQ + r) * BD + col];
        dst[int64_t(t0 + qp + r) * d + qcol + col] = v * c;
      }
    }
  }
}

__global__ void sum_splits_kernel(const float* __restrict__ part, int splits, int64_t n, float* __restrict__ out) {
  griddep_wait();
  griddep_launch();
  const int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n) return;
  float v = 0.f;
  for (int s = 0; s < splits; ++s) v += part[int64_t(s) * n + i];
  out[i] = v;
}

}  // namespace

int attention_bwd_bf16(const float* Q, const void* KV, const int32_t* hoff, const int32_t* toff, int B, int T, int d,
                       int H, int splits, int score, const float* O, const float* lse, const float* dO, float* dQ,
                       float* dKV, float* part_dq, void* dKV16, cudaStream_t s) {
  if (B == 0) return 0;
  if (d % H != 0 || d / H != BD) return STCA_ERR_UNSUPPORTED;
  BwdArgs a;
  a.Q = Q;
  a.KV = reinterpret_cast<const bf16*>(KV);
  a.hoff = hoff;
  a.toff = toff;
  a.O = O;
  a.lse = lse;
  a.dO = dO;
  a.dQ = dQ;
  a.dKV = dKV;
  a.dKV16 = reinterpret_cast<bf16*>(dKV16);
  a.part_dq = part_dq;
  a.B = B;
  a.T = T;
  a.d = d;
  a.H = H;
  a.splits = splits;
  const dim3 grid(B * splits, H);
  if (score == 0) {
    cudaFuncSetAttribute(attn_bwd_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, BWD_SMEM);
    launch_dep(attn_bwd_kernel<0>, grid, dim3(B_THREADS), BWD_SMEM, s, a);
  } else {
    cudaFuncSetAttribute(attn_bwd_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, BWD_SMEM);
    launch_dep(attn_bwd_kernel<1>, grid, dim3(B_THREADS), BWD_SMEM, s, a);
  }
  note_launch();
  if (cudaGetLastError() != cudaSuccess) return STCA_ERR_CUDA;
  if (splits > 1 && T > 0) {
    const int64_t n = int64_t(T) * d;
    launch_dep(sum_splits_kernel, dim3(unsigned((n + 255) / 256)), dim3(256), 0, s, part_dq, splits, n, dQ);
    note_launch();
    if (cudaGetLastError() != cudaSuccess) return STCA_ERR_CUDA;
  }
  return 0;
}

}  // namespace stca

// ------------------------------------------------------------------------------------
// C entry points of the training step (include/stca.h)

namespace {
int train_args_ok(const float* Q, const void* KV, const int32_t* hoff, const int32_t* toff, int B, int T, int d,
                  int H, int splits, int score) {
  if (B < 0 || T < 0 || d <= 0 || H <= 0 || d % H != 0 || splits < 1 || splits > 32 || (score != 0 && score != 1))
    return STCA_ERR_INVALID_ARG;
  if (B > 0 && (!hoff || !toff || (T > 0 && (!Q || !KV)))) return STCA_ERR_INVALID_ARG;
  if (d / H != 64 || d % 8 != 0) return STCA_ERR_UNSUPPORTED;
  return STCA_OK;
}
}  // namespace

extern "C" int stca_attention_train_forward(const float* Q, const void* KV, const int32_t* hoff,
                                            const int32_t* toff, int B, int T, int d, int H, int splits, int score,
                                            float* part_acc, float* part_ml, float* out, float* lse, int32_t* err,
                                            void* stream) {
  int rc = train_args_ok(Q, KV, hoff, toff, B, T, d, H, splits, score);
  if (rc != STCA_OK) return rc;
  if (B == 0 || T == 0) return STCA_OK;
  if (!out || (score == 0 && !lse) || (splits > 1 && (!part_acc || (score == 0 && !part_ml))))
    return STCA_ERR_INVALID_ARG;
  stca::AttnArgs a;
  a.Q = Q;
  a.KV = KV;
  a.hoff = hoff;
  a.toff = toff;
  a.kv_rows = nullptr;
  a.kv_len = nullptr;
  a.kv_mult = nullptr;
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
  a.lse_out = score == 0 ? lse : nullptr;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  rc = stca::attention_bf16(a, s);
  if (rc != STCA_OK) return rc;
  return stca::attention_needs_merge(a, true) ? stca::attention_merge(a, s) : STCA_OK;
}

extern "C" int stca_attention_backward(const float* Q, const void* KV, const int32_t* hoff, const int32_t* toff,
                                       int B, int T, int d, int H, int splits, int score, const float* out,
                                       const float* lse, const float* dout, float* dQ, float* dKV, float* part_dq,
                                       void* dkv_bf16, void* stream) {
  int rc = train_args_ok(Q, KV, hoff, toff, B, T, d, H, splits, score);
  if (rc != STCA_OK) return rc;
  if (B == 0) return STCA_OK;
  if (!dKV || (T > 0 && (!dout || !dQ || (score == 0 && (!out || !lse)))) || (splits > 1 && T > 0 && !part_dq) ||
      (reinterpret_cast<uintptr_t>(dkv_bf16) & 15))
    return STCA_ERR_INVALID_ARG;
  return stca::attention_bwd_bf16(Q, KV, hoff, toff, B, T, d, H, splits, score, out, lse, dout, dQ, dKV, part_dq,
                                  dkv_bf16, reinterpret_cast<cudaStream_t>(stream));
}

