// Attention with W_K and W_V folded into the queries (d = 256, d_h = 64).
//
// The review's core formula scores target query q_h against k_j = x~_j W_K,h and averages
// v_j = x~_j W_V,h.  By associativity
//   s_j = q_h . (x~_j W_K,h) = (q_h W_K,h^T) . x~_j = q~_h . x~_j
//   o_h = sum_j a_j x~_j W_V,h = (sum_j a_j x~_j) W_V,h = r_h W_V,h
// so the K/V projection of every history row can be skipped: the queries are folded once
// (q~ = Q_h W_K,h^T, a small target-side GEMM) and the weighted sum r_h of the d-wide rows
// x~_j is projected afterwards (another small GEMM).  x~_j itself is never formed either:
// the history FFN stores y'_j = y_j * gamma and the row moments (mean_j, rstd_j) of its
// LayerNorm, and x~_j = rstd_j (y'_j - mean_j gamma) + beta, so
//   s_j = rstd_j (q~ . y'_j - mean_j (q~ . gamma)) + q~ . beta
//   sum_j p_j x~_j = R1 - R2 gamma + (sum_j p_j) beta,
//   R1 = sum_j p_j rstd_j y'_j,  R2 = sum_j p_j rstd_j mean_j.
// Every (target, head) becomes one row of a [m H, d] query block per user; rows and keys go
// through mma.sync m16n8k16 tiles.  Softmax scores are kept in log2 units; the ReLU form uses
// relu(s_j); compacted keys weigh by their token counts, and a key past the slice gets count
// 0 (so no mask is needed).
//
// One CTA of 4 warps per (user, L-slice), 32 query rows per chunk.  Per 32-key tile (a
// 3-stage cp.async ring of y' rows and their moments): warp w scores keys 8w .. 8w + 7 of
// every row (K = d), the 4 warps agree on each row's running maximum through shared memory,
// write P' = p rstd as bf16, and then warp w accumulates R1 for output columns
// 64 w .. 64 w + 63 over all 32 keys.
#include "common.cuh"
#include "internal.h"

namespace stca {

namespace {

constexpr float F_LOG2E = 1.4426950408889634f;
constexpr int FD = 256;                 // d
constexpr int FDH = 64;                 // d_h
constexpr int FW = 4;                   // warps
constexpr int F_THREADS = 32 * FW;
constexpr int FR = 32;                  // query rows per chunk
constexpr int FKT = 32;                 // keys per tile
constexpr int FSTAGES = 3;
constexpr int FROW = FD * 2;            // 512-byte rows (bf16)
constexpr int F_Q = FR * FROW;          // 16 KB
constexpr int F_TILE = FKT * FROW;      // 16 KB
constexpr int F_META = FKT * 16;        // per key: mean, rstd, count (int), pad
constexpr int F_P = FR * FKT * 2;       // P' [32 rows x 32 keys] bf16, 64-byte rows
constexpr int OFF_RING = F_Q;
constexpr int OFF_META = OFF_RING + FSTAGES * F_TILE;
constexpr int OFF_P = OFF_META + FSTAGES * F_META;
constexpr int OFF_RED = OFF_P + F_P;    // [FW][FR] floats x 3 (max, sum, R2)
constexpr int OFF_CB = OFF_RED + 3 * FW * FR * 4;  // [FR] x 2 (q~ . gamma, q~ . beta)
constexpr int OFF_QLO = OFF_CB + 2 * FR * 4;       // ReLU: the low bf16 terms of q~
// The ReLU form's output is not normalised, so its score errors do not cancel: there q~ is
// carried as two bf16 terms hi + lo (hi = bf16(q~), lo = bf16(q~ - hi)), two MMAs per K
// step, which keeps the scores at fp32 accuracy (one bf16 rounding of the 256-wide q~ alone
// gave about 1e-2 of relative error at the output).  The softmax form stays at one term.
template <int SCORE>
constexpr int fold_smem() { return OFF_QLO + (SCORE == 1 ? F_Q : 0); }

// 16-byte chunk c (0..31) of row r of a tile with 512-byte rows, XOR-swizzled within
// each group of 8 chunks so the 8 rows an ldmatrix reads fall in different banks.
__device__ __forceinline__ int sw512(int r, int c) { return r * FROW + (((c & ~7) | ((c ^ r) & 7)) << 4); }
// chunk c (0..3) of row r of the 64-byte-row P' tile
__device__ __forceinline__ int sw64(int r, int c) { return r * 64 + ((c ^ ((r >> 1) & 3)) << 4); }

__device__ __forceinline__ void cp_async_8(void* smem_dst, const void* gsrc, uint32_t src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8, %2;" ::"r"(smem_u32(smem_dst)), "l"(gsrc), "r"(src_bytes)
               : "memory");
}

template <int SCORE>
__global__ void __launch_bounds__(F_THREADS, SCORE == 1 ? 2 : 3) attn_fold_kernel(FoldArgs a) {
  constexpr bool SPLIT = SCORE == 1;
  griddep_wait();
  griddep_launch();
  extern __shared__ __align__(128) uint8_t smem[];
  const int u = blockIdx.x / a.splits, s = blockIdx.x % a.splits;
  const int hbeg = a.hoff[u];
  const int64_t L = a.kv_len ? a.kv_len[u] : a.hoff[u + 1] - hbeg;
  const int64_t k0 = hbeg + (L * s) / a.splits;
  const int nk = int(hbeg + (L * (s + 1)) / a.splits - k0);
  const int t0 = a.toff[u], m = a.toff[u + 1] - t0;
  if (m <= 0) return;
  const int H = a.H, rows = m * H;  // this user's query rows: (t - t0) H + h
  const int64_t row0 = int64_t(t0) * H;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, tq = lane & 3;
  const float qscale = (SCORE == 0 ? F_LOG2E : 1.0f) * rsqrtf(float(FDH));
  const int n_tiles = (nk + FKT - 1) / FKT;
  float* red_max = reinterpret_cast<float*>(smem + OFF_RED);
  float* red_sum = red_max + FW * FR;
  float* red_r2 = red_sum + FW * FR;
  float* s_c = reinterpret_cast<float*>(smem + OFF_CB);
  float* s_b = s_c + FR;
  const uint32_t sQ = smem_u32(smem), sP = smem_u32(smem + OFF_P), sQlo = smem_u32(smem + OFF_QLO);
  const bf16* Yb = reinterpret_cast<const bf16*>(a.Y);

  // warp w copies keys w + 4 i (i < 8) of a tile: one 512-byte row per warp instruction;
  // lanes 0..7 also copy key w + 4 lane's moments and count
  auto key_row = [&](int tile, int i, int& valid) -> int64_t {
    const int key = tile * FKT + warp + 4 * i;
    valid = key < nk;
    return valid ? (a.kv_rows ? int64_t(a.kv_rows[k0 + key]) : k0 + key) : 0;
  };
  auto issue = [&](int tile, int64_t myrow, int myvalid) {
    if (tile >= n_tiles) return;
    const int st = tile % FSTAGES;
    uint8_t* ring = smem + OFF_RING + st * F_TILE;
    uint8_t* meta = smem + OFF_META + st * F_META;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int64_t r = __shfl_sync(0xffffffffu, myrow, i);
      const int v = __shfl_sync(0xffffffffu, myvalid, i);
      const int key = warp + 4 * i;
      cp_async_16(ring + sw512(key, lane), Yb + r * FD + lane * 8, v ? 16u : 0u);
    }
    if (lane < 8) {
      const int key = warp + 4 * lane;
      uint8_t* mk = meta + key * 16;
      cp_async_8(mk, a.stats + 2 * myrow, myvalid ? 8u : 0u);
      if (a.kv_mult) cp_async_4(mk + 8, a.kv_mult + k0 + tile * FKT + key, myvalid ? 4u : 0u);
      else *reinterpret_cast<int*>(mk + 8) = myvalid ? 1 : 0;
    }
  };

  for (int qp = 0; qp < rows; qp += FR) {
    const int nr = min(FR, rows - qp);
    __syncthreads();  // the previous chunk is done with every buffer
    // ---- folded queries of the chunk as bf16 (scaled), and q~ . gamma, q~ . beta per row
    for (int i = threadIdx.x; i < FR * (FD / 8); i += F_THREADS) {
      const int r = i / (FD / 8), c = i % (FD / 8);
      uint4 v = make_uint4(0, 0, 0, 0), vlo = v;
      if (r < nr) {
        const float* src = a.Qf + (row0 + qp + r) * FD + c * 8;
        const float4 x0 = *reinterpret_cast<const float4*>(src), x1 = *reinterpret_cast<const float4*>(src + 4);
        const float x[8] = {x0.x * qscale, x0.y * qscale, x0.z * qscale, x0.w * qscale,
                            x1.x * qscale, x1.y * qscale, x1.z * qscale, x1.w * qscale};
        uint32_t hi[4], lo[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          hi[e] = pack_bf16x2(x[2 * e], x[2 * e + 1]);
          const __nv_bfloat162 hb = *reinterpret_cast<const __nv_bfloat162*>(&hi[e]);
          const float2 hf = __bfloat1622float2(hb);
          lo[e] = pack_bf16x2(x[2 * e] - hf.x, x[2 * e + 1] - hf.y);
        }
        v = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        vlo = make_uint4(lo[0], lo[1], lo[2], lo[3]);
      }
      *reinterpret_cast<uint4*>(smem + sw512(r, c)) = v;
      if (SPLIT) *reinterpret_cast<uint4*>(smem + OFF_QLO + sw512(r, c)) = vlo;
    }
    __syncthreads();
    for (int r = warp; r < FR; r += FW) {  // from the rounded queries the MMAs use
      float cg = 0.f, cb = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int col = lane * 8 + e;
        const __nv_bfloat16 qv = *reinterpret_cast<const __nv_bfloat16*>(smem + sw512(r, lane) + e * 2);
        float q = __bfloat162float(qv);
        if (SPLIT) q += __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(smem + OFF_QLO + sw512(r, lane) + e * 2));
        cg = fmaf(q, a.gamma[col], cg);
        cb = fmaf(q, a.beta[col], cb);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        cg += __shfl_xor_sync(0xffffffffu, cg, o);
        cb += __shfl_xor_sync(0xffffffffu, cb, o);
      }
      if (lane == 0) {
        s_c[r] = cg;
        s_b[r] = cb;
      }
    }
    // running state of this thread's four rows (16 mt + g + 8 hr), R1 of its columns
    float mrow[2][2], lsum[2][2], r2[2][2];
    float acc[2][8][4];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int hr = 0; hr < 2; ++hr) {
        mrow[mt][hr] = -INFINITY;
        lsum[mt][hr] = 0.f;
        r2[mt][hr] = 0.f;
      }
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[mt][nt][e] = 0.f;

    // ---- the key ring: tiles 0 and 1 in flight, rows of the tile after them prefetched
    int64_t myrow;
    int myvalid;
    myrow = key_row(0, lane & 7, myvalid);
    issue(0, myrow, myvalid);
    cp_async_commit();
    myrow = key_row(1, lane & 7, myvalid);
    issue(1, myrow, myvalid);
    cp_async_commit();
    myrow = key_row(2, lane & 7, myvalid);
    __syncthreads();  // s_c, s_b
    float cr[2][2], br[2][2];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int hr = 0; hr < 2; ++hr) {
        cr[mt][hr] = s_c[16 * mt + g + 8 * hr];
        br[mt][hr] = s_b[16 * mt + g + 8 * hr];
      }

    for (int j = 0; j < n_tiles; ++j) {
      cp_async_wait<1>();
      __syncthreads();  // every thread's copies of tile j landed; tile j - 1 is done
      issue(j + 2, myrow, myvalid);
      cp_async_commit();
      myrow = key_row(j + 3, lane & 7, myvalid);
      const int st = j % FSTAGES;
      const uint32_t sY = smem_u32(smem + OFF_RING + st * F_TILE);
      const float4* meta = reinterpret_cast<const float4*>(smem + OFF_META + st * F_META);
      // ---- S = Q~ Y'^T for keys 8 warp .. 8 warp + 7 (one n8 tile), K = d
      float sc[2][4];
#pragma unroll
      for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int e = 0; e < 4; ++e) sc[mt][e] = 0.f;
      const int ar = (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll 4
      for (int kk = 0; kk < FD / 16; kk += 2) {
        uint32_t b[4], a0[4], a1[4], a2[4], a3[4];
        ldsm_x4(sY + sw512(8 * warp + (lane & 7), 2 * kk + (lane >> 3)), b);
        ldsm_x4(sQ + sw512(ar, 2 * kk + (lane >> 4)), a0);
        ldsm_x4(sQ + sw512(16 + ar, 2 * kk + (lane >> 4)), a1);
        ldsm_x4(sQ + sw512(ar, 2 * kk + 2 + (lane >> 4)), a2);
        ldsm_x4(sQ + sw512(16 + ar, 2 * kk + 2 + (lane >> 4)), a3);
        mma_bf16_16816(sc[0], a0, b[0], b[1]);
        mma_bf16_16816(sc[1], a1, b[0], b[1]);
        mma_bf16_16816(sc[0], a2, b[2], b[3]);
        mma_bf16_16816(sc[1], a3, b[2], b[3]);
        if (SPLIT) {
          ldsm_x4(sQlo + sw512(ar, 2 * kk + (lane >> 4)), a0);
          ldsm_x4(sQlo + sw512(16 + ar, 2 * kk + (lane >> 4)), a1);
          ldsm_x4(sQlo + sw512(ar, 2 * kk + 2 + (lane >> 4)), a2);
          ldsm_x4(sQlo + sw512(16 + ar, 2 * kk + 2 + (lane >> 4)), a3);
          mma_bf16_16816(sc[0], a0, b[0], b[1]);
          mma_bf16_16816(sc[1], a1, b[0], b[1]);
          mma_bf16_16816(sc[0], a2, b[2], b[3]);
          mma_bf16_16816(sc[1], a3, b[2], b[3]);
        }
      }
      // ---- scores with the LayerNorm of the keys: s = rstd (S - mean c) + b
      float4 km[2];
      km[0] = meta[8 * warp + 2 * tq];
      km[1] = meta[8 * warp + 2 * tq + 1];
      float cnt[2] = {float(__float_as_int(km[0].z)), float(__float_as_int(km[1].z))};
#pragma unroll
      for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int hr = e >> 1, kq = e & 1;
          sc[mt][e] = fmaf(km[kq].y, sc[mt][e] - km[kq].x * cr[mt][hr], br[mt][hr]);
        }
      float pw[2][4];  // weights p (count included)
      if (SCORE == 0) {
        // each row's maximum over this warp's keys, then over the four warps
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
          for (int hr = 0; hr < 2; ++hr) {
            float mx = fmaxf(cnt[0] > 0.f ? sc[mt][2 * hr] : -INFINITY, cnt[1] > 0.f ? sc[mt][2 * hr + 1] : -INFINITY);
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
            if (tq == 0) red_max[warp * FR + 16 * mt + g + 8 * hr] = mx;
          }
        __syncthreads();
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
          for (int hr = 0; hr < 2; ++hr) {
            const int r = 16 * mt + g + 8 * hr;
            float tmax = red_max[r];
#pragma unroll
            for (int w = 1; w < FW; ++w) tmax = fmaxf(tmax, red_max[w * FR + r]);
            const float mnew = fmaxf(mrow[mt][hr], tmax);
            const float corr = (mnew == mrow[mt][hr]) ? 1.f : exp2_approx(mrow[mt][hr] - mnew);
            mrow[mt][hr] = mnew;
            lsum[mt][hr] *= corr;
            r2[mt][hr] *= corr;
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
              acc[mt][nt][2 * hr] *= corr;
              acc[mt][nt][2 * hr + 1] *= corr;
            }
            const float muse = mnew == -INFINITY ? 0.f : mnew;
#pragma unroll
            for (int kq = 0; kq < 2; ++kq) pw[mt][2 * hr + kq] = exp2_approx(sc[mt][2 * hr + kq] - muse) * cnt[kq];
          }
      } else {
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
          for (int e = 0; e < 4; ++e) pw[mt][e] = fmaxf(sc[mt][e], 0.f) * cnt[e & 1];
      }
      // ---- row sums, P' = p rstd into the shared tile
#pragma unroll
      for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) {
          const float p0 = pw[mt][2 * hr], p1 = pw[mt][2 * hr + 1];
          lsum[mt][hr] += p0 + p1;
          r2[mt][hr] += p0 * km[0].y * km[0].x + p1 * km[1].y * km[1].x;
          const int r = 16 * mt + g + 8 * hr;
          *reinterpret_cast<uint32_t*>(smem + OFF_P + sw64(r, warp) + tq * 4) =
              pack_bf16x2(p0 * km[0].y, p1 * km[1].y);
        }
      __syncthreads();  // P' complete
      // ---- R1 += P' Y' for columns 64 warp .. 64 warp + 63 (k = the tile's 32 keys)
#pragma unroll
      for (int kk = 0; kk < 2; ++kk) {
        uint32_t pa0[4], pa1[4];
        ldsm_x4(sP + sw64(ar, 2 * kk + (lane >> 4)), pa0);
        ldsm_x4(sP + sw64(16 + ar, 2 * kk + (lane >> 4)), pa1);
        const int key = 16 * kk + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
        for (int np = 0; np < 4; ++np) {
          uint32_t b[4];
          ldsm_x4_t(sY + sw512(key, 8 * warp + 2 * np + (lane >> 4)), b);
          mma_bf16_16816(acc[0][2 * np], pa0, b[0], b[1]);
          mma_bf16_16816(acc[0][2 * np + 1], pa0, b[2], b[3]);
          mma_bf16_16816(acc[1][2 * np], pa1, b[0], b[1]);
          mma_bf16_16816(acc[1][2 * np + 1], pa1, b[2], b[3]);
        }
      }
    }
    cp_async_wait_all();

    // ---- row totals over the 4 lanes of a quad and the 4 warps
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int hr = 0; hr < 2; ++hr) {
        float l = lsum[mt][hr], q2 = r2[mt][hr];
        l += __shfl_xor_sync(0xffffffffu, l, 1);
        l += __shfl_xor_sync(0xffffffffu, l, 2);
        q2 += __shfl_xor_sync(0xffffffffu, q2, 1);
        q2 += __shfl_xor_sync(0xffffffffu, q2, 2);
        if (tq == 0) {
          red_sum[warp * FR + 16 * mt + g + 8 * hr] = l;
          red_r2[warp * FR + 16 * mt + g + 8 * hr] = q2;
        }
      }
    __syncthreads();
    const bool direct = a.splits == 1 && !a.partial_out;
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int hr = 0; hr < 2; ++hr) {
        const int r = 16 * mt + g + 8 * hr;
        if (r >= nr) continue;
        float l = 0.f, q2 = 0.f;
#pragma unroll
        for (int w = 0; w < FW; ++w) {
          l += red_sum[w * FR + r];
          q2 += red_r2[w * FR + r];
        }
        // sum_j p_j x~_j = R1 - R2 gamma + (sum p) beta, normalised here when final
        const float scale = (SCORE == 0 && direct) ? (l > 0.f ? 1.f / l : 0.f) : 1.f;
        const int64_t orow = row0 + qp + r;
        float* dst = direct ? a.out + orow * FD : a.part_acc + (int64_t(s) * a.T * H + orow) * FD;
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
          const int col = 64 * warp + 8 * nt + 2 * tq;
          const float v0 = (acc[mt][nt][2 * hr] - q2 * a.gamma[col] + l * a.beta[col]) * scale;
          const float v1 = (acc[mt][nt][2 * hr + 1] - q2 * a.gamma[col + 1] + l * a.beta[col + 1]) * scale;
          *reinterpret_cast<float2*>(dst + col) = make_float2(v0, v1);
        }
        if (SCORE == 0 && !direct && warp == 0 && tq == 0) {
          float* pml = a.part_ml + (int64_t(s) * a.T * H + orow) * 2;
          pml[0] = mrow[mt][hr];
          pml[1] = l;
        }
      }
  }
}

}  // namespace

int attention_fold_bf16(const FoldArgs& a, cudaStream_t s) {
  if (a.B == 0 || a.T == 0) return 0;
  if (a.d != FD || a.d / a.H != FDH) return STCA_ERR_UNSUPPORTED;
  const dim3 grid(a.B * a.splits);
  if (a.score == 0) {
    cudaFuncSetAttribute(attn_fold_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, fold_smem<0>());
    launch_dep(attn_fold_kernel<0>, grid, dim3(F_THREADS), fold_smem<0>(), s, a);
  } else {
    cudaFuncSetAttribute(attn_fold_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, fold_smem<1>());
    launch_dep(attn_fold_kernel<1>, grid, dim3(F_THREADS), fold_smem<1>(), s, a);
  }
  note_launch();
  return cudaGetLastError() == cudaSuccess ? 0 : STCA_ERR_CUDA;
}

}  // namespace stca
