// Backward (training) steps of the history side of one STCA layer, X -> Xt = LN(SwiGLU(X))
// -> [K | V] = Xt [W_K | W_V] (STCA notes, section "STCA"; review §三 核心公式), given the
// gradients of K and V from the attention backward:
//   dXt = dKV [W_K | W_V]^T            (a plain GEMM, the library's tensor-core kernels)
//   dW_KV = Xt^T dKV                   gemm_wgrad: a reduction over the tokens
//   dy, dgamma, dbeta = LN backward    layer_norm_bwd (Xt recomputed on the way)
//   dA = dy W2^T,  dW2 = A^T dy        plain GEMM + gemm_wgrad
//   dP = SwiGLU backward of A = SiLU(P1) * P3     swiglu_bwd
//   dX = dP [W1 | W3]^T, [dW1 | dW3] = X^T dP     plain GEMM + gemm_wgrad
//   dE[ids], dT[bucket] += dX          table_rows_bwd (the lookup's backward)
// The pages train at about 2K-long histories (STCA notes, "短序列训练，长序列推理").
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace stca {

namespace {

// ------------------------------------------------------------------ weight gradients
// C [K, N] = A^T G over the M tokens: A [M, K] and G [M, N] bf16 row-major (tokens by
// features), C fp32.  A CTA computes a 128 x 128 tile of C over one slice of the tokens,
// accumulating in registers with mma.sync m16n8k16 (both operands come out of the
// token-major tiles through ldmatrix.trans); slices write their partial tiles to a
// workspace that a second kernel adds up in a fixed order, so the result does not depend
// on scheduling.  Tokens stream through a 3-stage cp.async ring of 64-token stages
// (16 KB of A and 16 KB of G, 256-byte rows with the 16-byte chunks XOR-swizzled by row).
constexpr int WG_T = 128;       // C tile (K and N)
constexpr int WG_TK = 64;       // tokens per stage
constexpr int WG_STAGES = 3;
constexpr int WG_TILE_BYTES = WG_TK * WG_T * 2;  // 16 KB
constexpr int WG_SMEM = WG_STAGES * 2 * WG_TILE_BYTES;  // 96 KB: two CTAs per SM

__device__ __forceinline__ uint32_t wg_off(int tok, int chunk) {  // byte offset in a tile
  return uint32_t(tok * 256 + ((chunk ^ (tok & 7)) << 4));
}

__global__ void __launch_bounds__(256, 2) gemm_wgrad_kernel(const bf16* __restrict__ A, int64_t lda,
                                                            const bf16* __restrict__ G, int64_t ldg, int M, int K,
                                                            int N, int splits, float* __restrict__ part) {
  griddep_wait();
  extern __shared__ __align__(128) uint8_t wg_smem[];
  const int n0 = blockIdx.x * WG_T, k0 = blockIdx.y * WG_T, sl = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int wm = warp >> 2, wn = warp & 3;  // warp tile: rows 64 wm .. +64 of C, columns 32 wn .. +32
  const int m_lo = int(int64_t(M) * sl / splits), m_hi = int(int64_t(M) * (sl + 1) / splits);
  const int n_st = (m_hi - m_lo + WG_TK - 1) / WG_TK;
  const uint32_t base = smem_u32(wg_smem);

  // stage s: A tile at base + s * 2 * TILE, G tile right after; thread t copies chunks
  // t, t + 256, ... of each (token = chunk / 16, 16-byte chunk = chunk % 16)
  auto load = [&](int st, int slot) {
    if (st >= n_st) return;
    const int t0 = m_lo + st * WG_TK;
    uint8_t* sa = wg_smem + slot * 2 * WG_TILE_BYTES;
    uint8_t* sg = sa + WG_TILE_BYTES;
#pragma unroll
    for (int i = 0; i < WG_TK * 16 / 256; ++i) {
      const int c = tid + 256 * i, tok = c >> 4, ch = c & 15;
      const int m = t0 + tok;
      const bool ok = m < m_hi;
      const int64_t row = ok ? m : m_lo;
      cp_async_16(sa + wg_off(tok, ch), A + row * lda + k0 + ch * 8, ok ? 16u : 0u);
      cp_async_16(sg + wg_off(tok, ch), G + row * ldg + n0 + ch * 8, ok ? 16u : 0u);
    }
  };

  float acc[4][4][4];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[a][b][e] = 0.f;

#pragma unroll
  for (int s = 0; s < WG_STAGES - 1; ++s) {
    load(s, s);
    cp_async_commit();
  }
  for (int st = 0; st < n_st; ++st) {
    cp_async_wait<WG_STAGES - 2>();
    __syncthreads();  // stage st landed for every thread; stage st - 1 is free again
    load(st + WG_STAGES - 1, (st + WG_STAGES - 1) % WG_STAGES);
    cp_async_commit();
    const uint32_t sa = base + (st % WG_STAGES) * 2 * WG_TILE_BYTES, sg = sa + WG_TILE_BYTES;
#pragma unroll
    for (int kk = 0; kk < WG_TK / 16; ++kk) {
      // A^T fragments (rows = features of A, k = tokens): matrix q of lane l is rows
      // tok = 16 kk + (l & 7) + 8 ((l >> 4) & 1), features f0 + 8 ((l >> 3) & 1)
      uint32_t af[4][4];
#pragma unroll
      for (int mt = 0; mt < 4; ++mt) {
        const int tok = 16 * kk + (lane & 7) + 8 * ((lane >> 4) & 1);
        const int f = 64 * wm + 16 * mt + 8 * ((lane >> 3) & 1);
        ldsm_x4_t(sa + wg_off(tok, f >> 3), af[mt]);
      }
      // G fragments (k = tokens, columns = features of G), two 8-column tiles per load
      uint32_t bf[4][2];
#pragma unroll
      for (int np = 0; np < 2; ++np) {
        const int tok = 16 * kk + (lane & 7) + 8 * ((lane >> 3) & 1);
        const int f = 32 * wn + 16 * np + 8 * (lane >> 4);
        uint32_t r[4];
        ldsm_x4_t(sg + wg_off(tok, f >> 3), r);
        bf[2 * np][0] = r[0];
        bf[2 * np][1] = r[1];
        bf[2 * np + 1][0] = r[2];
        bf[2 * np + 1][1] = r[3];
      }
#pragma unroll
      for (int mt = 0; mt < 4; ++mt)
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) mma_bf16_16816(acc[mt][nt], af[mt], bf[nt][0], bf[nt][1]);
    }
  }
  cp_async_wait_all();
  griddep_launch();
  // partial tile of this token slice: part[sl][K][N]
  float* out = part + int64_t(sl) * K * N;
  const int g = lane >> 2, tq = lane & 3;
#pragma unroll
  for (int mt = 0; mt < 4; ++mt)
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
      const int r = k0 + 64 * wm + 16 * mt + g, c = n0 + 32 * wn + 8 * nt + 2 * tq;
      *reinterpret_cast<float2*>(out + int64_t(r) * N + c) = make_float2(acc[mt][nt][0], acc[mt][nt][1]);
      *reinterpret_cast<float2*>(out + int64_t(r + 8) * N + c) = make_float2(acc[mt][nt][2], acc[mt][nt][3]);
    }
}

// C[k][n] (+)= sum over slices s in order of part[s][k][n]; four columns per thread
__global__ void wgrad_reduce_kernel(const float* __restrict__ part, int splits, int K, int N, float* __restrict__ C,
                                    int64_t ldc, int accumulate) {
  griddep_wait();
  const int64_t i = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) * 4;
  if (i >= int64_t(K) * N) return;
  const int r = int(i / N), c = int(i % N);
  float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int s = 0; s < splits; ++s) {
    const float4 p = *reinterpret_cast<const float4*>(part + int64_t(s) * K * N + i);
    v.x += p.x;
    v.y += p.y;
    v.z += p.z;
    v.w += p.w;
  }
  float4* dst = reinterpret_cast<float4*>(C + int64_t(r) * ldc + c);
  if (accumulate) {
    const float4 o = *dst;
    v.x += o.x;
    v.y += o.y;
    v.z += o.z;
    v.w += o.w;
  }
  *dst = v;
}

// token slices: enough CTAs for two per SM, each slice at least 256 tokens
int wgrad_splits(int M, int K, int N) {
  const int tiles = (K / WG_T) * (N / WG_T);
  const int by_sm = std::max(1, (2 * sm_count() + tiles - 1) / tiles);
  const int by_rows = std::max(1, M / 256);
  return std::min(by_sm, by_rows);
}

// ------------------------------------------------------------------ LayerNorm backward
// One warp per row (d = 32 DPL columns, lane l holds columns l + 32 i).  With
// xhat = (y - mean) rstd and g = dxt * gamma:
//   dy = rstd (g - mean(g) - xhat mean(g xhat)),  xt = xhat gamma + beta,
//   dgamma += dxt xhat,  dbeta += dxt  (over the rows; per block, then added in order).
__device__ __forceinline__ float ld_f(const bf16* p) { return __bfloat162float(*p); }
__device__ __forceinline__ float ld_f(const float* p) { return *p; }
__device__ __forceinline__ void st_f(bf16* p, float v) { *p = __float2bfloat16(v); }
__device__ __forceinline__ void st_f(float* p, float v) { *p = v; }

// rows of bf16 (the history side) or fp32 (the target side, which keeps fp32 activations)
template <int DPL, typename T>
__global__ void __launch_bounds__(256) ln_bwd_kernel(const T* __restrict__ y, const T* __restrict__ dxt, int M,
                                                     const float* __restrict__ gamma, const float* __restrict__ beta,
                                                     float eps, T* __restrict__ dy, T* __restrict__ xt,
                                                     float* __restrict__ part) {
  griddep_wait();
  constexpr int D = 32 * DPL;
  __shared__ float red[8][2][D];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float gm[DPL], bt[DPL], sg[DPL], sb[DPL];
#pragma unroll
  for (int i = 0; i < DPL; ++i) {
    gm[i] = gamma[lane + 32 * i];
    bt[i] = beta ? beta[lane + 32 * i] : 0.f;
    sg[i] = 0.f;
    sb[i] = 0.f;
  }
  const int rows_per_block = (M + gridDim.x - 1) / gridDim.x;
  const int r0 = blockIdx.x * rows_per_block, r1 = min(M, r0 + rows_per_block);
  for (int r = r0 + warp; r < r1; r += 8) {
    float v[DPL], gv[DPL], dv[DPL];
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < DPL; ++i) {
      v[i] = ld_f(y + int64_t(r) * D + lane + 32 * i);
      dv[i] = ld_f(dxt + int64_t(r) * D + lane + 32 * i);
      s += v[i];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    const float mean = s / D;
    float q = 0.f;
#pragma unroll
    for (int i = 0; i < DPL; ++i) {
      v[i] -= mean;
      q += v[i] * v[i];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) q += __shfl_xor_sync(0xffffffffu, q, o);
    const float rstd = rsqrtf(q / D + eps);
    float m1 = 0.f, m2 = 0.f;
#pragma unroll
    for (int i = 0; i < DPL; ++i) {
      v[i] *= rstd;  // xhat
      gv[i] = dv[i] * gm[i];
      m1 += gv[i];
      m2 += gv[i] * v[i];
      sg[i] += dv[i] * v[i];
      sb[i] += dv[i];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      m1 += __shfl_xor_sync(0xffffffffu, m1, o);
      m2 += __shfl_xor_sync(0xffffffffu, m2, o);
    }
    m1 /= D;
    m2 /= D;
#pragma unroll
    for (int i = 0; i < DPL; ++i) {
      st_f(dy + int64_t(r) * D + lane + 32 * i, rstd * (gv[i] - m1 - v[i] * m2));
      if (xt) st_f(xt + int64_t(r) * D + lane + 32 * i, v[i] * gm[i] + bt[i]);
    }
  }
  griddep_launch();
#pragma unroll
  for (int i = 0; i < DPL; ++i) {
    red[warp][0][lane + 32 * i] = sg[i];
    red[warp][1][lane + 32 * i] = sb[i];
  }
  __syncthreads();
  for (int c = threadIdx.x; c < 2 * D; c += blockDim.x) {
    const int which = c / D, col = c % D;
    float t = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) t += red[w][which][col];
    part[(int64_t(blockIdx.x) * 2 + which) * D + col] = t;
  }
}

// dgamma[c] = sum_b part[b][0][c], dbeta[c] = sum_b part[b][1][c] (blocks in order)
__global__ void ln_bwd_reduce_kernel(const float* __restrict__ part, int blocks, int D, float* __restrict__ dgamma,
                                     float* __restrict__ dbeta, int accumulate) {
  griddep_wait();
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= 2 * D) return;
  const int which = c / D, col = c % D;
  float t = 0.f;
  for (int b = 0; b < blocks; ++b) t += part[(int64_t(b) * 2 + which) * D + col];
  float* dst = which == 0 ? dgamma : dbeta;
  dst[col] = accumulate ? dst[col] + t : t;
}

// ------------------------------------------------------------------ SwiGLU backward
// A = SiLU(P1) * P3 with P = [P1 | P3] ([M, 2h] bf16) and dA [M, h] bf16:
//   dP1 = dA P3 SiLU'(P1),  dP3 = dA SiLU(P1),  SiLU'(x) = s (1 + x (1 - s)), s = sigma(x)
// written to dP = [dP1 | dP3] ([M, 2h] bf16); optionally A itself (a_out [M, h]).
__global__ void swiglu_bwd_kernel(const bf16* __restrict__ P, const bf16* __restrict__ dA, int64_t M, int h,
                                  bf16* __restrict__ dP, bf16* __restrict__ a_out) {
  griddep_wait();
  const int64_t n8 = M * h / 8;
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n8; i += int64_t(gridDim.x) * blockDim.x) {
    const int64_t e = i * 8, r = e / h, c = e % h;
    const uint4 p1 = *reinterpret_cast<const uint4*>(P + r * 2 * h + c);
    const uint4 p3 = *reinterpret_cast<const uint4*>(P + r * 2 * h + h + c);
    const uint4 da = *reinterpret_cast<const uint4*>(dA + e);
    const __nv_bfloat162* x1 = reinterpret_cast<const __nv_bfloat162*>(&p1);
    const __nv_bfloat162* x3 = reinterpret_cast<const __nv_bfloat162*>(&p3);
    const __nv_bfloat162* g = reinterpret_cast<const __nv_bfloat162*>(&da);
    uint4 o1, o3, oa;
    __nv_bfloat162* w1 = reinterpret_cast<__nv_bfloat162*>(&o1);
    __nv_bfloat162* w3 = reinterpret_cast<__nv_bfloat162*>(&o3);
    __nv_bfloat162* wa = reinterpret_cast<__nv_bfloat162*>(&oa);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 a = __bfloat1622float2(x1[j]), b = __bfloat1622float2(x3[j]), d = __bfloat1622float2(g[j]);
      const float sa = 1.f / (1.f + __expf(-a.x)), sb = 1.f / (1.f + __expf(-a.y));
      const float fa = a.x * sa, fb = a.y * sb;  // SiLU
      w1[j] = __floats2bfloat162_rn(d.x * b.x * sa * (1.f + a.x * (1.f - sa)), d.y * b.y * sb * (1.f + a.y * (1.f - sb)));
      w3[j] = __floats2bfloat162_rn(d.x * fa, d.y * fb);
      wa[j] = __floats2bfloat162_rn(fa * b.x, fb * b.y);
    }
    *reinterpret_cast<uint4*>(dP + r * 2 * h + c) = o1;
    *reinterpret_cast<uint4*>(dP + r * 2 * h + h + c) = o3;
    if (a_out) *reinterpret_cast<uint4*>(a_out + e) = oa;
  }
}

// LayerNorm forward, one warp per row of d = 32 DPL (biased variance): the training step
// recomputes the forward's LayerNorm outputs with it (bf16 history rows, fp32 target rows).
template <int DPL, typename TI, typename TO>
__global__ void __launch_bounds__(256) ln_fwd_kernel(const TI* __restrict__ x, int64_t ldx, int M,
                                                     const float* __restrict__ gamma, const float* __restrict__ beta,
                                                     float eps, TO* __restrict__ y, int64_t ldy) {
  griddep_wait();
  constexpr int D = 32 * DPL;
  const int lane = threadIdx.x & 31;
  const int r = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (r < M) {
    float v[DPL];
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < DPL; ++i) {
      v[i] = ld_f(x + int64_t(r) * ldx + lane + 32 * i);
      s += v[i];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    const float mean = s / D;
    float q = 0.f;
#pragma unroll
    for (int i = 0; i < DPL; ++i) {
      v[i] -= mean;
      q += v[i] * v[i];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) q += __shfl_xor_sync(0xffffffffu, q, o);
    const float rstd = rsqrtf(q / D + eps);
#pragma unroll
    for (int i = 0; i < DPL; ++i)
      st_f(y + int64_t(r) * ldy + lane + 32 * i, v[i] * rstd * gamma[lane + 32 * i] + (beta ? beta[lane + 32 * i] : 0.f));
  }
  griddep_launch();
}

// SwiGLU backward on fp32 rows (the target side): as swiglu_bwd_kernel, one value per thread
__global__ void swiglu_bwd_f32_kernel(const float* __restrict__ P, const float* __restrict__ dA, int64_t M, int h,
                                      float* __restrict__ dP, float* __restrict__ a_out) {
  griddep_wait();
  const int64_t n = M * h;
  for (int64_t e = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; e < n; e += int64_t(gridDim.x) * blockDim.x) {
    const int64_t r = e / h, c = e % h;
    const float a = P[r * 2 * h + c], b = P[r * 2 * h + h + c], d = dA[e];
    const float sg = 1.f / (1.f + __expf(-a)), f = a * sg;
    dP[r * 2 * h + c] = d * b * sg * (1.f + a * (1.f - sg));
    dP[r * 2 * h + h + c] = d * f;
    if (a_out) a_out[e] = f * b;
  }
}

// dst [rows, cols] bf16 (ld ldd) = round-to-nearest-even of src [rows, cols] fp32 (ld lds)
__global__ void f32_to_bf16_kernel(const float* __restrict__ src, int64_t lds, int rows, int cols,
                                   bf16* __restrict__ dst, int64_t ldd) {
  griddep_wait();
  const int64_t n = int64_t(rows) * cols;
  for (int64_t e = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; e < n; e += int64_t(gridDim.x) * blockDim.x) {
    const int64_t r = e / cols, c = e % cols;
    dst[r * ldd + c] = __float2bfloat16(src[r * lds + c]);
  }
}

// ------------------------------------------------------------------ lookup backward
// dtable[ids[n]] += dX[n] (16-byte fp32 vector atomics, one warp per token, 8 values per
// lane per pass);
// with dt, dt_table[bucket(dt[n])] += dX[n] through a per-block [16, d] shared
// accumulator, so that the 16 bucket rows take one atomic per block and column.
__global__ void __launch_bounds__(256) table_rows_bwd_kernel(const bf16* __restrict__ dX, int M, int d,
                                                             const int32_t* __restrict__ ids,
                                                             const int32_t* __restrict__ dt, int64_t n_items,
                                                             float* __restrict__ dtable,
                                                             float* __restrict__ ddt_table, int32_t* err) {
  griddep_wait();
  extern __shared__ float bucket_acc[];  // [16][d] when ddt_table
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool with_dt = dt && ddt_table;
  if (with_dt)
    for (int i = threadIdx.x; i < 16 * d; i += blockDim.x) bucket_acc[i] = 0.f;
  __syncthreads();
  const int per_block = (M + gridDim.x - 1) / gridDim.x;
  const int r0 = blockIdx.x * per_block, r1 = min(M, r0 + per_block);
  for (int r = r0 + warp; r < r1; r += 8) {
    const int64_t id = ids[r];
    const bool ok = id >= 0 && id < n_items;
    if (!ok && lane == 0) set_error(err, STCA_ERR_ID_OUT_OF_RANGE);
    const int b = with_dt ? dt_bucket(dt[r]) : 0;
    for (int c = lane * 8; c < d; c += 256) {
      const uint4 u = *reinterpret_cast<const uint4*>(dX + int64_t(r) * d + c);
      const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&u);
      float f[8];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 t = __bfloat1622float2(h2[j]);
        f[2 * j] = t.x;
        f[2 * j + 1] = t.y;
      }
      if (ok) {  // 16-byte vector reductions: a quarter of the atomic operations on hot rows
        float4* row = reinterpret_cast<float4*>(dtable + id * d + c);
        atomicAdd(row, make_float4(f[0], f[1], f[2], f[3]));
        atomicAdd(row + 1, make_float4(f[4], f[5], f[6], f[7]));
      }
      if (with_dt) {
#pragma unroll
        for (int j = 0; j < 8; ++j) atomicAdd(bucket_acc + b * d + c + j, f[j]);
      }
    }
  }
  griddep_launch();
  if (!with_dt) return;
  __syncthreads();
  for (int i = threadIdx.x; i < 16 * d; i += blockDim.x)
    if (bucket_acc[i] != 0.f) atomicAdd(ddt_table + i, bucket_acc[i]);
}

// The same scatter with the tokens of each 1024-token chunk grouped by id first, for d a
// multiple of 256: a shared-memory hash table (2048 slots, linear probing, at most 1024
// keys) gives each token its group; a scan lays the groups' members out contiguously;
// then one warp per group sums the members' rows in registers (four rows in flight) and
// adds the sum to the id's row with one set of vector atomics.  A Zipf-popular id that
// appears 100 times in a chunk costs one row of atomics there instead of 100, which is
// what the atomics on hot rows were waiting on.
constexpr int TR_CH = 1024, TR_HS = 2048, TR_THREADS = 256;
constexpr size_t TR_SMEM_INT = size_t(4 * TR_HS + 3 * TR_CH + 4) * 4;  // keys cnt start fill | slot order gslot | misc

template <int DV>
__global__ void __launch_bounds__(TR_THREADS) table_rows_grouped_kernel(const bf16* __restrict__ dX, int M,
                                                                        const int32_t* __restrict__ ids,
                                                                        const int32_t* __restrict__ dt,
                                                                        int64_t n_items, float* __restrict__ dtable,
                                                                        float* __restrict__ ddt_table, int32_t* err) {
  constexpr int d = 256 * DV;
  griddep_wait();
  extern __shared__ __align__(16) int tr_smem[];
  int* keys = tr_smem;                // [TR_HS] id, -1 empty
  int* cnt = keys + TR_HS;            // [TR_HS] members per slot
  int* start = cnt + TR_HS;           // [TR_HS] first member position
  int* fill = start + TR_HS;          // [TR_HS] members placed so far
  int* slot_of = fill + TR_HS;        // [TR_CH] token -> slot (-1: skipped)
  int* order = slot_of + TR_CH;       // [TR_CH] tokens grouped by slot
  int* gslot = order + TR_CH;         // [TR_CH] slot of group g
  int* misc = gslot + TR_CH;          // [0] groups, [1] next group, [2..3] scan scratch
  float* bucket_acc = reinterpret_cast<float*>(misc + 4);  // [16][d] when ddt_table
  __shared__ int warp_sum[TR_THREADS / 32], warp_ne[TR_THREADS / 32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool with_dt = dt && ddt_table;
  if (with_dt)
    for (int i = threadIdx.x; i < 16 * d; i += TR_THREADS) bucket_acc[i] = 0.f;
  const int nchunks = (M + TR_CH - 1) / TR_CH;
  for (int chunk = blockIdx.x; chunk < nchunks; chunk += gridDim.x) {
    const int c0 = chunk * TR_CH;
    for (int i = threadIdx.x; i < TR_HS; i += TR_THREADS) {
      keys[i] = -1;
      cnt[i] = 0;
      fill[i] = 0;
    }
    if (threadIdx.x == 0) misc[1] = 0;
    __syncthreads();
    // ---- groups: insert each token's id (bounded probing; at most TR_CH < TR_HS keys)
    for (int t = threadIdx.x; t < TR_CH; t += TR_THREADS) {
      const int r = c0 + t;
      int slot = -1;
      if (r < M) {
        const int id = ids[r];
        if (id < 0 || int64_t(id) >= n_items) {
          set_error(err, STCA_ERR_ID_OUT_OF_RANGE);
        } else {
          uint32_t h = (uint32_t(id) * 2654435761u) >> (32 - 11);
          for (int p = 0; p < TR_HS; ++p, h = (h + 1) & (TR_HS - 1)) {
            const int k = atomicCAS(&keys[h], -1, id);
            if (k == -1 || k == id) {
              slot = int(h);
              break;
            }
          }
          if (slot >= 0) atomicAdd(&cnt[slot], 1);
          else set_error(err, STCA_ERR_CAPACITY);
        }
      }
      slot_of[t] = slot;
    }
    __syncthreads();
    // ---- exclusive scans of the member counts and of the non-empty slots (8 slots a thread)
    {
      const int s0 = threadIdx.x * (TR_HS / TR_THREADS);
      int sum = 0, ne = 0;
#pragma unroll
      for (int i = 0; i < TR_HS / TR_THREADS; ++i) {
        sum += cnt[s0 + i];
        ne += cnt[s0 + i] > 0;
      }
      int isum = sum, ine = ne;  // inclusive warp scans
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int a = __shfl_up_sync(0xffffffffu, isum, o), b = __shfl_up_sync(0xffffffffu, ine, o);
        if (lane >= o) {
          isum += a;
          ine += b;
        }
      }
      if (lane == 31) {
        warp_sum[warp] = isum;
        warp_ne[warp] = ine;
      }
      __syncthreads();
      int base = isum - sum, gbase = ine - ne;
      for (int w = 0; w < warp; ++w) {
        base += warp_sum[w];
        gbase += warp_ne[w];
      }
      if (threadIdx.x == TR_THREADS - 1) misc[0] = gbase + ne;
#pragma unroll
      for (int i = 0; i < TR_HS / TR_THREADS; ++i) {
        const int c = cnt[s0 + i];
        start[s0 + i] = base;
        base += c;
        if (c > 0) gslot[gbase++] = s0 + i;
      }
    }
    __syncthreads();
    for (int t = threadIdx.x; t < TR_CH; t += TR_THREADS) {
      const int slot = slot_of[t];
      if (slot >= 0) order[start[slot] + atomicAdd(&fill[slot], 1)] = t;
    }
    __syncthreads();
    // ---- one warp per group (taken in turn): sum the members' rows, then one add per id
    const int ngroups = misc[0];
    while (true) {
      int g = 0;
      if (lane == 0) g = atomicAdd(&misc[1], 1);
      g = __shfl_sync(0xffffffffu, g, 0);
      if (g >= ngroups) break;
      const int slot = gslot[g];
      const int64_t id = keys[slot];
      const int beg = start[slot], n = cnt[slot];
      float acc[DV][8];
#pragma unroll
      for (int v = 0; v < DV; ++v)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[v][j] = 0.f;
      for (int m = 0; m < n; m += 4) {
        uint4 u[4][DV];
        int rr[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          rr[q] = m + q < n ? c0 + order[beg + m + q] : -1;
#pragma unroll
          for (int v = 0; v < DV; ++v)
            u[q][v] = rr[q] >= 0 ? *reinterpret_cast<const uint4*>(dX + int64_t(rr[q]) * d + v * 256 + lane * 8)
                                 : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int b = (with_dt && rr[q] >= 0) ? dt_bucket(dt[rr[q]]) : 0;
#pragma unroll
          for (int v = 0; v < DV; ++v) {
            const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&u[q][v]);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const float2 f = __bfloat1622float2(h2[j]);
              acc[v][2 * j] += f.x;
              acc[v][2 * j + 1] += f.y;
              if (with_dt && rr[q] >= 0) {
                atomicAdd(bucket_acc + b * d + v * 256 + lane * 8 + 2 * j, f.x);
                atomicAdd(bucket_acc + b * d + v * 256 + lane * 8 + 2 * j + 1, f.y);
              }
            }
          }
        }
      }
#pragma unroll
      for (int v = 0; v < DV; ++v) {
        float4* row = reinterpret_cast<float4*>(dtable + id * d + v * 256 + lane * 8);
        atomicAdd(row, make_float4(acc[v][0], acc[v][1], acc[v][2], acc[v][3]));
        atomicAdd(row + 1, make_float4(acc[v][4], acc[v][5], acc[v][6], acc[v][7]));
      }
    }
    __syncthreads();  // the chunk's tables are reset next
  }
  griddep_launch();
  if (!with_dt) return;
  __syncthreads();
  for (int i = threadIdx.x; i < 16 * d; i += TR_THREADS)
    if (bucket_acc[i] != 0.f) atomicAdd(ddt_table + i, bucket_acc[i]);
}

// dst [K, 2N] from W [K, N] without transposing: mode 3 puts column n of W at column
// 128 (n / 64) + off + n % 64 (the head-interleaved [K_h | V_h] layout, d_h = 64), mode 4
// at column off + n (two blocks side by side)
__global__ void place_cols_kernel(const bf16* __restrict__ W, int K, int N, bf16* __restrict__ dst, int mode,
                                  int off) {
  const int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= int64_t(K) * N) return;
  const int k = int(i / N), n = int(i % N);
  const int col = mode == 3 ? 128 * (n / 64) + off + n % 64 : off + n;
  dst[int64_t(k) * 2 * N + col] = W[i];
}

}  // namespace

size_t gemm_wgrad_workspace_bytes(int M, int K, int N) {
  if (M <= 0 || K <= 0 || N <= 0 || K % WG_T || N % WG_T) return 0;
  return size_t(std::max(wgrad_splits(M, K, N), tc_wgrad_splits(M, K, N))) * K * N * 4;
}

int gemm_wgrad(const void* A, int64_t lda, const void* G, int64_t ldg, int M, int K, int N, float* C, int64_t ldc,
               int accumulate, int impl, void* ws, size_t ws_bytes, int32_t* err, cudaStream_t s) {
  if (M < 0 || K <= 0 || N <= 0 || K % WG_T || N % WG_T || lda % 8 || ldg % 8 || ldc % 4) return STCA_ERR_UNSUPPORTED;
  if (lda < K || ldg < N || ldc < N || impl < 0 || impl > 1) return STCA_ERR_INVALID_ARG;
  const uintptr_t al = reinterpret_cast<uintptr_t>(A) | reinterpret_cast<uintptr_t>(G) |
                       reinterpret_cast<uintptr_t>(C) | reinterpret_cast<uintptr_t>(ws);
  if (al & 15) return STCA_ERR_INVALID_ARG;
  // 0: the tensor-core (tcgen05) kernel; 1: the mma.sync kernel (both kept under test)
  const bool tc = impl != 1;
  const int splits = M > 0 ? (tc ? tc_wgrad_splits(M, K, N) : wgrad_splits(M, K, N)) : 1;
  if (M > 0 && ws_bytes < size_t(splits) * K * N * 4) return STCA_ERR_CAPACITY;
  float* part = static_cast<float*>(ws);
  if (M > 0 && tc) {
    const int rc = tc_wgrad_partials(A, lda, G, ldg, M, K, N, splits, part, err, s);
    if (rc != STCA_OK) return rc;
  } else if (M > 0) {
    cudaFuncSetAttribute(gemm_wgrad_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, WG_SMEM);
    if (launch_dep(gemm_wgrad_kernel, dim3(N / WG_T, K / WG_T, splits), dim3(256), WG_SMEM, s,
                   static_cast<const bf16*>(A), lda, static_cast<const bf16*>(G), ldg, M, K, N, splits,
                   part) != cudaSuccess)
      return STCA_ERR_CUDA;
    note_launch();
  } else if (!accumulate) {
    return cudaMemset2DAsync(C, size_t(ldc) * 4, 0, size_t(N) * 4, K, s) == cudaSuccess ? STCA_OK : STCA_ERR_CUDA;
  } else {
    return STCA_OK;
  }
  const int64_t n4 = int64_t(K) * N / 4;
  if (launch_dep(wgrad_reduce_kernel, dim3(unsigned((n4 + 255) / 256)), dim3(256), 0, s,
                 static_cast<const float*>(part), splits, K, N, C, ldc, accumulate) != cudaSuccess)
    return STCA_ERR_CUDA;
  note_launch();
  return STCA_OK;
}

// as many 256-thread blocks as fit on every SM at once (d = 256: 64 registers a thread, four
// blocks; d = 512: 128 registers, two), so that more rows are in flight
int ln_bwd_blocks(int M, int d) {
  return std::max(1, std::min((d == 256 ? 4 : 2) * sm_count(), (M + 31) / 32));
}

size_t layer_norm_bwd_workspace_bytes(int M, int d) { return size_t(ln_bwd_blocks(M, d)) * 2 * d * 4; }

template <typename T>
static cudaError_t launch_ln_bwd(int d, int blocks, cudaStream_t s, const void* y, const void* dxt, int M,
                                 const float* gamma, const float* beta, float eps, void* dy, void* xt, float* part) {
  auto kern = d == 256 ? ln_bwd_kernel<8, T> : ln_bwd_kernel<16, T>;
  return launch_dep(kern, dim3(blocks), dim3(256), 0, s, static_cast<const T*>(y), static_cast<const T*>(dxt), M,
                    gamma, beta, eps, static_cast<T*>(dy), static_cast<T*>(xt), part);
}

int layer_norm_bwd(const void* y, const void* dxt, int M, int d, int fp32, const float* gamma, const float* beta,
                   float eps, void* dy, void* xt, float* dgamma, float* dbeta, int accumulate, void* ws,
                   size_t ws_bytes, cudaStream_t s) {
  if (M < 0 || (d != 256 && d != 512)) return STCA_ERR_UNSUPPORTED;
  if (!gamma || !dgamma || !dbeta || (M > 0 && (!y || !dxt || !dy))) return STCA_ERR_INVALID_ARG;
  const int blocks = ln_bwd_blocks(M, d);
  if (ws_bytes < size_t(blocks) * 2 * d * 4 || !ws) return STCA_ERR_CAPACITY;
  float* part = static_cast<float*>(ws);
  const cudaError_t e = fp32 ? launch_ln_bwd<float>(d, blocks, s, y, dxt, M, gamma, beta, eps, dy, xt, part)
                             : launch_ln_bwd<bf16>(d, blocks, s, y, dxt, M, gamma, beta, eps, dy, xt, part);
  if (e != cudaSuccess) return STCA_ERR_CUDA;
  note_launch();
  if (launch_dep(ln_bwd_reduce_kernel, dim3((2 * d + 255) / 256), dim3(256), 0, s, static_cast<const float*>(part),
                 blocks, d, dgamma, dbeta, accumulate) != cudaSuccess)
    return STCA_ERR_CUDA;
  note_launch();
  return STCA_OK;
}

int swiglu_bwd(const void* P, const void* dA, int M, int h, int fp32, void* dP, void* a_out, cudaStream_t s) {
  if (M < 0 || h <= 0 || h % 8) return STCA_ERR_UNSUPPORTED;
  if (M == 0) return STCA_OK;
  if (!P || !dA || !dP) return STCA_ERR_INVALID_ARG;
  if (fp32) {
    const int64_t n = int64_t(M) * h;
    const int blocks = int(std::min<int64_t>((n + 255) / 256, int64_t(8) * sm_count()));
    if (launch_dep(swiglu_bwd_f32_kernel, dim3(blocks), dim3(256), 0, s, static_cast<const float*>(P),
                   static_cast<const float*>(dA), int64_t(M), h, static_cast<float*>(dP), static_cast<float*>(a_out)) !=
        cudaSuccess)
      return STCA_ERR_CUDA;
    note_launch();
    return STCA_OK;
  }
  const uintptr_t al = reinterpret_cast<uintptr_t>(P) | reinterpret_cast<uintptr_t>(dA) |
                       reinterpret_cast<uintptr_t>(dP) | reinterpret_cast<uintptr_t>(a_out);
  if (al & 15) return STCA_ERR_INVALID_ARG;
  const int64_t n8 = int64_t(M) * h / 8;
  const int blocks = int(std::min<int64_t>((n8 + 255) / 256, int64_t(8) * sm_count()));
  if (launch_dep(swiglu_bwd_kernel, dim3(blocks), dim3(256), 0, s, static_cast<const bf16*>(P),
                 static_cast<const bf16*>(dA), int64_t(M), h, static_cast<bf16*>(dP), static_cast<bf16*>(a_out)) !=
      cudaSuccess)
    return STCA_ERR_CUDA;
  note_launch();
  return STCA_OK;
}

int layer_norm_fwd(const void* x, int64_t ldx, int x_fp32, int M, int d, const float* gamma, const float* beta,
                   float eps, void* y, int64_t ldy, int y_fp32, cudaStream_t s) {
  if (M < 0 || (d != 256 && d != 512)) return STCA_ERR_UNSUPPORTED;
  if (M == 0) return STCA_OK;
  if (!x || !y || !gamma || ldx < d || ldy < d) return STCA_ERR_INVALID_ARG;
  const dim3 grid((M + 7) / 8), block(256);
  cudaError_t e;
  if (x_fp32 && y_fp32)
    e = launch_dep(d == 256 ? ln_fwd_kernel<8, float, float> : ln_fwd_kernel<16, float, float>, grid, block, 0, s,
                   static_cast<const float*>(x), ldx, M, gamma, beta, eps, static_cast<float*>(y), ldy);
  else if (!x_fp32 && !y_fp32)
    e = launch_dep(d == 256 ? ln_fwd_kernel<8, bf16, bf16> : ln_fwd_kernel<16, bf16, bf16>, grid, block, 0, s,
                   static_cast<const bf16*>(x), ldx, M, gamma, beta, eps, static_cast<bf16*>(y), ldy);
  else
    return STCA_ERR_UNSUPPORTED;
  if (e != cudaSuccess) return STCA_ERR_CUDA;
  note_launch();
  return STCA_OK;
}

int f32_to_bf16(const float* src, int64_t lds, int rows, int cols, void* dst, int64_t ldd, cudaStream_t s) {
  if (rows < 0 || cols < 0 || lds < cols || ldd < cols) return STCA_ERR_INVALID_ARG;
  if (rows == 0 || cols == 0) return STCA_OK;
  if (!src || !dst) return STCA_ERR_INVALID_ARG;
  const int64_t n = int64_t(rows) * cols;
  const int blocks = int(std::min<int64_t>((n + 255) / 256, int64_t(8) * sm_count()));
  if (launch_dep(f32_to_bf16_kernel, dim3(blocks), dim3(256), 0, s, src, lds, rows, cols, static_cast<bf16*>(dst),
                 ldd) != cudaSuccess)
    return STCA_ERR_CUDA;
  note_launch();
  return STCA_OK;
}

int table_rows_bwd(const void* dX, int M, int d, const int32_t* ids, const int32_t* dt, int64_t n_items,
                   float* dtable, float* ddt_table, int32_t* err, cudaStream_t s) {
  if (M < 0 || d <= 0 || d % 8 || n_items <= 0) return STCA_ERR_INVALID_ARG;
  if (M == 0) return STCA_OK;
  if (!dX || !ids || !dtable || ((reinterpret_cast<uintptr_t>(dX) | reinterpret_cast<uintptr_t>(dtable)) & 15))
    return STCA_ERR_INVALID_ARG;
  const bool with_dt = dt && ddt_table;
  if (d == 256 || d == 512) {  // tokens grouped by id per chunk
    const size_t smem = TR_SMEM_INT + (with_dt ? size_t(16) * d * 4 : 0);
    const int blocks = std::max(1, std::min(4 * sm_count(), (M + TR_CH - 1) / TR_CH));
    auto kern = d == 256 ? table_rows_grouped_kernel<1> : table_rows_grouped_kernel<2>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) != cudaSuccess)
      return STCA_ERR_CUDA;
    if (launch_dep(kern, dim3(blocks), dim3(TR_THREADS), smem, s, static_cast<const bf16*>(dX), M, ids,
                   with_dt ? dt : nullptr, n_items, dtable, with_dt ? ddt_table : nullptr, err) != cudaSuccess)
      return STCA_ERR_CUDA;
    note_launch();
    return STCA_OK;
  }
  const size_t smem = with_dt ? size_t(16) * d * 4 : 0;
  if (smem > 48 * 1024) return STCA_ERR_UNSUPPORTED;
  const int blocks = std::max(1, std::min(4 * sm_count(), (M + 7) / 8));
  if (launch_dep(table_rows_bwd_kernel, dim3(blocks), dim3(256), smem, s, static_cast<const bf16*>(dX), M, d, ids,
                 with_dt ? dt : nullptr, n_items, dtable, with_dt ? ddt_table : nullptr, err) != cudaSuccess)
    return STCA_ERR_CUDA;
  note_launch();
  return STCA_OK;
}

int place_cols(const void* W, int K, int N, void* dst, int mode, int off, cudaStream_t s) {
  if (!W || !dst || K <= 0 || N <= 0 || (mode != 3 && mode != 4)) return STCA_ERR_INVALID_ARG;
  if (mode == 3 && (N % 64 || (off != 0 && off != 64))) return STCA_ERR_INVALID_ARG;
  if (mode == 4 && off != 0 && off != N) return STCA_ERR_INVALID_ARG;
  const int64_t n = int64_t(K) * N;
  place_cols_kernel<<<unsigned((n + 255) / 256), 256, 0, s>>>(static_cast<const bf16*>(W), K, N,
                                                              static_cast<bf16*>(dst), mode, off);
  note_launch();
  return cudaGetLastError() == cudaSuccess ? STCA_OK : STCA_ERR_CUDA;
}

}  // namespace stca
