// Tensor-core GEMM for the target-side (query) path with bf16 weights.
//
// The query path keeps fp32 activations: each A element a is split into two bf16 terms
// a_hi = bf16(a), a_lo = bf16(a - a_hi), so a_hi + a_lo carries 16 significant bits, and
// the weights are bf16 already; the two products a_hi*w and a_lo*w are exact in the fp32
// accumulator.  The result matches an fp32 GEMM to ~2^-17 relative per product, well
// inside fp32 accumulation error over K >= 256.
//
// CTA tile 128 x 128, K step 32, 8 warps as 2 (M) x 4 (N), warp tile 64 x 32;
// mma.sync m16n8k16 with fragments from XOR-swizzled shared memory via ldmatrix.  Same
// argument struct as the SIMT kernel (row remaps, two-segment A, SwiGLU pair, residual,
// per-batch weights), minus the gathered-A form.
#include "common.cuh"
#include "internal.h"

namespace stca {

namespace {

constexpr int QM = 128, QN = 128, QK = 32;
constexpr int A_TILE = QM * QK * 2;  // one bf16 [128 x 32] tile: 8 KB
constexpr int B_TILE = QK * QN * 2;  // one bf16 [32 x 128] tile: 8 KB

__device__ __forceinline__ int64_t qremap(int r, int grp, int gstride, int goff) {
  return grp ? int64_t(r / grp) * gstride + goff + r % grp : int64_t(r);
}

// A tile [128 rows][32 k] bf16: 64-byte rows, 16-byte chunk c of row r at c ^ ((r >> 1) & 3)
__device__ __forceinline__ int a_off(int r, int c) { return r * 64 + ((c ^ ((r >> 1) & 3)) << 4); }
// B tile [32 k rows][128 n] bf16: 256-byte rows, 16-byte chunk c of row k at c ^ (k & 7)
__device__ __forceinline__ int b_off(int k, int c) { return k * 256 + ((c ^ (k & 7)) << 4); }

__device__ __forceinline__ float silu_acc(float x) { return x / (1.0f + expf(-x)); }

template <bool DUAL>
__global__ void __launch_bounds__(256, 1) query_gemm_kernel(SimtGemmArgs<float, bf16> a) {
  extern __shared__ __align__(128) uint8_t smem[];
  // [stage][A_hi | A_lo | B | B2]
  constexpr int STAGE = 2 * A_TILE + (DUAL ? 2 : 1) * B_TILE;
  const int z = blockIdx.z;
  const float* A = a.A + z * a.bsA;
  const bool per_batch = a.Bz[0] != nullptr;
  const bf16* Bm = per_batch ? a.Bz[z] : a.B + z * a.bsB;
  const bf16* Bm2 = DUAL ? (per_batch ? a.B2z[z] : a.B2 + z * a.bsB) : nullptr;
  float* C = a.C + z * a.bsC;
  const float* Rr = a.R ? a.R + z * a.bsR : nullptr;
  const int m0 = blockIdx.y * QM, n0 = blockIdx.x * QN;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int wm = warp >> 2, wn = warp & 3;  // warp tile: rows wm*64, cols wn*32

  // loader mapping: A: thread -> (row tid/2, 16 k = 4 float4 at (tid&1)*16);
  //                 B: thread -> (k row tid/8, 16 n = 2 x uint4 at (tid&7)*16)
  const int ar = tid >> 1, ak = (tid & 1) * 16;
  const int arow = m0 + ar;
  const float* arow_ptr = arow < a.M ? A + qremap(arow, a.a_grp, a.a_gstride, a.a_goff) * a.lda : nullptr;
  const int bk = tid >> 3, bn = (tid & 7) * 16;

  float4 ra[4];
  uint4 rb[2], rb2[2];
  auto load_global = [&](int k0) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int k = k0 + ak + i * 4;
      if (arow_ptr && k < a.K) {
        const int col = k < a.ksplit ? k : k + a.kshift;
        ra[i] = *reinterpret_cast<const float4*>(arow_ptr + col);
      } else {
        ra[i] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
    const int k = k0 + bk;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int n = n0 + bn + j * 8;
      const bool ok = k < a.K && n < a.N;
      rb[j] = ok ? *reinterpret_cast<const uint4*>(Bm + int64_t(k) * a.N + n) : make_uint4(0, 0, 0, 0);
      if (DUAL) rb2[j] = ok ? *reinterpret_cast<const uint4*>(Bm2 + int64_t(k) * a.N + n) : make_uint4(0, 0, 0, 0);
    }
  };
  auto store_smem = [&](int stage) {
    uint8_t* st = smem + stage * STAGE;
    uint8_t* sAh = st;
    uint8_t* sAl = st + A_TILE;
    uint8_t* sB = st + 2 * A_TILE;
    // A: 16 fp32 -> 16 bf16 hi + 16 bf16 lo = two 16-byte chunks each
    uint32_t hi[8], lo[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float v[4] = {ra[i].x, ra[i].y, ra[i].z, ra[i].w};
#pragma unroll
      for (int e = 0; e < 4; e += 2) {
        const __nv_bfloat162 h = __floats2bfloat162_rn(v[e], v[e + 1]);
        const float2 hf = __bfloat1622float2(h);
        const __nv_bfloat162 l = __floats2bfloat162_rn(v[e] - hf.x, v[e + 1] - hf.y);
        hi[i * 2 + e / 2] = *reinterpret_cast<const uint32_t*>(&h);
        lo[i * 2 + e / 2] = *reinterpret_cast<const uint32_t*>(&l);
      }
    }
    const int c0 = ak / 8;  // chunk index (8 bf16 per chunk)
    *reinterpret_cast<uint4*>(sAh + a_off(ar, c0)) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
    *reinterpret_cast<uint4*>(sAh + a_off(ar, c0 + 1)) = make_uint4(hi[4], hi[5], hi[6], hi[7]);
    *reinterpret_cast<uint4*>(sAl + a_off(ar, c0)) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
    *reinterpret_cast<uint4*>(sAl + a_off(ar, c0 + 1)) = make_uint4(lo[4], lo[5], lo[6], lo[7]);
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      *reinterpret_cast<uint4*>(sB + b_off(bk, bn / 8 + j)) = rb[j];
      if (DUAL) *reinterpret_cast<uint4*>(sB + B_TILE + b_off(bk, bn / 8 + j)) = rb2[j];
    }
  };

  float acc[4][4][4], acc2[DUAL ? 4 : 1][DUAL ? 4 : 1][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        acc[i][j][e] = 0.f;
        if (DUAL) acc2[i][j][e] = 0.f;
      }

  const int nk = (a.K + QK - 1) / QK;
  load_global(0);
  store_smem(0);
  __syncthreads();
  for (int kt = 0; kt < nk; ++kt) {
    const int cur = kt & 1;
    if (kt + 1 < nk) load_global((kt + 1) * QK);
    const uint32_t base = smem_u32(smem + cur * STAGE);
    const uint32_t sAh = base, sAl = base + A_TILE, sB = base + 2 * A_TILE;
#pragma unroll
    for (int kk = 0; kk < 2; ++kk) {  // two k16 steps per K step
      uint32_t bfr[4][2], bfr2[DUAL ? 4 : 1][2];
#pragma unroll
      for (int np = 0; np < 2; ++np) {  // pairs of n8 tiles
        const int krow = kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
        const int ch = (wn * 32 + np * 16) / 8 + (lane >> 4);
        uint32_t r[4];
        ldsm_x4_t(sB + b_off(krow, ch), r);
        bfr[2 * np][0] = r[0];
        bfr[2 * np][1] = r[1];
        bfr[2 * np + 1][0] = r[2];
        bfr[2 * np + 1][1] = r[3];
        if (DUAL) {
          ldsm_x4_t(sB + B_TILE + b_off(krow, ch), r);
          bfr2[2 * np][0] = r[0];
          bfr2[2 * np][1] = r[1];
          bfr2[2 * np + 1][0] = r[2];
          bfr2[2 * np + 1][1] = r[3];
        }
      }
#pragma unroll
      for (int mi = 0; mi < 4; ++mi) {
        const int row = wm * 64 + mi * 16 + (lane & 15);
        const int ch = kk * 2 + (lane >> 4);
        uint32_t ah[4], al[4];
        ldsm_x4(sAh + a_off(row, ch), ah);
        ldsm_x4(sAl + a_off(row, ch), al);
#pragma unroll
        for (int nj = 0; nj < 4; ++nj) {
          mma_bf16_16816(acc[mi][nj], ah, bfr[nj][0], bfr[nj][1]);
          mma_bf16_16816(acc[mi][nj], al, bfr[nj][0], bfr[nj][1]);
          if (DUAL) {
            mma_bf16_16816(acc2[mi][nj], ah, bfr2[nj][0], bfr2[nj][1]);
            mma_bf16_16816(acc2[mi][nj], al, bfr2[nj][0], bfr2[nj][1]);
          }
        }
      }
    }
    if (kt + 1 < nk) {
      store_smem(cur ^ 1);
    }
    __syncthreads();
  }

  // epilogue: c0,c1 -> (row g, cols 2t, 2t+1), c2,c3 -> (row g+8, ...)
  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int mi = 0; mi < 4; ++mi)
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
      const int m = m0 + wm * 64 + mi * 16 + g + hr * 8;
      if (m >= a.M) continue;
      float* crow = C + qremap(m, a.c_grp, a.c_gstride, a.c_goff) * a.ldc;
      const float* rrow = Rr ? Rr + int64_t(m) * a.ldr : nullptr;
#pragma unroll
      for (int nj = 0; nj < 4; ++nj) {
        const int n = n0 + wn * 32 + nj * 8 + 2 * t;
        if (n >= a.N) continue;
        float v0 = acc[mi][nj][2 * hr], v1 = acc[mi][nj][2 * hr + 1];
        if (DUAL) {
          v0 = silu_acc(v0) * acc2[mi][nj][2 * hr];
          v1 = silu_acc(v1) * acc2[mi][nj][2 * hr + 1];
        }
        if (rrow) {
          v0 += rrow[n];
          v1 += rrow[n + 1];
        }
        crow[n] = v0;
        crow[n + 1] = v1;
      }
    }
}

}  // namespace

bool query_gemm_supported(const SimtGemmArgs<float, bf16>& a) {
  const bool a_aligned = (reinterpret_cast<uintptr_t>(a.A) % 16 == 0) && a.lda % 4 == 0 && a.bsA % 4 == 0 &&
                         a.ksplit % 4 == 0 && a.kshift % 4 == 0;
  return a.gather.ids == nullptr && a_aligned && a.K % 16 == 0 && a.N % 8 == 0;
}

int query_gemm(const SimtGemmArgs<float, bf16>& a, cudaStream_t s) {
  dim3 grid((a.N + QN - 1) / QN, (a.M + QM - 1) / QM, a.batch);
  if (a.B2) {
    constexpr int smem = 2 * (2 * A_TILE + 2 * B_TILE);
    cudaFuncSetAttribute(query_gemm_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    query_gemm_kernel<true><<<grid, 256, smem, s>>>(a);
  } else {
    constexpr int smem = 2 * (2 * A_TILE + B_TILE);
    cudaFuncSetAttribute(query_gemm_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    query_gemm_kernel<false><<<grid, 256, smem, s>>>(a);
  }
  note_launch();
  return cudaGetLastError() == cudaSuccess ? 0 : STCA_ERR_CUDA;
}

}  // namespace stca
