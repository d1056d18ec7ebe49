// fp32-accumulating SIMT kernels: the whole path of the fp32 configuration, LayerNorm,
// the ragged-offset scan and the token mix.  The target-side GEMMs with bf16 weights go
// to the tensor-core form in query_gemm.cu when their shapes allow.
//
// The query path works on T_tot x d matrices (one row per target), which are small next
// to the history side; it keeps fp32 activations throughout.
#include <type_traits>

#include "common.cuh"
#include "internal.h"

namespace stca {

namespace {

constexpr int SB_M = 64, SB_N = 64, SB_K = 16;

__device__ __forceinline__ int64_t remap_row(int r, int grp, int gstride, int goff) {
  return grp ? int64_t(r / grp) * gstride + goff + r % grp : int64_t(r);
}

template <typename T>
__device__ __forceinline__ float ld_f(const T* p) {
  return to_f<T>(*p);
}

__device__ __forceinline__ float silu_exact(float x) { return x / (1.0f + expf(-x)); }

// C = A B (or SiLU(A B) * (A B2)), 64x64 tile per 256 threads, 4x4 per thread.
template <typename TA, typename TB, bool DUAL>
__global__ void __launch_bounds__(256) simt_gemm_kernel(SimtGemmArgs<TA, TB> a) {
  __shared__ float As[SB_K][SB_M + 4];
  __shared__ float Bs[SB_K][SB_N];
  __shared__ float Bs2[DUAL ? SB_K : 1][DUAL ? SB_N : 1];
  const int z = blockIdx.z;
  const TA* A = a.A + z * a.bsA;
  const bool per_batch = a.Bz[0] != nullptr;
  const TB* B = per_batch ? a.Bz[z] : a.B + z * a.bsB;
  const TB* B2 = DUAL ? (per_batch ? a.B2z[z] : a.B2 + z * a.bsB) : nullptr;
  float* C = a.C + z * a.bsC;
  const float* R = a.R ? a.R + z * a.bsR : nullptr;
  const int m0 = blockIdx.y * SB_M, n0 = blockIdx.x * SB_N;
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;

  // per-thread A-row source for the tile load: row m0 + tid/4, 4 consecutive k
  const int ar = tid >> 2, ac = (tid & 3) * 4;
  const int arow = m0 + ar;
  const TA* arow_ptr = nullptr;
  const TA* dtrow_ptr = nullptr;
  if (arow < a.M) {
    if (a.gather.ids) {
      int64_t id = a.gather.ids[arow];
      if (id < 0 || id >= a.gather.n_items) {
        set_error(a.err, STCA_ERR_ID_OUT_OF_RANGE);
      } else {
        arow_ptr = reinterpret_cast<const TA*>(a.gather.table) + id * a.K;
      }
      if (a.gather.dt && a.gather.dt_table) {
        const int32_t dt = a.gather.dt[arow];
        dtrow_ptr = reinterpret_cast<const TA*>(a.gather.dt_table) + int64_t(dt_bucket(dt < 0 ? 0 : dt)) * a.K;
      }
    } else {
      arow_ptr = A + remap_row(arow, a.a_grp, a.a_gstride, a.a_goff) * a.lda;
    }
  }
  const int br = tid >> 4, bc = (tid & 15) * 4;

  float acc[4][4], acc2[DUAL ? 4 : 1][DUAL ? 4 : 1];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      acc[i][j] = 0.f;
      if (DUAL) acc2[i][j] = 0.f;
    }

  for (int k0 = 0; k0 < a.K; k0 += SB_K) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int k = k0 + ac + i;
      float v = 0.f;
      if (arow_ptr && k < a.K) {
        const int col = (a.gather.ids || k < a.ksplit) ? k : k + a.kshift;
        v = ld_f(arow_ptr + col);
        if (dtrow_ptr) v += ld_f(dtrow_ptr + k);
      }
      As[ac + i][ar] = v;
    }
    {
      const int k = k0 + br;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int n = n0 + bc + j;
        const bool ok = k < a.K && n < a.N;
        Bs[br][bc + j] = ok ? ld_f(B + int64_t(k) * a.N + n) : 0.f;
        if (DUAL) Bs2[br][bc + j] = ok ? ld_f(B2 + int64_t(k) * a.N + n) : 0.f;
      }
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < SB_K; ++kk) {
      float av[4], bv[4], bv2[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) av[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        bv[j] = Bs[kk][tx * 4 + j];
        if (DUAL) bv2[j] = Bs2[kk][tx * 4 + j];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
          if (DUAL) acc2[i][j] = fmaf(av[i], bv2[j], acc2[i][j]);
        }
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + ty * 4 + i;
    if (m >= a.M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n >= a.N) continue;
      float v = DUAL ? silu_exact(acc[i][j]) * acc2[i][j] : acc[i][j];
      if (R) v += R[int64_t(m) * a.ldr + n];
      C[remap_row(m, a.c_grp, a.c_gstride, a.c_goff) * a.ldc + n] = v;
    }
  }
}

// LayerNorm, one warp per row, d <= 1024; two-pass variance.
__global__ void layer_norm_kernel(const float* __restrict__ x, int64_t ldx, float* __restrict__ y, int64_t ldy,
                                  int rows, int d, const float* __restrict__ gamma, const float* __restrict__ beta,
                                  float eps) {
  griddep_wait();
  griddep_launch();
  const int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  float v[32];
  const float* xr = x + int64_t(row) * ldx;
  float sum = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const int c = lane + 32 * i;
    v[i] = c < d ? xr[c] : 0.f;
    sum += v[i];
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
  const float mean = sum / d;
  float sq = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const int c = lane + 32 * i;
    if (c < d) {
      const float t = v[i] - mean;
      sq += t * t;
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, off);
  const float rstd = 1.0f / sqrtf(sq / d + eps);
  float* yr = y + int64_t(row) * ldy;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const int c = lane + 32 * i;
    if (c < d) yr[c] = (v[i] - mean) * rstd * gamma[c] + beta[c];
  }
}

// Exclusive scan of B lengths in one block; validates signs and the total. Every offset,
// offsets[B] included, is clamped to `expected` (the caller's declared total, which sized its
// buffers), so that lengths which sum above it are reported but can never send a later kernel
// past the end of an id, row or output buffer. Negative lengths count as 0.
__global__ void offsets_kernel(const int32_t* __restrict__ lengths, int B, int32_t* __restrict__ offsets,
                               int expected, int32_t* err) {
  griddep_wait();
  griddep_launch();
  __shared__ long long warp_sums[32];
  __shared__ long long carry;
  const long long cap = expected > 0 ? expected : 0;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) carry = 0;
  __syncthreads();
  for (int base = 0; base < B; base += blockDim.x) {
    const int i = base + tid;
    long long v = 0;
    if (i < B) {
      v = lengths[i];
      if (v < 0) {
        set_error(err, STCA_ERR_BAD_LENGTHS);
        v = 0;
      }
    }
    long long incl = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const long long n = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += n;
    }
    if (lane == 31) warp_sums[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      long long ws = lane < (blockDim.x >> 5) ? warp_sums[lane] : 0;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const long long n = __shfl_up_sync(0xffffffffu, ws, off);
        if (lane >= off) ws += n;
      }
      warp_sums[lane] = ws;
    }
    __syncthreads();
    const long long excl = carry + (warp > 0 ? warp_sums[warp - 1] : 0) + incl - v;
    if (i < B) offsets[i] = int32_t(excl < cap ? excl : cap);
    __syncthreads();
    if (tid == 0) carry += warp_sums[(blockDim.x >> 5) - 1];
    __syncthreads();
  }
  if (tid == 0) {
    offsets[B] = int32_t(carry < cap ? carry : cap);
    if (carry != expected) set_error(err, STCA_ERR_BAD_LENGTHS);
  }
}

template <typename T>
__global__ void copy_rows_kernel(const T* __restrict__ src, int rows, int d, float* __restrict__ dst, int64_t ldd,
                                 int col0) {
  griddep_wait();
  griddep_launch();
  const int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= int64_t(rows) * d) return;
  const int64_t r = i / d;
  const int c = int(i % d);
  dst[r * ldd + col0 + c] = to_f<T>(src[i]);
}

__global__ void token_mix_kernel(const float* __restrict__ Q, int B, int T, int d, float* __restrict__ out) {
  griddep_wait();
  griddep_launch();
  const int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= int64_t(B) * T * d) return;
  const int sub = d / T;
  const int64_t b = i / (int64_t(T) * d);
  const int rem = int(i % (int64_t(T) * d));
  const int hh = rem / d, col = rem % d;   // output token hh, column col = t*sub + j
  const int t = col / sub, j = col % sub;
  out[i] = Q[(b * T + t) * d + hh * sub + j];
}

__global__ void arange_kernel(int32_t* out, int n, int step) {
  griddep_wait();
  griddep_launch();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) out[i] = i * step;
}

}  // namespace

int fill_arange(int32_t* out, int n, int step, cudaStream_t s) {
  if (n <= 0) return 0;
  launch_dep(arange_kernel, dim3((n + 255) / 256), dim3(256), 0, s, out, n, step); note_launch();
  return cudaGetLastError() == cudaSuccess ? 0 : STCA_ERR_CUDA;
}

template <typename TA, typename TB>
int simt_gemm(const SimtGemmArgs<TA, TB>& a, cudaStream_t s) {
  if (a.M == 0 || a.N == 0 || a.batch == 0) return 0;
  if (a.M < 0 || a.N < 0 || a.K <= 0) return STCA_ERR_INVALID_ARG;
  if constexpr (std::is_same<TA, float>::value && std::is_same<TB, bf16>::value) {
    if (query_gemm_supported(a)) return query_gemm(a, s);
  }
  dim3 grid((a.N + SB_N - 1) / SB_N, (a.M + SB_M - 1) / SB_M, a.batch);
  if (a.B2) simt_gemm_kernel<TA, TB, true><<<grid, 256, 0, s>>>(a);
  else simt_gemm_kernel<TA, TB, false><<<grid, 256, 0, s>>>(a);
  note_launch();
  return cudaGetLastError() == cudaSuccess ? 0 : STCA_ERR_CUDA;
}

template int simt_gemm<float, float>(const SimtGemmArgs<float, float>&, cudaStream_t);
template int simt_gemm<float, bf16>(const SimtGemmArgs<float, bf16>&, cudaStream_t);
template int simt_gemm<bf16, bf16>(const SimtGemmArgs<bf16, bf16>&, cudaStream_t);

int layer_norm_f32(const float* x, int64_t ldx, float* y, int64_t ldy, int rows, int d, const float* gamma,
                   const float* beta, float eps, cudaStream_t s) {
  if (rows == 0) return 0;
  if (d > 1024) return STCA_ERR_UNSUPPORTED;
  launch_dep(layer_norm_kernel, dim3((rows + 7) / 8), dim3(256), 0, s, x, ldx, y, ldy, rows, d, gamma, beta, eps);
  note_launch();
  return cudaGetLastError() == cudaSuccess ? 0 : STCA_ERR_CUDA;
}

int exclusive_offsets(const int32_t* lengths, int B, int32_t* offsets, int expected, int32_t* err, cudaStream_t s) {
  launch_dep(offsets_kernel, dim3(1), dim3(1024), 0, s, lengths, B, offsets, expected, err); note_launch();
  return cudaGetLastError() == cudaSuccess ? 0 : STCA_ERR_CUDA;
}

int copy_rows_to_f32(const void* src, int src_bf16, int rows, int d, float* dst, int64_t ldd, int col0,
                     cudaStream_t s) {
  const int64_t n = int64_t(rows) * d;
  if (n == 0) return 0;
  const int blocks = int((n + 255) / 256);
  if (src_bf16)
    launch_dep(copy_rows_kernel<bf16>, dim3(blocks), dim3(256), 0, s, reinterpret_cast<const bf16*>(src), rows, d, dst,
               ldd, col0);
  else
    launch_dep(copy_rows_kernel<float>, dim3(blocks), dim3(256), 0, s, reinterpret_cast<const float*>(src), rows, d, dst,
               ldd, col0);
  note_launch();
  return cudaGetLastError() == cudaSuccess ? 0 : STCA_ERR_CUDA;
}

int token_mix(const float* Q, int B, int T, int d, float* mixed, cudaStream_t s) {
  const int64_t n = int64_t(B) * T * d;
  if (n == 0) return 0;
  launch_dep(token_mix_kernel, dim3(int((n + 255) / 256)), dim3(256), 0, s, Q, B, T, d, mixed); note_launch();
  return cudaGetLastError() == cudaSuccess ? 0 : STCA_ERR_CUDA;
}

}  // namespace stca
