// Pointwise ReLU target attention with the embedding lookup fused in (WeChat TA article,
// §1.1 low-memory TA operator and §1.2 element-wise ReLU scores):
//   out[b] = sum_{j < L_b} relu(q_b . e_j / sqrt(D)) e_j,   e_j = table[ids_b[j]]
// Each looked-up row is read once from HBM and used as both key and value; the
// gathered [B, L, D] matrix never exists.  D = 128 (256-byte bf16 rows): a half-warp
// holds one row, 16 bytes per lane, and reduces the dot product with 4 shuffles.
#include "common.cuh"
#include "internal.h"

namespace stca {

namespace {

constexpr int PD = 128;          // row width
constexpr int PW_THREADS = 256;  // 16 half-warps
constexpr int UNROLL = 4;

__device__ __forceinline__ void bf16x8_to_f32(const uint4& u, float (&f)[8]) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 t = __bfloat1622float2(h[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}

// One CTA per (sample b, slice s).  dst = partials + s*B*D (or out when splits == 1).
__global__ void __launch_bounds__(PW_THREADS) pointwise_kernel(const int32_t* __restrict__ ids,
                                                               const int32_t* __restrict__ offsets,
                                                               const bf16* __restrict__ q,
                                                               const bf16* __restrict__ table, int64_t n_items,
                                                               int B, int splits, float* __restrict__ dst,
                                                               int32_t* err) {
  __shared__ float red[PW_THREADS / 16][PD];
  const int b = blockIdx.x / splits, s = blockIdx.x % splits;
  const int tid = threadIdx.x, hw = tid >> 4, li = tid & 15;
  const int64_t beg = offsets[b], end = offsets[b + 1];
  const int64_t L = end - beg;
  const int64_t j0 = beg + (L * s) / splits, j1 = beg + (L * (s + 1)) / splits;

  float qf[8];
  {
    const uint4 qu = __ldg(reinterpret_cast<const uint4*>(q + int64_t(b) * PD) + li);
    bf16x8_to_f32(qu, qf);
    const float sc = rsqrtf(float(PD));
#pragma unroll
    for (int i = 0; i < 8; ++i) qf[i] *= sc;
  }
  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.f;

  const uint4* tab4 = reinterpret_cast<const uint4*>(table);
  // Rows j0 + 16*k + hw for k = 0, 1, ...; the loop bound is warp-uniform so both
  // half-warps run the same iterations (the shuffles below use the full mask).  The ids of
  // the next UNROLL rows are loaded while this iteration's rows are in flight, so a row
  // load waits on one memory latency, not on an id load and then a row load.
  constexpr int STEP = PW_THREADS / 16;
  const int warp_first = 2 * (tid >> 5);
  const int64_t first = j0 + warp_first + (hw & 1);
  int idn[UNROLL];
#pragma unroll
  for (int u = 0; u < UNROLL; ++u) {
    const int64_t jj = first + int64_t(u) * STEP;
    idn[u] = jj < j1 ? __ldg(ids + jj) : 0;
  }
  for (int64_t base = j0 + warp_first; base < j1; base += STEP * UNROLL) {
    uint4 row[UNROLL];
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      const int64_t jj = base + int64_t(u) * STEP + (hw & 1);
      bool ok = jj < j1;
      int64_t id = idn[u];
      if (ok && (id < 0 || id >= n_items)) {
        set_error(err, STCA_ERR_ID_OUT_OF_RANGE);
        ok = false;
      }
      row[u] = ok ? __ldg(tab4 + id * (PD / 8) + li) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      const int64_t jj = base + int64_t(STEP * UNROLL) + int64_t(u) * STEP + (hw & 1);
      idn[u] = jj < j1 ? __ldg(ids + jj) : 0;
    }
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      float e[8];
      bf16x8_to_f32(row[u], e);
      float dot = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) dot = fmaf(qf[i], e[i], dot);
      dot += __shfl_xor_sync(0xffffffffu, dot, 8);
      dot += __shfl_xor_sync(0xffffffffu, dot, 4);
      dot += __shfl_xor_sync(0xffffffffu, dot, 2);
      dot += __shfl_xor_sync(0xffffffffu, dot, 1);
      const float w = fmaxf(dot, 0.f);
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = fmaf(w, e[i], acc[i]);
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) red[hw][li * 8 + i] = acc[i];
  __syncthreads();
  if (tid < PD) {
    float v = 0.f;
#pragma unroll
    for (int r = 0; r < PW_THREADS / 16; ++r) v += red[r][tid];
    dst[(int64_t(s) * B + b) * PD + tid] = v;
  }
}

__global__ void pointwise_sum_kernel(const float* __restrict__ partials, int B, int splits, float* __restrict__ out) {
  const int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= int64_t(B) * PD) return;
  float v = 0.f;
  for (int s = 0; s < splits; ++s) v += partials[int64_t(s) * B * PD + i];
  out[i] = v;
}

}  // namespace

int pointwise_relu_ta(const int32_t* ids, const int32_t* offsets, const void* q, const void* table, int64_t n_items,
                      int B, int D, int splits, float* partials, float* out, int32_t* err, cudaStream_t s) {
  if (B == 0) return 0;
  if (D != PD || splits < 1) return STCA_ERR_UNSUPPORTED;
  float* dst = splits == 1 ? out : partials;
  pointwise_kernel<<<B * splits, PW_THREADS, 0, s>>>(ids, offsets, reinterpret_cast<const bf16*>(q),
                                                      reinterpret_cast<const bf16*>(table), n_items, B, splits, dst,
                                                      err); note_launch();
  if (cudaGetLastError() != cudaSuccess) return STCA_ERR_CUDA;
  if (splits > 1) {
    const int64_t n = int64_t(B) * PD;
    pointwise_sum_kernel<<<int((n + 255) / 256), 256, 0, s>>>(partials, B, splits, out); note_launch();
    if (cudaGetLastError() != cudaSuccess) return STCA_ERR_CUDA;
  }
  return 0;
}

}  // namespace stca
