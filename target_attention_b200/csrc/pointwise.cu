// Pointwise ReLU target attention with the embedding lookup fused in (WeChat TA article,
// §1.1 low-memory TA operator and §1.2 element-wise ReLU scores):
//   out[b] = sum_{j < L_b} relu(q_b . e_j / sqrt(D)) e_j,   e_j = table[ids_b[j]]
// Each looked-up row is read once from HBM and used as both key and value; the
// gathered [B, L, D] matrix never exists.  D = 128 (256-byte bf16 rows).
#include "common.cuh"
#include "internal.h"

namespace stca {

namespace {

constexpr int PD = 128;          // row width
constexpr int PW_THREADS = 256;  // 16 half-warps
constexpr int PW_RPS = 8;        // rows per half-warp per ring stage
constexpr int PW_STAGES = 3;     // ring stages (two in flight while one is read)
constexpr int PW_SMEM = PW_STAGES * PW_RPS * PW_THREADS * 16;  // 96 KB: two CTAs per SM

__device__ __forceinline__ void bf16x8_to_f32(const uint4& u, float (&f)[8]) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 t = __bfloat1622float2(h[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}

// 16-byte copy that also allocates in L1 (hot rows of a skewed id distribution are met
// again by the same SM).
__device__ __forceinline__ void cp_async_16_l1(void* smem_dst, const void* gsrc, uint32_t src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(smem_dst)), "l"(gsrc), "r"(src_bytes)
               : "memory");
}

// One CTA per (sample b, slice s).  dst = partials + s*B*D (or out when splits == 1).
//
// A half-warp holds one 256-byte row (16 bytes per lane) and reduces the dot product with
// 4 shuffles.  Rows travel through a ring of shared-memory stages: in stage k, half-warp hw
// takes rows base_k + hw + 16 r (r < PW_RPS) and lane li copies chunk li of each of them
// into its OWN slots, later reading back exactly what it copied, so no barrier is needed
// and the rows in flight per SM are set by the ring (about 128 KB), not by registers.  The
// ids of a stage are loaded (one per lane, coalesced across the CTA) one stage ahead and
// handed to the half-warp's lanes by shuffles.
__global__ void __launch_bounds__(PW_THREADS, 2) pointwise_kernel(const int32_t* __restrict__ ids,
                                                                  const int32_t* __restrict__ offsets,
                                                                  const bf16* __restrict__ q,
                                                                  const bf16* __restrict__ table, int64_t n_items,
                                                                  int B, int splits, float* __restrict__ dst,
                                                                  int32_t* err) {
  extern __shared__ __align__(16) uint4 ring[];  // [stage][r][thread]
  const int b = blockIdx.x / splits, s = blockIdx.x % splits;
  const int tid = threadIdx.x, hw = tid >> 4, li = tid & 15;
  const int64_t beg = offsets[b], end = offsets[b + 1];
  const int64_t L = end - beg;
  const int64_t j0 = beg + (L * s) / splits, j1 = beg + (L * (s + 1)) / splits;
  constexpr int ROWS_PER_STAGE = 16 * PW_RPS;
  const int n_st = int((j1 - j0 + ROWS_PER_STAGE - 1) / ROWS_PER_STAGE);

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

  // lane li < PW_RPS of half-warp hw loads the id of row hw + 16 li of stage k
  auto load_id = [&](int k) -> int {
    const int64_t jj = j0 + int64_t(k) * ROWS_PER_STAGE + hw + 16 * li;
    return (k < n_st && li < PW_RPS && jj < j1) ? __ldg(ids + jj) : 0;
  };
  auto issue = [&](int k, int myid) {
    if (k >= n_st) return;
    uint4* slot = ring + (k % PW_STAGES) * PW_RPS * PW_THREADS + tid;
#pragma unroll
    for (int r = 0; r < PW_RPS; ++r) {
      const int64_t id = __shfl_sync(0xffffffffu, myid, r, 16);
      const int64_t jj = j0 + int64_t(k) * ROWS_PER_STAGE + hw + 16 * r;
      bool ok = jj < j1;
      if (ok && (id < 0 || id >= n_items)) {
        set_error(err, STCA_ERR_ID_OUT_OF_RANGE);
        ok = false;
      }
      // rows past the slice or with a bad id land as zeros
      cp_async_16_l1(slot + r * PW_THREADS, tab4 + (ok ? id : 0) * (PD / 8) + li, ok ? 16u : 0u);
    }
  };

  int myid = load_id(0);
#pragma unroll
  for (int k = 0; k < PW_STAGES - 1; ++k) {
    issue(k, myid);
    myid = load_id(k + 1);
    cp_async_commit();
  }
  for (int k = 0; k < n_st; ++k) {
    cp_async_wait<PW_STAGES - 2>();  // this thread's copies of stage k have landed
    issue(k + PW_STAGES - 1, myid);
    myid = load_id(k + PW_STAGES);
    cp_async_commit();
    const uint4* slot = ring + (k % PW_STAGES) * PW_RPS * PW_THREADS + tid;
#pragma unroll
    for (int r = 0; r < PW_RPS; ++r) {
      float e[8];
      bf16x8_to_f32(slot[r * PW_THREADS], e);
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
  cp_async_wait_all();
  __syncthreads();
  float* red = reinterpret_cast<float*>(ring);  // [16 half-warps][PD]
#pragma unroll
  for (int i = 0; i < 8; ++i) red[hw * PD + li * 8 + i] = acc[i];
  __syncthreads();
  if (tid < PD) {
    float v = 0.f;
#pragma unroll
    for (int r = 0; r < PW_THREADS / 16; ++r) v += red[r * PD + tid];
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
  cudaFuncSetAttribute(pointwise_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, PW_SMEM);
  pointwise_kernel<<<B * splits, PW_THREADS, PW_SMEM, s>>>(ids, offsets, reinterpret_cast<const bf16*>(q),
                                                             reinterpret_cast<const bf16*>(table), n_items, B, splits,
                                                             dst, err); note_launch();
  if (cudaGetLastError() != cudaSuccess) return STCA_ERR_CUDA;
  if (splits > 1) {
    const int64_t n = int64_t(B) * PD;
    pointwise_sum_kernel<<<int((n + 255) / 256), 256, 0, s>>>(partials, B, splits, out); note_launch();
    if (cudaGetLastError() != cudaSuccess) return STCA_ERR_CUDA;
  }
  return 0;
}

}  // namespace stca
