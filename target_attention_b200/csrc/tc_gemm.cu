// tcgen05 / TMEM bf16 GEMMs for the history side of STCA.
//
// Per layer the history tokens go through (STCA notes, section "STCA"; review §三):
//   A  = SiLU(X W1) * (X W3)          X gathered from the item table, SwiGLU epilogue
//   X~ = LN(A W2)                     LayerNorm over the full d-wide row in the epilogue
//   [K | V] = X~ [W_K | W_V]          plain epilogue
// All three are dense bf16 contractions with fp32 accumulation in tensor memory.
//
// Tiles are 128 rows (one token per TMEM lane) by up to 512 columns.  Operands sit in
// shared memory as K-major rows of 128 bytes with the 128-byte swizzle; TMA writes that
// layout for dense operands, and the fused gather producer writes it with cp.async.
//
// Warp roles (384 threads): warp 0 lane 0 issues TMA, warp 1 owns TMEM and lane 0
// issues tcgen05.mma, warps 4..11 gather A rows and run the epilogue, two warps per TMEM
// lane quarter (warp w reads lanes 32 (w % 4) .. + 32), each on half of the columns.
// Waits are bounded (see common.cuh).
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace stca {

namespace {

constexpr int BM = 128;                        // tile rows = TMEM lanes
constexpr int A_CHUNK = BM * 64 * 2;           // one 64-wide K chunk of A: 16 KB
constexpr int B_BOX_ROWS = 256;                // TMA box height for weights
constexpr int B_STAGE_256 = B_BOX_ROWS * 128;  // 256 weight rows x 64 K: 32 KB
constexpr int MIN_SMEM = 120 * 1024;           // keeps one CTA per SM (TMEM is not shared)

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

__device__ __forceinline__ bool abort_set(volatile int* f) { return *f != 0; }

__device__ __forceinline__ void fail(volatile int* f, int32_t* err) {
  *f = 1;
  set_error(err, STCA_ERR_TIMEOUT);
}

// Waits for every load the producer issued into `stages` ring slots (bounded).
__device__ __forceinline__ void drain_ring(uint64_t* full, int stages, int issued) {
  for (int s = 0; s < stages && s < issued; ++s) {
    const int last = s + stages * ((issued - 1 - s) / stages);
    mbar_wait(&full[s], (last / stages) & 1);
  }
}

// Epilogue store of 32 consecutive fp32 values as bf16 (64 bytes, 16-byte aligned).
__device__ __forceinline__ void store_bf16x32(bf16* dst, const float (&v)[32]) {
  uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint4 u;
    u.x = pack_bf16x2(v[8 * q + 0], v[8 * q + 1]);
    u.y = pack_bf16x2(v[8 * q + 2], v[8 * q + 3]);
    u.z = pack_bf16x2(v[8 * q + 4], v[8 * q + 5]);
    u.w = pack_bf16x2(v[8 * q + 6], v[8 * q + 7]);
    d4[q] = u;
  }
}

// Gather producer, 256 threads: thread (r, half) loads 16-byte chunks [4 half, 4 half + 4)
// of row r of the A tile for every K chunk, with cp.async into the swizzled K-major
// layout, then (time feature) adds the bucket row, and releases chunk kc on a_full[kc]
// as soon as its own copies have landed.
__device__ __forceinline__ void gather_a_tile(const GatherSrc& g, uint8_t* sA, uint64_t* a_full, int m0,
                                              int M, int K, int r, int half, int32_t* err) {
  const int KC = K / 64;
  const int grow = m0 + r;
  bool valid = grow < M;
  int64_t id = 0;
  int bucket = 0;
  if (valid) {
    id = g.ids[grow];
    if (id < 0 || id >= g.n_items) {
      set_error(err, STCA_ERR_ID_OUT_OF_RANGE);
      valid = false;
      id = 0;
    }
    if (g.dt) {
      const int32_t dt = g.dt[grow];
      if (dt < 0) set_error(err, STCA_ERR_INVALID_ARG);
      bucket = dt_bucket(dt < 0 ? 0 : dt);
    }
  }
  const bf16* src = reinterpret_cast<const bf16*>(g.table) + id * int64_t(K) + half * 32;
  const uint32_t nbytes = valid ? 16u : 0u;
  for (int kc = 0; kc < KC; ++kc) {
    uint8_t* rowp = sA + kc * A_CHUNK + r * 128;
#pragma unroll
    for (int c = 0; c < 4; ++c)
      cp_async_16(rowp + (((half * 4 + c) ^ (r & 7)) << 4), src + kc * 64 + c * 8, nbytes);
    cp_async_commit();
  }
  const bf16* trow = (g.dt_table != nullptr && grow < M)
                         ? reinterpret_cast<const bf16*>(g.dt_table) + int64_t(bucket) * K + half * 32
                         : nullptr;
  uint4 t[4];
  if (trow != nullptr)
#pragma unroll
    for (int c = 0; c < 4; ++c) t[c] = __ldg(reinterpret_cast<const uint4*>(trow) + c);
  for (int kc = 0; kc < KC; ++kc) {
    cp_async_wait_dyn(KC - 1 - kc);
    if (trow != nullptr) {
      uint4 tn[4];
      if (kc + 1 < KC)
#pragma unroll
        for (int c = 0; c < 4; ++c) tn[c] = __ldg(reinterpret_cast<const uint4*>(trow + (kc + 1) * 64) + c);
      uint8_t* rowp = sA + kc * A_CHUNK + r * 128;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint4* p = reinterpret_cast<uint4*>(rowp + (((half * 4 + c) ^ (r & 7)) << 4));
        uint4 x = *p;
        const __nv_bfloat162* xa = reinterpret_cast<const __nv_bfloat162*>(&x);
        const __nv_bfloat162* ta = reinterpret_cast<const __nv_bfloat162*>(&t[c]);
        uint32_t o[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 xf = __bfloat1622float2(xa[e]);
          const float2 tf = __bfloat1622float2(ta[e]);
          o[e] = pack_bf16x2(xf.x + tf.x, xf.y + tf.y);
        }
        *p = make_uint4(o[0], o[1], o[2], o[3]);
      }
      if (kc + 1 < KC)
#pragma unroll
        for (int c = 0; c < 4; ++c) t[c] = tn[c];
    }
    fence_proxy_async_smem();
    mbar_arrive(&a_full[kc]);
  }
}

// SiLU(x) = x sigmoid(x) = h + h tanh(h) with h = x/2: one MUFU op per element.
__device__ __forceinline__ float silu_tanh(float x) {
  const float h = 0.5f * x;
  float t;
  asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(h));
  return fmaf(h, t, h);
}

// Named barrier over the 256 epilogue threads (warps 4..11).
__device__ __forceinline__ void epilogue_sync() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

// ------------------------------------------------------------------------------------
// Kernel R: A resident in shared memory (K <= 512), N walked in 256-column tiles with a
// double-buffered TMEM accumulator so the epilogue of tile n overlaps the MMAs of n+1.

template <int AMODE, int EPI, int STAGES>
__global__ void __launch_bounds__(384, 1)
    tc_gemm_resident_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                            GatherSrc g, int M, int K, int NT, bf16* __restrict__ C, int ldc, int32_t* err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  const int KC = K / 64;
  uint8_t* sA = smem;
  uint8_t* sB = smem + KC * A_CHUNK;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + STAGES * B_STAGE_256);
  uint64_t* a_full = bars;                 // [8]
  uint64_t* b_full = bars + 8;             // [STAGES]
  uint64_t* b_empty = b_full + STAGES;     // [STAGES]
  uint64_t* t_full = b_empty + STAGES;     // [2]
  uint64_t* t_empty = t_full + 2;          // [2]
  uint64_t* mma_done = t_empty + 2;        // [1]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * BM;

  if (threadIdx.x == 0) {
    for (int i = 0; i < KC; ++i) mbar_init(&a_full[i], AMODE == A_GATHER ? 256 : 1);
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&b_full[s], 1);
      mbar_init(&b_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&t_full[i], 1);
      mbar_init(&t_empty[i], 256);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      if (AMODE == A_TMA) prefetch_tmap(&tmA);
      prefetch_tmap(&tmB);
      if (AMODE == A_TMA) {
        for (int kc = 0; kc < KC; ++kc) {
          mbar_arrive_expect_tx(&a_full[kc], A_CHUNK);
          tma_load_2d(sA + kc * A_CHUNK, &tmA, kc * 64, m0, &a_full[kc]);
        }
      }
      int it = 0;
      const int total = NT * KC;
      for (; it < total; ++it) {
        const int s = it % STAGES;
        const int round = it / STAGES;
        if (round > 0 && !mbar_wait(&b_empty[s], (round - 1) & 1)) {
          fail(abort_flag, err);
          break;
        }
        if (abort_set(abort_flag)) break;
        const int nt = it / KC, kc = it % KC;
        mbar_arrive_expect_tx(&b_full[s], B_STAGE_256);
        tma_load_2d(sB + s * B_STAGE_256, &tmB, kc * 64, nt * 256, &b_full[s]);
      }
      drain_ring(b_full, STAGES, it);
      if (AMODE == A_TMA)
        for (int kc = 0; kc < KC; ++kc) mbar_wait(&a_full[kc], 0);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = umma_idesc_bf16(128, 256);
      int it = 0;
      bool ok = true;
      for (int nt = 0; nt < NT && ok; ++nt) {
        const int buf = nt & 1, use = nt >> 1;
        if (use > 0 && !mbar_wait(&t_empty[buf], (use - 1) & 1)) {
          fail(abort_flag, err);
          break;
        }
        tc_fence_after();
        const uint32_t dcol = tmem + buf * 256;
        for (int kc = 0; kc < KC; ++kc, ++it) {
          const int s = it % STAGES;
          if ((nt == 0 && !mbar_wait(&a_full[kc], 0)) || !mbar_wait(&b_full[s], (it / STAGES) & 1) ||
              abort_set(abort_flag)) {
            fail(abort_flag, err);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sA + kc * A_CHUNK);
          const uint32_t b_addr = smem_u32(sB + s * B_STAGE_256);
#pragma unroll
          for (int k = 0; k < 4; ++k)
            umma_bf16(dcol, umma_sdesc_sw128(a_addr + k * 32), umma_sdesc_sw128(b_addr + k * 32), idesc,
                      (kc | k) != 0);
          umma_commit(&b_empty[s]);
        }
        if (ok) umma_commit(&t_full[buf]);
      }
      umma_commit(mma_done);
      mbar_wait(mma_done, 0);
    }
  } else if (warp >= 4) {
    // two epilogue warps per TMEM lane quarter, each taking half of the columns
    const int quarter = warp & 3;
    const int half = (warp - 4) >> 2;
    const int r = quarter * 32 + lane;  // tile row == TMEM lane
    if (AMODE == A_GATHER) gather_a_tile(g, sA, a_full, m0, M, K, r, half, err);
    const int grow = m0 + r;
    const uint32_t lane_base = tmem + (uint32_t(quarter * 32) << 16);
    for (int nt = 0; nt < NT; ++nt) {
      const int buf = nt & 1, use = nt >> 1;
      if (!mbar_wait(&t_full[buf], use & 1) || abort_set(abort_flag)) {
        fail(abort_flag, err);
        break;
      }
      tc_fence_after();
      const uint32_t tb = lane_base + buf * 256;
      if (EPI == EPI_SWIGLU) {
#pragma unroll 1
        for (int j = 0; j < 2; ++j) {
          const int col = half * 64 + j * 32;
          float gv[32], uv[32];
          tmem_ld_32x32b_x32(tb + col, gv);
          tmem_ld_32x32b_x32(tb + 128 + col, uv);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) gv[e] = silu_tanh(gv[e]) * uv[e];
          if (grow < M) store_bf16x32(C + int64_t(grow) * ldc + nt * 128 + col, gv);
        }
      } else {
#pragma unroll 1
        for (int j = 0; j < 4; ++j) {
          const int col = half * 128 + j * 32;
          float v[32];
          tmem_ld_32x32b_x32(tb + col, v);
          tmem_ld_wait();
          if (grow < M) store_bf16x32(C + int64_t(grow) * ldc + nt * 256 + col, v);
        }
      }
      tc_fence_before();
      mbar_arrive(&t_empty[buf]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------------------------
// Kernel S: A and B streamed through a STAGES-deep ring, the full output row (NB x 256
// columns) accumulated in TMEM, then LayerNorm (or a plain store) per row.

template <int EPI, int NB, int STAGES>
__global__ void __launch_bounds__(384, 1)
    tc_gemm_rowwise_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                           int M, int K, bf16* __restrict__ C, int ldc, const float* __restrict__ gamma,
                           const float* __restrict__ beta, float eps, int32_t* err) {
  constexpr int N = NB * 256;
  constexpr int STAGE_BYTES = A_CHUNK + NB * B_STAGE_256;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
  uint64_t* full = bars;                  // [STAGES]
  uint64_t* empty = bars + STAGES;        // [STAGES]
  uint64_t* t_full = empty + STAGES;      // [1]
  uint64_t* mma_done = t_full + 1;        // [1]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* s_gamma = reinterpret_cast<float*>(bars + 2 * STAGES + 8);  // [N]
  float* s_beta = s_gamma + N;                                       // [N]
  float* s_red = s_beta + N;                                         // [2][128]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * BM;
  const int KC = K / 64;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(t_full, 1);
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, N);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      prefetch_tmap(&tmA);
      prefetch_tmap(&tmB);
      int it = 0;
      for (; it < KC; ++it) {
        const int s = it % STAGES, round = it / STAGES;
        if (round > 0 && !mbar_wait(&empty[s], (round - 1) & 1)) {
          fail(abort_flag, err);
          break;
        }
        if (abort_set(abort_flag)) break;
        uint8_t* st = smem + s * STAGE_BYTES;
        mbar_arrive_expect_tx(&full[s], STAGE_BYTES);
        tma_load_2d(st, &tmA, it * 64, m0, &full[s]);
#pragma unroll
        for (int nb = 0; nb < NB; ++nb)
          tma_load_2d(st + A_CHUNK + nb * B_STAGE_256, &tmB, it * 64, nb * 256, &full[s]);
      }
      drain_ring(full, STAGES, it);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = umma_idesc_bf16(128, 256);
      bool ok = true;
      for (int it = 0; it < KC; ++it) {
        const int s = it % STAGES;
        if (!mbar_wait(&full[s], (it / STAGES) & 1) || abort_set(abort_flag)) {
          fail(abort_flag, err);
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a_addr = smem_u32(smem + s * STAGE_BYTES);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
#pragma unroll
          for (int nb = 0; nb < NB; ++nb) {
            const uint32_t b_addr = a_addr + A_CHUNK + nb * B_STAGE_256;
            umma_bf16(tmem + nb * 256, umma_sdesc_sw128(a_addr + k * 32), umma_sdesc_sw128(b_addr + k * 32),
                      idesc, (it | k) != 0);
          }
        }
        umma_commit(&empty[s]);
      }
      if (ok) umma_commit(t_full);
      umma_commit(mma_done);
      mbar_wait(mma_done, 0);
    }
  } else if (warp >= 4) {
    const int quarter = warp & 3;
    const int half = (warp - 4) >> 2;
    const int r = quarter * 32 + lane;
    const int grow = m0 + r;
    const int et = threadIdx.x - 128;
    constexpr int HN = N / 2;  // columns per epilogue warp
    if (EPI == EPI_LN) {
      for (int c = et; c < N; c += 256) {
        s_gamma[c] = gamma[c];
        s_beta[c] = beta[c];
      }
    }
    const uint32_t tb = tmem + (uint32_t(quarter * 32) << 16) + half * HN;
    const bool ok = mbar_wait(t_full, 0) && !abort_set(abort_flag);
    if (!ok) fail(abort_flag, err);
    tc_fence_after();
    bf16* crow = C + int64_t(grow) * ldc + half * HN;
    if (EPI == EPI_LN) {
      float sum = 0.f;
      if (ok) {
#pragma unroll 1
        for (int j = 0; j < HN / 32; ++j) {
          float v[32];
          tmem_ld_32x32b_x32(tb + j * 32, v);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) sum += v[e];
        }
      }
      s_red[half * 128 + r] = sum;
      epilogue_sync();
      const float mean = (s_red[r] + s_red[128 + r]) * (1.0f / N);
      float sq = 0.f;
      if (ok) {
#pragma unroll 1
        for (int j = 0; j < HN / 32; ++j) {
          float v[32];
          tmem_ld_32x32b_x32(tb + j * 32, v);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const float t = v[e] - mean;
            sq = fmaf(t, t, sq);
          }
        }
      }
      epilogue_sync();  // everyone has read the sums before they are overwritten
      s_red[half * 128 + r] = sq;
      epilogue_sync();
      const float rstd = rsqrtf((s_red[r] + s_red[128 + r]) * (1.0f / N) + eps);
      if (ok) {
        const float* gm = s_gamma + half * HN;
        const float* bt = s_beta + half * HN;
#pragma unroll 1
        for (int j = 0; j < HN / 32; ++j) {
          float v[32];
          tmem_ld_32x32b_x32(tb + j * 32, v);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = fmaf((v[e] - mean) * rstd, gm[j * 32 + e], bt[j * 32 + e]);
          if (grow < M) store_bf16x32(crow + j * 32, v);
        }
      }
    } else if (ok) {
#pragma unroll 1
      for (int j = 0; j < HN / 32; ++j) {
        float v[32];
        tmem_ld_32x32b_x32(tb + j * 32, v);
        tmem_ld_wait();
        if (grow < M) store_bf16x32(crow + j * 32, v);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, N);
  }
}

// ------------------------------------------------------------------------------------
// weight packing: [K, N] row-major -> K-major rows

__global__ void pack_weight_kernel(const bf16* __restrict__ W, int K, int N, bf16* __restrict__ dst, int mode,
                                   int row_offset) {
  __shared__ bf16 tile[32][33];
  const int k0 = blockIdx.y * 32, n0 = blockIdx.x * 32;
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int k = k0 + i, n = n0 + threadIdx.x;
    tile[i][threadIdx.x] = (k < K && n < N) ? W[int64_t(k) * N + n] : __float2bfloat16(0.f);
  }
  __syncthreads();
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int n = n0 + i, k = k0 + threadIdx.x;
    if (n < N && k < K) {
      int row;
      if (mode == 0) row = row_offset + n;
      else row = (n / 128) * 256 + (mode == 2 ? 128 : 0) + (n % 128);
      dst[int64_t(row) * K + k] = tile[threadIdx.x][i];
    }
  }
}

// ------------------------------------------------------------------------------------
// host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D bf16 tensor map over a [rows, cols] row-major matrix (row stride ld elements),
// box = 64 columns x box_rows rows, 128-byte swizzle, zero fill outside the matrix.
bool make_tmap(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint64_t ld, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {ld * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

size_t resident_smem(int K, int stages) {
  size_t bytes = 1024 + size_t(K / 64) * A_CHUNK + size_t(stages) * B_STAGE_256 + 256;
  return bytes < MIN_SMEM ? MIN_SMEM : bytes;
}

size_t rowwise_smem(int nb, int stages) {
  size_t bytes = 1024 + size_t(stages) * (A_CHUNK + nb * B_STAGE_256) + 256 + 2 * nb * 256 * 4 + 2 * 128 * 4;
  return bytes < MIN_SMEM ? MIN_SMEM : bytes;
}

template <int AMODE, int EPI, int STAGES>
int run_resident(const CUtensorMap& ta, const CUtensorMap& tb, const GatherSrc& g, int M, int K, int NT, void* C,
                 int ldc, int32_t* err, cudaStream_t s) {
  auto kern = tc_gemm_resident_kernel<AMODE, EPI, STAGES>;
  const size_t smem = resident_smem(K, STAGES);
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) != cudaSuccess)
    return STCA_ERR_CUDA;
  const int grid = (M + BM - 1) / BM;
  kern<<<grid, 384, smem, s>>>(ta, tb, g, M, K, NT, reinterpret_cast<bf16*>(C), ldc, err); note_launch();
  return cudaGetLastError() == cudaSuccess ? 0 : STCA_ERR_CUDA;
}

template <int EPI, int NB, int STAGES>
int run_rowwise(const CUtensorMap& ta, const CUtensorMap& tb, int M, int K, void* C, int ldc, const float* gamma,
                const float* beta, float eps, int32_t* err, cudaStream_t s) {
  auto kern = tc_gemm_rowwise_kernel<EPI, NB, STAGES>;
  const size_t smem = rowwise_smem(NB, STAGES);
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) != cudaSuccess)
    return STCA_ERR_CUDA;
  const int grid = (M + BM - 1) / BM;
  kern<<<grid, 384, smem, s>>>(ta, tb, M, K, reinterpret_cast<bf16*>(C), ldc, gamma, beta, eps, err); note_launch();
  return cudaGetLastError() == cudaSuccess ? 0 : STCA_ERR_CUDA;
}

}  // namespace

int tc_pack_weight(const void* W, int K, int N, void* dst, int mode, int row_offset, cudaStream_t s) {
  if (K <= 0 || N <= 0) return STCA_ERR_INVALID_ARG;
  dim3 grid((N + 31) / 32, (K + 31) / 32), block(32, 8);
  pack_weight_kernel<<<grid, block, 0, s>>>(reinterpret_cast<const bf16*>(W), K, N, reinterpret_cast<bf16*>(dst),
                                            mode, row_offset); note_launch();
  return cudaGetLastError() == cudaSuccess ? 0 : STCA_ERR_CUDA;
}

int tc_gemm_resident(int amode, int epi, const void* A, GatherSrc g, int M, int K, const void* Wp, int Nout,
                     void* C, int ldc, int32_t* err, cudaStream_t s) {
  if (M == 0) return 0;
  if (M < 0 || (K != 256 && K != 512) || Nout <= 0 || ldc % 8 != 0) return STCA_ERR_UNSUPPORTED;
  const int N = epi == EPI_SWIGLU ? 2 * Nout : Nout;
  if (N % 256 != 0) return STCA_ERR_UNSUPPORTED;
  const int NT = N / 256;
  CUtensorMap ta, tb;
  memset(&ta, 0, sizeof(ta));
  if (!make_tmap(&tb, Wp, N, K, K, B_BOX_ROWS)) return STCA_ERR_CUDA;
  if (amode == A_TMA) {
    if (!make_tmap(&ta, A, M, K, K, BM)) return STCA_ERR_CUDA;
  } else {
    ta = tb;  // unused by the gather producer
  }
#define STCA_RES(AM, EP)                                                                  \
  (K == 512 ? run_resident<AM, EP, 3>(ta, tb, g, M, K, NT, C, ldc, err, s)               \
            : run_resident<AM, EP, 5>(ta, tb, g, M, K, NT, C, ldc, err, s))
  if (amode == A_TMA && epi == EPI_PLAIN) return STCA_RES(A_TMA, EPI_PLAIN);
  if (amode == A_TMA && epi == EPI_SWIGLU) return STCA_RES(A_TMA, EPI_SWIGLU);
  if (amode == A_GATHER && epi == EPI_PLAIN) return STCA_RES(A_GATHER, EPI_PLAIN);
  if (amode == A_GATHER && epi == EPI_SWIGLU) return STCA_RES(A_GATHER, EPI_SWIGLU);
#undef STCA_RES
  return STCA_ERR_UNSUPPORTED;
}

int tc_gemm_rowwise(int epi, const void* A, int M, int K, const void* Wp, int N, const float* gamma,
                    const float* beta, float eps, void* C, int ldc, int32_t* err, cudaStream_t s) {
  if (M == 0) return 0;
  if (M < 0 || K <= 0 || K % 64 != 0 || (N != 256 && N != 512) || ldc % 8 != 0) return STCA_ERR_UNSUPPORTED;
  if (epi == EPI_LN && (!gamma || !beta)) return STCA_ERR_INVALID_ARG;
  CUtensorMap ta, tb;
  if (!make_tmap(&ta, A, M, K, K, BM)) return STCA_ERR_CUDA;
  if (!make_tmap(&tb, Wp, N, K, K, B_BOX_ROWS)) return STCA_ERR_CUDA;
  if (N == 512) {
    return epi == EPI_LN ? run_rowwise<EPI_LN, 2, 2>(ta, tb, M, K, C, ldc, gamma, beta, eps, err, s)
                         : run_rowwise<EPI_PLAIN, 2, 2>(ta, tb, M, K, C, ldc, gamma, beta, eps, err, s);
  }
  return epi == EPI_LN ? run_rowwise<EPI_LN, 1, 4>(ta, tb, M, K, C, ldc, gamma, beta, eps, err, s)
                       : run_rowwise<EPI_PLAIN, 1, 4>(ta, tb, M, K, C, ldc, gamma, beta, eps, err, s);
}

}  // namespace stca
