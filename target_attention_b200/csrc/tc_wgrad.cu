// Weight gradients on the tensor cores (training): C [K, N] = A^T G, a reduction over the
// M token rows of two token-major bf16 matrices A [M, K] and G [M, N] (dW = X^T dY for
// every GEMM of the history side and the target side; the pages train STCA on ~2K-long
// histories: STCA notes, "短序列训练，长序列推理").
//
// Both operands are read as they lie in memory.  A TMA box of 64 tokens x 64 features
// with the 128-byte swizzle is, for the tensor cores, a canonical MN-major tile: the
// features (the MMA's M for A, N for G) run along the 128-byte rows and the tokens (the
// MMA's K) go down the rows, 8-row groups 1024 bytes apart.  The instruction descriptor
// marks A and B as MN-major, so no transpose is done anywhere.
//
// One CTA owns a 128 x BN tile of C (BN = 256 or 128 fp32 TMEM columns) and one slice of
// the tokens; slices start on 64-token stage boundaries, so only the last stage of the
// whole matrix is ragged (TMA fills rows past M with zeros).  Tokens stream through a
// 4-stage ring (16 KB of A + BN x 128 bytes of G per 64 tokens); warp 0 lane 0 issues TMA,
// warp 1 owns TMEM and its lane 0 issues four 128 x BN x 16 MMAs per stage.  The 4 warps
// then read the accumulator (warp w: rows 32 w .. 32 w + 31) and store the slice's
// partial tile; a second kernel adds the slices in a fixed order.  Every wait is bounded
// (common.cuh); a timeout sets STCA_ERR_TIMEOUT and the CTA winds down.
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace stca {

namespace {

constexpr int WT_M = 128;      // C rows per tile (features of A)
constexpr int WT_TOK = 64;     // tokens per stage
constexpr int WT_STAGES = 4;
constexpr int WT_BOX = WT_TOK * 64 * 2;  // one 64-token x 64-feature box: 8 KB
constexpr int WT_A = 2 * WT_BOX;         // A of one stage: 16 KB

template <int BN>
struct WtShape {
  static constexpr int B = (BN / 64) * WT_BOX;  // G of one stage
  static constexpr int STAGE = WT_A + B;
  static constexpr size_t SMEM = 1024 + size_t(WT_STAGES) * STAGE + 256;
};

// Shared-memory descriptor of an MN-major operand in 128-byte swizzled boxes: 64 features
// per 128-byte row, 8-token groups 1024 bytes apart (stride byte offset), 64-feature boxes
// WT_BOX bytes apart (leading byte offset).
__device__ __forceinline__ uint64_t sdesc_mn_sw128(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= uint64_t((smem_addr >> 4) & 0x3FFFu);
  d |= uint64_t(WT_BOX >> 4) << 16;
  d |= uint64_t(1024 >> 4) << 32;
  d |= uint64_t(1) << 46;
  d |= uint64_t(2) << 61;
  return d;
}

__device__ __forceinline__ uint8_t* wt_align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

template <int BN>
__global__ void __launch_bounds__(128, 1) tc_wgrad_kernel(const __grid_constant__ CUtensorMap tmA,
                                                          const __grid_constant__ CUtensorMap tmG, int M, int K,
                                                          int N, int splits, float* __restrict__ part,
                                                          int32_t* err) {
  constexpr int STAGE = WtShape<BN>::STAGE;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = wt_align1024(smem_raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + WT_STAGES * STAGE);
  uint64_t* full = bars;                   // [WT_STAGES] TMA bytes
  uint64_t* empty = bars + WT_STAGES;      // [WT_STAGES] MMA commit
  uint64_t* d_full = bars + 2 * WT_STAGES; // accumulator complete
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(d_full + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * BN, k0 = blockIdx.y * WT_M, z = blockIdx.z;
  const int S = (M + WT_TOK - 1) / WT_TOK;
  const int st0 = int(int64_t(S) * z / splits), nst = int(int64_t(S) * (z + 1) / splits) - st0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < WT_STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(d_full, 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmG);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, BN);
    tmem_relinquish();
  }
  griddep_wait();
  griddep_launch();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 && lane == 0) {
    int issued = 0;
    for (int i = 0; i < nst; ++i, ++issued) {
      const int s = i % WT_STAGES, round = i / WT_STAGES;
      if ((round > 0 && !mbar_wait(&empty[s], (round - 1) & 1)) || *abort_flag) {
        *abort_flag = 1;
        set_error(err, STCA_ERR_TIMEOUT);
        break;
      }
      uint8_t* sa = smem + s * STAGE;
      const int y = (st0 + i) * WT_TOK;
      mbar_arrive_expect_tx(&full[s], STAGE);
      tma_load_2d(sa, &tmA, k0, y, &full[s]);
      tma_load_2d(sa + WT_BOX, &tmA, k0 + 64, y, &full[s]);
#pragma unroll
      for (int c = 0; c < BN / 64; ++c) tma_load_2d(sa + WT_A + c * WT_BOX, &tmG, n0 + 64 * c, y, &full[s]);
    }
    // no copy may still be writing shared memory when the CTA exits
    for (int s = 0; s < WT_STAGES && s < issued; ++s) {
      const int last = s + WT_STAGES * ((issued - 1 - s) / WT_STAGES);
      mbar_wait(&full[s], (last / WT_STAGES) & 1);
    }
  } else if (warp == 1 && lane == 0) {
    // bf16 x bf16 -> fp32, M = 128, N = BN, A and B both MN-major
    constexpr uint32_t idesc = umma_idesc_bf16(WT_M, BN) | (1u << 15) | (1u << 16);
    const uint64_t desc0 = sdesc_mn_sw128(smem_u32(smem));
    bool ok = true;
    for (int i = 0; i < nst; ++i) {
      const int s = i % WT_STAGES;
      if (!mbar_wait(&full[s], (i / WT_STAGES) & 1) || *abort_flag) {
        *abort_flag = 1;
        set_error(err, STCA_ERR_TIMEOUT);
        ok = false;
        break;
      }
      tc_fence_after();
      const uint64_t a = desc0 + uint64_t((s * STAGE) >> 4);
      const uint64_t b = a + uint64_t(WT_A >> 4);
#pragma unroll
      for (int k = 0; k < WT_TOK / 16; ++k)  // 16 tokens = two 8-token groups = 2048 bytes
        umma_bf16(tmem, a + uint64_t(k * (2048 >> 4)), b + uint64_t(k * (2048 >> 4)), idesc, (i | k) != 0);
      umma_commit(&empty[s]);
    }
    if (ok && nst > 0) umma_commit(d_full);
  }
  __syncwarp();

  // ---- epilogue: warp w reads TMEM lanes 32 w .. 32 w + 31 (C rows k0 + 32 w + lane)
  bool ok = true;
  if (nst > 0 && !mbar_wait(d_full, 0)) {
    *abort_flag = 1;
    set_error(err, STCA_ERR_TIMEOUT);
    ok = false;
  }
  __syncwarp();
  if (ok) {
    tc_fence_after();
    float* dst = part + (int64_t(z) * K + k0 + warp * 32 + lane) * N + n0;
    const uint32_t tbase = tmem + (uint32_t(warp * 32) << 16);
#pragma unroll 1
    for (int j = 0; j < BN / 32; ++j) {
      float v[32];
      if (nst > 0) {
        tmem_ld_32x32b_x32(tbase + j * 32, v);
        tmem_ld_wait();
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] = 0.f;
      }
#pragma unroll
      for (int e = 0; e < 32; e += 4)
        *reinterpret_cast<float4*>(dst + j * 32 + e) = make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, BN);
  }
}

int wt_bn(int N) { return N % 256 == 0 ? 256 : 128; }

}  // namespace

// token slices: about one CTA per SM over the tiles of C, each slice at least 4 stages
int tc_wgrad_splits(int M, int K, int N) {
  const int tiles = (K / WT_M) * (N / wt_bn(N));
  const int S = (M + WT_TOK - 1) / WT_TOK;
  return std::max(1, std::min(sm_count() / std::max(tiles, 1), S / 4));
}

int tc_wgrad_partials(const void* A, int64_t lda, const void* G, int64_t ldg, int M, int K, int N, int splits,
                      float* part, int32_t* err, cudaStream_t s) {
  CUtensorMap ta, tg;
  if (!make_tmap(&ta, A, uint64_t(M), uint64_t(K), uint64_t(lda), WT_TOK)) return STCA_ERR_CUDA;
  if (!make_tmap(&tg, G, uint64_t(M), uint64_t(N), uint64_t(ldg), WT_TOK)) return STCA_ERR_CUDA;
  const dim3 grid(unsigned(N / wt_bn(N)), unsigned(K / WT_M), unsigned(splits));
  cudaError_t e;
  if (wt_bn(N) == 256) {
    cudaFuncSetAttribute(tc_wgrad_kernel<256>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         int(WtShape<256>::SMEM));
    e = launch_dep(tc_wgrad_kernel<256>, grid, dim3(128), WtShape<256>::SMEM, s, ta, tg, M, K, N, splits, part,
                   err);
  } else {
    cudaFuncSetAttribute(tc_wgrad_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         int(WtShape<128>::SMEM));
    e = launch_dep(tc_wgrad_kernel<128>, grid, dim3(128), WtShape<128>::SMEM, s, ta, tg, M, K, N, splits, part,
                   err);
  }
  if (e != cudaSuccess) return STCA_ERR_CUDA;
  note_launch();
  return STCA_OK;
}

}  // namespace stca
