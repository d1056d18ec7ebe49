// tcgen05 GEMMs for the target-side (query) path.
//
// C = A W (+ R) or C = SiLU(A W1) * (A W3), with fp32 activations A, bf16 weights and
// fp32 results: the query projection and W_O of every layer, the fusion W_C, W_Z and the
// target-side SwiGLU FFNs (STCA notes, section "STCA"; review §三 fusion formula).  The
// query path keeps fp32 activations: each activation a enters the tensor cores as two bf16
// terms hi = bf16(a) and lo = bf16(a - hi), both multiplied by the same bf16 weight and
// accumulated in fp32, so every product is within ~2^-17 relative of the fp32 product.
//
// One CTA computes a 128-row x BN-column tile with cta_group::1 MMAs (M = 128, N = BN,
// K = 16) into BN TMEM columns; BN = 256, or 128 / 64 for plain GEMMs whose 256-column
// grid would leave SMs idle (a few hundred target rows: every launch is then a chain of
// MMA latencies, and narrower tiles both spread it over more SMs and shorten each MMA).
// K streams through a 3-stage ring of 64-wide chunks: the
// weight chunk arrives by TMA (K-major packed weights, 128-byte swizzle); eight producer
// warps load the fp32 activation rows (three chunks in flight), split them and store the
// hi and lo tiles in the same swizzled layout.  Those warps then run the epilogue (two per
// TMEM lane quarter).
// Warp 0 lane 0 issues TMA, warp 1 owns TMEM and its lane 0 issues the MMAs.  Every wait
// is bounded (see common.cuh); a timeout sets STCA_ERR_TIMEOUT and the CTA winds down.
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace stca {

namespace {

constexpr int QBM = 128, QKC = 64, QSTAGES = 3;
constexpr int QA_TILE = QBM * QKC * 2;          // one bf16 activation tile: 16 KB
template <int BN>
struct QShape {
  static constexpr int B_TILE = BN * QKC * 2;            // one weight chunk: 8, 16 or 32 KB
  static constexpr int STAGE = 2 * QA_TILE + B_TILE;     // hi | lo | weights
  static constexpr size_t SMEM = 1024 + size_t(QSTAGES) * STAGE + 256;
  static_assert(QSTAGES * STAGE >= 8 * 8192, "the epilogue stages its blocks in the ring");
};

struct TcqArgs {
  const float* A;
  int64_t lda;
  int ksplit, kshift;
  int a_grp, a_gstride, a_goff;
  float* C;
  int64_t ldc;
  int c_grp, c_gstride, c_goff;
  const float* R;
  int64_t ldr;
  int M, N, K;  // N output columns
  int64_t bsA, bsC, bsR;  // element offsets per batch (grid z)
  int wrows;              // packed weight rows per batch
  int c_tma;              // C written by TMA tile stores (one batch, rows not remapped)
  int32_t* err;
};

__device__ __forceinline__ uint8_t* q_align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

__device__ __forceinline__ int64_t q_remap(int r, int grp, int gstride, int goff) {
  return grp ? int64_t(r / grp) * gstride + goff + r % grp : int64_t(r);
}

// SiLU(x) = x / (1 + e^-x) with the fast exponential and division intrinsics: a few
// ulp of fp32 (the target side keeps fp32 accuracy; the bf16 history side uses tanh.approx).
// For x below about -88, e^-x is +inf and the quotient is 0, the limit of SiLU.
__device__ __forceinline__ float silu_fast(float x) { return __fdividef(x, 1.0f + __expf(-x)); }

// hi and lo bf16 pairs of two fp32 values
__device__ __forceinline__ void split2(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
  const float2 hf = __bfloat1622float2(h);
  const __nv_bfloat162 l = __floats2bfloat162_rn(x0 - hf.x, x1 - hf.y);
  hi = *reinterpret_cast<const uint32_t*>(&h);
  lo = *reinterpret_cast<const uint32_t*>(&l);
}

template <bool DUAL, int BN>
__global__ void __launch_bounds__(384, 1) tc_query_kernel(const __grid_constant__ CUtensorMap tmB,
                                                          const __grid_constant__ CUtensorMap tmC, TcqArgs a) {
  static_assert(!DUAL || BN == 256, "the SwiGLU pair is packed as 128 gate + 128 up rows");
  constexpr int QB_TILE = QShape<BN>::B_TILE, QSTAGE = QShape<BN>::STAGE;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = q_align1024(smem_raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + QSTAGES * QSTAGE);
  uint64_t* a_full = bars;                 // [QSTAGES] 256 producer arrivals
  uint64_t* b_full = bars + QSTAGES;       // [QSTAGES] TMA bytes
  uint64_t* empty = bars + 2 * QSTAGES;    // [QSTAGES] MMA commit
  uint64_t* d_full = bars + 3 * QSTAGES;   // accumulator complete
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(d_full + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.y * QBM;
  const int z = blockIdx.z;
  const int wrow0 = z * a.wrows + blockIdx.x * BN;  // first packed weight row of this tile
  const int KC = a.K / QKC;
  const float* A = a.A + z * a.bsA;
  float* C = a.C + z * a.bsC;
  const float* R = a.R ? a.R + z * a.bsR : nullptr;

  if (threadIdx.x == 0) {
    for (int s = 0; s < QSTAGES; ++s) {
      mbar_init(&a_full[s], 256);
      mbar_init(&b_full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(d_full, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, BN);
    tmem_relinquish();
  }
  if (threadIdx.x == 0) prefetch_tmap(&tmB);
  // Launched as a programmatic dependent of the previous kernel on the stream: the setup
  // above overlaps that kernel's tail; nothing it writes (or anything before it) is touched
  // before this wait.  The next target-side GEMM may start its own setup now.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      int issued = 0;
      for (int kc = 0; kc < KC; ++kc, ++issued) {
        const int s = kc % QSTAGES, round = kc / QSTAGES;
        if ((round > 0 && !mbar_wait(&empty[s], (round - 1) & 1)) || *abort_flag) {
          *abort_flag = 1;
          set_error(a.err, STCA_ERR_TIMEOUT);
          break;
        }
        mbar_arrive_expect_tx(&b_full[s], QB_TILE);
        tma_load_2d(smem + s * QSTAGE + 2 * QA_TILE, &tmB, kc * QKC, wrow0, &b_full[s]);
      }
      // no copy may still be writing shared memory when the CTA exits
      for (int s = 0; s < QSTAGES && s < issued; ++s) {
        const int last = s + QSTAGES * ((issued - 1 - s) / QSTAGES);
        mbar_wait(&b_full[s], (last / QSTAGES) & 1);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = umma_idesc_bf16(QBM, BN);
      // lean issue loop: descriptor bases advance by constant steps (16-byte units)
      const uint64_t desc0 = umma_sdesc_sw128(smem_u32(smem));
      bool ok = true;
      int s = 0;
      uint32_t par = 0;
      for (int kc = 0; kc < KC; ++kc) {
        if (!mbar_wait(&a_full[s], par) || !mbar_wait(&b_full[s], par)) {
          *abort_flag = 1;
          set_error(a.err, STCA_ERR_TIMEOUT);
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t hi = desc0 + uint64_t(s * (QSTAGE >> 4));
        const uint64_t lo = hi + (QA_TILE >> 4);
        const uint64_t b = hi + ((2 * QA_TILE) >> 4);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          umma_bf16(tmem, hi + 2 * k, b + 2 * k, idesc, (kc | k) != 0);
          umma_bf16(tmem, lo + 2 * k, b + 2 * k, idesc, 1);
        }
        umma_commit(&empty[s]);
        if (++s == QSTAGES) {
          s = 0;
          par ^= 1;
        }
      }
      if (ok) umma_commit(d_full);
    }
  } else if (warp >= 4) {
    // ---- producers: lane -> (row sub = lane / 8, 8-column group c = lane % 8); warp pw
    // takes rows 16 pw + 4 i + sub, i = 0..3, so each load instruction covers 4 whole
    // 256-byte row segments of the chunk.  Three chunks are in flight per thread (register
    // buffers b0..b2 in turn): the loads of chunk kc + 3 go out once chunk kc is stored.
    const int pw = warp - 4;
    const int sub = lane >> 3, c = lane & 7;
    const float* rowp[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = m0 + pw * 16 + 4 * i + sub;
      rowp[i] = r < a.M ? A + q_remap(r, a.a_grp, a.a_gstride, a.a_goff) * a.lda : nullptr;
    }
    auto load = [&](int kc, float4 (&b)[8]) {
      if (kc >= KC) return;
      const int k = kc * QKC;
      const int col = k + (k >= a.ksplit ? a.kshift : 0) + c * 8;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        if (rowp[i]) {
          b[2 * i] = __ldg(reinterpret_cast<const float4*>(rowp[i] + col));
          b[2 * i + 1] = __ldg(reinterpret_cast<const float4*>(rowp[i] + col + 4));
        } else {
          b[2 * i] = b[2 * i + 1] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
    };
    bool ok = true;
    auto step = [&](int kc, float4 (&b)[8]) {
      if (kc >= KC || !ok) return;
      const int s = kc % QSTAGES, round = kc / QSTAGES;
      if ((round > 0 && !mbar_wait(&empty[s], (round - 1) & 1)) || *abort_flag) {
        *abort_flag = 1;
        set_error(a.err, STCA_ERR_TIMEOUT);
        ok = false;
        return;
      }
      uint8_t* hi_t = smem + s * QSTAGE;
      uint8_t* lo_t = hi_t + QA_TILE;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int rr = pw * 16 + 4 * i + sub;
        const int off = rr * 128 + ((c ^ (rr & 7)) << 4);
        uint4 h, l;
        split2(b[2 * i].x, b[2 * i].y, h.x, l.x);
        split2(b[2 * i].z, b[2 * i].w, h.y, l.y);
        split2(b[2 * i + 1].x, b[2 * i + 1].y, h.z, l.z);
        split2(b[2 * i + 1].z, b[2 * i + 1].w, h.w, l.w);
        *reinterpret_cast<uint4*>(hi_t + off) = h;
        *reinterpret_cast<uint4*>(lo_t + off) = l;
      }
      load(kc + 3, b);
      fence_proxy_async_smem();
      mbar_arrive(&a_full[s]);
    };
    float4 b0[8], b1[8], b2[8];
    load(0, b0);
    load(1, b1);
    load(2, b2);
    for (int kc = 0; kc < KC && ok; kc += 3) {
      step(kc, b0);
      step(kc + 1, b1);
      step(kc + 2, b2);
    }

    // ---- epilogue: two warps per TMEM lane quarter (warp % 4), each on half the columns;
    // lane l holds output row 32 quarter + l
    if (ok && !mbar_wait(d_full, 0)) {
      *abort_flag = 1;
      set_error(a.err, STCA_ERR_TIMEOUT);
      ok = false;
    }
    __syncwarp();
    if (ok) {
      tc_fence_after();
      fence_proxy_async_smem();  // the ring's last async reads come before the staging writes
      const int quarter = warp & 3, half = (warp - 4) >> 2;
      const int row = m0 + quarter * 32 + lane;
      const uint32_t tbase = tmem + (uint32_t(quarter * 32) << 16);
      float* crow = row < a.M ? C + q_remap(row, a.c_grp, a.c_gstride, a.c_goff) * a.ldc : nullptr;
      const float* rrow = (row < a.M && R) ? R + int64_t(row) * a.ldr : nullptr;
      // With tile stores, each warp stages its 32 x 32 blocks in two 4 KB buffers of the
      // (now idle) operand ring, rows 128-byte swizzled, and TMA writes whole rows; rows or
      // columns outside C are clipped.  Otherwise each lane stores its own row.
      uint8_t* stage = smem + (warp - 4) * 8192;
      constexpr int NCH = DUAL ? 2 : BN / 64;  // 32-column output chunks per warp
#pragma unroll 1
      for (int j = 0; j < NCH; ++j) {
        const int tc = half * NCH * 32 + j * 32;  // accumulator column (gate half when DUAL)
        float v[32];
        tmem_ld_32x32b_x32(tbase + tc, v);
        if (DUAL) {
          float u[32];
          tmem_ld_32x32b_x32(tbase + 128 + tc, u);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = silu_fast(v[e]) * u[e];
        } else {
          tmem_ld_wait();
        }
        const int col = (DUAL ? blockIdx.x * 128 : blockIdx.x * BN) + tc;
        if (col >= a.N) continue;  // warp-uniform
        if (rrow) {
#pragma unroll
          for (int e = 0; e < 32; e += 4) {
            const float4 r4 = *reinterpret_cast<const float4*>(rrow + col + e);
            v[e] += r4.x;
            v[e + 1] += r4.y;
            v[e + 2] += r4.z;
            v[e + 3] += r4.w;
          }
        }
        if (a.c_tma) {
          uint8_t* buf = stage + (j & 1) * 4096;
          if (lane == 0 && j >= 2) bulk_wait_read<1>();  // the store that read this buffer
          __syncwarp();
#pragma unroll
          for (int c = 0; c < 8; ++c)
            *reinterpret_cast<float4*>(buf + lane * 128 + ((c ^ (lane & 7)) << 4)) =
                make_float4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&tmC, col, m0 + quarter * 32, buf);
            bulk_commit();
          }
        } else if (crow) {
#pragma unroll
          for (int e = 0; e < 32; e += 4)
            *reinterpret_cast<float4*>(crow + col + e) = make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
        }
      }
      if (a.c_tma && lane == 0) bulk_wait_all();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, BN);
  }
}

}  // namespace

bool tc_query_supported(const SimtGemmArgs<float, bf16>& a) {
  auto al16 = [](const void* p) { return reinterpret_cast<uintptr_t>(p) % 16 == 0; };
  if (a.gather.ids || a.batch < 1) return false;
  if (a.K <= 0 || a.K % QKC != 0 || a.N <= 0 || a.N % (a.B2 ? 128 : 32) != 0) return false;
  if (a.ksplit < a.K && (a.ksplit % QKC != 0 || a.kshift % 4 != 0)) return false;
  if (!al16(a.A) || a.lda % 4 != 0 || !al16(a.C) || a.ldc % 4 != 0) return false;
  if (a.R && (!al16(a.R) || a.ldr % 4 != 0)) return false;
  if (a.batch > 1) {
    // per-batch weights sit back to back in the packed buffer, whole 256-row tiles each
    const int wrows = a.B2 ? 2 * a.N : a.N;
    if (wrows % 256 != 0 || a.bsA % 4 != 0 || a.bsC % 4 != 0 || a.bsR % 4 != 0) return false;
  }
  return true;
}

int tc_query_gemm(const SimtGemmArgs<float, bf16>& a, const void* Wp, cudaStream_t s) {
  if (a.M == 0) return 0;
  if (!tc_query_supported(a) || !Wp || a.M < 0) return STCA_ERR_UNSUPPORTED;
  const bool dual = a.B2 != nullptr;
  // packed rows: N (plain), or 256 per 128 output columns (gate and up halves)
  const int wrows = dual ? 2 * a.N : a.N;
  // column tile: 256, unless that grid would fill under ~4/5 of the SMs (plain GEMMs only)
  auto ctas = [&](int bn) { return int64_t((wrows + bn - 1) / bn) * ((a.M + QBM - 1) / QBM) * a.batch; };
  const int64_t fill = int64_t(sm_count()) * 4 / 5;
  const int bn = dual || ctas(256) >= fill ? 256 : (ctas(128) >= fill ? 128 : 64);
  CUtensorMap tb;
  if (!make_tmap(&tb, Wp, uint64_t(wrows) * a.batch, uint64_t(a.K), uint64_t(a.K), bn)) return STCA_ERR_CUDA;
  TcqArgs q;
  q.A = a.A;
  q.lda = a.lda;
  q.ksplit = a.ksplit;
  q.kshift = a.kshift;
  q.a_grp = a.a_grp;
  q.a_gstride = a.a_gstride;
  q.a_goff = a.a_goff;
  q.C = a.C;
  q.ldc = a.ldc;
  q.c_grp = a.c_grp;
  q.c_gstride = a.c_gstride;
  q.c_goff = a.c_goff;
  q.R = a.R;
  q.ldr = a.ldr;
  q.M = a.M;
  q.N = a.N;
  q.K = a.K;
  q.bsA = a.bsA;
  q.bsC = a.bsC;
  q.bsR = a.bsR;
  q.wrows = wrows;
  q.err = a.err;
  // tile stores need one contiguous [M, N] block: one batch, rows not remapped
  q.c_tma = a.batch == 1 && a.c_grp == 0;
  CUtensorMap tc;
  if (q.c_tma) {
    if (!make_tmap_f32_out(&tc, a.C, uint64_t(a.M), uint64_t(a.N), uint64_t(a.ldc))) return STCA_ERR_CUDA;
  } else {
    tc = tb;  // unused
  }
  const dim3 grid((wrows + bn - 1) / bn, (a.M + QBM - 1) / QBM, a.batch);
  auto kern = dual ? tc_query_kernel<true, 256>
                   : (bn == 256 ? tc_query_kernel<false, 256>
                                : (bn == 128 ? tc_query_kernel<false, 128> : tc_query_kernel<false, 64>));
  const size_t smem = bn == 256 ? QShape<256>::SMEM : (bn == 128 ? QShape<128>::SMEM : QShape<64>::SMEM);
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) != cudaSuccess)
    return STCA_ERR_CUDA;
  // programmatic dependent launch: the CTAs may start (barriers, TMEM, descriptor prefetch)
  // while the previous kernel on the stream drains; the kernel waits for it before any data
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = grid;
  cfg.blockDim = dim3(384);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, tb, tc, q) != cudaSuccess) return STCA_ERR_CUDA;
  note_launch();
  return cudaGetLastError() == cudaSuccess ? 0 : STCA_ERR_CUDA;
}

}  // namespace stca
