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
// A pair of CTAs (a cluster of 2) computes 256-row tiles with cta_group::2 MMAs: each CTA
// holds its 128 rows of A and half of each weight tile, so each SM streams half the
// weight bytes.  The kernels are persistent (one pair per two SMs).  Warp roles: warp 0
// lane 0 issues TMA, warp 1 owns TMEM and (leader CTA) lane 0 issues tcgen05.mma, warps
// 4..11 run the epilogue, two warps per TMEM lane quarter (warp w reads lanes
// 32 (w % 4) .. + 32), each on half of the columns; warps 12, 14, 15 and 2 gather A rows
// (none on the MMA warp's scheduler, warp % 4 == 1, whose issue slots stay free).
// Waits are bounded (see common.cuh).
#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "tc_tile.cuh"

namespace stca {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
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

// 2-D fp32 tensor map for tile stores of 32 x 32 values (128-byte rows, 128-byte swizzle).
bool make_tmap_f32_out(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint64_t ld) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {ld * 4};
  cuuint32_t box[2] = {32, 32};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Output map for the epilogue's TMA stores: 32 x 32 boxes, 64-byte swizzle.
bool make_tmap_out(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint64_t ld) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {ld * 2};
  cuuint32_t box[2] = {32, 32};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}


namespace {

// ------------------------------------------------------------------------------------
// Kernel R (persistent): each CTA pair walks 256-row tiles; each CTA keeps its 128 rows
// of A resident in shared memory (K <= 512) and streams its half of every 256-column
// weight tile.  N is walked in 256-column tiles with a double-buffered TMEM accumulator
// (the epilogue of one tile overlaps the MMAs of the next, across row tiles too), and
// chunk kc of the next row tile's A is loaded as soon as the last N tile has used it.
//
// Warps: 0 weight-tile TMA producer, 3 A-tile TMA producer (TMA mode), 1 TMEM owner + MMA
// issuer (leader CTA), 4..11 epilogue,
// 12, 14, 15, 2 gather producer (gather mode): cp.async of the CTA's A rows into the swizzled
// layout (8 lanes per 128-byte row segment), the time-bucket row added (from L1), and
// an L2 prefetch of the next tile's rows one tile ahead.  With store_x the
// gather warps also write the finished A rows to X (TMA tile stores straight from the
// swizzled chunks), so that later layers over the same rows read X with TMA instead of
// gathering again.

template <int AMODE, int EPI, int STAGES>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(512, 1)
    tc_gemm_resident_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                            const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmX,
                            const __grid_constant__ CUtensorMap tmP, GatherSrc g, int M_max, int K, int NT,
                            int store_x, int32_t* err, const int32_t* M_dev, EpiFold fold) {
  griddep_wait();
  griddep_launch();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  const int KC = K / 64;
  uint8_t* sA = smem;
  uint8_t* sB = sA + KC * A_CHUNK;
  uint8_t* sOut = sB + STAGES * B_HALF;               // 8 warps x 2 KB
  uint64_t* bars = reinterpret_cast<uint64_t*>(sOut + 8 * OUT_STAGE);
  uint64_t* a_full = bars;                 // [8]      leader
  uint64_t* a_empty = bars + 8;            // [8]      both
  uint64_t* b_full = bars + 16;            // [STAGES] leader
  uint64_t* b_empty = b_full + STAGES;     // [STAGES] both
  uint64_t* t_full = b_empty + STAGES;     // [2]      both
  uint64_t* t_empty = t_full + 2;          // [2]      leader
  uint64_t* mma_done = t_empty + 2;        // [1]      leader
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  // N tiles whose accumulators this CTA's epilogue has received (times the gather's L2
  // prefetch of the next row tile)
  volatile int* progress = abort_flag + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  const int M = M_dev ? min(M_max, *M_dev) : M_max;  // rows present in this call
  const int num_tiles = (M + 2 * BM - 1) / (2 * BM);
  const int cl = blockIdx.x >> 1, ncl = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    *progress = 0;
    for (int i = 0; i < KC; ++i) {
      mbar_init(&a_full[i], AMODE == A_GATHER ? 256 : 1);
      mbar_init(&a_empty[i], 1);
    }
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&b_full[s], 1);
      mbar_init(&b_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&t_full[i], 1);
      mbar_init(&t_empty[i], 512);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // the peer's barriers exist before anyone signals them
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      prefetch_tmap(&tmB);
      prefetch_tmap(&tmC);
      const uint32_t b_full0 = cluster_addr(&b_full[0], 0);
      int it = 0;
      bool ok = true;
      for (int tile = cl; tile < num_tiles && ok; tile += ncl) {
        for (int nt = 0; nt < NT && ok; ++nt) {
          for (int kc = 0; kc < KC; ++kc, ++it) {
            const int s = it % STAGES, round = it / STAGES;
            if ((round > 0 && !mbar_wait(&b_empty[s], (round - 1) & 1)) || abort_set(abort_flag)) {
              fail(abort_flag, err);
              ok = false;
              break;
            }
            if (leader) mbar_arrive_expect_tx(&b_full[s], 2 * B_HALF);
            tma_load_2d_pair(sB + s * B_HALF, &tmB, kc * 64, nt * 256 + int(rank) * BM, b_full0 + s * 8);
          }
        }
      }
      // the leader's full barriers count both CTAs' bytes
      if (leader) drain_ring(b_full, STAGES, it);
    }
  } else if (warp == 3) {
    // A producer (TMA mode): chunk kc of the next row tile is requested as soon as the last
    // column tile of the current one has consumed chunk kc, apart from the weight ring, so
    // the new rows arrive while the last column tile is still being multiplied
    if (AMODE == A_TMA && lane == 0) {
      prefetch_tmap(&tmA);
      const uint32_t a_full0 = cluster_addr(&a_full[0], 0);
      int li = 0;
      bool ok = true;
      for (int tile = cl; tile < num_tiles && ok; tile += ncl, ++li) {
        const int m0 = tile * 2 * BM + int(rank) * BM;
        for (int kc = 0; kc < KC; ++kc) {
          if ((li > 0 && !mbar_wait(&a_empty[kc], (li - 1) & 1)) || abort_set(abort_flag)) {
            fail(abort_flag, err);
            ok = false;
            break;
          }
          if (leader) mbar_arrive_expect_tx(&a_full[kc], 2 * A_CHUNK);
          tma_load_2d_pair(sA + kc * A_CHUNK, &tmA, kc * 64, m0, a_full0 + kc * 8);
        }
      }
      // no copy may still be writing shared memory when the pair exits
      if (leader && li > 0)
        for (int kc = 0; kc < KC; ++kc) mbar_wait(&a_full[kc], (li - 1) & 1);
    }
  } else if (warp == 1) {
    if (leader && lane == 0) {
      // The issue loop is the kernel's critical thread: everything per MMA is precomputed
      // (descriptor bases advance by constant steps; the ring slot and phase are counters).
      const uint32_t idesc = umma_idesc_bf16(256, 256);
      // descriptor start addresses are in 16-byte units: +2 per 16-element K step
      const uint64_t adesc0 = umma_sdesc_sw128(smem_u32(sA)), bdesc0 = umma_sdesc_sw128(smem_u32(sB));
      int s = 0, gnt = 0, li = 0;
      uint32_t bphase = 0;
      bool ok = true;
      for (int tile = cl; tile < num_tiles && ok; tile += ncl, ++li) {
        for (int nt = 0; nt < NT && ok; ++nt, ++gnt) {
          const int buf = gnt & 1, use = gnt >> 1;
          if (use > 0 && !mbar_wait_cluster(&t_empty[buf], (use - 1) & 1)) {
            fail(abort_flag, err);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t dcol = tmem + buf * 256;
          for (int kc = 0; kc < KC; ++kc) {
            if ((nt == 0 && !mbar_wait_cluster(&a_full[kc], li & 1)) || !mbar_wait(&b_full[s], bphase)) {
              fail(abort_flag, err);
              ok = false;
              break;
            }
            tc_fence_after();
            const uint64_t ad = adesc0 + uint64_t(kc * (A_CHUNK >> 4));
            const uint64_t bd = bdesc0 + uint64_t(s * (B_HALF >> 4));
            umma_bf16_pair(dcol, ad, bd, idesc, kc != 0);
            umma_bf16_pair(dcol, ad + 2, bd + 2, idesc, 1);
            umma_bf16_pair(dcol, ad + 4, bd + 4, idesc, 1);
            umma_bf16_pair(dcol, ad + 6, bd + 6, idesc, 1);
            umma_commit_pair_both(&b_empty[s], 0x3);
            if (nt == NT - 1) umma_commit_pair_both(&a_empty[kc], 0x3);
            if (++s == STAGES) {
              s = 0;
              bphase ^= 1;
            }
          }
          if (ok) {
            umma_commit_pair_both(&t_full[buf], 0x3);
          }
        }
      }
      umma_commit_pair(cluster_addr(mma_done, 0));
      mbar_wait(mma_done, 0);
    }
  } else if (warp == 2 || warp == 12 || warp >= 14) {
    // gather warps: warp gw copies rows 32 gw .. 32 gw + 31 of this CTA's A tile; in each
    // copy instruction 8 consecutive lanes take the 8 16-byte chunks of one row, so a warp
    // moves 4 whole 128-byte row segments per instruction (row r_i = 32 gw + 4 i + lane/8)
    if (AMODE == A_GATHER) {
      const int gw = warp == 2 ? 3 : (warp == 12 ? 0 : warp - 13);
      const int sub = lane >> 3, c = lane & 7;
      const bool with_dt = g.dt != nullptr && g.dt_table != nullptr;
      const bf16* dtt = reinterpret_cast<const bf16*>(g.dt_table);
      const bf16* table = reinterpret_cast<const bf16*>(g.table);
      const uint32_t a_full0 = cluster_addr(&a_full[0], 0);
      int32_t id[8], nid[8];
      int bk[8], nbk[8];
      uint32_t vmask = 0, nvmask = 0;
      auto rows_of = [&](int tile, int32_t (&ids)[8], int (&bks)[8], uint32_t& mask) {
        mask = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          int64_t idl;
          const bool v = gather_row(g, tile * 2 * BM + int(rank) * BM + gw * 32 + i * 4 + sub, M, idl, bks[i],
                                    c == 0 ? err : nullptr);
          ids[i] = int32_t(idl);
          if (v) mask |= 1u << i;
        }
      };
      auto prefetch_rows = [&](const int32_t (&ids)[8], uint32_t mask) {
        if (c != 0) return;
#pragma unroll
        for (int i = 0; i < 8; ++i)
          if ((mask >> i) & 1u) prefetch_l2_bulk(table + int64_t(ids[i]) * K, uint32_t(K) * 2);
      };
      if (cl < num_tiles) {
        rows_of(cl, id, bk, vmask);
        prefetch_rows(id, vmask);
      }
      if (store_x && lane == 0) prefetch_tmap(&tmX);
      int li = 0;
      bool ok = true;
      for (int tile = cl; tile < num_tiles && ok; tile += ncl, ++li) {
        // this lane's rows of the next tile while this one is in flight (prefetched into L2
        // below, a few N tiles before the gather needs them: prefetched a whole row tile
        // ahead, the rows were evicted by the hidden stream again and read from DRAM twice)
        const int next = tile + ncl;
        if (next < num_tiles) rows_of(next, nid, nbk, nvmask);
        else nvmask = 0;
        if (store_x && li > 0) {
          // the previous tile's X stores have read their chunks before the chunks refill
          if (lane == 0) bulk_wait_read<0>();
          __syncwarp();
        }
        // chunk kc - GATHER_LAG is completed and published right after chunk kc is issued,
        // so chunk 0 of a tile is ready while the MMAs still work through the previous
        // tile's last chunks (each chunk is only refilled once those MMAs released it)
        auto publish = [&](int kc) {
          if (with_dt) {
            uint8_t* chunk = sA + kc * A_CHUNK;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              if (!((vmask >> i) & 1u)) continue;
              const int r = gw * 32 + i * 4 + sub;
              uint4* p = reinterpret_cast<uint4*>(chunk + r * 128 + ((c ^ (r & 7)) << 4));
              const uint4 x = *p;
              // the 16-row time table (16 K bf16) stays in L1
              const uint4 t = __ldg(reinterpret_cast<const uint4*>(dtt + int64_t(bk[i]) * K + kc * 64 + c * 8));
              const __nv_bfloat162* xa = reinterpret_cast<const __nv_bfloat162*>(&x);
              const __nv_bfloat162* ta = reinterpret_cast<const __nv_bfloat162*>(&t);
              uint32_t o[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float2 xf = __bfloat1622float2(xa[e]);
                const float2 tf = __bfloat1622float2(ta[e]);
                o[e] = pack_bf16x2(xf.x + tf.x, xf.y + tf.y);
              }
              *p = make_uint4(o[0], o[1], o[2], o[3]);
            }
          }
          fence_proxy_async_smem();
          mbar_arrive_remote(a_full0 + kc * 8);  // the leader counts both CTAs' rows
          if (store_x) {
            __syncwarp();
            if (lane == 0) {
              tma_store_2d(&tmX, kc * 64, tile * 2 * BM + int(rank) * BM + gw * 32, sA + kc * A_CHUNK + gw * 32 * 128);
              bulk_commit();
            }
          }
        };
        for (int kc = 0; kc < KC; ++kc) {
          if (li > 0 && !mbar_wait(&a_empty[kc], (li - 1) & 1)) {
            fail(abort_flag, err);
            ok = false;
            break;
          }
          uint8_t* chunk = sA + kc * A_CHUNK;
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int r = gw * 32 + i * 4 + sub;
            const bool v = (vmask >> i) & 1u;
            cp_async_16(chunk + r * 128 + ((c ^ (r & 7)) << 4), table + int64_t(v ? id[i] : 0) * K + kc * 64 + c * 8,
                        v ? 16u : 0u);
          }
          cp_async_commit();
          if (kc >= GATHER_LAG) {
            cp_async_wait<GATHER_LAG>();
            publish(kc - GATHER_LAG);
          }
        }
        if (!ok) break;
        for (int kc = KC - GATHER_LAG; kc < KC; ++kc) {
          cp_async_wait_dyn(KC - 1 - kc);
          publish(kc);
        }
        if (nvmask) {
          // wait (bounded; the prefetch is only a hint) until all but the last few N tiles
          // of this row tile have left the tensor cores, then prefetch the next tile's rows
          const int target = li * NT + (NT > PREFETCH_LEAD ? NT - PREFETCH_LEAD : 0);
          for (int it = 0; it < 16384 && *progress < target && !abort_set(abort_flag); ++it) __nanosleep(256);
          prefetch_rows(nid, nvmask);
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          id[i] = nid[i];
          bk[i] = nbk[i];
        }
        vmask = nvmask;
      }
      cp_async_wait_all();
      if (store_x && lane == 0) bulk_wait_all();
    }
  } else if (warp >= 4 && warp < 12) {
    // two epilogue warps per TMEM lane quarter, each taking half of the columns
    const int quarter = warp & 3;
    const int half = (warp - 4) >> 2;
    uint8_t* stage = sOut + (warp - 4) * OUT_STAGE;
    const uint32_t lane_base = tmem + (uint32_t(quarter * 32) << 16);
    const uint32_t t_empty0 = cluster_addr(&t_empty[0], 0);
    int gnt = 0;
    bool ok = true;
    for (int tile = cl; tile < num_tiles && ok; tile += ncl) {
      const int y = tile * 2 * BM + int(rank) * BM + quarter * 32;
      for (int nt = 0; nt < NT; ++nt, ++gnt) {
        const int buf = gnt & 1, use = gnt >> 1;
        if (!mbar_wait(&t_full[buf], use & 1) || abort_set(abort_flag)) {
          fail(abort_flag, err);
          ok = false;
          break;
        }
        if (AMODE == A_GATHER && warp == 4 && lane == 0) *progress = gnt + 1;
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
            if (fold.p_out) {  // the pre-activations [A W1 | A W3], tile stores like C's
              epi_store(stage, gv, lane, &tmP, nt * 128 + col, y);
              epi_store(stage, uv, lane, &tmP, NT * 128 + nt * 128 + col, y);
            }
#pragma unroll
            for (int e = 0; e < 32; ++e) gv[e] = silu_tanh(gv[e]) * uv[e];
            epi_store(stage, gv, lane, &tmC, nt * 128 + col, y);
          }
        } else {
          float mean = 0.f, rstd = 1.f;
          if (EPI == EPI_LNFOLD) {  // row moments of the LayerNorm folded into this GEMM
            const int row = y + lane;
            if (row < M) {
              const float2 st = __ldg(reinterpret_cast<const float2*>(fold.stats) + row);
              mean = st.x;
              rstd = st.y;
            }
          }
#pragma unroll 1
          for (int j = 0; j < 4; ++j) {
            const int col = half * 128 + j * 32;
            float v[32];
            tmem_ld_32x32b_x32(tb + col, v);
            tmem_ld_wait();
            if (EPI == EPI_LNFOLD) {
              const float4* cv = reinterpret_cast<const float4*>(fold.cvec + nt * 256 + col);
              const float4* bv = reinterpret_cast<const float4*>(fold.bvec + nt * 256 + col);
#pragma unroll
              for (int q = 0; q < 8; ++q) {
                const float4 c4 = __ldg(cv + q), b4 = __ldg(bv + q);
                v[4 * q] = fmaf(rstd, fmaf(-mean, c4.x, v[4 * q]), b4.x);
                v[4 * q + 1] = fmaf(rstd, fmaf(-mean, c4.y, v[4 * q + 1]), b4.y);
                v[4 * q + 2] = fmaf(rstd, fmaf(-mean, c4.z, v[4 * q + 2]), b4.z);
                v[4 * q + 3] = fmaf(rstd, fmaf(-mean, c4.w, v[4 * q + 3]), b4.w);
              }
            }
            epi_store(stage, v, lane, &tmC, nt * 256 + col, y);
          }
        }
        tc_fence_before();
        mbar_arrive_remote_relaxed(t_empty0 + buf * 8);
      }
    }
    if (lane == 0) bulk_wait_all();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // neither CTA frees its memory while the pair still uses it
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

// ------------------------------------------------------------------------------------
// Kernel S (persistent): each CTA pair walks 256-row tiles, streaming A (its own 128
// rows each) and its half of every 256-row weight group through a STAGES-deep ring,
// accumulates the full output row (NB x 256 columns) in TMEM, then applies LayerNorm
// (or a plain store) per row.  The ring keeps loading the next tile during the epilogue.

template <int EPI, int NB, int STAGES>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(384, 1)
    tc_gemm_rowwise_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                           const __grid_constant__ CUtensorMap tmC, int M_max, int K,
                           const float* __restrict__ gamma, const float* __restrict__ beta, float eps, int32_t* err,
                           const int32_t* M_dev, float* __restrict__ stats) {
  griddep_wait();
  griddep_launch();
  constexpr int N = NB * 256;
  constexpr int STAGE_BYTES = A_CHUNK + NB * B_HALF;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sOut = smem + STAGES * STAGE_BYTES;            // 8 warps x 2 KB
  uint64_t* bars = reinterpret_cast<uint64_t*>(sOut + 8 * OUT_STAGE);
  uint64_t* full = bars;                  // [STAGES] leader
  uint64_t* empty = bars + STAGES;        // [STAGES] both
  uint64_t* t_full = empty + STAGES;      // [1]      both
  uint64_t* t_empty = t_full + 1;         // [1]      leader
  uint64_t* mma_done = t_empty + 1;       // [1]      leader
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* s_gamma = reinterpret_cast<float*>(bars + 2 * STAGES + 8);  // [N]
  float* s_beta = s_gamma + N;                                       // [N]
  float* s_sum = s_beta + N;                                         // [2][128]
  float* s_sq = s_sum + 256;                                         // [2][128]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  const int KC = K / 64;
  const int M = M_dev ? min(M_max, *M_dev) : M_max;  // rows present in this call
  const int num_tiles = (M + 2 * BM - 1) / (2 * BM);
  const int cl = blockIdx.x >> 1, ncl = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(t_full, 1);
    mbar_init(t_empty, 512);
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, N);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      prefetch_tmap(&tmA);
      prefetch_tmap(&tmB);
      prefetch_tmap(&tmC);
      const uint32_t full0 = cluster_addr(&full[0], 0);
      int it = 0;
      bool ok = true;
      for (int tile = cl; tile < num_tiles && ok; tile += ncl) {
        const int m0 = tile * 2 * BM + int(rank) * BM;
        for (int kc = 0; kc < KC; ++kc, ++it) {
          const int s = it % STAGES, round = it / STAGES;
          if ((round > 0 && !mbar_wait(&empty[s], (round - 1) & 1)) || abort_set(abort_flag)) {
            fail(abort_flag, err);
            ok = false;
            break;
          }
          uint8_t* st = smem + s * STAGE_BYTES;
          if (leader) mbar_arrive_expect_tx(&full[s], 2 * STAGE_BYTES);
          tma_load_2d_pair(st, &tmA, kc * 64, m0, full0 + s * 8);
#pragma unroll
          for (int nb = 0; nb < NB; ++nb)
            tma_load_2d_pair(st + A_CHUNK + nb * B_HALF, &tmB, kc * 64, nb * 256 + int(rank) * BM, full0 + s * 8);
        }
      }
      if (leader) drain_ring(full, STAGES, it);
    }
  } else if (warp == 1) {
    if (leader && lane == 0) {
      const uint32_t idesc = umma_idesc_bf16(256, 256);
      // lean issue loop: descriptor bases advance by constant steps (16-byte units)
      const uint64_t desc0 = umma_sdesc_sw128(smem_u32(smem));
      int s = 0, li = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = cl; tile < num_tiles && ok; tile += ncl, ++li) {
        if (li > 0 && !mbar_wait_cluster(t_empty, (li - 1) & 1)) {
          fail(abort_flag, err);
          break;
        }
        tc_fence_after();
        for (int kc = 0; kc < KC; ++kc) {
          if (!mbar_wait(&full[s], phase)) {
            fail(abort_flag, err);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t ad = desc0 + uint64_t(s * (STAGE_BYTES >> 4));
#pragma unroll
          for (int k = 0; k < 4; ++k) {
#pragma unroll
            for (int nb = 0; nb < NB; ++nb)
              umma_bf16_pair(tmem + nb * 256, ad + 2 * k, ad + ((A_CHUNK + nb * B_HALF) >> 4) + 2 * k, idesc,
                             (kc | k) != 0);
          }
          umma_commit_pair_both(&empty[s], 0x3);
          if (++s == STAGES) {
            s = 0;
            phase ^= 1;
          }
        }
        if (ok) {
          umma_commit_pair_both(t_full, 0x3);
        }
      }
      umma_commit_pair(cluster_addr(mma_done, 0));
      mbar_wait(mma_done, 0);
    }
  } else if (warp >= 4) {
    const int quarter = warp & 3;
    const int half = (warp - 4) >> 2;
    const int r = quarter * 32 + lane;
    const int et = threadIdx.x - 128;
    constexpr int HN = N / 2;  // columns per epilogue warp
    uint8_t* stage = sOut + (warp - 4) * OUT_STAGE;
    if (EPI == EPI_LN || EPI == EPI_LNSTAT) {
      for (int c = et; c < N; c += 256) {
        s_gamma[c] = gamma[c];
        s_beta[c] = beta[c];
      }
    }
    const uint32_t tb = tmem + (uint32_t(quarter * 32) << 16) + half * HN;
    const uint32_t t_empty_addr = cluster_addr(t_empty, 0);
    const float* gm = s_gamma + half * HN;
    const float* bt = s_beta + half * HN;
    int li = 0;
    for (int tile = cl; tile < num_tiles; tile += ncl, ++li) {
      const int y = tile * 2 * BM + int(rank) * BM + quarter * 32;
      const bool ok = !epilogue_any(!mbar_wait(t_full, li & 1) || abort_set(abort_flag));
      if (!ok) fail(abort_flag, err);
      tc_fence_after();
      if (EPI == EPI_LN) {
        // one pass for both moments, shifted by the row's first value c (a sample of the
        // row, so |mean - c| is of the order of the spread and the shifted sums do not cancel)
        float s1 = 0.f, s2 = 0.f, c0 = 0.f;
        if (ok) {
          {
            float v[32];
            tmem_ld_32x32b_x32(tb - half * HN, v);
            tmem_ld_wait();
            c0 = v[0];
          }
#pragma unroll 1
          for (int j = 0; j < HN / 32; ++j) {
            float v[32];
            tmem_ld_32x32b_x32(tb + j * 32, v);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const float dv = v[e] - c0;
              s1 += dv;
              s2 = fmaf(dv, dv, s2);
            }
          }
        }
        s_sum[half * 128 + r] = s1;
        s_sq[half * 128 + r] = s2;
        epilogue_sync();
        const float m1 = (s_sum[r] + s_sum[128 + r]) * (1.0f / N);
        const float mean = c0 + m1;
        const float var = fmaxf((s_sq[r] + s_sq[128 + r]) * (1.0f / N) - m1 * m1, 0.f);
        const float rstd = rsqrtf(var + eps);
        if (ok) {
#pragma unroll 1
          for (int j = 0; j < HN / 32; ++j) {
            float v[32];
            tmem_ld_32x32b_x32(tb + j * 32, v);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = fmaf((v[e] - mean) * rstd, gm[j * 32 + e], bt[j * 32 + e]);
            epi_store(stage, v, lane, &tmC, half * HN + j * 32, y);
          }
        }
      } else if (EPI == EPI_LNSTAT) {
        // one pass: the row moments (shifted by the row's first value c, as above) and
        // y * gamma stored; the next GEMM applies (mean, rstd) and beta (EpiFold)
        float s1 = 0.f, s2 = 0.f, c0 = 0.f;
        if (ok) {
          {
            float v[32];
            tmem_ld_32x32b_x32(tb - half * HN, v);
            tmem_ld_wait();
            c0 = v[0];
          }
#pragma unroll 1
          for (int j = 0; j < HN / 32; ++j) {
            float v[32];
            tmem_ld_32x32b_x32(tb + j * 32, v);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const float dv = v[e] - c0;
              s1 += dv;
              s2 = fmaf(dv, dv, s2);
              v[e] *= gm[j * 32 + e];
            }
            epi_store(stage, v, lane, &tmC, half * HN + j * 32, y);
          }
        }
        s_sum[half * 128 + r] = s1;
        s_sq[half * 128 + r] = s2;
        epilogue_sync();
        if (ok && half == 0 && y + lane < M) {
          const float m1 = (s_sum[r] + s_sum[128 + r]) * (1.0f / N);
          const float var = fmaxf((s_sq[r] + s_sq[128 + r]) * (1.0f / N) - m1 * m1, 0.f);
          reinterpret_cast<float2*>(stats)[y + lane] = make_float2(c0 + m1, rsqrtf(var + eps));
        }
      } else if (ok) {
#pragma unroll 1
        for (int j = 0; j < HN / 32; ++j) {
          float v[32];
          tmem_ld_32x32b_x32(tb + j * 32, v);
          tmem_ld_wait();
          epi_store(stage, v, lane, &tmC, half * HN + j * 32, y);
        }
      }
      tc_fence_before();
      mbar_arrive_remote_relaxed(t_empty_addr);
      if (!ok) break;
    }
    if (lane == 0) bulk_wait_all();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, N);
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

// many matrices in one launch: blockIdx.z picks the job, blocks past a job's extent return
struct PackJobs {
  PackJob j[PACK_MAX_JOBS];
};

__global__ void pack_many_kernel(PackJobs jobs) {
  const PackJob& jb = jobs.j[blockIdx.z];
  const int k0 = blockIdx.y * 32, n0 = blockIdx.x * 32;
  if (k0 >= jb.K || n0 >= jb.N) return;
  __shared__ bf16 tile[32][33];
  const bf16* W = reinterpret_cast<const bf16*>(jb.W);
  bf16* dst = reinterpret_cast<bf16*>(jb.dst);
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int k = k0 + i, n = n0 + threadIdx.x;
    tile[i][threadIdx.x] = (k < jb.K && n < jb.N) ? W[int64_t(k) * jb.N + n] : __float2bfloat16(0.f);
  }
  __syncthreads();
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int n = n0 + i, k = k0 + threadIdx.x;
    if (n < jb.N && k < jb.K) {
      if (jb.mode >= 4) {
        // block-diagonal folds of a [K, N] = [d, d] projection (g = group = d_h, H = N / g):
        // mode 4: dst [H K, N], dst[(n / g) K + k][n] = W[k][n]   (q~ = Q dst^T per head)
        // mode 5: dst [N, H K], dst[n][(n / g) K + k] = W[k][n]   (o = r dst^T per head)
        const int64_t hk = int64_t(n / jb.group) * jb.K + k;
        const int64_t at = jb.mode == 4 ? hk * jb.N + n : int64_t(n) * (int64_t(jb.N / jb.group) * jb.K) + hk;
        dst[at] = tile[threadIdx.x][i];
      } else {
        const int row = jb.mode == 0   ? jb.row_offset + n
                        : jb.mode == 3 ? (n / jb.group) * 2 * jb.group + jb.row_offset + n % jb.group
                                       : (n / 128) * 256 + (jb.mode == 2 ? 128 : 0) + (n % 128);
        dst[int64_t(row) * jb.K + k] = tile[threadIdx.x][i];
      }
    }
  }
}

// c = gamma^T [WK | WV], b = beta^T [WK | WV]: a block of 8 warps per 32 output columns;
// lane l takes column c0 + l, warp w the rows w, w + 8, ... (reads coalesced across lanes),
// and the 8 partial sums meet in shared memory.  Output column c is the K/V GEMM's: with
// dh > 0, head c / (2 dh), K for the first dh columns of the head's block and V after.
__global__ void __launch_bounds__(256) fold_consts_kernel(const float* __restrict__ gamma,
                                                          const float* __restrict__ beta,
                                                          const bf16* __restrict__ WK, const bf16* __restrict__ WV,
                                                          int d, int dh, float* __restrict__ out) {
  __shared__ float part[2][8][32];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int c = blockIdx.x * 32 + lane;
  float sc = 0.f, sb = 0.f;
  if (c < 2 * d) {
    bool is_k;
    int col;
    if (dh > 0) {
      const int j = c % (2 * dh);
      is_k = j < dh;
      col = (c / (2 * dh)) * dh + (is_k ? j : j - dh);
    } else {
      is_k = c < d;
      col = is_k ? c : c - d;
    }
    const bf16* W = is_k ? WK : WV;
    for (int k = w; k < d; k += 8) {
      const float x = __bfloat162float(W[int64_t(k) * d + col]);
      sc = fmaf(gamma[k], x, sc);
      sb = fmaf(beta[k], x, sb);
    }
  }
  part[0][w][lane] = sc;
  part[1][w][lane] = sb;
  __syncthreads();
  if (w == 0 && c < 2 * d) {
    float a = 0.f, b = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      a += part[0][i][lane];
      b += part[1][i][lane];
    }
    out[c] = a;
    out[2 * d + c] = b;
  }
}

// ------------------------------------------------------------------------------------
// host side

size_t resident_smem(int K, int stages, bool gather) {
  size_t bytes = 1024 + size_t(K / 64) * A_CHUNK + size_t(stages) * B_HALF + 8 * OUT_STAGE + 512;
  return bytes < MIN_SMEM ? MIN_SMEM : bytes;
}

size_t rowwise_smem(int nb, int stages) {
  size_t bytes = 1024 + size_t(stages) * (A_CHUNK + nb * B_HALF) + 8 * OUT_STAGE + 256 + 2 * nb * 256 * 4 + 4 * 128 * 4;
  return bytes < MIN_SMEM ? MIN_SMEM : bytes;
}

template <int AMODE, int EPI, int STAGES>
int run_resident(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tc, const CUtensorMap& tx,
                 const CUtensorMap& tp, int store_x, const GatherSrc& g, int M, int K, int NT, int32_t* err,
                 cudaStream_t s, const int32_t* M_dev, const EpiFold& fold, int max_pairs) {
  auto kern = tc_gemm_resident_kernel<AMODE, EPI, STAGES>;
  const size_t smem = resident_smem(K, STAGES, AMODE == A_GATHER);
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) != cudaSuccess)
    return STCA_ERR_CUDA;
  int pairs = std::min((M + 2 * BM - 1) / (2 * BM), sm_count() / 2);
  if (max_pairs > 0) pairs = std::min(pairs, max_pairs);
  const int grid = 2 * pairs;
  launch_dep(kern, dim3(grid), dim3(512), smem, s, ta, tb, tc, tx, tp, g, M, K, NT, store_x, err, M_dev, fold);
  note_launch();
  return cudaGetLastError() == cudaSuccess ? 0 : STCA_ERR_CUDA;
}

template <int EPI, int NB, int STAGES>
int run_rowwise(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tc, int M, int K,
                const float* gamma, const float* beta, float eps, int32_t* err, cudaStream_t s,
                const int32_t* M_dev, float* stats) {
  auto kern = tc_gemm_rowwise_kernel<EPI, NB, STAGES>;
  const size_t smem = rowwise_smem(NB, STAGES);
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) != cudaSuccess)
    return STCA_ERR_CUDA;
  const int grid = 2 * std::min((M + 2 * BM - 1) / (2 * BM), sm_count() / 2);
  launch_dep(kern, dim3(grid), dim3(384), smem, s, ta, tb, tc, M, K, gamma, beta, eps, err, M_dev, stats);
  note_launch();
  return cudaGetLastError() == cudaSuccess ? 0 : STCA_ERR_CUDA;
}

}  // namespace

// Streaming multiprocessors of the current device (persistent grids cover each SM once).
int sm_count() {
  int dev = 0, n = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n >= 2 ? n : 2;
}

int tc_pack_weight(const void* W, int K, int N, void* dst, int mode, int row_offset, cudaStream_t s) {
  if (K <= 0 || N <= 0) return STCA_ERR_INVALID_ARG;
  dim3 grid((N + 31) / 32, (K + 31) / 32), block(32, 8);
  pack_weight_kernel<<<grid, block, 0, s>>>(reinterpret_cast<const bf16*>(W), K, N, reinterpret_cast<bf16*>(dst),
                                            mode, row_offset); note_launch();
  return cudaGetLastError() == cudaSuccess ? 0 : STCA_ERR_CUDA;
}

int fold_consts(const float* gamma, const float* beta, const void* WK, const void* WV, int d, int dh, float* out,
                cudaStream_t s) {
  if (!gamma || !beta || !WK || !WV || !out || d <= 0 || dh < 0 || (dh > 0 && d % dh != 0))
    return STCA_ERR_INVALID_ARG;
  fold_consts_kernel<<<(2 * d + 31) / 32, 256, 0, s>>>(gamma, beta, reinterpret_cast<const bf16*>(WK),
                                                       reinterpret_cast<const bf16*>(WV), d, dh, out);
  note_launch();
  return cudaGetLastError() == cudaSuccess ? 0 : STCA_ERR_CUDA;
}

int tc_pack_weights(const PackJob* jobs, int n, cudaStream_t s) {
  for (int b = 0; b < n; b += PACK_MAX_JOBS) {
    PackJobs batch;
    memset(&batch, 0, sizeof(batch));
    const int cnt = std::min(PACK_MAX_JOBS, n - b);
    int gx = 1, gy = 1;
    for (int i = 0; i < cnt; ++i) {
      const PackJob& jb = jobs[b + i];
      if (jb.K <= 0 || jb.N <= 0 || !jb.W || !jb.dst || jb.mode < 0 || jb.mode > 5) return STCA_ERR_INVALID_ARG;
      if (jb.mode >= 3 && (jb.group <= 0 || jb.N % jb.group != 0)) return STCA_ERR_INVALID_ARG;
      batch.j[i] = jb;
      gx = std::max(gx, (jb.N + 31) / 32);
      gy = std::max(gy, (jb.K + 31) / 32);
    }
    pack_many_kernel<<<dim3(gx, gy, cnt), dim3(32, 8), 0, s>>>(batch);
    note_launch();
  }
  return cudaGetLastError() == cudaSuccess ? 0 : STCA_ERR_CUDA;
}

int tc_gemm_resident(int amode, int epi, const void* A, GatherSrc g, int M, int K, const void* Wp, int Nout,
                     void* C, int ldc, int32_t* err, cudaStream_t s, const int32_t* M_dev, void* x_out,
                     const EpiFold* fold, int max_pairs, void* p_out) {
  if (M == 0) return 0;
  if (M < 0 || (K != 256 && K != 512) || Nout <= 0 || ldc % 8 != 0) return STCA_ERR_UNSUPPORTED;
  const int N = epi == EPI_SWIGLU ? 2 * Nout : Nout;
  if (N % 256 != 0) return STCA_ERR_UNSUPPORTED;
  const int NT = N / 256;
  if (reinterpret_cast<uintptr_t>(C) % 16 != 0) return STCA_ERR_INVALID_ARG;
  if (x_out && (amode != A_GATHER || reinterpret_cast<uintptr_t>(x_out) % 16 != 0)) return STCA_ERR_INVALID_ARG;
  if (p_out && (epi != EPI_SWIGLU || reinterpret_cast<uintptr_t>(p_out) % 16 != 0)) return STCA_ERR_INVALID_ARG;
  if (epi == EPI_LNFOLD && (!fold || !fold->stats || !fold->cvec || !fold->bvec || amode != A_TMA))
    return STCA_ERR_INVALID_ARG;
  EpiFold fo;
  memset(&fo, 0, sizeof(fo));
  if (fold) fo = *fold;
  fo.p_out = p_out;
  CUtensorMap ta, tb, tc, tx, tp;
  memset(&ta, 0, sizeof(ta));
  if (!make_tmap(&tb, Wp, N, K, K, BM)) return STCA_ERR_CUDA;
  if (!make_tmap_out(&tc, C, M, Nout, ldc)) return STCA_ERR_CUDA;
  if (amode == A_TMA) {
    if (!make_tmap(&ta, A, M, K, K, BM)) return STCA_ERR_CUDA;
  } else {
    ta = tb;  // unused by the gather producer
  }
  // X [M, K] written by the gather warps: one 64-column x 32-row box per warp and chunk
  if (x_out) {
    if (!make_tmap(&tx, x_out, M, K, K, 32)) return STCA_ERR_CUDA;
  } else {
    tx = tb;  // unused
  }
  const int sx = x_out != nullptr;
  // P [M, 2 Nout] written by the SwiGLU epilogue: 32 x 32 boxes like C
  if (p_out) {
    if (!make_tmap_out(&tp, p_out, M, 2 * uint64_t(Nout), 2 * uint64_t(Nout))) return STCA_ERR_CUDA;
  } else {
    tp = tc;  // unused
  }
  // stage counts fill the 227 KB of shared memory (see resident_smem)
#define STCA_RES(AM, EP)                                                                                   \
  (K == 512 ? run_resident<AM, EP, 5>(ta, tb, tc, tx, tp, sx, g, M, K, NT, err, s, M_dev, fo, max_pairs)     \
            : run_resident<AM, EP, 9>(ta, tb, tc, tx, tp, sx, g, M, K, NT, err, s, M_dev, fo, max_pairs))
  if (amode == A_TMA && epi == EPI_PLAIN) return STCA_RES(A_TMA, EPI_PLAIN);
  if (amode == A_TMA && epi == EPI_LNFOLD) return STCA_RES(A_TMA, EPI_LNFOLD);
  if (amode == A_TMA && epi == EPI_SWIGLU) return STCA_RES(A_TMA, EPI_SWIGLU);
  if (amode == A_GATHER && epi == EPI_PLAIN) return STCA_RES(A_GATHER, EPI_PLAIN);
  if (amode == A_GATHER && epi == EPI_SWIGLU) return STCA_RES(A_GATHER, EPI_SWIGLU);
#undef STCA_RES
  return STCA_ERR_UNSUPPORTED;
}

int tc_gemm_rowwise(int epi, const void* A, int M, int K, const void* Wp, int N, const float* gamma,
                    const float* beta, float eps, void* C, int ldc, int32_t* err, cudaStream_t s,
                    const int32_t* M_dev, int lda, float* stats) {
  if (M == 0) return 0;
  if (lda == 0) lda = K;
  if (M < 0 || K <= 0 || K % 64 != 0 || (N != 256 && N != 512) || ldc % 8 != 0 || lda < K || lda % 8 != 0 ||
      reinterpret_cast<uintptr_t>(A) % 16 != 0)
    return STCA_ERR_UNSUPPORTED;
  if ((epi == EPI_LN || epi == EPI_LNSTAT) && (!gamma || !beta)) return STCA_ERR_INVALID_ARG;
  if (epi == EPI_LNSTAT && (!stats || reinterpret_cast<uintptr_t>(stats) % 8 != 0)) return STCA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(C) % 16 != 0) return STCA_ERR_INVALID_ARG;
  CUtensorMap ta, tb, tc;
  if (!make_tmap(&ta, A, M, K, lda, BM)) return STCA_ERR_CUDA;
  if (!make_tmap(&tb, Wp, N, K, K, BM)) return STCA_ERR_CUDA;
  if (!make_tmap_out(&tc, C, M, N, ldc)) return STCA_ERR_CUDA;
  if (N == 512) {
    if (epi == EPI_LN) return run_rowwise<EPI_LN, 2, 4>(ta, tb, tc, M, K, gamma, beta, eps, err, s, M_dev, stats);
    if (epi == EPI_LNSTAT)
      return run_rowwise<EPI_LNSTAT, 2, 4>(ta, tb, tc, M, K, gamma, beta, eps, err, s, M_dev, stats);
    return run_rowwise<EPI_PLAIN, 2, 4>(ta, tb, tc, M, K, gamma, beta, eps, err, s, M_dev, stats);
  }
  if (epi == EPI_LN) return run_rowwise<EPI_LN, 1, 6>(ta, tb, tc, M, K, gamma, beta, eps, err, s, M_dev, stats);
  if (epi == EPI_LNSTAT)
    return run_rowwise<EPI_LNSTAT, 1, 6>(ta, tb, tc, M, K, gamma, beta, eps, err, s, M_dev, stats);
  return run_rowwise<EPI_PLAIN, 1, 6>(ta, tb, tc, M, K, gamma, beta, eps, err, s, M_dev, stats);
}

}  // namespace stca
