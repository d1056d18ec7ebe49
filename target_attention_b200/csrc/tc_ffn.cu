// Fused history FFN for d = 256: gather -> X [W1 | W3] -> SwiGLU -> W2 -> LayerNorm
// moments, for every layer, with the SwiGLU hidden activations kept on chip.
//
// Per layer i the history side computes X~ = LN((SiLU(X W1) * (X W3)) W2) from the
// ORIGINAL X (STCA notes, section "STCA"; review §三), and the WeChat article's low-memory
// operator (§1.1, "lookup while computing") fuses the lookup into the computation.  Here
// the fusion is carried one step further: the hidden activation A = SiLU(X W1) * (X W3)
// (h wide) never goes to HBM.  A CTA pair walks 256-row tiles (cta_group::2 MMAs, each CTA
// holds 128 rows); the gathered X tile (K = 256) stays resident in shared memory for all
// layers.  Per layer l and hidden chunk j of 128 units:
//   GEMM1   acc1 = X [W1 | W3]_{l, j}          TMEM columns 0..255 (128 gates | 128 ups)
//   SwiGLU  the epilogue warps turn acc1 into the bf16 hidden chunk and write it straight
//           into shared memory, in the K-major 128-byte-swizzled layout an MMA operand
//           needs (two buffers)
//   GEMM2   acc2 += chunk W2_l[128 j .. 128 j + 128, :]   TMEM columns 256..511
// The MMA thread issues GEMM1 of chunk j + 1 before GEMM2 of chunk j, so the tensor cores
// multiply one chunk while the epilogue converts the other.  After a layer's last chunk the
// epilogue stores y' = (A W2) * gamma_l and the row moments; the K/V GEMM then applies the
// LayerNorm (rstd (y' W - mean gamma^T W) + beta^T W), as on the unfused path.  At d = 256
// the two accumulators fill the 512 TMEM columns exactly.
//
// Warps: 0 weight TMA (W1|W3 and W2 tiles through one ring, in the MMA thread's order),
// 1 TMEM owner + MMA issuer (leader CTA), 2, 12, 14, 15 gather A rows, 4..11 epilogue (two
// per TMEM lane quarter, each on half of the columns).  Every wait is bounded.
#include <algorithm>

#include "tc_tile.cuh"

namespace stca {

namespace {

constexpr int F_K = 256;                      // d: the GEMM1 K and the GEMM2 N
constexpr int F_KC = F_K / 64;                // A chunks
constexpr int F_HCH = 128;                    // hidden units per chunk
constexpr int F_HBUF = 2 * A_CHUNK;           // one hidden chunk: 128 rows x 128 K bf16 (32 KB)

struct FfnGammas {
  const float* g[STCA_MAX_LAYERS];
};

template <int STAGES>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(512, 1)
    tc_ffn_fused_kernel(const __grid_constant__ CUtensorMap tmW13, const __grid_constant__ CUtensorMap tmW2,
                        const __grid_constant__ CUtensorMap tmY, GatherSrc g, int M_max, int layers, int hidden,
                        int layer_stride, FfnGammas gam, float eps, float* __restrict__ stats, int32_t* err,
                        const int32_t* M_dev) {
  griddep_wait();
  griddep_launch();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sA = smem;                          // F_KC x 16 KB
  uint8_t* sB = sA + F_KC * A_CHUNK;           // STAGES x 16 KB
  uint8_t* sH = sB + STAGES * B_HALF;          // 2 x 32 KB
  uint8_t* sOut = sH + 2 * F_HBUF;             // 8 warps x 2 KB
  uint64_t* bars = reinterpret_cast<uint64_t*>(sOut + 8 * OUT_STAGE);
  uint64_t* a_full = bars;                     // [4]      leader (gather, both CTAs)
  uint64_t* a_empty = bars + 4;                // [4]      both
  uint64_t* b_full = bars + 8;                 // [STAGES] leader
  uint64_t* b_empty = b_full + STAGES;         // [STAGES] both
  uint64_t* acc1_full = b_empty + STAGES;      // [1]      both
  uint64_t* acc1_empty = acc1_full + 1;        // [1]      leader (epilogue, both CTAs)
  uint64_t* h_full = acc1_empty + 1;           // [2]      leader (epilogue, both CTAs)
  uint64_t* h_empty = h_full + 2;              // [2]      both
  uint64_t* acc2_full = h_empty + 2;           // [1]      both
  uint64_t* acc2_empty = acc2_full + 1;        // [1]      leader (epilogue, both CTAs)
  uint64_t* mma_done = acc2_empty + 1;         // [1]      leader
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* s_sum = reinterpret_cast<float*>(bars + 8 + 2 * STAGES + 16);  // [2][128]
  float* s_sq = s_sum + 256;                                             // [2][128]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  const int M = M_dev ? min(M_max, *M_dev) : M_max;  // rows present in this call
  const int num_tiles = (M + 2 * BM - 1) / (2 * BM);
  const int cl = blockIdx.x >> 1, ncl = gridDim.x >> 1;
  const int NJ = hidden / F_HCH;

  if (threadIdx.x == 0) {
    for (int i = 0; i < F_KC; ++i) {
      mbar_init(&a_full[i], 256);
      mbar_init(&a_empty[i], 1);
    }
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&b_full[s], 1);
      mbar_init(&b_empty[s], 1);
    }
    mbar_init(acc1_full, 1);
    mbar_init(acc1_empty, 512);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&h_full[i], 512);
      mbar_init(&h_empty[i], 1);
    }
    mbar_init(acc2_full, 1);
    mbar_init(acc2_empty, 512);
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
    // weights, in the order the MMA thread consumes them: per layer and chunk step j, the
    // four K chunks of W1|W3 rows for chunk j (j < NJ), then the two K chunks of W2 for
    // chunk j - 1 (j >= 1); each CTA loads its 128 of the 256 N rows
    if (lane == 0) {
      prefetch_tmap(&tmW13);
      prefetch_tmap(&tmW2);
      const uint32_t b_full0 = cluster_addr(&b_full[0], 0);
      int it = 0;
      bool ok = true;
      auto load = [&](const CUtensorMap* map, int x, int y) -> bool {
        const int s = it % STAGES, round = it / STAGES;
        if ((round > 0 && !mbar_wait(&b_empty[s], (round - 1) & 1)) || abort_set(abort_flag)) {
          fail(abort_flag, err);
          return false;
        }
        if (leader) mbar_arrive_expect_tx(&b_full[s], 2 * B_HALF);
        tma_load_2d_pair(sB + s * B_HALF, map, x, y, b_full0 + s * 8);
        ++it;
        return true;
      };
      for (int tile = cl; tile < num_tiles && ok; tile += ncl)
        for (int l = 0; l < layers && ok; ++l)
          for (int j = 0; j <= NJ && ok; ++j) {
            if (j < NJ)
              for (int kc = 0; kc < F_KC && ok; ++kc)
                ok = load(&tmW13, kc * 64, (l * 2 * hidden + j * 2 * F_HCH) + int(rank) * BM);
            if (j >= 1)
              for (int kc = 0; kc < F_HCH / 64 && ok; ++kc)
                ok = load(&tmW2, (j - 1) * F_HCH + kc * 64, l * F_K + int(rank) * BM);
          }
      if (leader) drain_ring(b_full, STAGES, it);
    }
  } else if (warp == 1) {
    if (leader && lane == 0) {
      const uint32_t idesc = umma_idesc_bf16(256, 256);
      const uint64_t adesc0 = umma_sdesc_sw128(smem_u32(sA)), bdesc0 = umma_sdesc_sw128(smem_u32(sB));
      const uint64_t hdesc0 = umma_sdesc_sw128(smem_u32(sH));
      const uint32_t acc1 = tmem, acc2 = tmem + 256;
      int s = 0, c1 = 0, c2 = 0, lm = 0, li = 0;
      uint32_t bphase = 0;
      bool ok = true;
      auto next_stage = [&]() {
        if (++s == STAGES) {
          s = 0;
          bphase ^= 1;
        }
      };
      for (int tile = cl; tile < num_tiles && ok; tile += ncl, ++li) {
        for (int l = 0; l < layers && ok; ++l) {
          for (int j = 0; j <= NJ && ok; ++j) {
            if (j < NJ) {  // GEMM1 of chunk j: acc1 = X [W1 | W3]_{l, j}
              if (c1 > 0 && !mbar_wait_cluster(acc1_empty, (c1 - 1) & 1)) {
                fail(abort_flag, err);
                ok = false;
                break;
              }
              tc_fence_after();
              for (int kc = 0; kc < F_KC; ++kc) {
                if ((l == 0 && j == 0 && !mbar_wait_cluster(&a_full[kc], li & 1)) || !mbar_wait(&b_full[s], bphase)) {
                  fail(abort_flag, err);
                  ok = false;
                  break;
                }
                tc_fence_after();
                const uint64_t ad = adesc0 + uint64_t(kc * (A_CHUNK >> 4));
                const uint64_t bd = bdesc0 + uint64_t(s * (B_HALF >> 4));
                umma_bf16_pair(acc1, ad, bd, idesc, kc != 0);
                umma_bf16_pair(acc1, ad + 2, bd + 2, idesc, 1);
                umma_bf16_pair(acc1, ad + 4, bd + 4, idesc, 1);
                umma_bf16_pair(acc1, ad + 6, bd + 6, idesc, 1);
                umma_commit_pair_both(&b_empty[s], 0x3);
                if (l == layers - 1 && j == NJ - 1) umma_commit_pair_both(&a_empty[kc], 0x3);
                next_stage();
              }
              if (!ok) break;
              umma_commit_pair_both(acc1_full, 0x3);
              ++c1;
            }
            if (j >= 1) {  // GEMM2 of chunk j - 1: acc2 += hidden chunk x W2 rows
              const int hb = c2 & 1;
              if (!mbar_wait_cluster(&h_full[hb], (c2 >> 1) & 1) ||
                  (j == 1 && lm > 0 && !mbar_wait_cluster(acc2_empty, (lm - 1) & 1))) {
                fail(abort_flag, err);
                ok = false;
                break;
              }
              tc_fence_after();
              for (int kc = 0; kc < F_HCH / 64; ++kc) {
                if (!mbar_wait(&b_full[s], bphase)) {
                  fail(abort_flag, err);
                  ok = false;
                  break;
                }
                tc_fence_after();
                const uint64_t ad = hdesc0 + uint64_t((hb * 2 + kc) * (A_CHUNK >> 4));
                const uint64_t bd = bdesc0 + uint64_t(s * (B_HALF >> 4));
                umma_bf16_pair(acc2, ad, bd, idesc, (j > 1 || kc > 0) ? 1u : 0u);
                umma_bf16_pair(acc2, ad + 2, bd + 2, idesc, 1);
                umma_bf16_pair(acc2, ad + 4, bd + 4, idesc, 1);
                umma_bf16_pair(acc2, ad + 6, bd + 6, idesc, 1);
                umma_commit_pair_both(&b_empty[s], 0x3);
                next_stage();
              }
              if (!ok) break;
              umma_commit_pair_both(&h_empty[hb], 0x3);
              ++c2;
            }
          }
          if (!ok) break;
          umma_commit_pair_both(acc2_full, 0x3);
          ++lm;
        }
      }
      umma_commit_pair(cluster_addr(mma_done, 0));
      mbar_wait(mma_done, 0);
    }
  } else if (warp == 2 || warp == 12 || warp >= 14) {
    // gather warps: warp gw copies rows 32 gw .. 32 gw + 31 of this CTA's A tile, 8 lanes per
    // 128-byte row segment; chunk kc - GATHER_LAG is completed and published (with the time
    // bucket row added) right after chunk kc is issued.  The next tile's rows are
    // prefetched into L2 once this tile is published.
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
        if ((mask >> i) & 1u) prefetch_l2_bulk(table + int64_t(ids[i]) * F_K, uint32_t(F_K) * 2);
    };
    auto publish = [&](int kc) {
      if (with_dt) {
        uint8_t* chunk = sA + kc * A_CHUNK;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          if (!((vmask >> i) & 1u)) continue;
          const int r = gw * 32 + i * 4 + sub;
          uint4* p = reinterpret_cast<uint4*>(chunk + r * 128 + ((c ^ (r & 7)) << 4));
          const uint4 x = *p;
          const uint4 t = __ldg(reinterpret_cast<const uint4*>(dtt + int64_t(bk[i]) * F_K + kc * 64 + c * 8));
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
    };
    if (cl < num_tiles) {
      rows_of(cl, id, bk, vmask);
      prefetch_rows(id, vmask);
    }
    int li = 0;
    bool ok = true;
    for (int tile = cl; tile < num_tiles && ok; tile += ncl, ++li) {
      const int next = tile + ncl;
      if (next < num_tiles) rows_of(next, nid, nbk, nvmask);
      else nvmask = 0;
      for (int kc = 0; kc < F_KC; ++kc) {
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
          cp_async_16(chunk + r * 128 + ((c ^ (r & 7)) << 4), table + int64_t(v ? id[i] : 0) * F_K + kc * 64 + c * 8,
                      v ? 16u : 0u);
        }
        cp_async_commit();
        if (kc >= GATHER_LAG) {
          cp_async_wait<GATHER_LAG>();
          publish(kc - GATHER_LAG);
        }
      }
      if (!ok) break;
      for (int kc = F_KC - GATHER_LAG; kc < F_KC; ++kc) {
        cp_async_wait_dyn(F_KC - 1 - kc);
        publish(kc);
      }
      prefetch_rows(nid, nvmask);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        id[i] = nid[i];
        bk[i] = nbk[i];
      }
      vmask = nvmask;
    }
    cp_async_wait_all();
  } else if (warp >= 4 && warp < 12) {
    // two epilogue warps per TMEM lane quarter: half 0 / 1 takes hidden units 0..63 /
    // 64..127 of a chunk and output columns 0..127 / 128..255 of a layer
    const int quarter = warp & 3;
    const int half = (warp - 4) >> 2;
    const int r = quarter * 32 + lane;           // this thread's row of the CTA's 128
    uint8_t* stage = sOut + (warp - 4) * OUT_STAGE;
    const uint32_t lane_base = tmem + (uint32_t(quarter * 32) << 16);
    const uint32_t acc1_empty0 = cluster_addr(acc1_empty, 0);
    const uint32_t h_full0 = cluster_addr(&h_full[0], 0);
    const uint32_t acc2_empty0 = cluster_addr(acc2_empty, 0);
    int ce = 0, le = 0;
    bool ok = true;
    for (int tile = cl; tile < num_tiles && ok; tile += ncl) {
      const int y0 = tile * 2 * BM + int(rank) * BM + quarter * 32;  // first row of this warp's block
      for (int l = 0; l < layers && ok; ++l) {
        for (int j = 0; j < NJ; ++j, ++ce) {
          const int hb = ce & 1, use = ce >> 1;
          // the hidden buffer is free (GEMM2 two chunks back is done) and acc1 holds chunk j
          ok = !epilogue_any((use > 0 && !mbar_wait(&h_empty[hb], (use - 1) & 1)) ||
                             !mbar_wait(acc1_full, ce & 1) || abort_set(abort_flag));
          if (!ok) {
            fail(abort_flag, err);
            break;
          }
          tc_fence_after();
          uint8_t* hrow = sH + hb * F_HBUF + half * A_CHUNK + r * 128;
#pragma unroll 1
          for (int part = 0; part < 2; ++part) {
            const int col = half * 64 + part * 32;
            float gv[32], uv[32];
            tmem_ld_32x32b_x32(lane_base + col, gv);
            tmem_ld_32x32b_x32(lane_base + 128 + col, uv);
            tmem_ld_wait();
            uint32_t pk[16];
#pragma unroll
            for (int e = 0; e < 16; ++e)
              pk[e] = pack_bf16x2(silu_tanh(gv[2 * e]) * uv[2 * e], silu_tanh(gv[2 * e + 1]) * uv[2 * e + 1]);
            // 16-byte chunk cc (8 hidden units) of the row at cc ^ (r % 8): the MMA's swizzle
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int cc = part * 4 + q;
              *reinterpret_cast<uint4*>(hrow + ((cc ^ (r & 7)) << 4)) =
                  make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
            }
          }
          tc_fence_before();
          mbar_arrive_remote_relaxed(acc1_empty0);  // acc1 read: GEMM1 of the next chunk may start
          fence_proxy_async_smem();                 // the chunk is visible to the tensor cores
          mbar_arrive_remote(h_full0 + hb * 8);
        }
        if (!ok) break;
        // ---- layer l done: y' = (A W2) * gamma_l and the row moments (shifted by the row's
        // first value, so the shifted sums do not cancel)
        ok = !epilogue_any(!mbar_wait(acc2_full, le & 1) || abort_set(abort_flag));
        if (!ok) {
          fail(abort_flag, err);
          break;
        }
        tc_fence_after();
        const uint32_t tb = lane_base + 256 + half * 128;
        const float* gm = gam.g[l] + half * 128;
        float s1 = 0.f, s2 = 0.f, c0;
        {
          float v[32];
          tmem_ld_32x32b_x32(lane_base + 256, v);
          tmem_ld_wait();
          c0 = v[0];
        }
#pragma unroll 1
        for (int jj = 0; jj < 4; ++jj) {
          float v[32];
          tmem_ld_32x32b_x32(tb + jj * 32, v);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const float dv = v[e] - c0;
            s1 += dv;
            s2 = fmaf(dv, dv, s2);
            v[e] *= __ldg(gm + jj * 32 + e);
          }
          epi_store(stage, v, lane, &tmY, half * 128 + jj * 32, l * layer_stride + y0);
        }
        tc_fence_before();
        mbar_arrive_remote_relaxed(acc2_empty0);  // acc2 read: the next layer's GEMM2 may start
        s_sum[half * 128 + r] = s1;
        s_sq[half * 128 + r] = s2;
        epilogue_sync();
        if (half == 0 && y0 + lane < M) {
          const float m1 = (s_sum[r] + s_sum[128 + r]) * (1.0f / F_K);
          const float var = fmaxf((s_sq[r] + s_sq[128 + r]) * (1.0f / F_K) - m1 * m1, 0.f);
          reinterpret_cast<float2*>(stats)[int64_t(l) * layer_stride + y0 + lane] =
              make_float2(c0 + m1, rsqrtf(var + eps));
        }
        epilogue_sync();  // s_sum / s_sq are reused by the next layer
        ++le;
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

constexpr int FFN_STAGES = 4;

size_t ffn_smem() {
  return 1024 + size_t(F_KC) * A_CHUNK + size_t(FFN_STAGES) * B_HALF + 2 * F_HBUF + 8 * OUT_STAGE + 512 + 2 * 256 * 4;
}

}  // namespace

int tc_ffn_fused(const GatherSrc& g, int M, const int32_t* M_dev, int layers, int hidden, const void* W13p,
                 const void* W2p, const float* const* gammas, float eps, void* Y, int layer_stride, float* stats,
                 int32_t* err, cudaStream_t s, int max_pairs) {
  if (M == 0) return 0;
  if (M < 0 || layers < 1 || layers > STCA_MAX_LAYERS || hidden < F_HCH || hidden % F_HCH != 0 ||
      layer_stride < M || layer_stride % (2 * BM) != 0 || !W13p || !W2p || !Y || !stats || !gammas ||
      reinterpret_cast<uintptr_t>(Y) % 16 != 0 || reinterpret_cast<uintptr_t>(stats) % 8 != 0 || !g.ids ||
      !g.table)
    return STCA_ERR_INVALID_ARG;
  FfnGammas gam;
  memset(&gam, 0, sizeof(gam));
  for (int l = 0; l < layers; ++l) {
    if (!gammas[l]) return STCA_ERR_INVALID_ARG;
    gam.g[l] = gammas[l];
  }
  CUtensorMap t13, t2, ty;
  if (!make_tmap(&t13, W13p, uint64_t(layers) * 2 * hidden, F_K, F_K, BM)) return STCA_ERR_CUDA;
  if (!make_tmap(&t2, W2p, uint64_t(layers) * F_K, hidden, hidden, BM)) return STCA_ERR_CUDA;
  if (!make_tmap_out(&ty, Y, uint64_t(layers) * layer_stride, F_K, F_K)) return STCA_ERR_CUDA;
  auto kern = tc_ffn_fused_kernel<FFN_STAGES>;
  const size_t smem = ffn_smem();
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) != cudaSuccess)
    return STCA_ERR_CUDA;
  int pairs = std::min((M + 2 * BM - 1) / (2 * BM), sm_count() / 2);
  if (max_pairs > 0) pairs = std::min(pairs, max_pairs);
  const int grid = 2 * pairs;
  launch_dep(kern, dim3(grid), dim3(512), smem, s, t13, t2, ty, g, M, layers, hidden, layer_stride, gam, eps, stats,
             err, M_dev);
  note_launch();
  return cudaGetLastError() == cudaSuccess ? 0 : STCA_ERR_CUDA;
}

}  // namespace stca
