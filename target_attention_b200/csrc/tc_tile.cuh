// Tile helpers shared by the tcgen05 history kernels (tc_gemm.cu, tc_ffn.cu): tile
// constants, the bounded-wait failure path, the epilogue's staged TMA store, SiLU, the
// epilogue warps' named barrier and the gathered-row lookup.  Everything here is device
// code in an anonymous namespace, so each translation unit gets its own copy.
#pragma once

#include "common.cuh"
#include "internal.h"

namespace stca {
namespace {

constexpr int BM = 128;                        // tile rows = TMEM lanes
constexpr int A_CHUNK = BM * 64 * 2;           // one 64-wide K chunk of A: 16 KB
constexpr int B_HALF = BM * 128;               // one CTA's 128 weight rows x 64 K: 16 KB
constexpr int OUT_STAGE = 32 * 64;             // one epilogue warp's 32 x 32 bf16 output tile
constexpr int MIN_SMEM = 120 * 1024;           // keeps one CTA per SM (TMEM is not shared)
constexpr int GATHER_LAG = 2;                  // gathered chunks in flight before one is published
// N tiles before the end of a row tile at which the gather prefetches the next row
// tile's table rows into L2
constexpr int PREFETCH_LEAD = 3;

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

// Epilogue store: lane r of a warp holds 32 consecutive fp32 values of output row r of
// the warp's 32-row block.  They are staged as bf16 in the warp's 2 KB shared buffer
// (64-byte rows with the 64-byte swizzle: 16-byte chunk c of row r sits at chunk
// c ^ ((r >> 1) & 3), which keeps the lanes' writes on distinct banks) and written with
// one TMA tile store of 32 x 32 at (x, y); rows or columns outside C are clipped by TMA.
// The buffer is reused once the previous store has read it.
__device__ __forceinline__ void epi_store(uint8_t* stage, const float (&v)[32], int lane, const CUtensorMap* tmC,
                                          int x, int y) {
  uint32_t packed[16];
#pragma unroll
  for (int q = 0; q < 16; ++q) packed[q] = pack_bf16x2(v[2 * q], v[2 * q + 1]);
  if (lane == 0) bulk_wait_read<0>();
  __syncwarp();
  uint8_t* rowp = stage + lane * 64;
#pragma unroll
  for (int c = 0; c < 4; ++c)
    *reinterpret_cast<uint4*>(rowp + ((c ^ ((lane >> 1) & 3)) << 4)) =
        make_uint4(packed[4 * c], packed[4 * c + 1], packed[4 * c + 2], packed[4 * c + 3]);
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) {
    tma_store_2d(tmC, x, y, stage);
    bulk_commit();
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

// Same barrier, returning whether any of the 256 epilogue threads passed `flag` != 0, so
// that they all take the same branch afterwards.
__device__ __forceinline__ bool epilogue_any(bool flag) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, 1, 256, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(uint32_t(flag))
      : "memory");
  return r != 0;
}


// Item id and time bucket of global row `grow`; false (and a zero row) when the row is
// past M or the id is out of range (recorded in the error word).
__device__ __forceinline__ bool gather_row(const GatherSrc& g, int grow, int M, int64_t& id, int& bucket,
                                           int32_t* err) {
  id = 0;
  bucket = 0;
  if (grow >= M) return false;
  const int tok = g.rows ? g.rows[grow] : grow;
  id = g.ids[tok];
  if (g.dt) {
    const int32_t dt = g.dt[tok];
    if (dt < 0) set_error(err, STCA_ERR_INVALID_ARG);
    bucket = dt_bucket(dt < 0 ? 0 : dt);
  }
  if (id < 0 || id >= g.n_items) {
    set_error(err, STCA_ERR_ID_OUT_OF_RANGE);
    id = 0;
    return false;
  }
  return true;
}

}  // namespace

}  // namespace stca
