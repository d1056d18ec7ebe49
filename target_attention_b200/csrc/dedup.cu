// Per-request deduplication of history rows (HyFormer page §3.8.1, GPU pooling: only a
// small fraction of the ids in long sequences is distinct, so the sequence is rebuilt on
// the GPU from a compressed table of distinct rows).
//
// X~, K and V of a history token depend only on its key (item id, time bucket), so the
// three per-token GEMMs run once per distinct key and every token reads its K/V row
// through uniq_idx.  Each distinct row is computed exactly as it would be per token, so
// the forward result does not change.
//
// Build, all on the stream, no host round trip:
//   1. clear an open-addressing table of 2^k slots (keys = all ones = empty);
//   2. insert every token's key (atomicCAS, linear probing), remember its slot, and keep
//      the smallest token index with that key (atomicMin);
//   3. number the keys in order of their first token (a prefix scan over the tokens that
//      are first occurrences): uniq_token[u] = first token of key u, count = number of keys;
//   4. uniq_idx[n] = number of token n's key.
// Numbering by first occurrence is deterministic and keeps a user's new items on
// consecutive K/V rows, while repeated items point at rows of popular (cache-resident)
// keys.
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace stca {

namespace {

constexpr unsigned long long EMPTY_KEY = ~0ull;

__device__ __forceinline__ unsigned long long mix64(unsigned long long x) {
  // splitmix64 finalizer (Steele, Lea, Flood: "Fast splittable pseudorandom number generators")
  x ^= x >> 30;
  x *= 0xbf58476d1ce4e5b9ull;
  x ^= x >> 27;
  x *= 0x94d049bb133111ebull;
  x ^= x >> 31;
  return x;
}

__device__ __forceinline__ unsigned long long row_key(const int32_t* ids, const int32_t* dt, int n) {
  const unsigned long long id = static_cast<unsigned long long>(static_cast<uint32_t>(ids[n]));
  const int b = dt ? dt_bucket(dt[n] < 0 ? 0 : dt[n]) : 0;
  return (id << 4) | unsigned(b);
}

__global__ void insert_kernel(const int32_t* __restrict__ ids, const int32_t* __restrict__ dt, int n,
                              unsigned long long* __restrict__ keys, int32_t* __restrict__ first,
                              int32_t* __restrict__ slot_of, unsigned mask, int32_t* err) {
  griddep_wait();
  griddep_launch();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const unsigned long long key = row_key(ids, dt, i);
  unsigned slot = unsigned(mix64(key)) & mask;
  for (unsigned probe = 0; probe <= mask; ++probe) {
    // Popular keys (Zipf ids) are met by thousands of tokens: a plain read finds a key
    // that is already in place without an atomic on its hot slot, and the first-token
    // minimum is only lowered when this token can lower it.  A stale read costs one
    // atomic more, never a wrong result (keys are only ever set once, minima only fall).
    unsigned long long prev = __ldcg(&keys[slot]);
    if (prev == EMPTY_KEY) prev = atomicCAS(&keys[slot], EMPTY_KEY, key);
    if (prev == EMPTY_KEY || prev == key) {
      if (__ldcg(&first[slot]) > i) atomicMin(&first[slot], i);
      slot_of[i] = int32_t(slot);
      return;
    }
    slot = (slot + 1) & mask;
  }
  set_error(err, STCA_ERR_CAPACITY);  // table full (cannot happen with capacity >= 2 n)
  slot_of[i] = 0;
}

constexpr int SCAN_THREADS = 1024, SCAN_ITEMS = 4, SCAN_TILE = SCAN_THREADS * SCAN_ITEMS;

__device__ __forceinline__ bool is_first(const int32_t* first, const int32_t* slot_of, int i) {
  return first[slot_of[i]] == i;
}

// Block-wide exclusive scan of one int per thread; returns the block total.
__device__ __forceinline__ int block_exclusive_scan(int v, int& excl) {
  __shared__ int warp_tot[SCAN_THREADS / 32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int x = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += x;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = lane < SCAN_THREADS / 32 ? warp_tot[lane] : 0;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int x = __shfl_up_sync(0xffffffffu, w, off);
      if (lane >= off) w += x;
    }
    warp_tot[lane] = w;
  }
  __syncthreads();
  excl = (warp > 0 ? warp_tot[warp - 1] : 0) + incl - v;
  const int total = warp_tot[SCAN_THREADS / 32 - 1];
  __syncthreads();
  return total;
}

// first-occurrence count per tile of SCAN_TILE tokens
__global__ void __launch_bounds__(SCAN_THREADS) count_kernel(const int32_t* __restrict__ first,
                                                             const int32_t* __restrict__ slot_of, int n,
                                                             int32_t* __restrict__ tile_counts) {
  griddep_wait();
  griddep_launch();
  const int base = blockIdx.x * SCAN_TILE + threadIdx.x * SCAN_ITEMS;
  int c = 0;
#pragma unroll
  for (int k = 0; k < SCAN_ITEMS; ++k)
    if (base + k < n && is_first(first, slot_of, base + k)) ++c;
  int excl;
  const int total = block_exclusive_scan(c, excl);
  if (threadIdx.x == 0) tile_counts[blockIdx.x] = total;
}

// exclusive scan of the tile counts in place (one block); count = grand total
__global__ void __launch_bounds__(SCAN_THREADS) scan_tiles_kernel(int32_t* __restrict__ tile_counts, int tiles,
                                                                  int32_t* __restrict__ count) {
  griddep_wait();
  griddep_launch();
  int carry = 0;
  for (int b = 0; b < tiles; b += SCAN_THREADS) {
    const int i = b + threadIdx.x;
    const int v = i < tiles ? tile_counts[i] : 0;
    int excl;
    const int total = block_exclusive_scan(v, excl);
    if (i < tiles) tile_counts[i] = carry + excl;
    carry += total;
  }
  if (threadIdx.x == 0) *count = carry;
}

// number of each first occurrence; uniq_token[number] = its token
__global__ void __launch_bounds__(SCAN_THREADS) number_kernel(const int32_t* __restrict__ first,
                                                              const int32_t* __restrict__ slot_of, int n,
                                                              const int32_t* __restrict__ tile_offsets,
                                                              int32_t* __restrict__ pos,
                                                              int32_t* __restrict__ uniq_token) {
  griddep_wait();
  griddep_launch();
  const int base = blockIdx.x * SCAN_TILE + threadIdx.x * SCAN_ITEMS;
  bool f[SCAN_ITEMS];
  int c = 0;
#pragma unroll
  for (int k = 0; k < SCAN_ITEMS; ++k) {
    f[k] = base + k < n && is_first(first, slot_of, base + k);
    c += f[k];
  }
  int excl;
  block_exclusive_scan(c, excl);
  int p = tile_offsets[blockIdx.x] + excl;
#pragma unroll
  for (int k = 0; k < SCAN_ITEMS; ++k)
    if (f[k]) {
      pos[base + k] = p;
      uniq_token[p] = base + k;
      ++p;
    }
}

__global__ void map_kernel(const int32_t* __restrict__ first, const int32_t* __restrict__ slot_of,
                           const int32_t* __restrict__ pos, int n, int32_t* __restrict__ uniq_idx) {
  griddep_wait();
  griddep_launch();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) uniq_idx[i] = pos[first[slot_of[i]]];
}

// ---- per-user compaction: one CTA per user, open-addressing table in shared memory.
// The user's tokens map to K/V rows; every distinct row of the user is kept once, in order
// of its first token, with its number of tokens.  The list overwrites nothing: it is
// written into the user's own token range [hoff[u], hoff[u] + len[u]).
constexpr int CU_SLOTS = 16384;  // table slots (a user with more tokens keeps them all)
constexpr size_t CU_SMEM = size_t(3) * CU_SLOTS * 4;

__device__ __forceinline__ uint32_t mix32(uint32_t x) {
  // the 32-bit finalizer of MurmurHash3 (Appleby)
  x ^= x >> 16;
  x *= 0x85ebca6bu;
  x ^= x >> 13;
  x *= 0xc2b2ae35u;
  x ^= x >> 16;
  return x;
}

// Every token as its own entry with multiplicity 1 (the same attention result, no saving).
__device__ void compact_per_token(const int32_t* __restrict__ rows, int h0, int L, int32_t* __restrict__ out_rows,
                                  int32_t* __restrict__ out_mult, int32_t* __restrict__ out_len, int u) {
  for (int i = threadIdx.x; i < L; i += blockDim.x) {
    out_rows[h0 + i] = rows[h0 + i];
    out_mult[h0 + i] = 1;
  }
  if (threadIdx.x == 0) out_len[u] = L;
}

// User u's compaction by the whole block, with cu_smem (CU_SMEM bytes) for its table.
__device__ void compact_user(int u, const int32_t* __restrict__ hoff, const int32_t* __restrict__ rows,
                             int32_t* __restrict__ out_rows, int32_t* __restrict__ out_mult,
                             int32_t* __restrict__ out_len, int32_t* cu_smem) {
  __shared__ int table_failed;
  __syncthreads();  // a block that runs several users: the previous one is done with the table
  const int h0 = hoff[u], L = hoff[u + 1] - h0;
  if (L >= CU_SLOTS) {  // too long for the table: every token is its own entry
    compact_per_token(rows, h0, L, out_rows, out_mult, out_len, u);
    return;
  }
  int cap = 64;
  while (cap < 2 * L && cap < CU_SLOTS) cap <<= 1;
  const uint32_t mask = uint32_t(cap - 1);
  int32_t* keys = cu_smem;
  int32_t* first = keys + CU_SLOTS;
  int32_t* cnt = first + CU_SLOTS;
  if (threadIdx.x == 0) table_failed = 0;
  for (int i = threadIdx.x; i < cap; i += blockDim.x) {
    keys[i] = -1;
    first[i] = 0x7fffffff;
    cnt[i] = 0;
  }
  __syncthreads();
  // insert: L < cap, so a free slot always exists within cap probes; the probe count is
  // bounded all the same, and a table that ran out sends the user to the per-token form
  for (int i = threadIdx.x; i < L; i += blockDim.x) {
    const int32_t r = rows[h0 + i];
    uint32_t slot = mix32(uint32_t(r)) & mask;
    int probe = 0;
    for (; probe < cap; ++probe) {
      const int32_t prev = atomicCAS(&keys[slot], -1, r);
      if (prev == -1 || prev == r) break;
      slot = (slot + 1) & mask;
    }
    if (probe == cap) {
      table_failed = 1;
      continue;
    }
    atomicMin(&first[slot], i);
    atomicAdd(&cnt[slot], 1);
  }
  __syncthreads();
  if (table_failed) {
    compact_per_token(rows, h0, L, out_rows, out_mult, out_len, u);
    return;
  }
  // first occurrences in token order, numbered by a block scan per chunk of tokens
  int base = 0;
  for (int c0 = 0; c0 < L; c0 += SCAN_THREADS) {
    const int i = c0 + threadIdx.x;
    int f = 0;
    int32_t r = 0, m = 0;
    if (i < L) {
      r = rows[h0 + i];
      uint32_t slot = mix32(uint32_t(r)) & mask;
      int probe = 0;
      while (keys[slot] != r && probe < cap) {  // every key was inserted: found within cap probes
        slot = (slot + 1) & mask;
        ++probe;
      }
      if (probe < cap) {
        f = first[slot] == i;
        m = cnt[slot];
      } else {
        table_failed = 1;
      }
    }
    int excl;
    const int total = block_exclusive_scan(f, excl);
    if (f) {
      out_rows[h0 + base + excl] = r;
      out_mult[h0 + base + excl] = m;
    }
    base += total;
  }
  __syncthreads();
  if (table_failed) {  // a lookup that could not happen did: rewrite the user per token
    compact_per_token(rows, h0, L, out_rows, out_mult, out_len, u);
    return;
  }
  if (threadIdx.x == 0) out_len[u] = base;
}

__global__ void __launch_bounds__(SCAN_THREADS) compact_user_kernel(const int32_t* __restrict__ hoff,
                                                                    const int32_t* __restrict__ rows,
                                                                    int32_t* __restrict__ out_rows,
                                                                    int32_t* __restrict__ out_mult,
                                                                    int32_t* __restrict__ out_len) {
  griddep_wait();
  griddep_launch();
  extern __shared__ int32_t cu_smem[];
  compact_user(blockIdx.x, hoff, rows, out_rows, out_mult, out_len, cu_smem);
}

// ---- everything above in one cooperative launch (one block per SM): clear the table,
// insert, count first occurrences per tile, number them, map every token, and (when hoff
// is given) compact every user, with a grid-wide barrier between the phases.  At short
// histories the separate launches (and their gaps) cost more than the work; a block
// numbers a tile from the sum of the earlier tiles' counts, so no scan pass is needed.

struct DedupFused {
  const int32_t* ids;
  const int32_t* dt;
  int n;
  unsigned long long* keys;
  int32_t* first;
  int32_t* slot_of;
  int32_t* pos;
  int32_t* tile_counts;
  unsigned mask;
  unsigned* barrier;  // zero at launch
  int32_t* uniq_idx;
  int32_t* uniq_token;
  int32_t* count;
  const int32_t* hoff;  // compaction when not null
  int B;
  int32_t* c_rows;
  int32_t* c_mult;
  int32_t* c_len;
  int32_t* err;
};

__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Grid-wide barrier number k (1, 2, ...): every block arrives once; bounded wait (records
// STCA_ERR_TIMEOUT and returns false when the other blocks do not arrive in time).
__device__ bool grid_barrier(unsigned* ctr, unsigned k, int32_t* err) {
  __shared__ int ok_s;
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    atomicAdd(ctr, 1u);
    const unsigned target = k * gridDim.x;
    int ok = 1;
    if (ld_acquire_gpu(ctr) < target) {
      const uint64_t t0 = global_timer_ns();
      while (ld_acquire_gpu(ctr) < target) {
        if (global_timer_ns() - t0 > STCA_WAIT_NS) {
          set_error(err, STCA_ERR_TIMEOUT);
          ok = 0;
          break;
        }
      }
    }
    __threadfence();
    ok_s = ok;
  }
  __syncthreads();
  return ok_s != 0;
}

__global__ void __launch_bounds__(SCAN_THREADS, 1) dedup_fused_kernel(DedupFused a) {
  extern __shared__ int32_t cu_smem[];
  const int tid = threadIdx.x, G = gridDim.x;
  const int64_t gthreads = int64_t(G) * SCAN_THREADS, gtid = int64_t(blockIdx.x) * SCAN_THREADS + tid;
  const int n = a.n;
  const int64_t cap = int64_t(a.mask) + 1;
  // 0. empty table
  for (int64_t i = gtid; i < cap; i += gthreads) {
    a.keys[i] = EMPTY_KEY;
    a.first[i] = 0x7fffffff;
  }
  if (!grid_barrier(a.barrier, 1, a.err)) return;
  // 1. insert every token's key
  for (int64_t i = gtid; i < n; i += gthreads) {
    const int ii = int(i);
    const unsigned long long key = row_key(a.ids, a.dt, ii);
    unsigned slot = unsigned(mix64(key)) & a.mask;
    bool placed = false;
    for (unsigned probe = 0; probe <= a.mask; ++probe) {
      unsigned long long prev = __ldcg(&a.keys[slot]);
      if (prev == EMPTY_KEY) prev = atomicCAS(&a.keys[slot], EMPTY_KEY, key);
      if (prev == EMPTY_KEY || prev == key) {
        if (__ldcg(&a.first[slot]) > ii) atomicMin(&a.first[slot], ii);
        a.slot_of[ii] = int32_t(slot);
        placed = true;
        break;
      }
      slot = (slot + 1) & a.mask;
    }
    if (!placed) {
      set_error(a.err, STCA_ERR_CAPACITY);
      a.slot_of[ii] = 0;
    }
  }
  if (!grid_barrier(a.barrier, 2, a.err)) return;
  // 2. first occurrences per tile of SCAN_TILE tokens
  const int tiles = (n + SCAN_TILE - 1) / SCAN_TILE;
  for (int t = blockIdx.x; t < tiles; t += G) {
    const int base = t * SCAN_TILE + tid * SCAN_ITEMS;
    int c = 0;
#pragma unroll
    for (int k = 0; k < SCAN_ITEMS; ++k)
      if (base + k < n && is_first(a.first, a.slot_of, base + k)) ++c;
    int excl;
    const int total = block_exclusive_scan(c, excl);
    if (tid == 0) a.tile_counts[t] = total;
  }
  if (!grid_barrier(a.barrier, 3, a.err)) return;
  // 3. number the first occurrences: tile t starts at the sum of the earlier tiles' counts
  for (int t = blockIdx.x; t < tiles; t += G) {
    int before = 0;
    for (int i = tid; i < t; i += SCAN_THREADS) before += a.tile_counts[i];
    int excl0;
    const int start = block_exclusive_scan(before, excl0);  // the block total
    const int base = t * SCAN_TILE + tid * SCAN_ITEMS;
    bool f[SCAN_ITEMS];
    int c = 0;
#pragma unroll
    for (int k = 0; k < SCAN_ITEMS; ++k) {
      f[k] = base + k < n && is_first(a.first, a.slot_of, base + k);
      c += f[k];
    }
    int excl;
    const int total = block_exclusive_scan(c, excl);
    int p = start + excl;
#pragma unroll
    for (int k = 0; k < SCAN_ITEMS; ++k)
      if (f[k]) {
        a.pos[base + k] = p;
        a.uniq_token[p] = base + k;
        ++p;
      }
    if (t == tiles - 1 && tid == 0) *a.count = start + total;
  }
  if (tiles == 0 && blockIdx.x == 0 && tid == 0) *a.count = 0;
  if (!grid_barrier(a.barrier, 4, a.err)) return;
  // 4. token -> number of its key
  for (int64_t i = gtid; i < n; i += gthreads) a.uniq_idx[i] = a.pos[a.first[a.slot_of[i]]];
  if (!a.hoff) return;
  if (!grid_barrier(a.barrier, 5, a.err)) return;
  // 5. per-user compaction of the K/V rows
  for (int u = blockIdx.x; u < a.B; u += G) compact_user(u, a.hoff, a.uniq_idx, a.c_rows, a.c_mult, a.c_len, cu_smem);
}

}  // namespace

int compact_user_rows(const int32_t* hoff, int B, const int32_t* rows, int32_t* out_rows, int32_t* out_mult,
                      int32_t* out_len, cudaStream_t s) {
  if (B <= 0) return STCA_OK;
  if (cudaFuncSetAttribute(compact_user_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(CU_SMEM)) !=
      cudaSuccess)
    return STCA_ERR_CUDA;
  launch_dep(compact_user_kernel, dim3(B), dim3(SCAN_THREADS), CU_SMEM, s, hoff, rows, out_rows, out_mult, out_len);
  note_launch();
  return cudaGetLastError() == cudaSuccess ? STCA_OK : STCA_ERR_CUDA;
}

size_t dedup_table_slots(int max_tokens) {
  size_t cap = 1024;
  while (cap < size_t(2) * size_t(max_tokens)) cap <<= 1;
  return cap;
}

namespace {
// keys [cap] u64 | first [cap] i32 | slot_of [n] i32 | pos [n] i32 | tile offsets |
// the fused kernel's barrier counter (16-byte aligned)
size_t layout_bytes(size_t cap, int n) {
  const size_t tiles = (size_t(n) + SCAN_TILE - 1) / SCAN_TILE + 1;
  return cap * 8 + cap * 4 + size_t(n) * 8 + tiles * 4 + 64 + 64;
}
}  // namespace

size_t dedup_workspace_bytes(int max_tokens) { return layout_bytes(dedup_table_slots(max_tokens), max_tokens); }

int dedup_rows(const int32_t* ids, const int32_t* dt, int n, void* ws, size_t ws_bytes, int32_t* uniq_idx,
               int32_t* uniq_token, int32_t* count, int32_t* err, cudaStream_t s) {
  if (n < 0) return STCA_ERR_INVALID_ARG;
  const size_t cap = dedup_table_slots(n);
  if (layout_bytes(cap, n) > ws_bytes) return STCA_ERR_CAPACITY;
  uint8_t* p = reinterpret_cast<uint8_t*>(ws);
  unsigned long long* keys = reinterpret_cast<unsigned long long*>(p);
  int32_t* first = reinterpret_cast<int32_t*>(p + cap * 8);
  int32_t* slot_of = first + cap;
  int32_t* pos = slot_of + n;
  int32_t* tile_off = pos + n;
  if (cudaMemsetAsync(count, 0, sizeof(int32_t), s) != cudaSuccess) return STCA_ERR_CUDA;
  if (n == 0) return STCA_OK;
  const int tiles = (n + SCAN_TILE - 1) / SCAN_TILE;
  if (cudaMemsetAsync(keys, 0xFF, cap * 8, s) != cudaSuccess) return STCA_ERR_CUDA;
  if (cudaMemsetAsync(first, 0x7F, cap * 4, s) != cudaSuccess) return STCA_ERR_CUDA;  // INT_MAX-like
  launch_dep(insert_kernel, dim3((n + 255) / 256), dim3(256), 0, s, ids, dt, n, keys, first, slot_of,
             unsigned(cap - 1), err);
  note_launch();
  launch_dep(count_kernel, dim3(tiles), dim3(SCAN_THREADS), 0, s, first, slot_of, n, tile_off);
  note_launch();
  launch_dep(scan_tiles_kernel, dim3(1), dim3(SCAN_THREADS), 0, s, tile_off, tiles, count);
  note_launch();
  launch_dep(number_kernel, dim3(tiles), dim3(SCAN_THREADS), 0, s, first, slot_of, n, tile_off, pos, uniq_token);
  note_launch();
  launch_dep(map_kernel, dim3((n + 255) / 256), dim3(256), 0, s, first, slot_of, pos, n, uniq_idx);
  note_launch();
  return cudaGetLastError() == cudaSuccess ? STCA_OK : STCA_ERR_CUDA;
}

int dedup_fused(const int32_t* ids, const int32_t* dt, int n, void* ws, size_t ws_bytes, int32_t* uniq_idx,
                int32_t* uniq_token, int32_t* count, const int32_t* hoff, int B, int32_t* c_rows, int32_t* c_mult,
                int32_t* c_len, int32_t* err, cudaStream_t s) {
  if (n < 0 || B < 0) return STCA_ERR_INVALID_ARG;
  const size_t cap = dedup_table_slots(n);
  if (layout_bytes(cap, n) > ws_bytes) return STCA_ERR_CAPACITY;
  uint8_t* p = reinterpret_cast<uint8_t*>(ws);
  DedupFused a;
  a.ids = ids;
  a.dt = dt;
  a.n = n;
  a.keys = reinterpret_cast<unsigned long long*>(p);
  a.first = reinterpret_cast<int32_t*>(p + cap * 8);
  a.slot_of = a.first + cap;
  a.pos = a.slot_of + n;
  a.tile_counts = a.pos + n;
  const size_t tiles = (size_t(n) + SCAN_TILE - 1) / SCAN_TILE + 1;
  const uintptr_t bar = (reinterpret_cast<uintptr_t>(a.tile_counts + tiles) + 15) & ~uintptr_t(15);
  a.barrier = reinterpret_cast<unsigned*>(bar);
  a.mask = unsigned(cap - 1);
  a.uniq_idx = uniq_idx;
  a.uniq_token = uniq_token;
  a.count = count;
  a.hoff = (hoff && B > 0) ? hoff : nullptr;
  a.B = B;
  a.c_rows = c_rows;
  a.c_mult = c_mult;
  a.c_len = c_len;
  a.err = err;
  if (a.hoff && (!c_rows || !c_mult || !c_len)) return STCA_ERR_INVALID_ARG;
  static int blocks_per_sm = -1;
  if (blocks_per_sm < 0) {
    if (cudaFuncSetAttribute(dedup_fused_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(CU_SMEM)) !=
            cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&blocks_per_sm, dedup_fused_kernel, SCAN_THREADS, CU_SMEM) !=
            cudaSuccess || blocks_per_sm < 1)
      return STCA_ERR_CUDA;
  }
  if (cudaMemsetAsync(a.barrier, 0, sizeof(unsigned), s) != cudaSuccess) return STCA_ERR_CUDA;
  int grid = sm_count() * blocks_per_sm;
  const int64_t want = std::max<int64_t>(std::max<int64_t>((int64_t(n) + SCAN_THREADS - 1) / SCAN_THREADS, B), 1);
  if (grid > want) grid = int(want);
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(SCAN_THREADS);
  cfg.dynamicSmemBytes = CU_SMEM;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;  // every block resident at once: the barriers need it
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, dedup_fused_kernel, a) != cudaSuccess) return STCA_ERR_CUDA;
  note_launch();
  return STCA_OK;
}

}  // namespace stca
