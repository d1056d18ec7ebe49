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
//   2. insert every token's key (atomicCAS, linear probing), remember its slot and, for
//      the token that created the slot, that token;
//   3. number the occupied slots (warp-aggregated atomicAdd): uniq_token[u] = a token with
//      that key, count = number of distinct keys;
//   4. uniq_idx[n] = number of token n's slot.
// The numbering order depends on scheduling; results do not, because each distinct row
// is computed independently of where it sits.
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
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const unsigned long long key = row_key(ids, dt, i);
  unsigned slot = unsigned(mix64(key)) & mask;
  for (unsigned probe = 0; probe <= mask; ++probe) {
    const unsigned long long prev = atomicCAS(&keys[slot], EMPTY_KEY, key);
    if (prev == EMPTY_KEY) {
      first[slot] = i;
      slot_of[i] = int32_t(slot);
      return;
    }
    if (prev == key) {
      slot_of[i] = int32_t(slot);
      return;
    }
    slot = (slot + 1) & mask;
  }
  set_error(err, STCA_ERR_CAPACITY);  // table full (cannot happen with capacity >= 2 n)
  slot_of[i] = 0;
}

__global__ void number_kernel(const unsigned long long* __restrict__ keys, const int32_t* __restrict__ first,
                              unsigned cap, int32_t* __restrict__ slot_index, int32_t* __restrict__ uniq_token,
                              int32_t* __restrict__ count) {
  const unsigned s = blockIdx.x * blockDim.x + threadIdx.x;
  const bool occ = s < cap && keys[s] != EMPTY_KEY;
  const unsigned ballot = __ballot_sync(0xffffffffu, occ);
  if (ballot == 0) return;
  const int lane = threadIdx.x & 31;
  int base = 0;
  if (lane == 0) base = atomicAdd(count, __popc(ballot));
  base = __shfl_sync(0xffffffffu, base, 0);
  if (occ) {
    const int idx = base + __popc(ballot & ((1u << lane) - 1u));
    slot_index[s] = idx;
    uniq_token[idx] = first[s];
  }
}

__global__ void map_kernel(const int32_t* __restrict__ slot_of, const int32_t* __restrict__ slot_index, int n,
                           int32_t* __restrict__ uniq_idx) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) uniq_idx[i] = slot_index[slot_of[i]];
}

}  // namespace

size_t dedup_table_slots(int max_tokens) {
  size_t cap = 1024;
  while (cap < size_t(2) * size_t(max_tokens)) cap <<= 1;
  return cap;
}

size_t dedup_workspace_bytes(int max_tokens) {
  const size_t cap = dedup_table_slots(max_tokens);
  return cap * 8 + cap * 4 * 2 + size_t(max_tokens) * 4 + 16;
}

int dedup_rows(const int32_t* ids, const int32_t* dt, int n, void* ws, size_t ws_bytes, int32_t* uniq_idx,
               int32_t* uniq_token, int32_t* count, int32_t* err, cudaStream_t s) {
  if (n < 0) return STCA_ERR_INVALID_ARG;
  size_t cap = 1024;
  while (cap < size_t(2) * size_t(n)) cap <<= 1;
  if (cap * 8 + cap * 8 + size_t(n) * 4 + 16 > ws_bytes) return STCA_ERR_CAPACITY;
  uint8_t* p = reinterpret_cast<uint8_t*>(ws);
  unsigned long long* keys = reinterpret_cast<unsigned long long*>(p);
  int32_t* first = reinterpret_cast<int32_t*>(p + cap * 8);
  int32_t* slot_index = first + cap;
  int32_t* slot_of = slot_index + cap;
  if (cudaMemsetAsync(count, 0, sizeof(int32_t), s) != cudaSuccess) return STCA_ERR_CUDA;
  if (n == 0) return STCA_OK;
  if (cudaMemsetAsync(keys, 0xFF, cap * 8, s) != cudaSuccess) return STCA_ERR_CUDA;
  insert_kernel<<<(n + 255) / 256, 256, 0, s>>>(ids, dt, n, keys, first, slot_of, unsigned(cap - 1), err);
  note_launch();
  number_kernel<<<unsigned((cap + 255) / 256), 256, 0, s>>>(keys, first, unsigned(cap), slot_index, uniq_token,
                                                             count);
  note_launch();
  map_kernel<<<(n + 255) / 256, 256, 0, s>>>(slot_of, slot_index, n, uniq_idx);
  note_launch();
  return cudaGetLastError() == cudaSuccess ? STCA_OK : STCA_ERR_CUDA;
}

}  // namespace stca
