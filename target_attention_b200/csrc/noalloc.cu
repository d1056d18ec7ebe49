// stca_pointwise_forward_noalloc: the pointwise ReLU target attention without a handle
// and without any device allocation.
//
// Some callers cannot call cudaMalloc: plugins that run inside a host runtime which owns
// the whole device memory pool and forbids other allocations, and latency-critical
// request paths where an allocation (which may synchronise the device) is not allowed.
// This entry point keeps its scratch (the ragged offsets and the per-slice partial sums)
// in a fixed-size array in device memory that belongs to the library image; the caller
// passes only inputs and outputs.
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace {

constexpr int NOALLOC_MAX_USERS = STCA_NOALLOC_MAX_USERS;
constexpr int NOALLOC_MAX_SPLITS = 4;
constexpr int NOALLOC_D = 128;

struct NoallocScratch {
  int32_t offsets[NOALLOC_MAX_USERS + 1];
  int32_t err;
  float partials[NOALLOC_MAX_SPLITS * NOALLOC_MAX_USERS * NOALLOC_D];
};

// Every GPU that loads the library holds this array (about 4.2 MB) until the process
// exits.  All calls share it and it keeps the last call's contents: each call rewrites
// the offsets and every partial slot it reads, so nothing has to start at zero.
static __device__ __align__(256) unsigned char g_noalloc_scratch[sizeof(NoallocScratch)];

constexpr int MAX_DEVICES = 64;
std::mutex g_mutex;

// The address is looked up once per device and context: it is kept with the id of the
// context it was found in, and looked up again when the device's current context has
// another id (after a cudaDeviceReset, the primary context is a new one and the array has
// a new address).  Context ids come from the driver (cuCtxGetCurrent, cuCtxGetId), reached
// through the runtime's entry-point query so the library needs no link against libcuda.
struct ScratchAddr {
  unsigned long long ctx_id;
  void* addr;
};
ScratchAddr g_addr[MAX_DEVICES] = {};

typedef int (*CtxGetCurrentFn)(void**);
typedef int (*CtxGetIdFn)(void*, unsigned long long*);

bool current_context_id(unsigned long long* id) {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static bool looked_up = false;
  if (!looked_up) {
    looked_up = true;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
    cudaGetLastError();
  }
  void* ctx = nullptr;
  if (!get_current || !get_id || get_current(&ctx) != 0 || !ctx) return false;
  return get_id(ctx, id) == 0;
}

// Device address of the scratch array on the current device.  In host code the array's
// name is only a host-side stand-in, so its device address is asked of the runtime, once
// per device and context (see above; where the driver gives no context id, every call
// asks).
NoallocScratch* scratch_on_current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_DEVICES) return nullptr;
  unsigned long long ctx_id = 0;
  const bool have_id = current_context_id(&ctx_id);
  std::lock_guard<std::mutex> lock(g_mutex);
  if (!have_id || g_addr[dev].addr == nullptr || g_addr[dev].ctx_id != ctx_id) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) {
      cudaGetLastError();
      return nullptr;
    }
    g_addr[dev].addr = p;
    g_addr[dev].ctx_id = have_id ? ctx_id : 0;
  }
  return reinterpret_cast<NoallocScratch*>(g_addr[dev].addr);
}

__global__ void copy_error_word(const int32_t* src, int32_t* dst) {
  if (threadIdx.x == 0 && blockIdx.x == 0 && *src != 0) atomicCAS(dst, 0, *src);
}

__global__ void clear_error_word(int32_t* e) {
  if (threadIdx.x == 0 && blockIdx.x == 0) *e = 0;
}

}  // namespace

extern "C" int stca_pointwise_forward_noalloc(const int32_t* ids, const int32_t* lengths, const void* q,
                                              const void* table, int64_t n_items, int B, int n_tok, float* out,
                                              int32_t* err_out, void* stream) {
  if (B < 0 || n_tok < 0 || n_items <= 0) return STCA_ERR_INVALID_ARG;
  if (B > NOALLOC_MAX_USERS) return STCA_ERR_CAPACITY;
  if (B > 0 && (!lengths || !q || !table || !out)) return STCA_ERR_INVALID_ARG;
  if (n_tok > 0 && !ids) return STCA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(table)) & 15) return STCA_ERR_INVALID_ARG;
  if (B == 0) return STCA_OK;
  NoallocScratch* sc = scratch_on_current_device();
  if (!sc) return STCA_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int splits = int((int64_t(n_tok) / B + 2047) / 2048);
  splits = splits < 1 ? 1 : (splits > NOALLOC_MAX_SPLITS ? NOALLOC_MAX_SPLITS : splits);
  clear_error_word<<<1, 32, 0, s>>>(&sc->err);
  stca::note_launch();
  int rc = stca::exclusive_offsets(lengths, B, sc->offsets, n_tok, &sc->err, s);
  if (rc != STCA_OK) return rc;
  rc = stca::pointwise_relu_ta(ids, sc->offsets, q, table, n_items, B, NOALLOC_D, splits, sc->partials, out, &sc->err,
                               s);
  if (rc != STCA_OK) return rc;
  if (err_out) {
    copy_error_word<<<1, 32, 0, s>>>(&sc->err, err_out);
    stca::note_launch();
  }
  return cudaGetLastError() == cudaSuccess ? STCA_OK : STCA_ERR_CUDA;
}
