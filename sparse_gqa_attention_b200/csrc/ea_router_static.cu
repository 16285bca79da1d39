// ea_router_static.cu — ea_router_static_scratch: the router with scratch memory that
// the library owns, for callers that cannot allocate device memory.
//
// Some callers of this router cannot call cudaMalloc, for instance an inference runtime
// or plugin host that hands out all device memory through its own allocator.  This
// entry point takes the same inputs and outputs as ea_router but keeps its pooling
// partial sums and pooled hidden states in a fixed array compiled into the library, so
// it allocates nothing.
//
// The array is a file-scope __device__ variable: every GPU that loads the library holds
// kStaticScratchBytes of it until the process exits.  Host code cannot use the array's
// name as a device address, so the first call on each device looks the address up with
// cudaGetSymbolAddress (that device current) and caches it together with the context it
// was found in; a later call in another context (after a device reset, or from a caller's
// own context) looks it up again.  All calls share the one array, so calls whose kernels
// overlap on the GPU (different streams, or different host threads) race on it; order
// them on one stream.  Nothing in it needs to start at zero: every byte a call reads was
// written earlier in the same call.
#include <cuda_runtime.h>
#include <cstdint>
#include <mutex>
#include "ea_common.cuh"
#include "ea_internal.h"

namespace {

constexpr size_t kStaticScratchBytes = EA_ROUTER_STATIC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_router_scratch[kStaticScratchBytes];

std::mutex g_scratch_mu;
// One cached address per device, valid for the context it was looked up in (by the
// context's unique id, which the driver never reuses within a process): a different
// current context (after a device reset, or a caller's own non-primary context) gets
// the address looked up again.
struct CachedAddress {
  unsigned long long ctx_id;
  void* ptr;
};
CachedAddress g_scratch[kMaxDevices] = {};

typedef int (*CtxGetCurrentFn)(void**);                    // the driver's cuCtxGetCurrent
typedef int (*CtxGetIdFn)(void*, unsigned long long*);     // the driver's cuCtxGetId

template <typename F>
F driver_fn(const char* name) {
  void* f = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPointByVersion(name, &f, 12000, cudaEnableDefault, &q) == cudaSuccess &&
      q == cudaDriverEntryPointSuccess)
    return reinterpret_cast<F>(f);
  return nullptr;
}

// Unique id of the calling thread's current context; false when there is none yet.
bool current_context_id(unsigned long long* id) {
  static CtxGetCurrentFn get_ctx = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    get_ctx = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
    get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
  });
  void* ctx = nullptr;
  if (!get_ctx || !get_id || get_ctx(&ctx) != 0 || ctx == nullptr) return false;
  return get_id(ctx, id) == 0;
}

// Device address of g_router_scratch in the current device's current context.
ea_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return EA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return EA_ERR_UNSUPPORTED;
  unsigned long long id = 0;
  const bool have_ctx = current_context_id(&id);
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (have_ctx && g_scratch[dev].ptr != nullptr && g_scratch[dev].ctx_id == id) {
    *out = g_scratch[dev].ptr;
    return EA_OK;
  }
  // First call in this context (the lookup also starts the runtime's context on a thread
  // that has none yet, so the context is read again afterwards).
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_router_scratch) != cudaSuccess || p == nullptr) return EA_ERR_CUDA;
  if (!current_context_id(&id)) return EA_ERR_CUDA;
  g_scratch[dev].ctx_id = id;
  g_scratch[dev].ptr = p;
  *out = p;
  return EA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" ea_status ea_router_static_scratch(const void* hidden, ea_dtype dtype, int B, int S, int D, int H_kv,
                                              int d, const ea_router_weights* w, const ea_router_params* prm,
                                              int32_t* head_mode, float* logits, void* stream) {
  if (!hidden || !w || !prm || !head_mode) return EA_ERR_INVALID_ARG;
  if (!w->w_k || !w->w_t1 || !w->b_t1 || !w->w_t2 || !w->b_t2 || !w->w_r1 || !w->b_r1 || !w->w_o || !w->b_o)
    return EA_ERR_INVALID_ARG;
  if (B < 1 || S < 1 || D < 1 || H_kv < 1) return EA_ERR_INVALID_ARG;
  if (H_kv > EA_MAX_KV_HEADS) return EA_ERR_UNSUPPORTED;
  if (d != 64 && d != 128) return EA_ERR_UNSUPPORTED;
  if (dtype != EA_DT_BF16 && dtype != EA_DT_F32) return EA_ERR_INVALID_ARG;
  if (D % (dtype == EA_DT_BF16 ? 8 : 4) != 0 || (reinterpret_cast<uintptr_t>(hidden) & 15u) != 0)
    return EA_ERR_INVALID_ARG;
  if ((size_t)D * sizeof(float) + 12u * d * sizeof(float) > 200u * 1024u) return EA_ERR_UNSUPPORTED;
  if (!aligned16(w->w_k) || !aligned16(w->w_t1) || !aligned16(w->w_t2) || !aligned16(w->w_r1) || !aligned16(w->w_o))
    return EA_ERR_INVALID_ARG;
  // The problem's scratch must fit the fixed array.
  if (ea::router_workspace_bytes(B, S, D, H_kv, d, prm->n_boundary) > kStaticScratchBytes) return EA_ERR_INVALID_ARG;
  void* scratch = nullptr;
  if (ea_status s = scratch_address(&scratch)) return s;
  return ea::launch_router(hidden, dtype, B, S, D, H_kv, d, w, prm, head_mode, logits, scratch,
                           static_cast<cudaStream_t>(stream));
}
