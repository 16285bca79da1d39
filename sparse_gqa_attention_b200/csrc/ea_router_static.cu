// ea_router_static.cu — ea_router_static_scratch: the router with scratch memory that
// the library owns, for callers that cannot allocate device memory.
//
// Some callers of this router cannot call cudaMalloc: an inference runtime or plugin
// host that hands out all device memory through its own allocator, or code that runs
// while a stream is being captured (a global-mode capture rejects cudaMalloc, and
// cudaMalloc/cudaFree can synchronise the device).  This entry point takes the same
// inputs and outputs as ea_router but keeps its pooling partial sums and pooled
// hidden states in a fixed array compiled into the library, so it allocates nothing.
//
// The array is a file-scope __device__ variable: every GPU that loads the library holds
// kStaticScratchBytes of it until the process exits.  Host code cannot use the array's
// name as a device address, so the first call on each device looks the address up with
// cudaGetSymbolAddress (that device current) and caches it; that first call should come
// before any stream capture.  All calls share the one array, so calls whose kernels
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
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_router_scratch on the current device (looked up once per device).
ea_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return EA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return EA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_router_scratch) != cudaSuccess || p == nullptr) return EA_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return EA_OK;
}

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
  // The problem's scratch must fit the fixed array.
  if (ea::router_workspace_bytes(B, S, D, H_kv, d, prm->n_boundary) > kStaticScratchBytes) return EA_ERR_INVALID_ARG;
  void* scratch = nullptr;
  if (ea_status s = scratch_address(&scratch)) return s;
  return ea::launch_router(hidden, dtype, B, S, D, H_kv, d, w, prm, head_mode, logits, scratch,
                           static_cast<cudaStream_t>(stream));
}
