// ea_router.cu — the Attention Router: boundary pooling and the per-head MLP.
//
// "Elastic Attention: Test-time Adaptive Sparsity Ratios for Efficient
// Transformers" (paperlayer.ai summary): section 3 "Attention Router" (pooled key
// states -> task MLP -> router MLP -> head-wise logit, hard decision), appendix
// H.4 "Router Input Length" (first and last 100 tokens), section 5 (x4 width).
//
// Kernels:
//   pool_partial   HBM-bound streaming reduction of hidden rows: 16-byte vector
//                  loads, fp32 accumulation, one partial sum per (split, b, column).
//   pool_finish    sums the partials in a fixed order and divides by |pooled rows|.
//   router_mlp     one CTA per (KV head, sample): key projection GEMV over D, task
//                  MLP, router MLP, output row, threshold.  Warp-per-row dot products.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>
#include "ea_common.cuh"
#include "ea_internal.h"

namespace ea {
namespace {

constexpr int kPoolThreads = 256;

template <typename T> struct Vec;
template <> struct Vec<float> { static constexpr int N = 4; };
template <> struct Vec<__nv_bfloat16> { static constexpr int N = 8; };

__device__ __forceinline__ uint4 ld_stream(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}

template <typename T>
__device__ __forceinline__ void add_vec(float* acc, uint4 raw) {
  if constexpr (Vec<T>::N == 4) {
    acc[0] += __uint_as_float(raw.x); acc[1] += __uint_as_float(raw.y);
    acc[2] += __uint_as_float(raw.z); acc[3] += __uint_as_float(raw.w);
  } else {
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      acc[2 * e] += __uint_as_float(w[e] << 16);
      acc[2 * e + 1] += __uint_as_float(w[e] & 0xffff0000u);
    }
  }
}

// Pooled row n (0 <= n < n_rows) -> token index: [0, a_len) then [b_start, b_start + ...).
__device__ __forceinline__ int pooled_token(int n, int a_len, int b_start) {
  return n < a_len ? n : b_start + (n - a_len);
}

// grid (column chunks, splits, B); each thread sums VEC consecutive columns over the
// split's rows with 4 independent 16-byte loads in flight.
template <typename T>
__global__ void __launch_bounds__(kPoolThreads)
pool_partial_kernel(const T* __restrict__ hidden, int S, int D, int n_rows, int a_len, int b_start,
                    int rows_per_split, float* __restrict__ partial) {
  constexpr int V = Vec<T>::N;
  const int b = blockIdx.z, split = blockIdx.y;
  const int col = (blockIdx.x * kPoolThreads + threadIdx.x) * V;
  const int r0 = split * rows_per_split;
  const int r1 = min(n_rows, r0 + rows_per_split);
  float acc[V];
#pragma unroll
  for (int e = 0; e < V; ++e) acc[e] = 0.f;
  if (col < D) {
    const T* base = hidden + (size_t)b * S * D + col;
    int n = r0;
    for (; n + 4 <= r1; n += 4) {
      uint4 x0 = ld_stream(base + (size_t)pooled_token(n, a_len, b_start) * D);
      uint4 x1 = ld_stream(base + (size_t)pooled_token(n + 1, a_len, b_start) * D);
      uint4 x2 = ld_stream(base + (size_t)pooled_token(n + 2, a_len, b_start) * D);
      uint4 x3 = ld_stream(base + (size_t)pooled_token(n + 3, a_len, b_start) * D);
      add_vec<T>(acc, x0); add_vec<T>(acc, x1); add_vec<T>(acc, x2); add_vec<T>(acc, x3);
    }
    for (; n < r1; ++n) add_vec<T>(acc, ld_stream(base + (size_t)pooled_token(n, a_len, b_start) * D));
    float* out = partial + ((size_t)split * gridDim.z + b) * D + col;
#pragma unroll
    for (int e = 0; e < V; e += 4)
      *reinterpret_cast<float4*>(out + e) = make_float4(acc[e], acc[e + 1], acc[e + 2], acc[e + 3]);
  }
}

__global__ void pool_finish_kernel(const float* __restrict__ partial, int n_splits, int B, int D,
                                   float inv_rows, float* __restrict__ hbar) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= B * D) return;
  float s = 0.f;
  for (int sp = 0; sp < n_splits; ++sp) s += partial[(size_t)sp * B * D + idx];
  hbar[idx] = s * inv_rows;
}

constexpr int kMlpThreads = 256;
constexpr int kMlpWarps = kMlpThreads / 32;

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// y[r] = act(W[r, :] . x + bias[r]) for r in [0, rows): one warp per row.
template <bool kRelu>
__device__ void gemv_rows(const float* __restrict__ W, const float* __restrict__ bias,
                          const float* x, int rows, int cols, float* y) {
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  for (int r = warp; r < rows; r += kMlpWarps) {
    const float* w = W + (size_t)r * cols;
    float s = 0.f;
    for (int c = lane; c < cols; c += 32) s += w[c] * x[c];
    s = warp_sum(s) + bias[r];
    if (lane == 0) y[r] = kRelu ? fmaxf(s, 0.f) : s;
  }
}

template <typename T>
__device__ __forceinline__ float to_f(T x);
template <> __device__ __forceinline__ float to_f<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

// grid (H_kv, B).  Dynamic shared memory: hbar [D] + projection partials [kMlpThreads]
// + p [d] + tau [d] + hidden [4d] + u [4d] + reduction [kMlpWarps].
template <typename T>
__global__ void __launch_bounds__(kMlpThreads)
router_mlp_kernel(const float* __restrict__ hbar, const T* __restrict__ w_k, ea_router_weights w,
                  int D, int H_kv, int d, int32_t* __restrict__ head_mode, float* __restrict__ logits) {
  extern __shared__ float sm[];
  const int h = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
  float* hb = sm;                 // [D]
  float* part = hb + D;           // [kMlpThreads]
  float* p = part + kMlpThreads;  // [2d]: p then tau (the router MLP input [p; tau])
  float* tau = p + d;
  float* hid = p + 2 * d;         // [4d]
  float* u = hid + 4 * d;         // [4d]
  float* red = u + 4 * d;         // [kMlpWarps]
  for (int i = tid; i < D; i += kMlpThreads) hb[i] = hbar[(size_t)b * D + i];
  __syncthreads();
  // Key projection p[c] = sum_i W_k[i, h*d + c] * hbar[i]: column c = tid % d, row lane
  // tid / d strides over D; consecutive threads read consecutive columns of a row.
  const int lanes = kMlpThreads / d;
  {
    const int c = tid % d, rl = tid / d;
    const T* col = w_k + (size_t)h * d + c;
    const size_t ld = (size_t)H_kv * d;
    float s0 = 0.f, s1 = 0.f;
    int i = rl;
    for (; i + lanes < D; i += 2 * lanes) {
      s0 += to_f(col[(size_t)i * ld]) * hb[i];
      s1 += to_f(col[(size_t)(i + lanes) * ld]) * hb[i + lanes];
    }
    if (i < D) s0 += to_f(col[(size_t)i * ld]) * hb[i];
    part[tid] = s0 + s1;
  }
  __syncthreads();
  if (tid < d) {
    float s = 0.f;
    for (int rl = 0; rl < lanes; ++rl) s += part[rl * d + tid];
    p[tid] = s;
  }
  __syncthreads();
  gemv_rows<true>(w.w_t1, w.b_t1, p, 4 * d, d, hid);       // task MLP, hidden layer
  __syncthreads();
  gemv_rows<false>(w.w_t2, w.b_t2, hid, d, 4 * d, tau);    // task representation tau
  __syncthreads();
  gemv_rows<true>(w.w_r1, w.b_r1, p, 4 * d, 2 * d, u);     // router MLP on [p; tau]
  __syncthreads();
  float s = 0.f;
  for (int j = tid; j < 4 * d; j += kMlpThreads) s += w.w_o[(size_t)h * 4 * d + j] * u[j];
  s = warp_sum(s);
  if (tid % 32 == 0) red[tid / 32] = s;
  __syncthreads();
  if (tid == 0) {
    float z = w.b_o[h];
    for (int i = 0; i < kMlpWarps; ++i) z += red[i];
    head_mode[b * H_kv + h] = z > 0.f ? 1 : 0;
    if (logits) logits[b * H_kv + h] = z;
  }
}

struct PoolPlan {
  int n_rows, a_len, b_start, n_splits, rows_per_split, n_chunks;
};

PoolPlan plan_pool(int B, int S, int D, int n_boundary, int vec) {
  PoolPlan pl;
  if (n_boundary <= 0 || S <= 2 * n_boundary) {
    pl.n_rows = S; pl.a_len = S; pl.b_start = 0;
  } else {
    pl.n_rows = 2 * n_boundary; pl.a_len = n_boundary; pl.b_start = S - n_boundary;
  }
  pl.n_chunks = cdiv(D, kPoolThreads * vec);
  // About four CTAs per SM in total, at least 8 rows per split.
  const int target = 148 * 4;
  int splits = cdiv(target, pl.n_chunks * B);
  splits = max(1, min(splits, cdiv(pl.n_rows, 8)));
  pl.rows_per_split = cdiv(pl.n_rows, splits);
  pl.n_splits = cdiv(pl.n_rows, pl.rows_per_split);
  return pl;
}

}  // namespace

size_t router_workspace_bytes(int B, int S, int D, int n_boundary) {
  PoolPlan pl = plan_pool(B, S, D, n_boundary, 4);  // f32 plan has the most chunks; splits match
  PoolPlan pl8 = plan_pool(B, S, D, n_boundary, 8);
  const int splits = max(pl.n_splits, pl8.n_splits);
  size_t partial = (size_t)splits * B * D * sizeof(float);
  size_t hb = (size_t)B * D * sizeof(float);
  return ((partial + 255) / 256) * 256 + ((hb + 255) / 256) * 256;
}

ea_status launch_router(const void* hidden, ea_dtype dtype, int B, int S, int D, int H_kv, int d,
                        const ea_router_weights* w, const ea_router_params* prm, int32_t* head_mode,
                        float* logits, void* workspace, cudaStream_t st) {
  const int vec = dtype == EA_DT_BF16 ? 8 : 4;
  PoolPlan pl = plan_pool(B, S, D, prm->n_boundary, vec);
  float* partial = reinterpret_cast<float*>(workspace);
  size_t partial_bytes = (size_t)pl.n_splits * B * D * sizeof(float);
  float* hbar = reinterpret_cast<float*>(reinterpret_cast<char*>(workspace) + ((partial_bytes + 255) / 256) * 256);
  dim3 g1(pl.n_chunks, pl.n_splits, B);
  if (dtype == EA_DT_BF16)
    pool_partial_kernel<__nv_bfloat16><<<g1, kPoolThreads, 0, st>>>(
        static_cast<const __nv_bfloat16*>(hidden), S, D, pl.n_rows, pl.a_len, pl.b_start, pl.rows_per_split, partial);
  else
    pool_partial_kernel<float><<<g1, kPoolThreads, 0, st>>>(
        static_cast<const float*>(hidden), S, D, pl.n_rows, pl.a_len, pl.b_start, pl.rows_per_split, partial);
  pool_finish_kernel<<<cdiv(B * D, 256), 256, 0, st>>>(partial, pl.n_splits, B, D, 1.0f / (float)pl.n_rows, hbar);
  const size_t smem = sizeof(float) * ((size_t)D + kMlpThreads + 2 * d + 8 * d + kMlpWarps);
  dim3 g2(H_kv, B);
  if (dtype == EA_DT_BF16) {
    auto k = router_mlp_kernel<__nv_bfloat16>;
    if (smem > 48 * 1024 && cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
      return EA_ERR_CUDA;
    k<<<g2, kMlpThreads, smem, st>>>(hbar, static_cast<const __nv_bfloat16*>(w->w_k), *w, D, H_kv, d, head_mode, logits);
  } else {
    auto k = router_mlp_kernel<float>;
    if (smem > 48 * 1024 && cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
      return EA_ERR_CUDA;
    k<<<g2, kMlpThreads, smem, st>>>(hbar, static_cast<const float*>(w->w_k), *w, D, H_kv, d, head_mode, logits);
  }
  return cudaGetLastError() == cudaSuccess ? EA_OK : EA_ERR_CUDA;
}

}  // namespace ea
