// ea_router.cu — the Attention Router: boundary pooling and the per-head MLP.
//
// "Elastic Attention: Test-time Adaptive Sparsity Ratios for Efficient
// Transformers" (paperlayer.ai summary): section 3 "Attention Router" (pooled key
// states -> task MLP -> router MLP -> head-wise logit, hard decision), appendix
// H.4 "Router Input Length" (first and last 100 tokens), section 5 (x4 width).
//
// Kernels (all fp32 arithmetic, fixed summation orders, so results are reproducible):
//   pool_partial   HBM-bound streaming reduction of the pooled hidden rows: 16-byte
//                  loads, 8 in flight per thread, one partial sum per (split, b, column).
//   project        one CTA per 64 rows of W_k: finishes the pooled mean of its rows,
//                  then the partial key projections of those rows for every column.
//   router_mlp     one CTA per (KV head, sample): sums the projection partials of its
//                  head, task MLP, router MLP on [p; tau], output row, threshold.
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
// split's rows with 8 independent 16-byte loads in flight.
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
    for (; n + 8 <= r1; n += 8) {
      uint4 x[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) x[u] = ld_stream(base + (size_t)pooled_token(n + u, a_len, b_start) * D);
#pragma unroll
      for (int u = 0; u < 8; ++u) add_vec<T>(acc, x[u]);
    }
    for (; n < r1; ++n) add_vec<T>(acc, ld_stream(base + (size_t)pooled_token(n, a_len, b_start) * D));
    float* out = partial + ((size_t)split * gridDim.z + b) * D + col;
#pragma unroll
    for (int e = 0; e < V; e += 4)
      *reinterpret_cast<float4*>(out + e) = make_float4(acc[e], acc[e + 1], acc[e + 2], acc[e + 3]);
  }
}

constexpr int kProjRows = 64;      // rows of W_k per projection CTA
constexpr int kProjThreads = 256;
constexpr int kProjB = 4;          // samples per pass over a W_k chunk

template <typename T>
__device__ __forceinline__ void fma_vec(float* acc, uint4 raw, float x) {
  if constexpr (Vec<T>::N == 4) {
    acc[0] = fmaf(__uint_as_float(raw.x), x, acc[0]); acc[1] = fmaf(__uint_as_float(raw.y), x, acc[1]);
    acc[2] = fmaf(__uint_as_float(raw.z), x, acc[2]); acc[3] = fmaf(__uint_as_float(raw.w), x, acc[3]);
  } else {
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      acc[2 * e] = fmaf(__uint_as_float(w[e] << 16), x, acc[2 * e]);
      acc[2 * e + 1] = fmaf(__uint_as_float(w[e] & 0xffff0000u), x, acc[2 * e + 1]);
    }
  }
}

// grid (ceil(D / kProjRows)).  For rows [r0, r0 + 64) of W_k:
//   hbar[b][r] = (sum over splits of the pooling partial sums) / n_rows      (fixed order)
//   pp[chunk][b][n] = sum_{r in chunk} W_k[r, n] * hbar[b][r]   for every column n < N = H_kv*d
template <typename T>
__global__ void __launch_bounds__(kProjThreads)
project_kernel(const float* __restrict__ partial, int n_splits, int B, int D, float inv_rows,
               const T* __restrict__ w_k, int N, float* __restrict__ pp) {
  constexpr int V = Vec<T>::N;
  __shared__ float hb[kProjB][kProjRows];
  __shared__ float red[kProjThreads / kProjRows][kProjRows];
  __shared__ float accs[kProjThreads * V];
  const int r0 = blockIdx.x * kProjRows, tid = threadIdx.x;
  const int rows = min(kProjRows, D - r0);
  const int col_threads = N / V;                          // N % V == 0 (d in {64, 128})
  for (int b0 = 0; b0 < B; b0 += kProjB) {
    const int nb = min(kProjB, B - b0);
    // Pooled hidden states of this chunk: thread = (row, split lane).
    {
      const int rl = tid % kProjRows, sl = tid / kProjRows, lanes = kProjThreads / kProjRows;
      for (int bb = 0; bb < nb; ++bb) {
        float s0 = 0.f, s1 = 0.f;
        if (rl < rows) {
          const float* src = partial + (size_t)(b0 + bb) * D + r0 + rl;
          int sp = sl;
          for (; sp + lanes < n_splits; sp += 2 * lanes) {
            s0 += src[(size_t)sp * B * D];
            s1 += src[(size_t)(sp + lanes) * B * D];
          }
          if (sp < n_splits) s0 += src[(size_t)sp * B * D];
        }
        red[sl][rl] = s0 + s1;
        __syncthreads();
        if (tid < kProjRows) {
          float t = 0.f;
          for (int l = 0; l < lanes; ++l) t += red[l][tid];
          hb[bb][tid] = t * inv_rows;
        }
        __syncthreads();
      }
    }
    // Partial projections: thread = (column group of V, row lane); columns loop when N/V > threads.
    for (int c0 = 0; c0 < col_threads; c0 += kProjThreads) {
      const int cgroups = min(kProjThreads, col_threads - c0);
      const int lanes = max(1, kProjThreads / cgroups);
      const int cg = tid % cgroups, rl = tid / cgroups;
      float acc[kProjB][V];
#pragma unroll
      for (int bb = 0; bb < kProjB; ++bb)
#pragma unroll
        for (int e = 0; e < V; ++e) acc[bb][e] = 0.f;
      if (rl < lanes) {
        const T* col = w_k + (size_t)r0 * N + (size_t)(c0 + cg) * V;
        int r = rl;
        for (; r + 3 * lanes < rows; r += 4 * lanes) {
          const uint4 x0 = *reinterpret_cast<const uint4*>(col + (size_t)r * N);
          const uint4 x1 = *reinterpret_cast<const uint4*>(col + (size_t)(r + lanes) * N);
          const uint4 x2 = *reinterpret_cast<const uint4*>(col + (size_t)(r + 2 * lanes) * N);
          const uint4 x3 = *reinterpret_cast<const uint4*>(col + (size_t)(r + 3 * lanes) * N);
#pragma unroll
          for (int bb = 0; bb < kProjB; ++bb) {
            if (bb < nb) {
              fma_vec<T>(acc[bb], x0, hb[bb][r]);
              fma_vec<T>(acc[bb], x1, hb[bb][r + lanes]);
              fma_vec<T>(acc[bb], x2, hb[bb][r + 2 * lanes]);
              fma_vec<T>(acc[bb], x3, hb[bb][r + 3 * lanes]);
            }
          }
        }
        for (; r < rows; r += lanes) {
          const uint4 x0 = *reinterpret_cast<const uint4*>(col + (size_t)r * N);
#pragma unroll
          for (int bb = 0; bb < kProjB; ++bb)
            if (bb < nb) fma_vec<T>(acc[bb], x0, hb[bb][r]);
        }
      }
      // Sum the row lanes (fixed order) and write this chunk's partial projections.
      for (int bb = 0; bb < nb; ++bb) {
#pragma unroll
        for (int e = 0; e < V; ++e) accs[tid * V + e] = acc[bb][e];
        __syncthreads();
        if (tid < cgroups) {
          float* out = pp + ((size_t)blockIdx.x * B + b0 + bb) * N + (size_t)(c0 + tid) * V;
#pragma unroll
          for (int e = 0; e < V; ++e) {
            float t = 0.f;
            for (int l = 0; l < lanes; ++l) t += accs[(l * cgroups + tid) * V + e];
            out[e] = t;
          }
        }
        __syncthreads();
      }
    }
  }
}

constexpr int kMlpThreads = 512;
constexpr int kMlpWarps = kMlpThreads / 32;
constexpr int kGemvRows = 8;       // rows per warp per pass: their loads are issued together

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// y[r] = act(W[r, :] . x + bias[r]) for r < rows (W row-major fp32, cols % 4 == 0, x in shared
// memory).  Each warp takes kGemvRows rows per pass; a lane reads float4s at columns
// 4*lane + 128*k, so all loads of a pass are in flight together.
template <bool kRelu>
__device__ void gemv_rows(const float* __restrict__ W, const float* __restrict__ bias, const float* x, int rows,
                          int cols, float* y) {
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  for (int r = kGemvRows * warp; r < rows; r += kGemvRows * kMlpWarps) {
    float s[kGemvRows];
#pragma unroll
    for (int u = 0; u < kGemvRows; ++u) s[u] = 0.f;
    for (int c = 4 * lane; c < cols; c += 128) {
      const float4 xv = *reinterpret_cast<const float4*>(x + c);
      float4 wv[kGemvRows];
#pragma unroll
      for (int u = 0; u < kGemvRows; ++u)
        wv[u] = r + u < rows ? __ldg(reinterpret_cast<const float4*>(W + (size_t)(r + u) * cols + c))
                             : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int u = 0; u < kGemvRows; ++u)
        s[u] += wv[u].x * xv.x + wv[u].y * xv.y + wv[u].z * xv.z + wv[u].w * xv.w;
    }
#pragma unroll
    for (int u = 0; u < kGemvRows; ++u) {
      const float t = warp_sum(s[u]);
      if (lane == 0 && r + u < rows) y[r + u] = kRelu ? fmaxf(t + bias[r + u], 0.f) : t + bias[r + u];
    }
  }
}

// grid (H_kv, B): p = sum of the projection partials of head h, then the task MLP,
// the router MLP on [p; tau], the head's output row and the threshold.
__global__ void __launch_bounds__(kMlpThreads)
router_mlp_kernel(const float* __restrict__ pp, int n_chunks, int B, int H_kv, int d, ea_router_weights w,
                  int32_t* __restrict__ head_mode, float* __restrict__ logits) {
  extern __shared__ __align__(16) float sm[];
  const int h = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
  const int N = H_kv * d;
  float* p = sm;                  // [2d]: p then tau (the router MLP input [p; tau])
  float* tau = p + d;
  float* hid = p + 2 * d;         // [4d]
  float* u = hid + 4 * d;         // [4d]
  float* part = u + 4 * d;        // [kMlpThreads]
  float* red = part + kMlpThreads;  // [kMlpWarps]
  {
    const int lanes = kMlpThreads / d, c = tid % d, cl = tid / d;
    const float* src = pp + (size_t)b * N + (size_t)h * d + c;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    int ch = cl;
    for (; ch + 7 * lanes < n_chunks; ch += 8 * lanes) {
#pragma unroll
      for (int k = 0; k < 8; ++k) acc[k] += src[(size_t)(ch + k * lanes) * B * N];
    }
    for (; ch < n_chunks; ch += lanes) acc[0] += src[(size_t)ch * B * N];
    part[tid] = ((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]));
  }
  __syncthreads();
  if (tid < d) {
    float s = 0.f;
    for (int l = 0; l < kMlpThreads / d; ++l) s += part[l * d + tid];
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

static size_t align256(size_t x) { return (x + 255) / 256 * 256; }

// Workspace: pooling partial sums [n_splits][B][D], then projection partials
// [ceil(D/64)][B][H_kv*d].
static size_t partial_bytes(int B, int S, int D, int n_boundary) {
  PoolPlan pl4 = plan_pool(B, S, D, n_boundary, 4), pl8 = plan_pool(B, S, D, n_boundary, 8);
  return align256((size_t)max(pl4.n_splits, pl8.n_splits) * B * D * sizeof(float));
}
static size_t proj_bytes(int B, int D, int N) { return align256((size_t)cdiv(D, kProjRows) * B * N * sizeof(float)); }

size_t router_workspace_bytes(int B, int S, int D, int H_kv, int d, int n_boundary) {
  return partial_bytes(B, S, D, n_boundary) + proj_bytes(B, D, H_kv * d);
}

ea_status launch_router(const void* hidden, ea_dtype dtype, int B, int S, int D, int H_kv, int d,
                        const ea_router_weights* w, const ea_router_params* prm, int32_t* head_mode,
                        float* logits, void* workspace, cudaStream_t st) {
  const int vec = dtype == EA_DT_BF16 ? 8 : 4;
  PoolPlan pl = plan_pool(B, S, D, prm->n_boundary, vec);
  float* partial = reinterpret_cast<float*>(workspace);
  float* pp = reinterpret_cast<float*>(reinterpret_cast<char*>(workspace) + partial_bytes(B, S, D, prm->n_boundary));
  const int N = H_kv * d, n_chunks = cdiv(D, kProjRows);
  dim3 g1(pl.n_chunks, pl.n_splits, B);
  if (dtype == EA_DT_BF16) {
    pool_partial_kernel<__nv_bfloat16><<<g1, kPoolThreads, 0, st>>>(
        static_cast<const __nv_bfloat16*>(hidden), S, D, pl.n_rows, pl.a_len, pl.b_start, pl.rows_per_split, partial);
    project_kernel<__nv_bfloat16><<<n_chunks, kProjThreads, 0, st>>>(
        partial, pl.n_splits, B, D, 1.0f / (float)pl.n_rows, static_cast<const __nv_bfloat16*>(w->w_k), N, pp);
  } else {
    pool_partial_kernel<float><<<g1, kPoolThreads, 0, st>>>(
        static_cast<const float*>(hidden), S, D, pl.n_rows, pl.a_len, pl.b_start, pl.rows_per_split, partial);
    project_kernel<float><<<n_chunks, kProjThreads, 0, st>>>(
        partial, pl.n_splits, B, D, 1.0f / (float)pl.n_rows, static_cast<const float*>(w->w_k), N, pp);
  }
  const size_t smem = sizeof(float) * ((size_t)10 * d + kMlpThreads + kMlpWarps);
  router_mlp_kernel<<<dim3(H_kv, B), kMlpThreads, smem, st>>>(pp, n_chunks, B, H_kv, d, *w, head_mode, logits);
  return cudaGetLastError() == cudaSuccess ? EA_OK : EA_ERR_CUDA;
}

}  // namespace ea
