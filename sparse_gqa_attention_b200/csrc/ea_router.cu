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
//   project        one CTA per 32 rows of W_k: finishes the pooled mean of its rows,
//                  then the partial key projections of those rows for every column.
//   proj_reduce    p[b][h*d + c] = sum over the row chunks of the partial projections.
//   mlp_layer x3   the task MLP's two layers and the router MLP, each a batched GEMV over
//                  all (sample, KV head) vectors (the MLP weights are shared by the heads):
//                  one warp per output row, the row held in registers, every vector of
//                  the batch streamed past it.
//   router_out     the head's output row, bias and threshold (one warp per (b, h)).
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

constexpr int kProjRows = 32;      // rows of W_k per projection CTA
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

// grid (ceil(D / kProjRows)).  For rows [r0, r0 + kProjRows) of W_k:
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

constexpr int kMlpThreads = 256;   // 8 warps, one output row each
constexpr int kMlpWarps = kMlpThreads / 32;

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// p[i] = sum over the row chunks of pp[chunk][i] (fixed order), i < B * H_kv * d.
__global__ void __launch_bounds__(256)
proj_reduce_kernel(const float* __restrict__ pp, int n_chunks, int total, float* __restrict__ p) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= total) return;
  float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
  int ch = 0;
  for (; ch + 4 <= n_chunks; ch += 4) {
    a0 += pp[(size_t)ch * total + i];
    a1 += pp[(size_t)(ch + 1) * total + i];
    a2 += pp[(size_t)(ch + 2) * total + i];
    a3 += pp[(size_t)(ch + 3) * total + i];
  }
  for (; ch < n_chunks; ++ch) a0 += pp[(size_t)ch * total + i];
  p[i] = (a0 + a1) + (a2 + a3);
}

// Y[v][r] = act(W[r, :] . [Xa[v]; Xb[v]] + bias[r]) for every vector v < nv and output row
// r < rows; the input of vector v is Xa[v] (na values) followed by Xb[v] (nb values, may be
// 0).  W is row-major fp32 with na + nb <= 512 columns, na and nb multiples of 4.  Warp w of
// CTA c takes row r = 8c + w: its W row stays in registers (lane: columns 4*lane + 128*k).
template <bool kRelu>
__global__ void __launch_bounds__(kMlpThreads)
mlp_layer_kernel(const float* __restrict__ Xa, int na, const float* __restrict__ Xb, int nb,
                 const float* __restrict__ W, const float* __restrict__ bias, int rows, int nv,
                 float* __restrict__ Y) {
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int r = blockIdx.x * kMlpWarps + warp;
  if (r >= rows) return;
  const int in = na + nb;
  float4 w[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int c = 4 * lane + 128 * k;
    w[k] = c < in ? __ldg(reinterpret_cast<const float4*>(W + (size_t)r * in + c)) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  const float br = bias[r];
  for (int v = 0; v < nv; ++v) {
    float s = 0.f;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int c = 4 * lane + 128 * k;
      if (c < in) {
        const float4 x = c < na ? *reinterpret_cast<const float4*>(Xa + (size_t)v * na + c)
                                : *reinterpret_cast<const float4*>(Xb + (size_t)v * nb + (c - na));
        s += w[k].x * x.x + w[k].y * x.y + w[k].z * x.z + w[k].w * x.w;
      }
    }
    s = warp_sum(s);
    if (lane == 0) Y[(size_t)v * rows + r] = kRelu ? fmaxf(s + br, 0.f) : s + br;
  }
}

// z[b][h] = w_o[h] . u[b*H_kv + h] + b_o[h]; head_mode = (z > 0).  One warp per (b, h).
__global__ void __launch_bounds__(kMlpThreads)
router_out_kernel(const float* __restrict__ u, int n4, int BH, int H_kv, const float* __restrict__ w_o,
                  const float* __restrict__ b_o, int32_t* __restrict__ head_mode, float* __restrict__ logits) {
  const int v = blockIdx.x * kMlpWarps + threadIdx.x / 32, lane = threadIdx.x % 32;
  if (v >= BH) return;
  const int h = v % H_kv;
  float s = 0.f;
  for (int j = lane; j < n4; j += 32) s += w_o[(size_t)h * n4 + j] * u[(size_t)v * n4 + j];
  s = warp_sum(s);
  if (lane == 0) {
    const float z = s + b_o[h];
    head_mode[v] = z > 0.f ? 1 : 0;
    if (logits) logits[v] = z;
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

// Workspace: pooling partial sums [n_splits][B][D], projection partials
// [ceil(D/32)][B][H_kv*d], then the MLP vectors p [B*H_kv][d], hid [.][4d], tau [.][d],
// u [.][4d].
static size_t partial_bytes(int B, int S, int D, int n_boundary) {
  PoolPlan pl4 = plan_pool(B, S, D, n_boundary, 4), pl8 = plan_pool(B, S, D, n_boundary, 8);
  return align256((size_t)max(pl4.n_splits, pl8.n_splits) * B * D * sizeof(float));
}
static size_t proj_bytes(int B, int D, int N) { return align256((size_t)cdiv(D, kProjRows) * B * N * sizeof(float)); }
static size_t mlp_bytes(int B, int N) { return align256((size_t)B * N * 10 * sizeof(float)); }

size_t router_workspace_bytes(int B, int S, int D, int H_kv, int d, int n_boundary) {
  return partial_bytes(B, S, D, n_boundary) + proj_bytes(B, D, H_kv * d) + mlp_bytes(B, H_kv * d);
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
  if (cudaGetLastError() != cudaSuccess) return EA_ERR_CUDA;
  float* p = reinterpret_cast<float*>(reinterpret_cast<char*>(pp) + proj_bytes(B, D, N));
  const int BH = B * H_kv;
  float* hid = p + (size_t)BH * d;
  float* tau = hid + (size_t)BH * 4 * d;
  float* u = tau + (size_t)BH * d;
  proj_reduce_kernel<<<cdiv(B * N, 256), 256, 0, st>>>(pp, n_chunks, B * N, p);
  mlp_layer_kernel<true><<<cdiv(4 * d, kMlpWarps), kMlpThreads, 0, st>>>(p, d, nullptr, 0, w->w_t1, w->b_t1, 4 * d,
                                                                        BH, hid);      // task MLP, hidden layer
  mlp_layer_kernel<false><<<cdiv(d, kMlpWarps), kMlpThreads, 0, st>>>(hid, 4 * d, nullptr, 0, w->w_t2, w->b_t2, d,
                                                                      BH, tau);        // task representation
  mlp_layer_kernel<true><<<cdiv(4 * d, kMlpWarps), kMlpThreads, 0, st>>>(p, d, tau, d, w->w_r1, w->b_r1, 4 * d,
                                                                        BH, u);        // router MLP on [p; tau]
  router_out_kernel<<<cdiv(BH, kMlpWarps), kMlpThreads, 0, st>>>(u, 4 * d, BH, H_kv, w->w_o, w->b_o, head_mode,
                                                                 logits);
  return cudaGetLastError() == cudaSuccess ? EA_OK : EA_ERR_CUDA;
}

}  // namespace ea
