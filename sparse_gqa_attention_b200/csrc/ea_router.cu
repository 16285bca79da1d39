// ea_router.cu — the Attention Router: boundary pooling, key projection and the
// per-head MLP with its hard threshold.
//
// "Elastic Attention: Test-time Adaptive Sparsity Ratios for Efficient
// Transformers" (paperlayer.ai summary): section 3 "Attention Router" (pooled key
// states -> task MLP -> router MLP -> head-wise logit, hard decision), appendix
// H.4 "Router Input Length" (first and last 100 tokens), section 5 (x4 width).
//
// Kernels (all fp32 arithmetic in fixed summation orders, so results are reproducible):
//   pool_partial   (whole-sequence pooling only) HBM-bound streaming reduction of the
//                  pooled rows: 16-byte loads, 8 in flight per thread, one partial sum
//                  per (split, b, column).
//   project        one CTA per 32 rows of W_k, clusters of 8 CTAs: the pooled mean of its
//                  rows (straight from the hidden states for boundary pooling, or from the
//                  partial sums), the partial key projections of those rows for every
//                  column, summed over the cluster through distributed shared memory.
//   router_head    one cluster of 8 CTAs for every (sample, KV head) vector: the key
//                  projection (sum of the clusters' partials), task MLP (two layers),
//                  router MLP, per-head output row and threshold.  Each CTA keeps its
//                  slice of the MLP rows in shared memory (loaded while the projection
//                  still runs) and sends the layer outputs to every CTA of the cluster.
// Launches after the first use programmatic dependent launch, so each kernel's launch
// and prologue overlap the previous kernel.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <atomic>
#include <cstdint>
#include "ea_common.cuh"
#include "ea_internal.h"
#include "ea_sm100.cuh"

namespace ea {
namespace {

using namespace sm100;

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
  launch_dependents();
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

// Sum of the splits sp = first, first + step, ... < n of partial[sp * stride + i], in that
// order, 8 loads in flight.
__device__ __forceinline__ float sum_splits(const float* __restrict__ partial, size_t stride, int first, int step,
                                            int n, size_t i) {
  float t = 0.f;
  int sp = first;
  for (; sp + 7 * step < n; sp += 8 * step) {
    float y[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) y[u] = partial[(size_t)(sp + u * step) * stride + i];
#pragma unroll
    for (int u = 0; u < 8; ++u) t += y[u];
  }
  for (; sp < n; sp += step) t += partial[(size_t)sp * stride + i];
  return t;
}

// hbar[b][c] = (sum over splits of the partial sums) / n_rows (ea_router_pool).  A CTA takes 32
// consecutive entries of [B, D]; warp w sums splits w, w+8, ...; the 8 warp sums are added in
// warp order.
__global__ void __launch_bounds__(256)
pool_finish_kernel(const float* __restrict__ partial, int n_splits, int B, int D, float inv_rows,
                   float* __restrict__ hbar) {
  __shared__ float red[8][32];
  grid_dependency_wait();
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const size_t i = (size_t)blockIdx.x * 32 + lane;
  const bool in = i < (size_t)B * D;
  red[warp][lane] = in ? sum_splits(partial, (size_t)B * D, warp, 8, n_splits, i) : 0.f;
  __syncthreads();
  if (warp == 0 && in) {
    float t = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) t += red[w][lane];
    hbar[i] = t * inv_rows;
  }
}

constexpr int kProjRows = 32;      // rows of W_k per projection CTA
constexpr int kProjThreads = 256;
constexpr int kProjB = 4;          // samples per pass over a W_k chunk (at most)
constexpr int kCluster = 8;        // CTAs per cluster (projection and router head)
constexpr int kStageFloats = 8192; // projection partials staged per CTA for the cluster sum

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

// grid (clusters of 8 CTAs along x, one CTA per 32 rows of W_k, padded to a multiple of 8).
// For rows [r0, r0 + 32) of W_k and each sample b:
//   hbar[b][r] = mean over the pooled tokens of hidden[b][t][r]: straight from hidden when
//                `partial` is null (boundary pooling), else (sum of the splits' partials) / n_rows
//   part[n]    = sum_{r in chunk} W_k[r, n] * hbar[b][r]              for every column n < N
//   pp[cluster][b][n] = sum over the cluster's 8 CTAs of part[n]      (fixed rank order)
// When its 32 rows of W_k fit (wk_smem), the CTA first copies them into shared memory
// with asynchronous 16-byte copies, so that the W_k stream overlaps the pooling.
template <typename T>
__global__ void __cluster_dims__(kCluster, 1, 1) __launch_bounds__(kProjThreads)
project_kernel(const T* __restrict__ hidden, int S, int n_rows, int a_len, int b_start,
               const float* __restrict__ partial, int n_splits, int B, int D, float inv_rows,
               const T* __restrict__ w_k, int N, int batch, float* __restrict__ pp, int wk_smem) {
  constexpr int V = Vec<T>::N;
  extern __shared__ __align__(16) uint8_t wk_s[];
  constexpr int kColVecs = kProjRows / V;              // 16-byte vectors per pooled row chunk
  constexpr int kTokLanes = kProjThreads / kColVecs;   // token lanes of the fused pooling
  constexpr int kRedRows = kTokLanes > kProjThreads / kProjRows ? kTokLanes : kProjThreads / kProjRows;
  constexpr int kScratch = kRedRows * kProjRows > kProjThreads * V ? kRedRows * kProjRows : kProjThreads * V;
  __shared__ float hb[kProjB][kProjRows];
  __shared__ float scratch[kScratch];   // pooling lane sums, then projection row-lane sums
  __shared__ __align__(16) float stage[kStageFloats];
  float (*red)[kProjRows] = reinterpret_cast<float (*)[kProjRows]>(scratch);
  float* accs = scratch;
  launch_dependents();
  const int r0 = blockIdx.x * kProjRows, tid = threadIdx.x;
  const int rows = max(0, min(kProjRows, D - r0));
  const uint32_t rank = cluster_rank();
  if (wk_smem) {   // W_k is an input, not the previous kernel's output: copy before waiting
    const int n16 = rows * N * (int)sizeof(T) / 16;
    const char* src = reinterpret_cast<const char*>(w_k + (size_t)r0 * N);
    for (int i = tid; i < n16; i += kProjThreads)
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(wk_s + 16 * i)), "l"(src + 16 * i)
                   : "memory");
    asm volatile("cp.async.commit_group;" ::: "memory");
  }
  grid_dependency_wait();   // the pooling partial sums (whole-sequence pooling)
  const int col_threads = N / V;                          // N % V == 0 (d in {64, 128})
  for (int b0 = 0; b0 < B; b0 += batch) {
    const int nb = min(batch, B - b0);
    for (int bb = 0; bb < nb; ++bb) {
      if (partial == nullptr) {
        // Pooled mean straight from hidden: thread = (token lane, 16-byte column vector).
        const int vl = tid % kColVecs, tl = tid / kColVecs;
        float acc[V];
#pragma unroll
        for (int e = 0; e < V; ++e) acc[e] = 0.f;
        if (vl * V < rows) {
          const T* base = hidden + (size_t)(b0 + bb) * S * D + r0 + vl * V;
          int n = tl;
          for (; n + 3 * kTokLanes < n_rows; n += 4 * kTokLanes) {
            uint4 x[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) x[u] = ld_stream(base + (size_t)pooled_token(n + u * kTokLanes, a_len, b_start) * D);
#pragma unroll
            for (int u = 0; u < 4; ++u) add_vec<T>(acc, x[u]);
          }
          for (; n < n_rows; n += kTokLanes) add_vec<T>(acc, ld_stream(base + (size_t)pooled_token(n, a_len, b_start) * D));
        }
#pragma unroll
        for (int e = 0; e < V; ++e) red[tl][vl * V + e] = acc[e];
        __syncthreads();
        if (tid < kProjRows) {
          float t = 0.f;
          for (int l = 0; l < kTokLanes; ++l) t += red[l][tid];
          hb[bb][tid] = t * inv_rows;
        }
        __syncthreads();
      } else {
        // From the splits' partial sums: thread = (row, split lane).
        const int rl = tid % kProjRows, sl = tid / kProjRows, lanes = kProjThreads / kProjRows;
        red[sl][rl] = rl < rows ? sum_splits(partial, (size_t)B * D, sl, lanes, n_splits,
                                             (size_t)(b0 + bb) * D + r0 + rl)
                                : 0.f;
        __syncthreads();
        if (tid < kProjRows) {
          float t = 0.f;
          for (int l = 0; l < lanes; ++l) t += red[l][tid];
          hb[bb][tid] = t * inv_rows;
        }
        __syncthreads();
      }
    }
    if (wk_smem && b0 == 0) {
      asm volatile("cp.async.wait_all;" ::: "memory");
      __syncthreads();
    }
    // Partial projections: thread = (column group of V, row lane); columns loop when N/V > threads.
    const T* wk_base = wk_smem ? reinterpret_cast<const T*>(wk_s) : w_k + (size_t)r0 * N;
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
        const T* col = wk_base + (size_t)(c0 + cg) * V;
        int r = rl;
        for (; r + 7 * lanes < rows; r += 8 * lanes) {   // 8 loads in flight
          uint4 x[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) x[u] = *reinterpret_cast<const uint4*>(col + (size_t)(r + u * lanes) * N);
#pragma unroll
          for (int bb = 0; bb < kProjB; ++bb) {
            if (bb < nb) {
#pragma unroll
              for (int u = 0; u < 8; ++u) fma_vec<T>(acc[bb], x[u], hb[bb][r + u * lanes]);
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
      // Sum the row lanes (fixed order) into this CTA's staged partials.
#pragma unroll
      for (int bb = 0; bb < kProjB; ++bb) {
        if (bb >= nb) break;
#pragma unroll
        for (int e = 0; e < V; ++e) accs[tid * V + e] = acc[bb][e];
        __syncthreads();
        if (tid < cgroups) {
#pragma unroll
          for (int e = 0; e < V; ++e) {
            float t = 0.f;
            for (int l = 0; l < lanes; ++l) t += accs[(l * cgroups + tid) * V + e];
            stage[bb * N + (c0 + tid) * V + e] = t;
          }
        }
        __syncthreads();
      }
    }
    // Sum over the cluster's CTAs: rank r owns columns [r*N/8, (r+1)*N/8) of every sample.
    cluster_sync();
    {
      const int per = N / kCluster;
      const uint32_t st0 = smem_u32(stage);
      for (int x = tid; x < nb * per; x += kProjThreads) {
        const int bb = x / per, n = (int)rank * per + x % per;
        float t = 0.f;
#pragma unroll
        for (int q = 0; q < kCluster; ++q) t += ld_cluster(map_rank(st0 + 4u * (uint32_t)(bb * N + n), (uint32_t)q));
        pp[((size_t)(blockIdx.x / kCluster) * B + b0 + bb) * N + n] = t;
      }
    }
    cluster_sync();   // the stage may be rewritten by the next batch
  }
}

constexpr int kVC = 16;            // (sample, KV head) vectors per pass through the MLP
constexpr int kSub = 8;            // vectors per register pass of a warp

// Sum of each of the warp's N per-lane values over the 32 lanes.  Each step halves the
// values a lane keeps while there is more than one (lanes with the step's bit set keep
// the upper half), then adds plainly; rs_index gives the original index of a kept value.
template <int N>
__device__ __forceinline__ void warp_reduce_scatter(float (&v)[N], int lane) {
  int n = N;
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    if (n > 1) {
      const bool up = (lane & o) != 0;
#pragma unroll
      for (int i = 0; i < N / 2; ++i) {
        if (i < n / 2) {
          const float send = up ? v[i] : v[i + n / 2];
          const float keep = up ? v[i + n / 2] : v[i];
          v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
      }
      n /= 2;
    } else {
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], o);
    }
  }
}
template <int N>
__device__ __forceinline__ int rs_index(int lane, int i) {
  int idx = i, n = N;
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1)
    if (n > 1) {
      if (lane & o) idx += n / 2;
      n /= 2;
    }
  return idx;
}
template <int N>
__device__ __forceinline__ bool rs_owner(int lane) {   // one lane per replicated result
  int n = N;
  bool own = true;
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    if (n > 1) n /= 2;
    else if (lane & o) own = false;
  }
  return own;
}

// Threads of the router head: 16 warps at head dim 128 (each layer's rows split 4 / 1 / 4 per
// warp), 8 at head dim 64.
template <int HD> struct HeadThreads { static constexpr int N = HD == 128 ? 512 : 256; };

// Rows [r0, r0 + RW) of a layer for kSub vectors: acc[r * kSub + v] = W[r] . x_v over K
// inputs, where x_v = X1[v] (K1 values) followed by X2[v] (K - K1 values).  W: shared
// memory, rows of K floats; X1 / X2: shared memory, vector strides K1 / K - K1.
template <int RW, int K, int K1>
__device__ __forceinline__ void warp_rows(const float* W, int r0, const float* X1, const float* X2, int nsub,
                                          int lane, float (&acc)[RW * kSub]) {
#pragma unroll
  for (int i = 0; i < RW * kSub; ++i) acc[i] = 0.f;
#pragma unroll
  for (int j = 0; j < K / 32; ++j) {
    const int k = lane + 32 * j;
    float w[RW];
#pragma unroll
    for (int r = 0; r < RW; ++r) w[r] = W[(r0 + r) * K + k];
#pragma unroll
    for (int v = 0; v < kSub; ++v) {
      if (v < nsub) {
        const float x = k < K1 ? X1[v * K1 + k] : X2[v * (K - K1) + (k - K1)];
#pragma unroll
        for (int r = 0; r < RW; ++r) acc[r * kSub + v] = fmaf(w[r], x, acc[r * kSub + v]);
      }
    }
  }
}

// Shared-memory layout of router_head_kernel for head dim HD (floats).
template <int HD>
struct HeadSmem {
  static constexpr int R1 = 4 * HD / kCluster;   // task-MLP hidden rows per CTA
  static constexpr int R2 = HD / kCluster;       // task-representation rows per CTA
  static constexpr int R3 = 4 * HD / kCluster;   // router-MLP rows per CTA
  static constexpr int W1 = 0;                   // [R1][HD]
  static constexpr int W2 = W1 + R1 * HD;        // [R2][4HD]
  static constexpr int W3 = W2 + R2 * 4 * HD;    // [R3][2HD]
  static constexpr int B1 = W3 + R3 * 2 * HD;    // [R1]
  static constexpr int B2 = B1 + R1;             // [R2]
  static constexpr int B3 = B2 + R2;             // [R3]
  static constexpr int WO = B3 + R3;             // [H_kv max][R3]: this CTA's columns of w_o
  static constexpr int P = WO + EA_MAX_KV_HEADS * R3;   // [kVC][HD]
  static constexpr int HID = P + kVC * HD;       // [kVC][4HD]
  static constexpr int TAU = HID + kVC * 4 * HD; // [kVC][HD]
  static constexpr int U = TAU + kVC * HD;       // [kVC][R3] this CTA's rows of u
  static constexpr int Z = U + kVC * R3;         // [kCluster][kVC] partial logits (used in rank 0)
  static constexpr int TOTAL = Z + kCluster * kVC;
  static constexpr size_t BYTES = (size_t)TOTAL * 4;
};

// One cluster of 8 CTAs for all B*H_kv vectors v = b*H_kv + h (kVC per pass):
//   p_v   = sum of the projection clusters' partials               (key projection, d)
//   hid_v = relu(W_t1 p_v + b_t1)                                    (4d; rank r: rows r*4d/8..)
//   tau_v = W_t2 hid_v + b_t2                                        (d)
//   u_v   = relu(W_r1 [p_v; tau_v] + b_r1)                           (4d)
//   z_v   = w_o[h] . u_v + b_o[h];  head_mode = (z_v > 0)
// Layer outputs go to every CTA's shared memory; the final dot product is summed over the
// CTAs' rows of u in rank order.
template <int HD>
__global__ void __cluster_dims__(kCluster, 1, 1) __launch_bounds__(HeadThreads<HD>::N, 1)
router_head_kernel(const float* __restrict__ pp, int n_pp, int BH, int H_kv, const float* __restrict__ w_t1,
                   const float* __restrict__ b_t1, const float* __restrict__ w_t2, const float* __restrict__ b_t2,
                   const float* __restrict__ w_r1, const float* __restrict__ b_r1, const float* __restrict__ w_o,
                   const float* __restrict__ b_o, int32_t* __restrict__ head_mode, float* __restrict__ logits) {
  using L = HeadSmem<HD>;
  constexpr int kHeadThreads = HeadThreads<HD>::N, kHeadWarps = kHeadThreads / 32;
  extern __shared__ __align__(16) float sm[];
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const uint32_t rank = cluster_rank();
  // This CTA's slices of the MLP weights (inputs, not outputs of the previous kernel:
  // loaded before waiting for it).
  {
    // 16-byte asynchronous copies, all in flight at once (completed before the first layer).
    auto copy4 = [&](float* dst, const float* src, int n) {
      for (int i = tid; i < n / 4; i += kHeadThreads)
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst + 4 * i)), "l"(src + 4 * i)
                     : "memory");
    };
    copy4(sm + L::W1, w_t1 + (size_t)rank * L::R1 * HD, L::R1 * HD);
    copy4(sm + L::W2, w_t2 + (size_t)rank * L::R2 * 4 * HD, L::R2 * 4 * HD);
    copy4(sm + L::W3, w_r1 + (size_t)rank * L::R3 * 2 * HD, L::R3 * 2 * HD);
    auto copy1 = [&](float* dst, const float* src) {   // 4-byte asynchronous copy
      asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
    };
    for (int i = tid; i < L::R1; i += kHeadThreads) copy1(sm + L::B1 + i, b_t1 + rank * L::R1 + i);
    for (int i = tid; i < L::R2; i += kHeadThreads) copy1(sm + L::B2 + i, b_t2 + rank * L::R2 + i);
    for (int i = tid; i < L::R3; i += kHeadThreads) copy1(sm + L::B3 + i, b_r1 + rank * L::R3 + i);
    for (int i = tid; i < H_kv * L::R3; i += kHeadThreads)
      copy1(sm + L::WO + i, w_o + (size_t)(i / L::R3) * 4 * HD + rank * L::R3 + i % L::R3);
    asm volatile("cp.async.commit_group;" ::: "memory");
  }
  grid_dependency_wait();   // the projection partials
  const uint32_t sbase = smem_u32(sm);
  auto bcast = [&](int off, float x) {   // the same float into every CTA of the cluster
#pragma unroll
    for (int q = 0; q < kCluster; ++q) st_cluster(map_rank(sbase + 4u * (uint32_t)off, (uint32_t)q), x);
  };
  for (int v0 = 0; v0 < BH; v0 += kVC) {
    const int nv = min(kVC, BH - v0);
    // p: rank r sums elements [r*E/8, (r+1)*E/8) of the pass over the projection clusters.
    {
      const int E = nv * HD, per = (E + kCluster - 1) / kCluster;
      for (int x = (int)rank * per + tid; x < min(E, ((int)rank + 1) * per); x += kHeadThreads) {
        const float* src = pp + (size_t)v0 * HD + x;
        float t = 0.f;
        int c = 0;
        for (; c + 8 <= n_pp; c += 8) {     // 8 loads in flight, summed in order
          float y[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) y[u] = src[(size_t)(c + u) * BH * HD];
#pragma unroll
          for (int u = 0; u < 8; ++u) t += y[u];
        }
        for (; c < n_pp; ++c) t += src[(size_t)c * BH * HD];
        bcast(L::P + x, t);
      }
    }
    if (v0 == 0) asm volatile("cp.async.wait_all;" ::: "memory");   // this thread's weight copies
    __syncthreads();
    cluster_sync();
    // Task MLP hidden layer: this CTA's R1 rows, split over the warps.
    for (int s0 = 0; s0 < nv; s0 += kSub) {
      constexpr int RW = L::R1 / kHeadWarps > 0 ? L::R1 / kHeadWarps : 1;
      if (warp * RW >= L::R1) continue;
      float acc[RW * kSub];
      const int ns = min(kSub, nv - s0);
      warp_rows<RW, HD, HD>(sm + L::W1, warp * RW, sm + L::P + s0 * HD, nullptr, ns, lane, acc);
      warp_reduce_scatter<RW * kSub>(acc, lane);
      if (rs_owner<RW * kSub>(lane)) {
#pragma unroll
        for (int i = 0; i < (RW * kSub >= 32 ? RW * kSub / 32 : 1); ++i) {
          const int idx = rs_index<RW * kSub>(lane, i), r = idx / kSub, v = idx % kSub;
          const int lr = warp * RW + r;
          if (v < ns) bcast(L::HID + (s0 + v) * 4 * HD + (int)rank * L::R1 + lr, fmaxf(acc[i] + sm[L::B1 + lr], 0.f));
        }
      }
    }
    cluster_sync();
    // Task representation: R2 rows.
    for (int s0 = 0; s0 < nv; s0 += kSub) {
      constexpr int RW = L::R2 / kHeadWarps > 0 ? L::R2 / kHeadWarps : 1;
      if (warp * RW >= L::R2) continue;
      float acc[RW * kSub];
      const int ns = min(kSub, nv - s0);
      warp_rows<RW, 4 * HD, 4 * HD>(sm + L::W2, warp * RW, sm + L::HID + s0 * 4 * HD, nullptr, ns, lane, acc);
      warp_reduce_scatter<RW * kSub>(acc, lane);
      if (rs_owner<RW * kSub>(lane)) {
#pragma unroll
        for (int i = 0; i < (RW * kSub >= 32 ? RW * kSub / 32 : 1); ++i) {
          const int idx = rs_index<RW * kSub>(lane, i), r = idx / kSub, v = idx % kSub;
          const int lr = warp * RW + r;
          if (v < ns) bcast(L::TAU + (s0 + v) * HD + (int)rank * L::R2 + lr, acc[i] + sm[L::B2 + lr]);
        }
      }
    }
    cluster_sync();
    // Router MLP hidden layer on [p; tau]: R3 rows, kept in this CTA.
    for (int s0 = 0; s0 < nv; s0 += kSub) {
      constexpr int RW = L::R3 / kHeadWarps > 0 ? L::R3 / kHeadWarps : 1;
      if (warp * RW >= L::R3) continue;
      float acc[RW * kSub];
      const int ns = min(kSub, nv - s0);
      warp_rows<RW, 2 * HD, HD>(sm + L::W3, warp * RW, sm + L::P + s0 * HD, sm + L::TAU + s0 * HD, ns, lane, acc);
      warp_reduce_scatter<RW * kSub>(acc, lane);
      if (rs_owner<RW * kSub>(lane)) {
#pragma unroll
        for (int i = 0; i < (RW * kSub >= 32 ? RW * kSub / 32 : 1); ++i) {
          const int idx = rs_index<RW * kSub>(lane, i), r = idx / kSub, v = idx % kSub;
          const int lr = warp * RW + r;
          if (v < ns) sm[L::U + (s0 + v) * L::R3 + lr] = fmaxf(acc[i] + sm[L::B3 + lr], 0.f);
        }
      }
    }
    __syncthreads();
    // This CTA's share of z_v = w_o[h] . u_v: one warp per vector, lanes over its rows.
    for (int v = warp; v < nv; v += kHeadWarps) {
      const int h = (v0 + v) % H_kv;
      float t = 0.f;
      for (int r = lane; r < L::R3; r += 32) t = fmaf(sm[L::WO + h * L::R3 + r], sm[L::U + v * L::R3 + r], t);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
      if (lane == 0) st_cluster(map_rank(sbase + 4u * (uint32_t)(L::Z + (int)rank * kVC + v), 0u), t);
    }
    cluster_sync();
    if (rank == 0 && tid < nv) {
      const int vg = v0 + tid, h = vg % H_kv;
      float z = 0.f;
#pragma unroll
      for (int q = 0; q < kCluster; ++q) z += sm[L::Z + q * kVC + tid];
      z += b_o[h];
      head_mode[vg] = z > 0.f ? 1 : 0;
      if (logits) logits[vg] = z;
    }
  }
  cluster_sync();   // no CTA leaves while another may still write into its shared memory
}

// Launch with programmatic dependent launch after the previous kernel of this call.
template <typename... KArgs, typename... Args>
cudaError_t launch_after(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, bool pdl,
                         Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
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

// Boundary pooling reads at most this many rows per sample; it is fused into the projection.
bool fused_pooling(const PoolPlan& pl) { return pl.n_rows <= 4096; }
int proj_ctas(int D) { return cdiv(cdiv(D, kProjRows), kCluster) * kCluster; }
int proj_batch(int N) { return max(1, min(kProjB, kStageFloats / N)); }

}  // namespace

static size_t align256(size_t x) { return (x + 255) / 256 * 256; }

// Raise a kernel's dynamic shared-memory limit once per device (host-side cost off the calls).
template <auto kern>
static bool attr_once(int bytes) {
  static std::atomic<uint64_t> done{0};   // bit per device, one set of bits per kernel
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  const uint64_t bit = dev < 64 ? (1ull << dev) : 0ull;
  if (bit && (done.load() & bit)) return true;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess) return false;
  done.fetch_or(bit);
  return true;
}

// Workspace: pooling partial sums [n_splits][B][D] (whole-sequence pooling), then the
// projection clusters' partials [n_clusters][B][H_kv*d].  The MLP vectors stay in the
// router head's shared memory.
static size_t partial_bytes(int B, int S, int D, int n_boundary) {
  PoolPlan pl4 = plan_pool(B, S, D, n_boundary, 4), pl8 = plan_pool(B, S, D, n_boundary, 8);
  return align256((size_t)max(pl4.n_splits, pl8.n_splits) * B * D * sizeof(float));
}
static size_t proj_bytes(int B, int D, int N) {
  return align256((size_t)(proj_ctas(D) / kCluster) * B * N * sizeof(float));
}

size_t router_workspace_bytes(int B, int S, int D, int H_kv, int d, int n_boundary) {
  return partial_bytes(B, S, D, n_boundary) + proj_bytes(B, D, H_kv * d);
}

size_t router_pool_workspace_bytes(int B, int S, int D, int n_boundary) { return partial_bytes(B, S, D, n_boundary); }

template <int HD>
static ea_status launch_head(const float* pp, int n_pp, int BH, int H_kv, const ea_router_weights* w,
                             int32_t* head_mode, float* logits, cudaStream_t st) {
  auto kern = router_head_kernel<HD>;
  constexpr size_t bytes = HeadSmem<HD>::BYTES;
  static_assert(bytes <= 232448, "router head shared memory beyond the 227 KB a CTA may use");
  if (!attr_once<router_head_kernel<HD>>((int)bytes)) return EA_ERR_CUDA;
  return launch_after(kern, dim3(kCluster), dim3(HeadThreads<HD>::N), bytes, st, true, pp, n_pp, BH, H_kv, w->w_t1,
                      w->b_t1, w->w_t2, w->b_t2, w->w_r1, w->b_r1, w->w_o, w->b_o, head_mode, logits) == cudaSuccess
             ? EA_OK
             : EA_ERR_CUDA;
}

template <typename T>
static ea_status launch_pool_project(const T* hidden, int B, int S, int D, int N, const T* w_k, int n_boundary,
                                     void* workspace, float* pp, cudaStream_t st) {
  const PoolPlan pl = plan_pool(B, S, D, n_boundary, Vec<T>::N);
  const bool fused = fused_pooling(pl);
  float* partial = reinterpret_cast<float*>(workspace);
  if (!fused) {
    dim3 g1(pl.n_chunks, pl.n_splits, B);
    pool_partial_kernel<T><<<g1, kPoolThreads, 0, st>>>(hidden, S, D, pl.n_rows, pl.a_len, pl.b_start,
                                                         pl.rows_per_split, partial);
    if (cudaGetLastError() != cudaSuccess) return EA_ERR_CUDA;
  }
  // W_k rows staged in shared memory when they fit next to the static buffers.
  const size_t wk_bytes = (size_t)kProjRows * N * sizeof(T);
  const int wk_smem = wk_bytes <= 96 * 1024 && (N * sizeof(T)) % 16 == 0 ? 1 : 0;
  const size_t dyn = wk_smem ? wk_bytes : 0;
  if (!attr_once<project_kernel<T>>(96 * 1024)) return EA_ERR_CUDA;
  const cudaError_t e = launch_after(project_kernel<T>, dim3(proj_ctas(D)), dim3(kProjThreads), dyn, st, !fused,
                                     hidden, S, pl.n_rows, pl.a_len, pl.b_start, fused ? nullptr : partial,
                                     pl.n_splits, B, D, 1.0f / (float)pl.n_rows, w_k, N, proj_batch(N), pp, wk_smem);
  return e == cudaSuccess ? EA_OK : EA_ERR_CUDA;
}

ea_status launch_router(const void* hidden, ea_dtype dtype, int B, int S, int D, int H_kv, int d,
                        const ea_router_weights* w, const ea_router_params* prm, int32_t* head_mode,
                        float* logits, void* workspace, cudaStream_t st) {
  const int N = H_kv * d;
  float* pp = reinterpret_cast<float*>(reinterpret_cast<char*>(workspace) + partial_bytes(B, S, D, prm->n_boundary));
  ea_status s = dtype == EA_DT_BF16
                    ? launch_pool_project(static_cast<const __nv_bfloat16*>(hidden), B, S, D, N,
                                          static_cast<const __nv_bfloat16*>(w->w_k), prm->n_boundary, workspace, pp, st)
                    : launch_pool_project(static_cast<const float*>(hidden), B, S, D, N,
                                          static_cast<const float*>(w->w_k), prm->n_boundary, workspace, pp, st);
  if (s != EA_OK) return s;
  const int n_pp = proj_ctas(D) / kCluster;
  return d == 128 ? launch_head<128>(pp, n_pp, B * H_kv, H_kv, w, head_mode, logits, st)
                  : launch_head<64>(pp, n_pp, B * H_kv, H_kv, w, head_mode, logits, st);
}

ea_status launch_router_pool(const void* hidden, ea_dtype dtype, int B, int S, int D, int n_boundary, float* hbar,
                             void* workspace, cudaStream_t st) {
  const int vec = dtype == EA_DT_BF16 ? 8 : 4;
  const PoolPlan pl = plan_pool(B, S, D, n_boundary, vec);
  float* partial = reinterpret_cast<float*>(workspace);
  dim3 g1(pl.n_chunks, pl.n_splits, B);
  if (dtype == EA_DT_BF16)
    pool_partial_kernel<__nv_bfloat16><<<g1, kPoolThreads, 0, st>>>(static_cast<const __nv_bfloat16*>(hidden), S, D,
                                                                     pl.n_rows, pl.a_len, pl.b_start,
                                                                     pl.rows_per_split, partial);
  else
    pool_partial_kernel<float><<<g1, kPoolThreads, 0, st>>>(static_cast<const float*>(hidden), S, D, pl.n_rows,
                                                             pl.a_len, pl.b_start, pl.rows_per_split, partial);
  if (cudaGetLastError() != cudaSuccess) return EA_ERR_CUDA;
  return launch_after(pool_finish_kernel, dim3(cdiv(B * D, 32)), dim3(256), 0, st, true, partial, pl.n_splits, B, D,
                      1.0f / (float)pl.n_rows, hbar) == cudaSuccess
             ? EA_OK
             : EA_ERR_CUDA;
}

}  // namespace ea
