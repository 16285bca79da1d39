// ea_assign.cu — retrieval scores and the static retrieval-head assignment.
//
// "Elastic Attention: Test-time Adaptive Sparsity Ratios for Efficient Transformers",
// appendix C.1 "Retrieval Score Calculation": a needle sits in a long haystack and the
// retrieval score of a head is the attention mass its last token puts on the needle
// positions; "Sparsity Assignment": for a target Omega_MSR the
// k = floor((1 - Omega_MSR) * L * H) best-scoring heads keep full attention and the
// rest use streaming sparse attention.  The assignment is per KV head (the unit the
// router assigns), a KV head's score being the mean of its G query heads' scores over
// the probe samples; ties go to the lower flat index l * H_kv + h.
//
//   retrieval_partial_kernel  grid (splits, H_q, B): the last query row against a slice
//                             of the keys, online (max, total mass, needle mass) in log2
//                             units; K is streamed once per query head in 16-byte loads
//   retrieval_finish_kernel   combines the slices: score = needle mass / total mass
//   assign_kernel             one CTA: KV-head means, rank of every head, head_mode
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cmath>
#include <cstdint>
#include "ea_common.cuh"
#include "ea_internal.h"

namespace ea {
namespace {

constexpr int kRetThreads = 256;
constexpr int kAssignThreads = 1024;
constexpr int kMaxAssignHeads = 8192;   // L * H_kv

struct Triple {
  float m, l, n;   // running max (log2 units), total mass and needle mass relative to 2^m
};
__device__ __forceinline__ Triple combine(Triple a, Triple b) {
  if (b.m == -INFINITY) return a;
  if (a.m == -INFINITY) return b;
  const float m = fmaxf(a.m, b.m);
  const float fa = exp2f(a.m - m), fb = exp2f(b.m - m);
  return {m, a.l * fa + b.l * fb, a.n * fa + b.n * fb};
}

__device__ __forceinline__ float dot_row(const float* qs, const float* k, int d) {
  float acc = 0.f;
  for (int e = 0; e < d; e += 4) {
    const float4 x = *reinterpret_cast<const float4*>(k + e);
    acc = fmaf(qs[e], x.x, acc);
    acc = fmaf(qs[e + 1], x.y, acc);
    acc = fmaf(qs[e + 2], x.z, acc);
    acc = fmaf(qs[e + 3], x.w, acc);
  }
  return acc;
}
__device__ __forceinline__ float dot_row(const float* qs, const __nv_bfloat16* k, int d) {
  float acc = 0.f;
  for (int e = 0; e < d; e += 8) {
    const uint4 x = *reinterpret_cast<const uint4*>(k + e);
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      acc = fmaf(qs[e + 2 * t], __uint_as_float(w[t] << 16), acc);
      acc = fmaf(qs[e + 2 * t + 1], __uint_as_float(w[t] & 0xffff0000u), acc);
    }
  }
  return acc;
}
__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__global__ void __launch_bounds__(kRetThreads)
retrieval_partial_kernel(const T* __restrict__ q, const T* __restrict__ k, int S, int H_q, int H_kv, int d,
                         int needle_begin, int needle_end, float scale_log2, int splits,
                         float* __restrict__ partial) {
  __shared__ float qs[128];
  __shared__ Triple red[kRetThreads / 32];
  const int sp = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int hk = h / (H_q / H_kv);
  const T* qrow = q + (((size_t)b * S + (S - 1)) * H_q + h) * d;
  for (int e = threadIdx.x; e < d; e += kRetThreads) qs[e] = to_f(qrow[e]) * scale_log2;
  __syncthreads();
  const int chunk = cdiv(S, splits);
  const int j0 = sp * chunk, j1 = min(S, j0 + chunk);
  Triple t{-INFINITY, 0.f, 0.f};
  for (int j = j0 + (int)threadIdx.x; j < j1; j += kRetThreads) {
    const float x = dot_row(qs, k + (((size_t)b * S + j) * H_kv + hk) * d, d);
    const float in = (j >= needle_begin && j < needle_end) ? 1.f : 0.f;
    if (x > t.m) {
      const float f = exp2f(t.m - x);   // 0 while t.m is -inf
      t.l = t.l * f + 1.f;
      t.n = t.n * f + in;
      t.m = x;
    } else {
      const float e = exp2f(x - t.m);
      t.l += e;
      t.n += in * e;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    Triple u{__shfl_xor_sync(0xffffffffu, t.m, o), __shfl_xor_sync(0xffffffffu, t.l, o),
             __shfl_xor_sync(0xffffffffu, t.n, o)};
    t = combine(t, u);
  }
  if (threadIdx.x % 32 == 0) red[threadIdx.x / 32] = t;
  __syncthreads();
  if (threadIdx.x == 0) {
    Triple a = red[0];
    for (int w = 1; w < kRetThreads / 32; ++w) a = combine(a, red[w]);
    float* out = partial + (((size_t)b * H_q + h) * splits + sp) * 3;
    out[0] = a.m;
    out[1] = a.l;
    out[2] = a.n;
  }
}

__global__ void retrieval_finish_kernel(const float* __restrict__ partial, int n_heads, int splits,
                                        float* __restrict__ scores) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n_heads) return;
  Triple a{-INFINITY, 0.f, 0.f};
  for (int sp = 0; sp < splits; ++sp) {
    const float* p = partial + ((size_t)i * splits + sp) * 3;
    a = combine(a, Triple{p[0], p[1], p[2]});
  }
  scores[i] = a.l > 0.f ? a.n / a.l : 0.f;
}

__global__ void __launch_bounds__(kAssignThreads)
assign_kernel(const float* __restrict__ scores, int L, int B, int H_q, int H_kv, int k_full,
              int32_t* __restrict__ head_mode) {
  extern __shared__ float kv[];
  const int n = L * H_kv, G = H_q / H_kv;
  for (int i = threadIdx.x; i < n; i += kAssignThreads) {
    const int l = i / H_kv, h = i % H_kv;
    float acc = 0.f;
    for (int b = 0; b < B; ++b)
      for (int g = 0; g < G; ++g) acc += scores[((size_t)l * B + b) * H_q + h * G + g];
    kv[i] = acc / (float)(B * G);
  }
  __syncthreads();
  for (int i = threadIdx.x; i < n; i += kAssignThreads) {
    const float si = kv[i];
    int rank = 0;
    for (int j = 0; j < n; ++j) {
      const float sj = kv[j];
      rank += (sj > si || (sj == si && j < i)) ? 1 : 0;
    }
    const int mode = rank < k_full ? 0 : 1;
    const int l = i / H_kv, h = i % H_kv;
    for (int b = 0; b < B; ++b) head_mode[((size_t)l * B + b) * H_kv + h] = mode;
  }
}

int retrieval_splits(int B, int S, int H_q) {
  const long long heads = (long long)B * H_q;
  long long sp = (4LL * 148 + heads - 1) / heads;
  sp = std::min<long long>(sp, std::max(1, cdiv(S, kRetThreads)));
  return (int)std::max<long long>(1, std::min<long long>(sp, 1024));
}

}  // namespace

size_t retrieval_workspace_bytes(int B, int S, int H_q) {
  return ((size_t)B * H_q * retrieval_splits(B, S, H_q) * 3 * sizeof(float) + 255) / 256 * 256;
}

ea_status launch_retrieval(const void* q, const void* k, ea_dtype dtype, int B, int S, int H_q, int H_kv, int d,
                           int needle_begin, int needle_end, float scale_log2, float* scores, void* workspace,
                           cudaStream_t st) {
  const int splits = retrieval_splits(B, S, H_q);
  float* partial = static_cast<float*>(workspace);
  dim3 grid(splits, H_q, B);
  if (dtype == EA_DT_BF16)
    retrieval_partial_kernel<__nv_bfloat16><<<grid, kRetThreads, 0, st>>>(
        static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k), S, H_q, H_kv, d, needle_begin,
        needle_end, scale_log2, splits, partial);
  else
    retrieval_partial_kernel<float><<<grid, kRetThreads, 0, st>>>(
        static_cast<const float*>(q), static_cast<const float*>(k), S, H_q, H_kv, d, needle_begin, needle_end,
        scale_log2, splits, partial);
  if (cudaGetLastError() != cudaSuccess) return EA_ERR_CUDA;
  const int n = B * H_q;
  retrieval_finish_kernel<<<cdiv(n, 256), 256, 0, st>>>(partial, n, splits, scores);
  return cudaGetLastError() == cudaSuccess ? EA_OK : EA_ERR_CUDA;
}

bool assignment_shape_ok(int L, int H_kv) { return (long long)L * H_kv <= kMaxAssignHeads; }

ea_status launch_assignment(const float* scores, int L, int B, int H_q, int H_kv, int k_full, int32_t* head_mode,
                            cudaStream_t st) {
  const size_t smem = (size_t)L * H_kv * sizeof(float);
  assign_kernel<<<1, kAssignThreads, smem, st>>>(scores, L, B, H_q, H_kv, k_full, head_mode);
  return cudaGetLastError() == cudaSuccess ? EA_OK : EA_ERR_CUDA;
}

}  // namespace ea
