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
//   retrieval_partial_kernel  grid (splits, H_kv, B): the last query rows of a KV group's G
//                             heads against a slice of the keys, online (max, total mass,
//                             needle mass) in log2 units; each key row is read once, in
//                             16-byte loads
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

// x[g] = qs[g] . krow for the ng (<= NG) heads at qs (rows of d floats); the key row is read once.
template <int NG, int D>
__device__ __forceinline__ void dot_rows(const float* qs, const float* krow, int ng, float (&x)[NG]) {
  constexpr int d = D;
#pragma unroll
  for (int g = 0; g < NG; ++g) x[g] = 0.f;
#pragma unroll
  for (int e = 0; e < d; e += 4) {
    const float4 v = *reinterpret_cast<const float4*>(krow + e);
#pragma unroll
    for (int g = 0; g < NG; ++g) {
      if (g >= ng) break;
      const float* qg = qs + g * d + e;
      x[g] = fmaf(qg[0], v.x, fmaf(qg[1], v.y, fmaf(qg[2], v.z, fmaf(qg[3], v.w, x[g]))));
    }
  }
}
template <int NG, int D>
__device__ __forceinline__ void dot_rows(const float* qs, const __nv_bfloat16* krow, int ng, float (&x)[NG]) {
  constexpr int d = D;
#pragma unroll
  for (int g = 0; g < NG; ++g) x[g] = 0.f;
#pragma unroll
  for (int e = 0; e < d; e += 8) {
    const uint4 v = *reinterpret_cast<const uint4*>(krow + e);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    float kf[8];
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      kf[2 * t] = __uint_as_float(w[t] << 16);
      kf[2 * t + 1] = __uint_as_float(w[t] & 0xffff0000u);
    }
#pragma unroll
    for (int g = 0; g < NG; ++g) {
      if (g >= ng) break;
      const float* qg = qs + g * d + e;
#pragma unroll
      for (int t = 0; t < 8; ++t) x[g] = fmaf(qg[t], kf[t], x[g]);
    }
  }
}
__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }

// One CTA per (key slice, KV head, sample) serves all G query heads of the group, so every
// key row is read once; heads are taken in groups of kHeadChunk (registers per thread).
constexpr int kHeadChunk = 8;

template <typename T, int d>
__global__ void __launch_bounds__(kRetThreads)
retrieval_partial_kernel(const T* __restrict__ q, const T* __restrict__ k, int S, int H_q, int H_kv,
                         int needle_begin, int needle_end, float scale_log2, int splits,
                         float* __restrict__ partial) {
  extern __shared__ float qs[];                    // [G][d], scaled to log2 units
  __shared__ Triple red[kRetThreads / 32][kHeadChunk];
  const int sp = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
  const int G = H_q / H_kv;
  for (int e = threadIdx.x; e < G * d; e += kRetThreads) {
    const int g = e / d;
    qs[e] = to_f(q[(((size_t)b * S + (S - 1)) * H_q + hk * G + g) * d + e % d]) * scale_log2;
  }
  __syncthreads();
  const int chunk = cdiv(S, splits);
  const int j0 = sp * chunk, j1 = min(S, j0 + chunk);
  for (int g0 = 0; g0 < G; g0 += kHeadChunk) {
    const int ng = min(kHeadChunk, G - g0);
    Triple t[kHeadChunk];
#pragma unroll
    for (int g = 0; g < kHeadChunk; ++g) t[g] = Triple{-INFINITY, 0.f, 0.f};
    for (int j = j0 + (int)threadIdx.x; j < j1; j += kRetThreads) {
      const T* krow = k + (((size_t)b * S + j) * H_kv + hk) * d;
      float x[kHeadChunk];
      dot_rows<kHeadChunk, d>(qs + (size_t)g0 * d, krow, ng, x);
      const float in = (j >= needle_begin && j < needle_end) ? 1.f : 0.f;
#pragma unroll
      for (int g = 0; g < kHeadChunk; ++g) {
        if (g >= ng) break;
        if (x[g] > t[g].m) {
          const float f = exp2f(t[g].m - x[g]);   // 0 while the max is -inf
          t[g].l = t[g].l * f + 1.f;
          t[g].n = t[g].n * f + in;
          t[g].m = x[g];
        } else {
          const float e = exp2f(x[g] - t[g].m);
          t[g].l += e;
          t[g].n += in * e;
        }
      }
    }
#pragma unroll
    for (int g = 0; g < kHeadChunk; ++g) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        Triple u{__shfl_xor_sync(0xffffffffu, t[g].m, o), __shfl_xor_sync(0xffffffffu, t[g].l, o),
                 __shfl_xor_sync(0xffffffffu, t[g].n, o)};
        t[g] = combine(t[g], u);
      }
      if (threadIdx.x % 32 == 0) red[threadIdx.x / 32][g] = t[g];
    }
    __syncthreads();
    if ((int)threadIdx.x < ng) {
      const int g = threadIdx.x;
      Triple a = red[0][g];
      for (int w = 1; w < kRetThreads / 32; ++w) a = combine(a, red[w][g]);
      float* out = partial + (((size_t)b * H_q + hk * G + g0 + g) * splits + sp) * 3;
      out[0] = a.m;
      out[1] = a.l;
      out[2] = a.n;
    }
    __syncthreads();
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

int retrieval_splits(int B, int S, int H_kv) {
  const long long heads = (long long)B * H_kv;
  long long sp = (4LL * 148 + heads - 1) / heads;
  sp = std::min<long long>(sp, std::max(1, cdiv(S, kRetThreads)));
  return (int)std::max<long long>(1, std::min<long long>(sp, 1024));
}

}  // namespace

size_t retrieval_workspace_bytes(int B, int S, int H_q, int H_kv) {
  return ((size_t)B * H_q * retrieval_splits(B, S, H_kv) * 3 * sizeof(float) + 255) / 256 * 256;
}

ea_status launch_retrieval(const void* q, const void* k, ea_dtype dtype, int B, int S, int H_q, int H_kv, int d,
                           int needle_begin, int needle_end, float scale_log2, float* scores, void* workspace,
                           cudaStream_t st) {
  const int splits = retrieval_splits(B, S, H_kv);
  float* partial = static_cast<float*>(workspace);
  dim3 grid(splits, H_kv, B);
  const size_t smem = (size_t)H_q / H_kv * d * sizeof(float);
  const auto* qb = static_cast<const __nv_bfloat16*>(q);
  const auto* kb = static_cast<const __nv_bfloat16*>(k);
  const auto* qf = static_cast<const float*>(q);
  const auto* kf = static_cast<const float*>(k);
  if (dtype == EA_DT_BF16 && d == 128)
    retrieval_partial_kernel<__nv_bfloat16, 128><<<grid, kRetThreads, smem, st>>>(
        qb, kb, S, H_q, H_kv, needle_begin, needle_end, scale_log2, splits, partial);
  else if (dtype == EA_DT_BF16)
    retrieval_partial_kernel<__nv_bfloat16, 64><<<grid, kRetThreads, smem, st>>>(
        qb, kb, S, H_q, H_kv, needle_begin, needle_end, scale_log2, splits, partial);
  else if (d == 128)
    retrieval_partial_kernel<float, 128><<<grid, kRetThreads, smem, st>>>(
        qf, kf, S, H_q, H_kv, needle_begin, needle_end, scale_log2, splits, partial);
  else
    retrieval_partial_kernel<float, 64><<<grid, kRetThreads, smem, st>>>(
        qf, kf, S, H_q, H_kv, needle_begin, needle_end, scale_log2, splits, partial);
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
