// ea_attn_simt.cu — fp32 hybrid-head attention on CUDA cores.
//
// Same per-head rule as the tensor-core kernel ("Elastic Attention: Test-time
// Adaptive Sparsity Ratios for Efficient Transformers", section 2 "Hybrid Head
// Mechanism", appendix D.1 "Sparse Inference"), in plain fp32 so fp32 inputs keep
// fp32 accuracy (tf32 tensor cores would not).  One CTA per (64 query rows, query
// head, sample); 8 warps x 8 rows; keys in 64-key tiles staged in shared memory;
// online softmax with accurate expf; key tiles with no live pair are skipped.
#include <cuda_runtime.h>
#include <cstdint>
#include "ea_common.cuh"
#include "ea_internal.h"

namespace ea {
namespace {

constexpr int kRows = 64, kKeys = 64, kThreads = 256, kRowsPerWarp = kRows / (kThreads / 32);

// Does key tile [c0, c0+64) hold a live pair for query rows [r0, r1]?
__device__ __forceinline__ bool simt_tile_live(const PatternDev& p, int kind, int H_kv, int b, int h,
                                               int r0, int r1, int c0) {
  if (c0 > r1) return false;
  if (kind == EA_STREAMING) {
    if (c0 < p.n_sink) return true;
    return r0 - (c0 + kKeys - 1) < p.window;  // smallest distance i - j over the tile pair
  }
  const int B = p.block;   // 64 or 128: the 64-row and 64-key tiles sit in one block each
  if (kind == EA_STREAMING_BLOCKS)
    return c0 / B < cdiv(p.n_sink, B) || r0 / B - c0 / B < cdiv(p.window, B);
  if (kind == EA_BLOCK_SPARSE) {   // (r0 is a sequence position; chunks start on a multiple of 128)
    long long a, e;
    csr_row(p, H_kv, b, h, r0 / B, a, e);
    for (long long x = a; x < e; ++x)
      if (p.cols[x] == c0 / B) return true;
    return false;
  }
  return true;
}

template <int HD>
__global__ void __launch_bounds__(kThreads)
attn_simt_kernel(const float* __restrict__ q, const float* __restrict__ k, const float* __restrict__ v,
                 float* __restrict__ o, const int32_t* __restrict__ head_mode, PatternDev p,
                 int S, int S_k, int H_q, int H_kv) {
  constexpr int NC = HD / 32;  // output columns per lane
  extern __shared__ float smem[];
  float (*Ks)[HD + 1] = reinterpret_cast<float (*)[HD + 1]>(smem);
  float (*Vs)[HD] = reinterpret_cast<float (*)[HD]>(smem + kKeys * (HD + 1));
  float (*Qs)[HD] = reinterpret_cast<float (*)[HD]>(smem + kKeys * (HD + 1) + kKeys * HD);
  // r0 / r1: first and last query row of this CTA in the call (q, o); g0 / g1 in the sequence.
  const int r0 = blockIdx.x * kRows, h_q = blockIdx.y, b = blockIdx.z;
  const int G = H_q / H_kv, h = h_q / G;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int kind = head_kind(p, head_mode, H_kv, b, h);
  const int r1 = min(S, r0 + kRows) - 1;
  const int q0 = p.q_tile0 * kTile, g0 = q0 + r0, g1 = q0 + r1;
  for (int x = threadIdx.x; x < kRows * HD; x += kThreads) {
    const int r = x / HD, c = x % HD;
    Qs[r][c] = (r0 + r < S) ? q[(((size_t)b * S + r0 + r) * H_q + h_q) * HD + c] : 0.f;
  }
  float m[kRowsPerWarp], l[kRowsPerWarp], acc[kRowsPerWarp][NC];
#pragma unroll
  for (int rr = 0; rr < kRowsPerWarp; ++rr) {
    m[rr] = -INFINITY;
    l[rr] = 0.f;
#pragma unroll
    for (int c = 0; c < NC; ++c) acc[rr][c] = 0.f;
  }
  for (int c0 = 0; c0 <= g1; c0 += kKeys) {
    if (!simt_tile_live(p, kind, H_kv, b, h, g0, g1, c0)) continue;
    __syncthreads();
    for (int x = threadIdx.x; x < kKeys * HD; x += kThreads) {
      const int j = x / HD, c = x % HD;
      const bool in = c0 + j < S_k;
      const size_t off = (((size_t)b * S_k + c0 + j) * H_kv + h) * HD + c;
      Ks[j][c] = in ? k[off] : 0.f;
      Vs[j][c] = in ? v[off] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int rr = 0; rr < kRowsPerWarp; ++rr) {
      const int rl = warp * kRowsPerWarp + rr, i = g0 + rl;   // query position in the sequence
      float s[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int j = lane + 32 * u;
        float dot = 0.f;
#pragma unroll 16
        for (int c = 0; c < HD; ++c) dot = fmaf(Qs[rl][c], Ks[j][c], dot);
        const int kind_el = (kind == EA_BLOCK_SPARSE) ? EA_FULL : kind;  // block listed: causal only
        s[u] = (r0 + rl < S && c0 + j < S_k && key_live(p, kind_el, i, c0 + j)) ? dot * p.scale : -INFINITY;
      }
      float mt = fmaxf(s[0], s[1]);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, off));
      const float m_new = fmaxf(m[rr], mt);
      if (m_new == -INFINITY) continue;  // no live key for this row yet
      const float corr = expf(m[rr] - m_new);
      const float p0 = expf(s[0] - m_new), p1 = expf(s[1] - m_new);
      float ps = p0 + p1;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
      l[rr] = l[rr] * corr + ps;
      m[rr] = m_new;
#pragma unroll
      for (int c = 0; c < NC; ++c) acc[rr][c] *= corr;
#pragma unroll 8
      for (int j = 0; j < kKeys; ++j) {
        const float pj = __shfl_sync(0xffffffffu, j < 32 ? p0 : p1, j & 31);
#pragma unroll
        for (int c = 0; c < NC; ++c) acc[rr][c] = fmaf(pj, Vs[j][lane + 32 * c], acc[rr][c]);
      }
    }
  }
#pragma unroll
  for (int rr = 0; rr < kRowsPerWarp; ++rr) {
    const int i = r0 + warp * kRowsPerWarp + rr;
    if (i >= S) continue;
    const float inv = l[rr] > 0.f ? 1.f / l[rr] : 0.f;
#pragma unroll
    for (int c = 0; c < NC; ++c) o[(((size_t)b * S + i) * H_q + h_q) * HD + lane + 32 * c] = acc[rr][c] * inv;
  }
}

}  // namespace

ea_status launch_attn_simt(const float* q, const float* k, const float* v, float* o, const int32_t* head_mode,
                           const PatternDev& pat, int B, int S, int S_k, int H_q, int H_kv, int d, cudaStream_t st) {
  dim3 grid(cdiv(S, kRows), H_q, B);
  const size_t smem = sizeof(float) * ((size_t)kKeys * (d + 1) + (size_t)kKeys * d + (size_t)kRows * d);
  auto kern = d == 64 ? attn_simt_kernel<64> : d == 128 ? attn_simt_kernel<128> : nullptr;
  if (!kern) return EA_ERR_UNSUPPORTED;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return EA_ERR_CUDA;
  kern<<<grid, kThreads, smem, st>>>(q, k, v, o, head_mode, pat, S, S_k, H_q, H_kv);
  return cudaGetLastError() == cudaSuccess ? EA_OK : EA_ERR_CUDA;
}

}  // namespace ea
