// ea_xattn.cu — XAttention block selection for the block-sparse heads, on the device.
//
// "Elastic Attention: Test-time Adaptive Sparsity Ratios for Efficient Transformers",
// section 4 "Evaluation Setting", runs its block-sparse heads with XAttention
// (threshold tau = 0.9); appendix G.2 "Efficiency Results" pairs it with full heads
// (FA-XA) and with streaming heads (XA-SSA).  The method (Xu et al., "XAttention:
// Block Sparse Attention with Antidiagonal Scoring", 2025), as computed here:
//   R[i, j] = sum_m q[i*st + m] . k[j*st + st-1-m]      (antidiagonal scoring, stride st)
//   P       = causal row softmax of R / (sqrt(d) * st)   (reduced columns j <= i)
//   A[qb,kb] = mean over the KV group's query heads of the P mass of tile (qb, kb)
//   row qb keeps its diagonal block, then blocks by descending A while the kept mass
//   is below tau x the row's total.
// The output is the CSR layout the hybrid attention reads for its BLOCK_SPARSE heads.
//
// Kernels, in stream order:
//   xattn_plan_kernel    the (b, h_q) whose KV head is BLOCK_SPARSE under head_mode;
//   xattn_score_kernel   R on the tensor cores, 128 reduced rows x 256 reduced columns per
//                        MMA (one q chunk feeds two key tiles; tcgen05, TMEM accumulators,
//                        TMA 5-D maps that split the sequence into (reduced row, m)), and
//                        per reduced row and 128-key block the partial softmax sums
//                        relative to the tile's row maximum;
//   xattn_select_kernel  per (b, h_kv, query block): row maxima and sums, the group-mean
//                        block masses, the sorted cumulative selection -> bitmap;
//   xattn_scan_kernel    row counts -> row_ptr;  xattn_fill_kernel  bitmap -> cols.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include "ea_common.cuh"
#include "ea_internal.h"
#include "ea_sm100.cuh"

namespace ea {
namespace {
using namespace sm100;

constexpr int XT = 128;                       // reduced rows (and columns) per tile
constexpr int XN = 256;                       // reduced key columns per MMA: a pair of tiles
constexpr int XNS = 4;                        // K-chunk stages
constexpr uint32_t kChunkBytes = 16384;       // 128 rows x 64 bf16 (q chunk)
constexpr uint32_t kBChunkBytes = 32768;      // 256 rows x 64 bf16 (k chunk)
constexpr uint32_t X_OFF_A = 0;
constexpr uint32_t X_OFF_B = XNS * kChunkBytes;
constexpr uint32_t X_OFF_BAR = XNS * (kChunkBytes + kBChunkBytes);
enum : int { X_FULL = 0, X_EMPTY = XNS, X_AFULL = 2 * XNS, X_AEMPTY = X_AFULL + 2, X_FIN = X_AEMPTY + 2,
             X_NEVER = X_FIN + 1, X_NBAR = X_NEVER + 1 };
constexpr uint32_t X_OFF_TMEM = X_OFF_BAR + X_NBAR * 8;
constexpr uint32_t X_OFF_ABORT = X_OFF_TMEM + 4;
constexpr uint32_t kXSmemBytes = X_OFF_ABORT + 4 + 1024;   // + slack to align the base to 1024
static_assert(kXSmemBytes <= 232448, "shared memory beyond the 227 KB a CTA may use");
constexpr int kXThreads = 192;                // warp 0 TMA, warp 1 TMEM + MMA, warps 2-5 epilogue
constexpr uint32_t kXTmemCols = 512;          // two 256-column accumulators
constexpr uint32_t IDESC_X = idesc_bf16(128, XN, false);
constexpr unsigned long long kXWaitLimitNs = 2000000000ull;

constexpr int kSelThreads = 256;
constexpr int kMaxQb = 2048;                  // query blocks (S <= 262144)
constexpr int kMaxSelRows = 1024;             // G x reduced rows per block

// Workspace (bytes from its base): status word at 0 (as every attention workspace), live
// (b, h_q) count at 8, then the plan, m_part, s_part, counts, bitmap.
constexpr size_t kXsLive = 8;
constexpr size_t kXsHeader = 256;

struct XLayout {
  int n_red, n_rt, n_qb, words;
  size_t plan, m_part, s_part, counts, bitmap, total;
};
size_t up256(size_t x) { return (x + 255) / 256 * 256; }
// blk: the layout's block edge (64 or 128); a 128-column reduced tile holds 128*st/blk blocks.
XLayout x_layout(int B, int S, int H_q, int H_kv, int st, int blk) {
  XLayout L;
  L.n_red = S / st;
  L.n_rt = cdiv(L.n_red, XT);
  L.n_qb = cdiv(S, blk);
  L.words = cdiv(L.n_qb, 32);
  const size_t rows_red = (size_t)B * H_q * L.n_red;
  const size_t n_rows = (size_t)B * H_kv * L.n_qb;
  L.plan = kXsHeader;
  L.m_part = L.plan + up256((size_t)B * H_q * 4);
  L.s_part = L.m_part + up256(rows_red * L.n_rt * 4);
  L.counts = L.s_part + up256(rows_red * L.n_rt * (XT * st / blk) * 4);
  L.bitmap = L.counts + up256(n_rows * 4);
  L.total = L.bitmap + up256(n_rows * L.words * 4);
  return L;
}

// ---- bounded waits (a CTA that waits 2 s raises its abort flag and the status word) ----
struct XCtx {
  uint32_t bar0;
  volatile int* abort_flag;
  uint32_t* status;
  __device__ uint32_t bar(int i) const { return bar0 + 8u * i; }
};
__device__ __noinline__ bool xwait_slow(const XCtx& c, uint32_t bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (*c.abort_flag) return false;
    if (globaltimer_ns() - t0 > kXWaitLimitNs) {
      *c.abort_flag = 1;
      atomicOr(c.status, kStatusTimeout);
      return false;
    }
  }
  return true;
}
__device__ __forceinline__ bool xwait(const XCtx& c, uint32_t bar, uint32_t parity) {
  return mbar_try_wait(bar, parity) || xwait_slow(c, bar, parity);
}
__device__ __noinline__ void xwait_drain(const XCtx& c, uint32_t bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > kXWaitLimitNs) {
      atomicOr(c.status, kStatusTimeout);
      return;
    }
  }
}

__device__ __forceinline__ void tma_load_5d(uint32_t dst, const CUtensorMap* map, uint32_t bar, int x, int y,
                                            int z, int w, int v) {
  asm volatile(
      "cp.async.bulk.tensor.5d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6, %7}], [%2];"
      ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y), "r"(z), "r"(w), "r"(v)
      : "memory");
}

// K-major 128-byte-swizzled chunk: 128 rows of 128 bytes, 8-row atoms 1024 bytes apart;
// K step kk (16 elements) = +32 bytes.
__device__ __forceinline__ uint64_t x_desc(uint32_t chunk, int kk) {
  return sdesc_sw128(chunk + (uint32_t)kk * 32u, 16u, 1024u);
}

struct XItem {
  int b, h, hk, r, bh;
};
__device__ __forceinline__ int x_item_index(int it, int cta, int ncta) {
  return it * ncta + ((it & 1) ? (ncta - 1 - cta) : cta);
}
// Work k -> (reduced query tile r, longest first; live head pi).
__device__ __forceinline__ XItem x_item(const int* plan, int idx, int n_live, int n_rt, int H_q, int G) {
  XItem I;
  const int rr = idx / n_live, pi = idx % n_live;
  I.r = n_rt - 1 - rr;
  I.bh = plan[pi];
  I.b = I.bh / H_q;
  I.h = I.bh % H_q;
  I.hk = I.h / G;
  return I;
}

__global__ void xattn_plan_kernel(const int32_t* __restrict__ head_mode, PatternDev p, int B, int H_q, int H_kv,
                                  uint32_t* __restrict__ hdr, int* __restrict__ plan) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  const int G = H_q / H_kv;
  int n = 0;
  uint32_t bad = 0;
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < H_kv; ++h) {
      const int m = head_mode[b * H_kv + h];
      if (m != 0 && m != 1) bad |= kStatusBadMode;
      if (head_kind(p, head_mode, H_kv, b, h) == EA_BLOCK_SPARSE)
        for (int g = 0; g < G; ++g) plan[n++] = b * H_q + h * G + g;
    }
  hdr[kXsLive / 4] = (uint32_t)n;
  if (bad) atomicOr(hdr + kWsStatus / 4, bad);
}

// Partial softmax sums of one reduced row over one 128-column tile holding NB blocks:
// sg[g] = sum of exp2(x*sl2 - ms) over the live columns of block g, ms = sl2 * (max over
// live columns).
template <int NB, bool kDiag>
__device__ __forceinline__ float x_row_tile(const float (&x)[XT], int lim, float sl2, float (&sg)[NB]) {
  constexpr int BW = XT / NB;
  float mx = -INFINITY;
#pragma unroll
  for (int e = 0; e < XT; ++e)
    if (!kDiag || e <= lim) mx = fmaxf(mx, x[e]);
  const float ms = mx * sl2;
#pragma unroll
  for (int g = 0; g < NB; ++g) {
    float a0 = 0.f, a1 = 0.f;
#pragma unroll
    for (int e = 0; e < BW; e += 2) {
      const int e0 = g * BW + e;
      a0 += (!kDiag || e0 <= lim) ? ex2(fmaf(x[e0], sl2, -ms)) : 0.f;
      a1 += (!kDiag || e0 + 1 <= lim) ? ex2(fmaf(x[e0 + 1], sl2, -ms)) : 0.f;
    }
    sg[g] = a0 + a1;
  }
  return ms;
}

// ST: antidiagonal stride; NB: blocks per 128-column reduced tile (ST at block 128, 2*ST at 64).
template <int ST, int NB>
__global__ void __launch_bounds__(kXThreads, 1)
xattn_score_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k, int H_q,
                   int H_kv, int n_red, int n_rt, float sl2, const int* __restrict__ plan,
                   uint32_t* __restrict__ hdr, float* __restrict__ m_part, float* __restrict__ s_part,
                   int inject_stall) {
  constexpr int NCH = 2 * ST;   // K chunks per tile: ST row offsets x two 64-column halves of d
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int G = H_q / H_kv;
  XCtx c;
  c.bar0 = base + X_OFF_BAR;
  c.abort_flag = reinterpret_cast<volatile int*>(gbase + X_OFF_ABORT);
  c.status = hdr + kWsStatus / 4;
  const int n_live = (int)hdr[kXsLive / 4];
  const int n_work = n_live * n_rt;

  if (threadIdx.x == 0) {
    tma_prefetch_map(&tm_q);
    tma_prefetch_map(&tm_k);
    for (int i = 0; i < X_NBAR; ++i) mbar_init(c.bar(i), (i == X_AEMPTY || i == X_AEMPTY + 1) ? 128u : 1u);
    *c.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(base + X_OFF_TMEM, kXTmemCols);
    tmem_relinquish();
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(gbase + X_OFF_TMEM);

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int ch = 0;
      bool ok = true;
      for (int it = 0; ok; ++it) {
        const int idx = x_item_index(it, blockIdx.x, gridDim.x);
        if (idx >= n_work) break;
        const XItem I = x_item(plan, idx, n_live, n_rt, H_q, G);
        for (int pp = 0; pp <= I.r / 2 && ok; ++pp) {   // key tiles 2pp, 2pp+1
          for (int q = 0; q < NCH; ++q) {
            const int s = ch % XNS, m = q >> 1, half = q & 1;
            ok = xwait(c, c.bar(X_EMPTY + s), ((ch / XNS) & 1) ^ 1);
            if (!ok) break;
            mbar_expect_tx(c.bar(X_FULL + s), kChunkBytes + kBChunkBytes);
            tma_load_5d(base + X_OFF_A + s * kChunkBytes, &tm_q, c.bar(X_FULL + s), 64 * half, I.h, m, XT * I.r, I.b);
            tma_load_5d(base + X_OFF_B + s * kBChunkBytes, &tm_k, c.bar(X_FULL + s), 64 * half, I.hk, ST - 1 - m,
                        XN * pp, I.b);
            ++ch;
          }
        }
      }
      for (int s = 0; s < XNS; ++s) {   // the last copy armed on every stage has landed
        const int uses = ch / XNS + (s < ch % XNS ? 1 : 0);
        if (uses > 0) xwait_drain(c, c.bar(X_FULL + s), (uses - 1) & 1);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int ch = 0, tile = 0;
      // Test hook for the timeout path: CTA 0 first waits on a barrier nothing arrives on.
      bool ok = !(inject_stall && blockIdx.x == 0) || xwait(c, c.bar(X_NEVER), 0);
      for (int it = 0; ok; ++it) {
        const int idx = x_item_index(it, blockIdx.x, gridDim.x);
        if (idx >= n_work) break;
        const XItem I = x_item(plan, idx, n_live, n_rt, H_q, G);
        for (int pp = 0; pp <= I.r / 2 && ok; ++pp) {
          const int a = tile & 1;
          ok = xwait(c, c.bar(X_AEMPTY + a), ((tile >> 1) & 1) ^ 1);
          if (!ok) break;
          fence_after_sync();
          for (int q = 0; q < NCH && ok; ++q) {
            const int s = ch % XNS;
            ok = xwait(c, c.bar(X_FULL + s), (ch / XNS) & 1);
            if (!ok) break;
            fence_after_sync();
            const uint32_t at = base + X_OFF_A + s * kChunkBytes, bt = base + X_OFF_B + s * kBChunkBytes;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_ss(tmem + (uint32_t)XN * a, x_desc(at, kk), x_desc(bt, kk), IDESC_X, (q > 0 || kk > 0) ? 1u : 0u);
            commit(c.bar(X_EMPTY + s));
            ++ch;
          }
          if (!ok) break;
          commit(c.bar(X_AFULL + a));
          ++tile;
        }
      }
      commit(c.bar(X_FIN));   // every MMA issued here has completed
      xwait_drain(c, c.bar(X_FIN), 0);
    }
  } else {
    // ------------------------------------------------------------ epilogue (one reduced row per thread)
    const int wq = warp % 4;
    const int row = wq * 32 + lane;
    const uint32_t lane_addr = tmem + ((uint32_t)(wq * 32) << 16);
    const int pitch = n_rt * NB;
    int tile = 0;
    bool ok = true;
    for (int it = 0; ok; ++it) {
      const int idx = x_item_index(it, blockIdx.x, gridDim.x);
      if (idx >= n_work) break;
      const XItem I = x_item(plan, idx, n_live, n_rt, H_q, G);
      const int i = XT * I.r + row;
      const size_t rrow = (size_t)I.bh * n_red + i;
      for (int pp = 0; pp <= I.r / 2; ++pp) {
        const int a = tile & 1;
        ok = xwait(c, c.bar(X_AFULL + a), (tile >> 1) & 1);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        ++tile;
        fence_after_sync();
        for (int hf = 0; hf < 2; ++hf) {   // key tiles 2pp and 2pp+1 (the second may lie past the diagonal)
          const int ct = 2 * pp + hf;
          float x[XT];
          {
            uint32_t rr[XT];
#pragma unroll
            for (int q4 = 0; q4 < XT / 32; ++q4)
              tmem_ld32(lane_addr + (uint32_t)XN * a + 128u * hf + 32 * q4, rr + 32 * q4);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < XT; ++e) x[e] = __uint_as_float(rr[e]);
          }
          if (hf == 1) {   // the accumulator is free once both halves are in registers
            fence_before_sync();
            mbar_arrive(c.bar(X_AEMPTY + a));
          }
          if (i < n_red && ct <= I.r) {
            float sg[NB];
            const float ms =
                ct < I.r ? x_row_tile<NB, false>(x, XT - 1, sl2, sg) : x_row_tile<NB, true>(x, row, sl2, sg);
            float* sp = s_part + rrow * pitch + ct * NB;
#pragma unroll
            for (int g = 0; g < NB; g += 4)
              *reinterpret_cast<float4*>(sp + g) = make_float4(sg[g], sg[g + 1], sg[g + 2], sg[g + 3]);
            m_part[rrow * n_rt + ct] = ms;
          }
        }
      }
    }
  }

  fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    fence_after_sync();
    tmem_dealloc(tmem, kXTmemCols);
  }
}

// One CTA per (query block qb, KV head h, sample b).
template <int ST, int NB>
__global__ void __launch_bounds__(kSelThreads)
xattn_select_kernel(const int32_t* __restrict__ head_mode, PatternDev p, int H_q, int H_kv, int n_red, int n_rt,
                    float tau, const float* __restrict__ m_part, const float* __restrict__ s_part,
                    uint32_t* __restrict__ counts, uint32_t* __restrict__ bitmap, float* __restrict__ scores) {
  constexpr int BW = XT / NB;                  // reduced rows (and columns) per block
  __shared__ float a[kMaxQb];
  __shared__ unsigned long long keys[kMaxQb];
  __shared__ float rowM[kMaxSelRows], rowInvL[kMaxSelRows];
  __shared__ float part[kSelThreads];
  __shared__ uint32_t bits[kMaxQb / 32];
  __shared__ float total_s;
  const int qb = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int n_qb = p.n_qb, words = cdiv(n_qb, 32);
  const size_t row = ((size_t)b * H_kv + h) * n_qb + qb;
  const int kind = head_kind(p, head_mode, H_kv, b, h);
  if (kind != EA_BLOCK_SPARSE) {
    for (int w = tid; w < words; w += kSelThreads) bitmap[row * words + w] = 0u;
    if (scores)
      for (int kb = tid; kb < n_qb; kb += kSelThreads) scores[row * n_qb + kb] = 0.f;
    if (tid == 0) counts[row] = 0u;
    return;
  }
  const int G = H_q / H_kv;
  const int i0 = qb * BW, nr = min(BW, n_red - i0), rows = G * nr;
  const int pitch = n_rt * NB;

  // Row maxima M (log2 units) and 1 / row sums, one warp per reduced row.
  for (int rr = warp; rr < rows; rr += kSelThreads / 32) {
    const int g = rr / nr, i = i0 + rr % nr;
    const size_t rrow = ((size_t)b * H_q + h * G + g) * n_red + i;
    const int n_t = i / XT + 1;
    const float* mrow = m_part + rrow * n_rt;
    const float* srow = s_part + rrow * pitch;
    float M = -INFINITY;
    for (int t = lane; t < n_t; t += 32) M = fmaxf(M, mrow[t]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float L = 0.f;
    for (int kb = lane; kb < n_t * NB; kb += 32) L += srow[kb] * ex2(mrow[kb / NB] - M);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
    if (lane == 0) {
      rowM[rr] = M;
      rowInvL[rr] = L > 0.f ? 1.f / L : 0.f;
    }
  }
  for (int w = tid; w < words; w += kSelThreads) bits[w] = 0u;
  __syncthreads();

  // Group-mean block masses A[kb], kb <= qb.
  const float inv_g = 1.f / (float)G;
  for (int kb = tid; kb <= qb; kb += kSelThreads) {
    float acc = 0.f;
    for (int rr = 0; rr < rows; ++rr) {
      const int g = rr / nr, i = i0 + rr % nr;
      const size_t rrow = ((size_t)b * H_q + h * G + g) * n_red + i;
      acc += s_part[rrow * pitch + kb] * ex2(m_part[rrow * n_rt + kb / NB] - rowM[rr]) * rowInvL[rr];
    }
    a[kb] = acc * inv_g;
    if (scores) scores[row * n_qb + kb] = acc * inv_g;
  }
  if (scores)
    for (int kb = qb + 1 + tid; kb < n_qb; kb += kSelThreads) scores[row * n_qb + kb] = 0.f;
  __syncthreads();

  // Row total.
  {
    float t = 0.f;
    for (int kb = tid; kb <= qb; kb += kSelThreads) t += a[kb];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
    if (lane == 0) part[warp] = t;
    __syncthreads();
    if (tid == 0) {
      float s = 0.f;
      for (int w = 0; w < kSelThreads / 32; ++w) s += part[w];
      total_s = s;
    }
    __syncthreads();
  }
  const float need = tau * total_s;

  // Off-diagonal blocks sorted by descending mass, ties by ascending index: ascending
  // order of (~bits(mass), index) for masses >= 0.
  const int n_el = qb;
  int n2 = 1;
  while (n2 < n_el) n2 <<= 1;
  for (int e = tid; e < n2; e += kSelThreads)
    keys[e] = e < n_el ? ((unsigned long long)(~__float_as_uint(fmaxf(a[e], 0.f))) << 32) | (unsigned)e
                       : ~0ull;
  __syncthreads();
  for (int k = 2; k <= n2; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int e = tid; e < n2; e += kSelThreads) {
        const int partner = e ^ j;
        if (partner > e) {
          const bool up = (e & k) == 0;
          const unsigned long long x = keys[e], y = keys[partner];
          if ((x > y) == up) {
            keys[e] = y;
            keys[partner] = x;
          }
        }
      }
      __syncthreads();
    }
  }

  // Keep sorted position q while (diagonal mass + mass of positions before q) < need.
  const int per = cdiv(max(n_el, 1), kSelThreads);
  const int p0 = min(tid * per, n_el), p1 = min(p0 + per, n_el);
  float local = 0.f;
  for (int q = p0; q < p1; ++q) local += a[(int)(keys[q] & 0xffffffffu)];
  part[tid] = local;
  __syncthreads();
  if (tid == 0) {
    float run = 0.f;
    for (int t = 0; t < kSelThreads; ++t) {
      const float v = part[t];
      part[t] = run;
      run += v;
    }
  }
  __syncthreads();
  float run = a[qb] + part[tid];
  for (int q = p0; q < p1; ++q) {
    const int kb = (int)(keys[q] & 0xffffffffu);
    if (!(run < need)) break;
    atomicOr(&bits[kb >> 5], 1u << (kb & 31));
    run += a[kb];
  }
  if (tid == 0) atomicOr(&bits[qb >> 5], 1u << (qb & 31));
  __syncthreads();
  int cnt = 0;
  for (int w = tid; w < words; w += kSelThreads) {
    bitmap[row * words + w] = bits[w];
    cnt += __popc(bits[w]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
  if (lane == 0) part[warp] = (float)cnt;
  __syncthreads();
  if (tid == 0) {
    int s = 0;
    for (int w = 0; w < kSelThreads / 32; ++w) s += (int)part[w];
    counts[row] = (uint32_t)s;
  }
}

// Exclusive scan of the row counts into row_ptr (one CTA of 1024 threads).
__global__ void __launch_bounds__(1024)
xattn_scan_kernel(const uint32_t* __restrict__ counts, int n_rows, int32_t* __restrict__ row_ptr) {
  __shared__ int warp_sum[32];
  __shared__ int carry;
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  if (tid == 0) {
    carry = 0;
    row_ptr[0] = 0;
  }
  __syncthreads();
  for (int base = 0; base < n_rows; base += 1024) {
    const int idx = base + tid;
    int v = idx < n_rows ? (int)counts[idx] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += y;
    }
    if (lane == 31) warp_sum[warp] = v;
    __syncthreads();
    if (warp == 0) {
      int w = warp_sum[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, w, o);
        if (lane >= o) w += y;
      }
      warp_sum[lane] = w;
    }
    __syncthreads();
    const int incl = carry + v + (warp > 0 ? warp_sum[warp - 1] : 0);
    if (idx < n_rows) row_ptr[idx + 1] = incl;
    __syncthreads();
    if (tid == 1023) carry = incl;
    __syncthreads();
  }
}

// Bitmap rows -> ascending column lists (one warp per row).
__global__ void __launch_bounds__(256)
xattn_fill_kernel(const uint32_t* __restrict__ bitmap, const int32_t* __restrict__ row_ptr, int n_rows, int words,
                  int32_t* __restrict__ cols) {
  const int row = blockIdx.x * 8 + threadIdx.x / 32, lane = threadIdx.x % 32;
  if (row >= n_rows) return;
  int pos0 = row_ptr[row];
  for (int w0 = 0; w0 < words; w0 += 32) {
    const int w = w0 + lane;
    uint32_t bm = w < words ? bitmap[(size_t)row * words + w] : 0u;
    const int n = __popc(bm);
    int incl = n;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    int pos = pos0 + incl - n;
    while (bm) {
      const int bit = __ffs(bm) - 1;
      cols[pos++] = w * 32 + bit;
      bm &= bm - 1;
    }
    pos0 += __shfl_sync(0xffffffffu, incl, 31);
  }
}

typedef CUresult (*XEncodeFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                              const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                              CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
XEncodeFn x_encode_fn() {
  static XEncodeFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<XEncodeFn>(ptr);
  });
  return fn;
}

// [B, S, H, 128] bf16 viewed as 5-D (d, H, st, S/st, B): coordinate (x, h, m, i, b) is
// element x of head h at sequence row i*st + m.  Box: 64 columns x 1 x 1 x box_rows reduced rows
// (128 for q, 256 for k).
bool make_map5(CUtensorMap* m, const void* ptr, int B, int S, int H, int st, int box_rows) {
  XEncodeFn fn = x_encode_fn();
  if (!fn) return false;
  const cuuint64_t row = (cuuint64_t)H * 128 * 2;
  const cuuint64_t dims[5] = {128, (cuuint64_t)H, (cuuint64_t)st, (cuuint64_t)(S / st), (cuuint64_t)B};
  const cuuint64_t strides[4] = {256, row, row * st, row * S};
  const cuuint32_t box[5] = {64, 1, 1, (cuuint32_t)box_rows, 1};
  const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int x_sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
  return n;
}

template <int ST, int NB>
ea_status launch_st(const void* q, const void* k, const int32_t* head_mode, const PatternDev& pd, int B, int S,
                    int H_q, int H_kv, float tau, int32_t* row_ptr, int32_t* cols, float* scores, void* workspace,
                    cudaStream_t st) {
  const XLayout L = x_layout(B, S, H_q, H_kv, ST, XT * ST / NB);
  CUtensorMap mq, mk;
  if (!make_map5(&mq, q, B, S, H_q, ST, XT) || !make_map5(&mk, k, B, S, H_kv, ST, XN)) return EA_ERR_CUDA;
  char* ws = static_cast<char*>(workspace);
  uint32_t* hdr = reinterpret_cast<uint32_t*>(ws);
  int* plan = reinterpret_cast<int*>(ws + L.plan);
  float* m_part = reinterpret_cast<float*>(ws + L.m_part);
  float* s_part = reinterpret_cast<float*>(ws + L.s_part);
  uint32_t* counts = reinterpret_cast<uint32_t*>(ws + L.counts);
  uint32_t* bitmap = reinterpret_cast<uint32_t*>(ws + L.bitmap);
  const float sl2 = (float)((double)pd.scale / ST * 1.4426950408889634);

  xattn_plan_kernel<<<1, 32, 0, st>>>(head_mode, pd, B, H_q, H_kv, hdr, plan);
  if (cudaGetLastError() != cudaSuccess) return EA_ERR_CUDA;
  auto kern = xattn_score_kernel<ST, NB>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kXSmemBytes) != cudaSuccess)
    return EA_ERR_CUDA;
  const long long max_work = (long long)B * H_q * L.n_rt;
  const int grid = (int)std::min<long long>(max_work, x_sm_count());
  const int inject = take_inject_stall() ? 1 : 0;
  kern<<<grid, kXThreads, kXSmemBytes, st>>>(mq, mk, H_q, H_kv, L.n_red, L.n_rt, sl2, plan, hdr, m_part, s_part,
                                             inject);
  if (cudaGetLastError() != cudaSuccess) return EA_ERR_CUDA;
  dim3 sgrid(L.n_qb, H_kv, B);
  xattn_select_kernel<ST, NB><<<sgrid, kSelThreads, 0, st>>>(head_mode, pd, H_q, H_kv, L.n_red, L.n_rt, tau, m_part,
                                                         s_part, counts, bitmap, scores);
  if (cudaGetLastError() != cudaSuccess) return EA_ERR_CUDA;
  const int n_rows = B * H_kv * L.n_qb;
  xattn_scan_kernel<<<1, 1024, 0, st>>>(counts, n_rows, row_ptr);
  if (cudaGetLastError() != cudaSuccess) return EA_ERR_CUDA;
  xattn_fill_kernel<<<cdiv(n_rows, 8), 256, 0, st>>>(bitmap, row_ptr, n_rows, L.words, cols);
  return cudaGetLastError() == cudaSuccess ? EA_OK : EA_ERR_CUDA;
}

}  // namespace

bool xattn_shape_ok(int S, int H_q, int H_kv, int stride, int block) {
  if (stride != 4 && stride != 8 && stride != 16) return false;
  if (block != 64 && block != kTile) return false;
  if (S % stride != 0 || cdiv(S, block) > kMaxQb) return false;
  return (long long)(H_q / H_kv) * (block / stride) <= kMaxSelRows;
}

size_t xattn_workspace_bytes(int B, int S, int H_q, int H_kv, int stride, int block) {
  return x_layout(B, S, H_q, H_kv, stride, block).total;
}

ea_status launch_xattn(const void* q, const void* k, const int32_t* head_mode, const PatternDev& pd, int B, int S,
                       int H_q, int H_kv, int stride, float tau, int32_t* row_ptr, int32_t* cols, float* scores,
                       void* workspace, cudaStream_t st) {
  const bool b64 = pd.block == 64;
#define EA_XATTN_CASE(STRIDE)                                                                                  \
  case STRIDE:                                                                                                 \
    return b64 ? launch_st<STRIDE, 2 * STRIDE>(q, k, head_mode, pd, B, S, H_q, H_kv, tau, row_ptr, cols, scores, \
                                               workspace, st)                                                  \
               : launch_st<STRIDE, STRIDE>(q, k, head_mode, pd, B, S, H_q, H_kv, tau, row_ptr, cols, scores,   \
                                           workspace, st);
  switch (stride) {
    EA_XATTN_CASE(4)
    EA_XATTN_CASE(8)
    EA_XATTN_CASE(16)
    default: return EA_ERR_UNSUPPORTED;
  }
#undef EA_XATTN_CASE
}

}  // namespace ea
