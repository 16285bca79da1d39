// ea_attn_tc.cuh — pieces shared by the two tensor-core attention kernels (ea_attn_tc.cu,
// block-128 layouts; ea_attn_tc64.cu, block-64 layouts): tile and shared-memory layout,
// barrier indices, bounded waits, work items and their run-time claiming, the MMA issue
// helpers and descriptors, the row softmax with its MUFU turns, and the host-side tensor
// maps.  The kernel bodies stay in their own files (their tile walks differ).
//
// The attention these kernels compute is stated in "Elastic Attention: Test-time Adaptive
// Sparsity Ratios for Efficient Transformers", section 2 "Hybrid Head Mechanism" and
// appendix D.1 "Sparse Inference" (one launch for every head kind).
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>
#include <mutex>
#include "ea_common.cuh"
#include "ea_sm100.cuh"

namespace ea {
namespace tc {

using namespace sm100;

constexpr int BM = 128, BN = 128, HD = 128;
constexpr int NKV = 3;                                 // K/V ring slots
constexpr int kThreads = 384;
constexpr uint32_t kTileBytes = BM * HD * 2;           // 32 KB per 128x128 bf16 tile
constexpr uint32_t kBoxBytes = kTileBytes / 2;         // one 64-column box
constexpr uint32_t OFF_Q = 0;
constexpr uint32_t OFF_P = 2 * kTileBytes;
constexpr uint32_t OFF_KV = 4 * kTileBytes;
constexpr uint32_t OFF_BAR = OFF_KV + NKV * kTileBytes;
enum : int {
  B_QFULL = 0, B_QEMPTY = 2, B_KVFULL = 4, B_KVEMPTY = B_KVFULL + NKV, B_SFULL = B_KVEMPTY + NKV,
  B_SFREE = B_SFULL + 2, B_PFULL = B_SFREE + 2, B_PVDONE = B_PFULL + 2, B_OFULL = B_PVDONE + 2,
  B_FIN = B_OFULL + 2, B_FIN2 = B_FIN + 1, B_TOK = B_FIN2 + 1, B_IFULL = B_TOK + 8, B_IEMPTY = B_IFULL + 2,
  B_NEVER = B_IEMPTY + 2, N_BAR = B_NEVER + 1
};
constexpr uint32_t OFF_TMEM = OFF_BAR + N_BAR * 8;
constexpr uint32_t OFF_ABORT = OFF_TMEM + 4;
constexpr uint32_t OFF_IRING = OFF_ABORT + 4;          // 2 claimed items, kItemWords ints each
constexpr int kItemWords = 12;
constexpr uint32_t kSmemBytes = OFF_IRING + 2 * kItemWords * 4 + 1024;  // + slack to align the base to 1024
// Roles that read every claimed item: Q K^T issuer, P V issuer and the 8 softmax warps.
constexpr uint32_t kItemReaders = 10;
static_assert(kSmemBytes <= 232448, "shared memory beyond the 227 KB a CTA may use");
constexpr uint32_t kTmemCols = 512;
__device__ __forceinline__ uint32_t col_s(int s) { return 128u * s; }        // S_s (and P_s) columns
__device__ __forceinline__ uint32_t col_o(int s) { return 256u + 128u * s; } // O_s columns
constexpr uint32_t IDESC_QK = idesc_bf16(BM, BN, false);
constexpr uint32_t IDESC_PV = idesc_bf16(BM, HD, true);
constexpr unsigned long long kWaitLimitNs = 2000000000ull;  // 2 s
constexpr float kRescaleLog2 = 8.0f;

// Register split: the launch gives 384 x 168 = 64512 registers; warpgroup 0 (producer,
// MMA, two idle warps) drops to 88 and the two softmax warpgroups rise to 208:
// 128 x 88 + 256 x 208 = 64512.
constexpr int kRegsCtl = 88, kRegsSoftmax = 208;
static_assert(128 * kRegsCtl + 256 * kRegsSoftmax <= kThreads * 168, "register split exceeds the launch");

struct Ctx {
  uint32_t bar0;                 // shared address of barrier 0
  volatile int* abort_flag;
  uint32_t* status;
  __device__ uint32_t bar(int i) const { return bar0 + 8u * i; }
};

__device__ __forceinline__ bool wait_slow(const Ctx& c, uint32_t bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (*c.abort_flag) return false;
    if (globaltimer_ns() - t0 > kWaitLimitNs) {
      *c.abort_flag = 1;
      atomicOr(c.status, kStatusTimeout);
      return false;
    }
  }
  return true;
}
__device__ __forceinline__ bool wait(const Ctx& c, uint32_t bar, uint32_t parity) {
  return mbar_try_wait(bar, parity) || wait_slow(c, bar, parity);
}
// Drain wait: also after an abort, wait (bounded) for this CTA's own copies and MMAs.
__device__ __forceinline__ void wait_drain(const Ctx& c, uint32_t bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > kWaitLimitNs) {
      atomicOr(c.status, kStatusTimeout);
      return;
    }
  }
}

struct Item {
  int b, h, t, T, pr, kind, n, sink_end, win_lo;   // t: query tile of this call, T: of the sequence
  long long csr_beg;
  bool two;
};

// Work items are claimed at run time: the producer takes the next index of the cost-sorted
// list (longest first) from a counter in the workspace whenever its CTA can start another
// item, decodes it (load_item: the item word, the head's routed kind, its live-tile range)
// and passes the decoded item to the other roles through a 2-entry ring in shared memory,
// so that they start the item without global loads of their own; index -1 ends the list.
// Greedy longest-first claiming keeps the CTAs' finishing times close.
__device__ __forceinline__ void put_item(volatile int* e, int idx, const Item& I) {
  e[0] = idx; e[1] = I.b; e[2] = I.h; e[3] = I.t; e[4] = I.T; e[5] = I.pr; e[6] = I.kind; e[7] = I.n;
  e[8] = I.sink_end; e[9] = I.win_lo; e[10] = (int)I.csr_beg; e[11] = (int)(I.csr_beg >> 32) * 2 + (I.two ? 1 : 0);
}
__device__ __forceinline__ int get_item(const volatile int* e, Item& I) {
  I.b = e[1]; I.h = e[2]; I.t = e[3]; I.T = e[4]; I.pr = e[5]; I.kind = e[6]; I.n = e[7];
  I.sink_end = e[8]; I.win_lo = e[9];
  const int hi = e[11];
  I.two = (hi & 1) != 0;
  I.csr_beg = (long long)(unsigned)e[10] | ((long long)(hi >> 1) << 32);
  return e[0];
}
struct ItemRing {
  volatile int* slot;   // 2 entries of kItemWords ints
  int k;                // items read so far
  // Next item for a reader role (index -1: done or aborted).  `arrive` is true for the one
  // thread of the role that signals the entry as read.
  __device__ int next(const Ctx& c, bool arrive, Item& I) {
    const int e = k & 1;
    const bool ok = wait(c, c.bar(B_IFULL + e), (k >> 1) & 1);
    const int idx = ok ? get_item(slot + e * kItemWords, I) : -1;
    if (ok && arrive) mbar_arrive(c.bar(B_IEMPTY + e));
    ++k;
    return idx;
  }
  // The index alone, for a ring whose producer publishes indices before decoding them (the
  // block-64 kernel: there every role walks the item's layout rows itself, in parallel).
  __device__ int next_idx(const Ctx& c, bool arrive) {
    const int e = k & 1;
    const bool ok = wait(c, c.bar(B_IFULL + e), (k >> 1) & 1);
    const int idx = ok ? slot[e * kItemWords] : -1;
    if (ok && arrive) mbar_arrive(c.bar(B_IEMPTY + e));
    ++k;
    return idx;
  }
};

// kBlock64: the block-64 kernel's items (block-sparse heads walk the union of two CSR rows;
// their live-tile count is read from the schedule's cost pass, `cost`, instead of walking
// the rows once more).
template <bool kBlock64 = false>
__device__ __forceinline__ Item load_item(const int4* items, int idx, const PatternDev& p,
                                          const int32_t* head_mode, int H_kv, int G,
                                          const int* cost = nullptr) {
  const int4 w = items[idx];
  Item I;
  I.b = w.x; I.h = w.y; I.t = w.z; I.pr = w.w;
  I.T = I.t + p.q_tile0;
  I.kind = head_kind(p, head_mode, H_kv, I.b, I.h);
  I.two = 2 * I.pr + 1 < G;
  I.sink_end = I.win_lo = 0;
  I.csr_beg = 0;
  if (is_streaming(I.kind)) {
    stream_ranges(p, I.kind, I.T, I.sink_end, I.win_lo);
    I.n = I.sink_end + max(0, I.T - I.win_lo + 1);
  } else if (kBlock64 && bs64_kind(p, I.kind)) {
    I.n = cost[((size_t)I.b * H_kv + I.h) * p.n_qt + I.t];
  } else if (I.kind == EA_BLOCK_SPARSE) {
    long long a, e;
    csr_row(p, H_kv, I.b, I.h, I.T, a, e);
    I.csr_beg = a;
    I.n = (int)(e - a);
  } else {
    I.n = I.T + 1;
  }
  return I;
}

__device__ __forceinline__ uint64_t qk_desc(uint32_t tile, int kk) {
  // K-major operand: rows of 128 bytes, 8-row swizzle atoms 1024 bytes apart (SBO);
  // K step kk of 16 elements = +32 bytes inside a 64-column box, boxes 16 KB apart.
  return sdesc_sw128(tile + (uint32_t)(kk >> 2) * kBoxBytes + (uint32_t)(kk & 3) * 32u, 16u, 1024u);
}
__device__ __forceinline__ uint64_t v_desc(uint32_t tile, int kk) {
  // MN-major operand (N = head dim, contiguous): 64-column boxes 16 KB apart (LBO),
  // 8-key groups 1024 bytes apart (SBO); K step kk of 16 keys = +2048 bytes.
  return sdesc_sw128(tile + (uint32_t)kk * 2048u, kBoxBytes, 1024u);
}

// S_s = Q_s K^T for the key tile at kt, once the softmax has loaded the previous S_s.  After
// the item's last key tile (last), Q_s is released once the product has read it.
__device__ __forceinline__ bool issue_qk(const Ctx& c, uint32_t tmem, uint32_t base, int s, uint32_t kt,
                                         int& s_cnt, bool last) {
  if (s_cnt > 0 && !wait(c, c.bar(B_SFREE + s), (s_cnt - 1) & 1)) return false;
  fence_after_sync();
  const uint32_t qt = base + OFF_Q + s * kTileBytes;
#pragma unroll
  for (int kk = 0; kk < HD / 16; ++kk)
    mma_ss(tmem + col_s(s), qk_desc(qt, kk), qk_desc(kt, kk), IDESC_QK, kk > 0 ? 1u : 0u);
  commit(c.bar(B_SFULL + s));
  if (last) commit(c.bar(B_QEMPTY + s));
  ++s_cnt;
  return true;
}

// O_s (+)= P_s V for the V tile at vt, once the softmax has written P_s.
__device__ __forceinline__ bool issue_pv(const Ctx& c, uint32_t tmem, uint32_t base, int s, uint32_t vt,
                                         bool accumulate, bool last, int& p_cnt) {
  if (!wait(c, c.bar(B_PFULL + s), p_cnt & 1)) return false;
  ++p_cnt;
  fence_after_sync();
  const uint32_t pt = base + OFF_P + s * kTileBytes;
#pragma unroll
  for (int kk = 0; kk < BN / 16; ++kk)
    mma_ss(tmem + col_o(s), qk_desc(pt, kk), v_desc(vt, kk), IDESC_PV, (accumulate || kk > 0) ? 1u : 0u);
  commit(c.bar(B_PVDONE + s));
  if (last) commit(c.bar(B_OFULL + s));
  return true;
}

// Share of the exponentials taken on the FMA pipe instead of the MUFU unit: one key
// pair in EA_POLY_EVERY (0: none).  The two softmax warps of an SM sub-partition share
// its MUFU unit, which each keeps busy for most of a tile.
#ifndef EA_POLY_EVERY
#define EA_POLY_EVERY 0
#endif
constexpr int kPolyEvery = EA_POLY_EVERY;

// 2^t for a pair of arguments on the FMA/ALU pipes: t = n + f with n the nearest integer
// (added to and subtracted from 1.5 * 2^23) and f in [-1/2, 1/2]; 2^f from the degree-3
// polynomial interpolating it at the four Chebyshev nodes of [-1/2, 1/2] (coefficients
// computed for this kernel; max relative error 1.0e-4); 2^n added into the exponent
// bits.  Arguments are clamped below at -126 (the result is then 2^-126, not 0).
__device__ __forceinline__ void ex2_pair_fma(uint64_t t2, float& r0, float& r1) {
  constexpr float kMagic = 12582912.0f;                  // 1.5 * 2^23, bits 0x4B400000
  constexpr float c0 = 0.99992454052f, c1 = 0.69313675165f, c2 = 0.24263948202f, c3 = 0.05583828315f;
  float a0, a1;
  f2_unpack(t2, a0, a1);
  const uint64_t t = f2_pack(fmaxf(a0, -126.f), fmaxf(a1, -126.f));
  const uint64_t j = f2_add(t, f2_pack(kMagic, kMagic));
  const uint64_t n = f2_add(j, f2_pack(-kMagic, -kMagic));
  const uint64_t fr = f2_fma(n, f2_pack(-1.f, -1.f), t);
  uint64_t q = f2_fma(f2_pack(c3, c3), fr, f2_pack(c2, c2));
  q = f2_fma(q, fr, f2_pack(c1, c1));
  q = f2_fma(q, fr, f2_pack(c0, c0));
  float q0, q1, j0, j1;
  f2_unpack(q, q0, q1);
  f2_unpack(j, j0, j1);
  r0 = __uint_as_float(__float_as_uint(q0) + ((__float_as_uint(j0) - 0x4B400000u) << 23));
  r1 = __uint_as_float(__float_as_uint(q1) + ((__float_as_uint(j1) - 0x4B400000u) << 23));
}

// One 128-key tile of one query row: running max (raised only past kRescaleLog2),
// row sum, and P = exp2(scale*log2e*s - max) as bf16 pairs in pk (pk[j] holds keys
// 2j, 2j+1).  kMode 0: every key live; 1: causal rule; 2: streaming rule; 3: causal rule
// within the enabled 64-key halves (block-64 kinds; sink_lim holds the half bits).  The
// exponentials run inside this warp's MUFU turn (tok).  Returns the factor O must be
// multiplied by (1 when the max was not raised).
template <int kMode, typename Tok>
__device__ __forceinline__ float softmax_tile(const float (&x)[BN], int lim, int sink_lim, int win_lim,
                                              float scale_log2, float& m_ref, float& l, uint32_t (&pk)[BN / 2],
                                              Tok& tok) {
  auto live = [&](int e) {
    if (kMode == 0) return true;
    if (kMode == 1) return e <= lim;
    if (kMode == 3) return e <= lim && ((sink_lim >> (e >> 6)) & 1) != 0;   // sink_lim: key-half bits
    return e <= lim && (e < sink_lim || e > win_lim);
  };
  auto xm = [&](int e) { return live(e) ? x[e] : -INFINITY; };
  // Row max as 8 independent 3-input chains over 16 columns each, then a short tree.
  float m8[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    m8[c] = xm(16 * c);
#pragma unroll
    for (int e = 1; e + 1 < 16; e += 2) m8[c] = fmax3(m8[c], xm(16 * c + e), xm(16 * c + e + 1));
    m8[c] = fmaxf(m8[c], xm(16 * c + 15));
  }
  const float mt = fmaxf(fmax3(m8[0], m8[1], m8[2]), fmax3(fmax3(m8[3], m8[4], m8[5]), m8[6], m8[7]));
  const float mts = mt * scale_log2;
  float f = 1.f;
  if (mts > m_ref + kRescaleLog2) {
    f = ex2(m_ref - mts);  // 0 while m_ref is still -inf
    l *= f;
    m_ref = mts;
  }
  // The exponentials start once this warp holds its sub-partition's MUFU turn; `sub` takes
  // a zero that only exists after the wait, so no exponential is scheduled before it.
  const float sub = ((m_ref == -INFINITY) ? 0.f : m_ref) + tok.acquire();
  const uint64_t scale2 = f2_pack(scale_log2, scale_log2), nsub2 = f2_pack(-sub, -sub);
  uint64_t l2 = f2_pack(0.f, 0.f);
#pragma unroll
  for (int e = 0; e < BN; e += 2) {
    const uint64_t t2 = f2_fma(f2_pack(x[e], x[e + 1]), scale2, nsub2);
    float p0, p1;
    if (kPolyEvery > 0 && (e / 2) % (kPolyEvery > 0 ? kPolyEvery : 1) == kPolyEvery - 1) {
      float e0, e1;
      ex2_pair_fma(t2, e0, e1);
      p0 = live(e) ? e0 : 0.f;
      p1 = live(e + 1) ? e1 : 0.f;
    } else {   // dead keys skip the MUFU (a whole warp past the diagonal skips it)
      float t0, t1;
      f2_unpack(t2, t0, t1);
      p0 = live(e) ? ex2(t0) : 0.f;
      p1 = live(e + 1) ? ex2(t1) : 0.f;
    }
    l2 = f2_add(l2, f2_pack(p0, p1));
    pk[e / 2] = pack_bf16x2(p0, p1);
  }
  float la, lb;
  f2_unpack(l2, la, lb);
  l += la + lb;
  tok.release(l);   // after the last exponential (the row sum depends on all of them)
  return f;
}

// softmax_tile for the block-64 kinds' tiles (kMode 3 mostly): the same results, with the
// masks applied per 32-key chunk with a decision that is the same for the whole
// warp: a chunk dead for every lane is skipped (no exponentials), one live for every lane
// runs without per-key tests, and only a mixed chunk tests each key (it computes every
// exponential and selects, so the MUFU stays pipelined; per-key branches around the
// exponentials would serialise them).  The exponentials run inside this warp's MUFU turn
// (tok).  Returns the factor O must be multiplied by (1 when the max was not raised).
template <int kMode, typename Tok>
__device__ __forceinline__ float softmax_tile_chunked(const float (&x)[BN], int lim, int sink_lim, int win_lim,
                                              float scale_log2, float& m_ref, float& l, uint32_t (&pk)[BN / 2],
                                              Tok& tok) {
  auto live = [&](int e) {
    if (kMode == 0) return true;
    if (kMode == 1) return e <= lim;
    if (kMode == 3) return e <= lim && ((sink_lim >> (e >> 6)) & 1) != 0;   // sink_lim: key-half bits
    return e <= lim && (e < sink_lim || e > win_lim);
  };
  // Chunk classes (0 dead, 1 live, 2 mixed) from the warp's extremes of the per-lane limits.
  int cls[4] = {1, 1, 1, 1};
  if (kMode != 0) {
    const int lo = __reduce_min_sync(0xffffffffu, lim), hi = __reduce_max_sync(0xffffffffu, lim);
    int wlo = 0, whi = 0;
    if (kMode == 2) {
      wlo = __reduce_min_sync(0xffffffffu, win_lim);
      whi = __reduce_max_sync(0xffffffffu, win_lim);
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int a = 32 * c, b = a + 31;
      int k = a > hi ? 0 : (b <= lo ? 1 : 2);                     // causal part
      if (kMode == 3 && ((sink_lim >> (a >> 6)) & 1) == 0) k = 0;  // disabled 64-key half
      if (kMode == 2 && k != 0) {
        if (a >= sink_lim && b <= wlo) k = 0;                      // between sinks and window, every lane
        else if (!(b < sink_lim || a > whi)) k = 2;                // sink/window edge inside the chunk
      }
      cls[c] = k;
    }
  }
  // Row max: per chunk two 3-input chains of 16 columns.
  float mc[4];
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    float m0 = -INFINITY, m1 = -INFINITY;
    if (cls[c] == 1) {
#pragma unroll
      for (int e = 0; e < 16; e += 2) {
        m0 = fmax3(m0, x[32 * c + e], x[32 * c + e + 1]);
        m1 = fmax3(m1, x[32 * c + 16 + e], x[32 * c + 16 + e + 1]);
      }
    } else if (cls[c] == 2) {
      auto xm = [&](int e) { return live(e) ? x[e] : -INFINITY; };
#pragma unroll
      for (int e = 0; e < 16; e += 2) {
        m0 = fmax3(m0, xm(32 * c + e), xm(32 * c + e + 1));
        m1 = fmax3(m1, xm(32 * c + 16 + e), xm(32 * c + 16 + e + 1));
      }
    }
    mc[c] = fmaxf(m0, m1);
  }
  const float mt = fmaxf(fmaxf(mc[0], mc[1]), fmaxf(mc[2], mc[3]));
  const float mts = mt * scale_log2;
  float f = 1.f;
  if (mts > m_ref + kRescaleLog2) {
    f = ex2(m_ref - mts);  // 0 while m_ref is still -inf
    l *= f;
    m_ref = mts;
  }
  // The exponentials start once this warp holds its sub-partition's MUFU turn; `sub` takes
  // a zero that only exists after the wait, so no exponential is scheduled before it.
  const float sub = ((m_ref == -INFINITY) ? 0.f : m_ref) + tok.acquire();
  const uint64_t scale2 = f2_pack(scale_log2, scale_log2), nsub2 = f2_pack(-sub, -sub);
  uint64_t l2 = f2_pack(0.f, 0.f);
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    if (cls[c] == 0) {
#pragma unroll
      for (int e = 32 * c; e < 32 * c + 32; e += 2) pk[e / 2] = 0u;
    } else if (cls[c] == 1) {
#pragma unroll
      for (int e = 32 * c; e < 32 * c + 32; e += 2) {
        const uint64_t t2 = f2_fma(f2_pack(x[e], x[e + 1]), scale2, nsub2);
        float p0, p1;
        if (kPolyEvery > 0 && (e / 2) % (kPolyEvery > 0 ? kPolyEvery : 1) == kPolyEvery - 1) {
          ex2_pair_fma(t2, p0, p1);
        } else {
          float t0, t1;
          f2_unpack(t2, t0, t1);
          p0 = ex2(t0);
          p1 = ex2(t1);
        }
        l2 = f2_add(l2, f2_pack(p0, p1));
        pk[e / 2] = pack_bf16x2(p0, p1);
      }
    } else {
#pragma unroll
      for (int e = 32 * c; e < 32 * c + 32; e += 2) {
        float t0, t1;
        f2_unpack(f2_fma(f2_pack(x[e], x[e + 1]), scale2, nsub2), t0, t1);
        const float e0 = ex2(t0), e1 = ex2(t1);
        const float p0 = live(e) ? e0 : 0.f, p1 = live(e + 1) ? e1 : 0.f;
        l2 = f2_add(l2, f2_pack(p0, p1));
        pk[e / 2] = pack_bf16x2(p0, p1);
      }
    }
  }
  float la, lb;
  f2_unpack(l2, la, lb);
  l += la + lb;
  tok.release(l);   // after the last exponential (the row sum depends on all of them)
  return f;
}

// Row `row` of P into the K-major, 128-byte-swizzled tile at p_tile: keys 64b..64b+63
// in box b, 16-byte chunk c of a row at chunk position c ^ (row % 8).
__device__ __forceinline__ void store_p_row(uint32_t p_tile, int row, const uint32_t (&pk)[BN / 2]) {
#pragma unroll
  for (int bx = 0; bx < 2; ++bx) {
#pragma unroll
    for (int ch = 0; ch < 8; ++ch) {
      const uint32_t addr = p_tile + bx * kBoxBytes + (uint32_t)row * 128u + (uint32_t)((ch ^ (row & 7)) << 4);
      const int j = 32 * bx + 4 * ch;
      asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(pk[j]), "r"(pk[j + 1]),
                   "r"(pk[j + 2]), "r"(pk[j + 3])
                   : "memory");
    }
  }
}

// MUFU turns of the two softmax warps that share an SM sub-partition (slot 0 and slot 1 of
// TMEM lane quadrant q): their exponential phases alternate, so each warp's loads, row max
// and P stores overlap the other's exponentials instead of both contending for the MUFU unit
// at once and leaving it idle together.  Slot 0 goes first; turn k of slot 0 waits for turn
// k-1 of slot 1, turn k of slot 1 for turn k of slot 0 (bounded waits, so a warp is never
// more than one phase ahead).  Items with a single query head take no turns.
struct MufuTurn {
  const Ctx* c;
  uint32_t mine, theirs;   // barrier this warp arrives on / waits on
  int slot, n;             // turns taken so far
  bool on, ok;
  __device__ float acquire() {
    if (on && (slot == 1 || n > 0)) ok = wait(*c, theirs, (slot == 1 ? n : n - 1) & 1) && ok;
    float z;
    asm volatile("mov.b32 %0, 0;" : "=f"(z) :: "memory");
    return z;
  }
  __device__ void release(float dep) {
    if (!on) return;
    asm volatile("" ::"f"(dep) : "memory");
    mbar_arrive(mine);
    ++n;
  }
};

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// [B, S, H, 128] bf16 viewed as 4-D (d, H, S, B); box = 64 columns x 1 head x 128 rows.
inline bool make_map(CUtensorMap* m, const void* ptr, int B, int S, int H) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[4] = {(cuuint64_t)HD, (cuuint64_t)H, (cuuint64_t)S, (cuuint64_t)B};
  const cuuint64_t strides[3] = {(cuuint64_t)HD * 2, (cuuint64_t)H * HD * 2, (cuuint64_t)S * H * HD * 2};
  const cuuint32_t box[4] = {64, 1, (cuuint32_t)BM, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

inline int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
  return n;
}


}  // namespace tc
}  // namespace ea
