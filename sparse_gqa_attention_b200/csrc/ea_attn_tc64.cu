// ea_attn_tc64.cu — the hybrid-head attention kernel for block-64 layouts (the pages'
// block edge: "Elastic Attention: Test-time Adaptive Sparsity Ratios for Efficient
// Transformers", appendix D.1 "Sparse Inference", block size 64).
// Same design and pipeline as ea_attn_tc.cu (read its header for the warp roles, TMEM and
// shared-memory layout, the MUFU turns, run-time item claims and bounded waits; the shared
// pieces are in ea_attn_tc.cuh); the differences are the tile walk and the masking.
// Tiles stay 128 x 128; each holds 2 x 2 blocks of 64:
//   block-sparse heads   the live key tiles of query tile t are the union of the key
//                        blocks listed for query blocks 2t and 2t+1 (block kb lies in tile
//                        kb/2); each tile carries the 2x2 map of its live blocks;
//   streaming-block heads sink blocks kb < ceil(n_sink/64) and local blocks
//                        qb - kb < ceil(window/64);
// every role walks the same tile sequence; on a tile that is not fully live (or on the
// diagonal) the softmax applies the causal rule within the 64-key halves its query
// half may read.  It is a separate kernel (not a template parameter of the block-128
// one) so that the block-128 kernel keeps its measured code.
#include <atomic>
#include "ea_attn_tc.cuh"
#include "ea_internal.h"

namespace ea {

namespace {

using namespace tc;

// Sequential walk over an item's live key tiles: the tile index (-1: nothing live) and,
// for block-64 block-sparse heads, the 2x2 map of its live blocks (0xF otherwise).
struct Walk {
  Bs64 w;
  int jj;
  __device__ __forceinline__ int next(const PatternDev& p, const Item& I, uint32_t& map) {
    map = 0xFu;
    int c;
    if (bs64_kind(p, I.kind)) {
      c = bs64_next(p, w, map);
      if (c > I.T) c = -1;   // a block above the diagonal (malformed layout): skipped
    } else {
      c = live_tile(p, I.kind, I.T, jj, I.sink_end, I.win_lo, I.csr_beg);
    }
    ++jj;
    return c;
  }
};
__device__ __forceinline__ Walk start_walk(const PatternDev& p, const Item& I, int H_kv) {
  Walk k;
  k.jj = 0;
  k.w.a0 = k.w.e0 = k.w.a1 = k.w.e1 = 0;
  if (bs64_kind(p, I.kind)) bs64_rows(p, H_kv, I.b, I.h, I.T, k.w);
  return k;
}

__global__ void __launch_bounds__(kThreads, 1)
hybrid_attn_tc64_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, __nv_bfloat16* __restrict__ o,
                      const int32_t* __restrict__ head_mode, const PatternDev p, int S, int H_q, int H_kv,
                      const int4* __restrict__ items, uint32_t* __restrict__ hdr, int inject_stall,
                      const int* __restrict__ cost) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int G = H_q / H_kv;
  Ctx c;
  c.bar0 = base + OFF_BAR;
  c.abort_flag = reinterpret_cast<volatile int*>(gbase + OFF_ABORT);
  c.status = hdr + kWsStatus / 4;
  const int n_items = (int)hdr[kWsNItems / 4];

  if (threadIdx.x == 0) {
    tma_prefetch_map(&tm_q);
    tma_prefetch_map(&tm_k);
    tma_prefetch_map(&tm_v);
    for (int i = 0; i < N_BAR; ++i) {
      const bool softmax_arrive = (i >= B_SFREE && i < B_SFREE + 2) || (i >= B_PFULL && i < B_PFULL + 2);
      const bool token = i >= B_TOK && i < B_TOK + 8;   // one softmax warp arrives
      const bool item_read = i >= B_IEMPTY && i < B_IEMPTY + 2;
      mbar_init(c.bar(i), softmax_arrive ? 128u : token ? 32u : item_read ? kItemReaders : 1u);
    }
    *c.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(base + OFF_TMEM, kTmemCols);
    tmem_relinquish();
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(gbase + OFF_TMEM);
  if (warp < 4) regs_dec<kRegsCtl>();
  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int q_use[2] = {0, 0};
      int kv = 0;
      bool ok = true;
      // One K or V tile into the next ring slot.
      auto load_tile = [&](const CUtensorMap* map, int h, int ct, int b) -> bool {
        const int slot = kv % NKV;
        if (!wait(c, c.bar(B_KVEMPTY + slot), ((kv / NKV) & 1) ^ 1)) return false;
        const uint32_t dst = base + OFF_KV + slot * kTileBytes;
        mbar_expect_tx(c.bar(B_KVFULL + slot), kTileBytes);
        tma_load_4d(dst, map, c.bar(B_KVFULL + slot), 0, h, ct * BN, b);
        tma_load_4d(dst + kBoxBytes, map, c.bar(B_KVFULL + slot), 64, h, ct * BN, b);
        ++kv;
        return true;
      };
      volatile int* ring = reinterpret_cast<volatile int*>(gbase + OFF_IRING);
      for (int it = 0; ok; ++it) {
        // Claim the next item once the readers are done with this ring entry's last use.
        const int e = it & 1;
        ok = wait(c, c.bar(B_IEMPTY + e), ((it >> 1) & 1) ^ 1);
        if (!ok) break;
        int idx = (int)atomicAdd(hdr + kWsClaim / 4, 1u);
        if (idx >= n_items) idx = -1;
        ring[e * kItemWords] = idx;
        mbar_arrive(c.bar(B_IFULL + e));
        if (idx < 0) break;
        const Item I = load_item<true>(items, idx, p, head_mode, H_kv, G, cost);
        if (I.n == 0) continue;
#pragma unroll
        for (int s = 0; s < 2; ++s) {
          if (!ok || (s == 1 && !I.two)) continue;
          ok = wait(c, c.bar(B_QEMPTY + s), (q_use[s] & 1) ^ 1);
          if (!ok) continue;
          const int h_q = I.h * G + 2 * I.pr + s;
          const uint32_t dst = base + OFF_Q + s * kTileBytes;
          mbar_expect_tx(c.bar(B_QFULL + s), kTileBytes);
          tma_load_4d(dst, &tm_q, c.bar(B_QFULL + s), 0, h_q, I.t * BM, I.b);
          tma_load_4d(dst + kBoxBytes, &tm_q, c.bar(B_QFULL + s), 64, h_q, I.t * BM, I.b);
          ++q_use[s];
        }
        // Ring order = MMA order: K0, then per tile jj: K(jj+1), V(jj).  The K walk runs
        // one tile ahead of the V walk.
        Walk kw = start_walk(p, I, H_kv), vw = start_walk(p, I, H_kv);
        uint32_t map;
        for (int jj = 0; jj < I.n && ok; ++jj) {
          if (jj == 0) ok = load_tile(&tm_k, I.h, max(0, kw.next(p, I, map)), I.b);
          if (ok && jj + 1 < I.n) ok = load_tile(&tm_k, I.h, max(0, kw.next(p, I, map)), I.b);
          if (ok) ok = load_tile(&tm_v, I.h, max(0, vw.next(p, I, map)), I.b);
        }
      }
      // Drain: the last copy armed on every barrier has landed before the CTA exits.
      for (int st = 0; st < NKV; ++st) {
        const int uses = kv / NKV + (st < kv % NKV ? 1 : 0);
        if (uses > 0) wait_drain(c, c.bar(B_KVFULL + st), (uses - 1) & 1);
      }
#pragma unroll
      for (int s = 0; s < 2; ++s)
        if (q_use[s] > 0) wait_drain(c, c.bar(B_QFULL + s), (q_use[s] - 1) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ Q K^T issuer
    // Walks the ring in the producer's order; takes the K entries, skips the V entries.
    if (lane == 0) {
      int q_use[2] = {0, 0}, s_cnt[2] = {0, 0};
      int kv = 0;
      // Test hook for the timeout path: CTA 0 first waits on a barrier nothing arrives on.
      bool ok = !(inject_stall && blockIdx.x == 0) || wait(c, c.bar(B_NEVER), 0);
      // S of key tile jj (both slots); the ring slot is released once both products finish.
      auto qk_tile = [&](const Item& I, int jj) -> bool {
        const int slot = kv % NKV;
        if (!wait(c, c.bar(B_KVFULL + slot), (kv / NKV) & 1)) return false;
        const uint32_t kt = base + OFF_KV + slot * kTileBytes;
        const bool last = jj + 1 == I.n;
        if (!issue_qk(c, tmem, base, 0, kt, s_cnt[0], last)) return false;
        if (I.two && !issue_qk(c, tmem, base, 1, kt, s_cnt[1], last)) return false;
        commit(c.bar(B_KVEMPTY + slot));
        ++kv;
        return true;
      };
      ItemRing ir{reinterpret_cast<volatile int*>(gbase + OFF_IRING), 0};
      while (ok) {
        const int idx = ir.next_idx(c, true);
        if (idx < 0) break;
        const Item I = load_item<true>(items, idx, p, head_mode, H_kv, G, cost);
        if (I.n == 0) continue;
        ok = wait(c, c.bar(B_QFULL + 0), q_use[0] & 1);
        ++q_use[0];
        if (I.two) {
          ok = ok && wait(c, c.bar(B_QFULL + 1), q_use[1] & 1);
          ++q_use[1];
        }
        ok = ok && qk_tile(I, 0);
        for (int jj = 0; jj < I.n && ok; ++jj) {
          if (jj + 1 < I.n) ok = qk_tile(I, jj + 1);   // ring order: K(jj+1), then V(jj)
          ++kv;                                       // V(jj): the P V issuer's entry
        }
      }
      commit(c.bar(B_FIN));                       // every MMA issued here has completed
      wait_drain(c, c.bar(B_FIN), 0);
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------ P V issuer
    // Walks the ring in the producer's order; takes the V entries, skips the K entries.
    if (lane == 0) {
      int p_cnt[2] = {0, 0};
      int kv = 0;
      bool ok = true;
      ItemRing ir{reinterpret_cast<volatile int*>(gbase + OFF_IRING), 0};
      while (ok) {
        const int idx = ir.next_idx(c, true);
        if (idx < 0) break;
        const Item I = load_item<true>(items, idx, p, head_mode, H_kv, G, cost);
        if (I.n == 0) continue;
        ++kv;                                         // K(0)
        for (int jj = 0; jj < I.n && ok; ++jj) {
          if (jj + 1 < I.n) ++kv;                     // K(jj+1)
          const int slot = kv % NKV;
          ok = wait(c, c.bar(B_KVFULL + slot), (kv / NKV) & 1);
          if (!ok) break;
          const uint32_t vt = base + OFF_KV + slot * kTileBytes;
          const bool last = jj + 1 == I.n;
          ok = issue_pv(c, tmem, base, 0, vt, jj > 0, last, p_cnt[0]);
          if (ok && I.two) ok = issue_pv(c, tmem, base, 1, vt, jj > 0, last, p_cnt[1]);
          if (!ok) break;
          commit(c.bar(B_KVEMPTY + slot));
          ++kv;
        }
      }
      commit(c.bar(B_FIN2));
      wait_drain(c, c.bar(B_FIN2), 0);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax slots
    regs_inc<kRegsSoftmax>();
    const int s = (warp - 4) / 4;
    const int row = (warp % 4) * 32 + lane;
    const uint32_t lane_addr = tmem + ((uint32_t)((warp % 4) * 32) << 16);
    const uint32_t p_tile = base + OFF_P + s * kTileBytes;
    int s_cnt = 0, p_cnt = 0, o_cnt = 0;
    bool ok = true;
    MufuTurn turn;
    turn.c = &c;
    turn.slot = s;
    turn.n = 0;
    turn.mine = c.bar(B_TOK + 4 * s + warp % 4);
    turn.theirs = c.bar(B_TOK + 4 * (1 - s) + warp % 4);
    ItemRing ir{reinterpret_cast<volatile int*>(gbase + OFF_IRING), 0};
    while (ok) {
      const int idx = ir.next_idx(c, false);   // every lane reads the entry, then lane 0 releases it
      __syncwarp();
      if (lane == 0 && idx >= 0) mbar_arrive(c.bar(B_IEMPTY + ((ir.k - 1) & 1)));
      if (idx < 0) break;
      const Item I = load_item<true>(items, idx, p, head_mode, H_kv, G, cost);
      if (I.n == 0 || (s == 1 && !I.two)) continue;
      turn.on = I.two;
      turn.ok = true;
      const int i = I.T * BM + row;        // query position in the sequence
      const int i_out = I.t * BM + row;    // row of q and o in this call
      const int kind_el = I.kind == EA_STREAMING ? EA_STREAMING : EA_FULL;
      const bool blk64 = p.block == 64 && (I.kind == EA_BLOCK_SPARSE || I.kind == EA_STREAMING_BLOCKS);
      Walk walk = start_walk(p, I, H_kv);
      float m_ref = -INFINITY, l = 0.f;
      for (int jj = 0; jj < I.n; ++jj) {
        uint32_t map;
        const int ct = walk.next(p, I, map);
        ok = wait(c, c.bar(B_SFULL + s), s_cnt & 1);
        ok = __all_sync(0xffffffffu, ok);
        ++s_cnt;
        if (!ok) break;
        fence_after_sync();
        float x[BN];
        {
          uint32_t r[BN];
#pragma unroll
          for (int q4 = 0; q4 < BN / 32; ++q4) tmem_ld32(lane_addr + col_s(s) + 32 * q4, r + 32 * q4);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < BN; ++e) x[e] = __uint_as_float(r[e]);
        }
        fence_before_sync();
        mbar_arrive(c.bar(B_SFREE + s));   // S_s may be overwritten by the next Q K^T
        // Key j = 128*ct + e is live iff e <= lim (causal) and, for a streaming head,
        // e < sink_lim or e > win_lim.  Unmasked tiles skip the test.
        uint32_t pk[BN / 2];
        float f;
        if (ct < 0) {
          f = softmax_tile<1>(x, -1, 0, 0, p.scale_log2, m_ref, l, pk, turn);
        } else if (blk64) {   // 64x64 blocks: the key halves this warp's query half may read
          const int hb = (int)half_bits(p, I.kind, I.T, ct, row >> 6, map);
          if (hb == 3 && ct < I.T)
            f = softmax_tile<0>(x, 0, 0, 0, p.scale_log2, m_ref, l, pk, turn);
          else
            f = softmax_tile_chunked<3>(x, i - ct * BN, hb, 0, p.scale_log2, m_ref, l, pk, turn);
        } else if (tile_needs_mask(p, I.kind, I.T, ct)) {
          const int lim = i - ct * BN;
          if (kind_el == EA_STREAMING)
            f = softmax_tile<2>(x, lim, p.n_sink - ct * BN, lim - p.window, p.scale_log2, m_ref, l, pk, turn);
          else
            f = softmax_tile<1>(x, lim, 0, 0, p.scale_log2, m_ref, l, pk, turn);
        } else {
          f = softmax_tile<0>(x, 0, 0, 0, p.scale_log2, m_ref, l, pk, turn);
        }
        if (!__all_sync(0xffffffffu, turn.ok)) {
          ok = false;
          break;
        }
        // The previous P_s V product must be done before P_s is rewritten and before O_s
        // (which it accumulates into) is rescaled.
        if (p_cnt > 0) {
          ok = wait(c, c.bar(B_PVDONE + s), (p_cnt - 1) & 1);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          fence_after_sync();
        }
        if (jj > 0 && __any_sync(0xffffffffu, f != 1.f)) {   // O (complete up to tile jj-1) *= f
#pragma unroll 1
          for (int q4 = 0; q4 < HD / 32; ++q4) {
            uint32_t r[32];
            tmem_ld32(lane_addr + col_o(s) + 32 * q4, r);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * f);
            tmem_st32(lane_addr + col_o(s) + 32 * q4, r);
          }
          tmem_st_wait();
        }
        store_p_row(p_tile, row, pk);
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // P visible to the tensor core
        fence_before_sync();
        mbar_arrive(c.bar(B_PFULL + s));
        ++p_cnt;
      }
      if (!ok) break;
      ok = wait(c, c.bar(B_OFULL + s), o_cnt & 1);
      ok = __all_sync(0xffffffffu, ok);
      ++o_cnt;
      if (!ok) break;
      fence_after_sync();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      const int h_q = I.h * G + 2 * I.pr + s;
      __nv_bfloat16* orow = o + (((size_t)I.b * S + i_out) * H_q + h_q) * HD;
#pragma unroll
      for (int q4 = 0; q4 < HD / 32; ++q4) {
        uint32_t r[32];
        tmem_ld32(lane_addr + col_o(s) + 32 * q4, r);
        tmem_ld_wait();
        if (i_out < S) {
#pragma unroll
          for (int e = 0; e < 32; e += 8) {
            uint4 w;
            w.x = pack_bf16x2(__uint_as_float(r[e]) * inv, __uint_as_float(r[e + 1]) * inv);
            w.y = pack_bf16x2(__uint_as_float(r[e + 2]) * inv, __uint_as_float(r[e + 3]) * inv);
            w.z = pack_bf16x2(__uint_as_float(r[e + 4]) * inv, __uint_as_float(r[e + 5]) * inv);
            w.w = pack_bf16x2(__uint_as_float(r[e + 6]) * inv, __uint_as_float(r[e + 7]) * inv);
            *reinterpret_cast<uint4*>(orow + 32 * q4 + e) = w;
          }
        }
      }
      fence_before_sync();
    }
  }

  fence_before_sync();
  __syncthreads();
  if (threadIdx.x == 0) {   // the last CTA to finish rewinds the claim counter for the next launch
    __threadfence();
    if (atomicAdd(hdr + kWsDone / 4, 1u) == gridDim.x - 1) {
      atomicExch(hdr + kWsClaim / 4, 0u);
      atomicExch(hdr + kWsDone / 4, 0u);
    }
  }
  if (warp == 1) {
    __syncwarp();
    fence_after_sync();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

ea_status launch_attn_tc64(const void* q, const void* k, const void* v, void* o, const int32_t* head_mode,
                           const PatternDev& pat, int B, int S, int S_k, int H_q, int H_kv, void* workspace,
                           cudaStream_t st) {
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, q, B, S, H_q) || !make_map(&mk, k, B, S_k, H_kv) || !make_map(&mv, v, B, S_k, H_kv))
    return EA_ERR_CUDA;
  const long long n_items = (long long)B * H_kv * pat.n_qt * n_pairs(H_q, H_kv);
  const int grid = (int)std::min<long long>(n_items, sm_count());
  auto kern = hybrid_attn_tc64_kernel;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes) != cudaSuccess)
    return EA_ERR_CUDA;
  char* ws = static_cast<char*>(workspace);
  const size_t items_off = kWsHeader + ((size_t)B * 4 + 255) / 256 * 256;
  const int inject = take_inject_stall() ? 1 : 0;
  kern<<<grid, kThreads, kSmemBytes, st>>>(mq, mk, mv, static_cast<__nv_bfloat16*>(o), head_mode, pat, S, H_q,
                                           H_kv, reinterpret_cast<const int4*>(ws + items_off),
                                           reinterpret_cast<uint32_t*>(ws), inject,
                                           reinterpret_cast<const int*>(ws + attn_costs_offset(B, S, H_q, H_kv)));
  return cudaGetLastError() == cudaSuccess ? EA_OK : EA_ERR_CUDA;
}

}  // namespace ea

