// ea_common.cuh — device-side definitions shared by the schedule builder, the
// attention kernels and the sparsity counter.
//
// Live key tiles per head kind, for a 128-row query tile t (rows 128t..128t+127 of the
// sequence: t is the global tile index, so a prefill chunk starting at row q_offset
// uses t = q_offset/128 + local tile) and 128-key tiles c (keys 128c..128c+127); the
// element rules follow section 2
// "Hybrid Head Mechanism" and appendix D.1 "Sparse Inference" of "Elastic
// Attention: Test-time Adaptive Sparsity Ratios for Efficient Transformers":
//   FULL          tiles 0..t; only the diagonal tile t needs the causal mask.
//   STREAMING     sink tiles 0..ceil(n_sink/128)-1 (at most t), then window tiles
//                 floor(max(0, 128t - window + 1)/128)..t (not repeating sink tiles).
//                 Every enumerated tile holds at least one live pair.
//   BLOCK_SPARSE  block 128: the listed key blocks of CSR row (b*H_kv + h)*n_qb + t;
//                 the diagonal tile needs the causal mask.  Block 64: the union of
//                 the key tiles of CSR rows 2t and 2t+1 (key block kb lies in tile
//                 kb/2), each with a 2x2 map of its live 64x64 blocks.
//   STREAMING_BLOCKS sink blocks kb < sb = ceil(n_sink/block) and local blocks
//                 qb - kb < lb = ceil(window/block): sink tiles up to
//                 ceil(sb*block/128)-1 (at most t), then tiles from
//                 floor(max(0, q0 - lb + 1)*block/128) to t, q0 = 128t/block the
//                 tile's first query block.  Block 128: only the diagonal tile needs
//                 the causal mask; block 64: boundary tiles use the 2x2 block map.
#pragma once
#include <cstdint>
#include <cuda_runtime.h>
#include "../../include/ea.h"

namespace ea {

constexpr int kTile = 128;

// Workspace layout of the attention calls (bytes from the workspace base).
constexpr size_t kWsStatus = 0;        // uint32 sticky status bits
constexpr size_t kWsNItems = 4;        // uint32 items in the schedule
constexpr size_t kWsClaim = 8;         // uint32 next item to claim (attention launch)
constexpr size_t kWsDone = 12;         // uint32 CTAs of the attention launch that finished
constexpr size_t kWsLivePairs = 16;    // uint64
constexpr size_t kWsLiveTiles = 24;    // uint64
constexpr size_t kWsHeader = 256;
// then int32 sparse-head count per sample, padded to 256 bytes, then int4 items.

// Device status bits.
constexpr uint32_t kStatusTimeout = 1u << 0;
constexpr uint32_t kStatusBadLayout = 1u << 1;
constexpr uint32_t kStatusBadMode = 1u << 2;

struct PatternDev {
  int n_sink;
  int window;
  int block;
  int n_qt;                 // query tiles of this call: ceil(S_q / 128)
  int q_tile0;              // global index of the call's first query tile (q_offset / 128)
  int n_qb;                 // CSR rows per (b, h_kv): ceil(S_k / block)
  const int32_t* row_ptr;
  const int32_t* cols;
  long long nnz;
  float scale;              // softmax scale
  float scale_log2;         // softmax scale * log2(e)
  int8_t kind_dense[EA_MAX_KV_HEADS];
  int8_t kind_sparse[EA_MAX_KV_HEADS];
};

__host__ __device__ __forceinline__ int cdiv(int a, int b) { return (a + b - 1) / b; }

__device__ __forceinline__ int head_kind(const PatternDev& p, const int32_t* head_mode, int H_kv,
                                         int b, int h) {
  return head_mode[b * H_kv + h] != 0 ? p.kind_sparse[h] : p.kind_dense[h];
}

__device__ __forceinline__ bool is_streaming(int kind) { return kind == EA_STREAMING || kind == EA_STREAMING_BLOCKS; }

// Tile ranges of query tile t for the two streaming kinds: [0, sink_end) and [win_lo, t].
__device__ __forceinline__ void stream_ranges(const PatternDev& p, int kind, int t, int& sink_end, int& win_lo) {
  if (kind == EA_STREAMING_BLOCKS) {
    const int B = p.block, sb = cdiv(p.n_sink, B), lb = cdiv(p.window, B);
    sink_end = min(cdiv(sb * B, kTile), t + 1);
    const int q0 = t * (kTile / B);                       // the tile's first query block
    win_lo = max(max(0, q0 - lb + 1) * B / kTile, sink_end);
  } else {
    sink_end = min(cdiv(p.n_sink, kTile), t + 1);
    win_lo = max(max(0, t * kTile - p.window + 1) / kTile, sink_end);
  }
}

// CSR row [beg, end) of (b, h, global query tile t), clamped so a malformed row never
// reads outside bs_col.
__device__ __forceinline__ void csr_row(const PatternDev& p, int H_kv, int b, int h, int t,
                                        long long& beg, long long& end) {
  long long r = ((long long)b * H_kv + h) * p.n_qb + t;
  long long a = p.row_ptr[r], e = p.row_ptr[r + 1];
  a = max(0LL, min(a, p.nnz));
  e = max(a, min(e, p.nnz));
  beg = a;
  end = e;
}

// Block-sparse rows of a 128-row query tile at block 64: CSR rows 2t and 2t+1.
struct Bs64 {
  long long a0, e0, a1, e1;
};
__device__ __forceinline__ void bs64_rows(const PatternDev& p, int H_kv, int b, int h, int t, Bs64& w) {
  csr_row(p, H_kv, b, h, 2 * t, w.a0, w.e0);
  if (2 * t + 1 < p.n_qb) {
    csr_row(p, H_kv, b, h, 2 * t + 1, w.a1, w.e1);
  } else {
    w.a1 = w.e1 = 0;
  }
}
// Next key tile of the union of the two rows (ascending), with its 2x2 map: bit
// 2*qsub + ksub for query half qsub (row 2t+qsub) and key half ksub (block 2c+ksub).
// Returns -1 when both rows are done.  Every walker over the same rows visits the
// same sequence, so producer, MMA issuer, softmax and schedule stay in step.
__device__ __forceinline__ int bs64_next(const PatternDev& p, Bs64& w, uint32_t& map) {
  const int k0 = w.a0 < w.e0 ? p.cols[w.a0] : 0x7fffffff;
  const int k1 = w.a1 < w.e1 ? p.cols[w.a1] : 0x7fffffff;
  const int kmin = min(k0, k1);
  if (kmin == 0x7fffffff) return -1;
  const int c = kmin >> 1;
  map = 0;
  while (w.a0 < w.e0 && (p.cols[w.a0] >> 1) == c) {
    map |= 1u << (p.cols[w.a0] & 1);
    ++w.a0;
  }
  while (w.a1 < w.e1 && (p.cols[w.a1] >> 1) == c) {
    map |= 4u << (p.cols[w.a1] & 1);
    ++w.a1;
  }
  return c;
}

__device__ __forceinline__ bool bs64_kind(const PatternDev& p, int kind) {
  return kind == EA_BLOCK_SPARSE && p.block == 64;
}

// Number of live key tiles of query tile t.
__device__ __forceinline__ int n_live_tiles(const PatternDev& p, int kind, int H_kv, int b, int h, int t) {
  if (is_streaming(kind)) {
    int se, wl;
    stream_ranges(p, kind, t, se, wl);
    return se + max(0, t - wl + 1);
  }
  if (bs64_kind(p, kind)) {
    Bs64 w;
    bs64_rows(p, H_kv, b, h, t, w);
    uint32_t map;
    int n = 0;
    while (bs64_next(p, w, map) >= 0) ++n;
    return n;
  }
  if (kind == EA_BLOCK_SPARSE) {
    long long a, e;
    csr_row(p, H_kv, b, h, t, a, e);
    return (int)(e - a);
  }
  return t + 1;
}

// For block-64 kinds: the enabled key halves (bit ksub) of key tile c for the query
// half qsub of tile t, from the 2x2 map (block-sparse) or the streaming-block rule.
__device__ __forceinline__ uint32_t half_bits(const PatternDev& p, int kind, int t, int c, int qsub, uint32_t map) {
  if (kind == EA_BLOCK_SPARSE) return (map >> (2 * qsub)) & 3u;
  const int sb = cdiv(p.n_sink, 64), lb = cdiv(p.window, 64), q = 2 * t + qsub;
  uint32_t bits = 0;
#pragma unroll
  for (int ks = 0; ks < 2; ++ks) {
    const int kb = 2 * c + ks;
    if (kb <= q && (kb < sb || q - kb < lb)) bits |= 1u << ks;
  }
  return bits;
}

// Key tile index of the jj-th live tile (0 <= jj < n_live_tiles).  For block-sparse
// heads a listed column outside [0, t] (a malformed layout) maps to -1: skip it.
__device__ __forceinline__ int live_tile(const PatternDev& p, int kind, int t, int jj,
                                         int sink_end, int win_lo, long long csr_beg) {
  if (is_streaming(kind)) return jj < sink_end ? jj : win_lo + (jj - sink_end);
  if (kind == EA_BLOCK_SPARSE) {
    int c = p.cols[csr_beg + jj];
    return (c >= 0 && c <= t) ? c : -1;
  }
  return jj;
}

// True when some pair of (query tile t, key tile c) may be dead, so the element rule
// must run; false when every pair with a real query row is live.
__device__ __forceinline__ bool tile_needs_mask(const PatternDev& p, int kind, int t, int c) {
  if (c >= t) return true;                              // diagonal (causal) tile
  if (kind != EA_STREAMING) return false;
  if (c * kTile + kTile - 1 < p.n_sink) return false;   // all sink keys
  return (t * kTile + kTile - 1) - c * kTile >= p.window;
}

// Element rule: is key j live for query row i.
__device__ __forceinline__ bool key_live(const PatternDev& p, int kind, int i, int j) {
  if (j > i) return false;
  if (kind == EA_STREAMING) return j < p.n_sink || i - j < p.window;
  if (kind == EA_STREAMING_BLOCKS)
    return j / p.block < cdiv(p.n_sink, p.block) || i / p.block - j / p.block < cdiv(p.window, p.block);
  return true;  // FULL, and BLOCK_SPARSE inside a listed block
}

}  // namespace ea
