// ea_schedule.cu — device-side work list for the hybrid attention launch, and the
// sparsity counters.
//
// The routing metadata (head_mode plus the per-head patterns) is turned into the
// list of live work items on the device, with no host round trip, so that one
// attention launch serves every head kind ("Elastic Attention: Test-time Adaptive
// Sparsity Ratios for Efficient Transformers", appendix D.1 "Sparse Inference":
// one unified launch fed by the routing metadata; section 3 "Efficient
// Deployment").  A work item is (b, h_kv, query tile t, head pair): the pair is
// query heads 2p and 2p+1 of the KV group, which read the same key tiles.  Items
// are sorted by cost (live tiles x heads), longest first.
//
// The sparsity counters follow section 2 "Sparsity Ratio Computation": sparse
// heads per sample (Omega_MSR), live query-key pairs and live 128x128 tiles.
#include <cuda_runtime.h>
#include <cstdint>
#include "ea_common.cuh"
#include "ea_internal.h"

namespace ea {
namespace {

constexpr int kSchedThreads = 1024;
constexpr int kMaxBins = 8192;

__device__ __forceinline__ void decode_item(int x, int np, int n_qt, int H_kv, int& b, int& h, int& t, int& pr) {
  pr = x % np;
  int r = x / np;
  t = r % n_qt;
  r /= n_qt;
  h = r % H_kv;
  b = r / H_kv;
}

// One thread per (b, h_kv, query tile of the call): the tile's live key tiles, and the
// device checks of head_mode and of the tile's block-layout rows.
__global__ void __launch_bounds__(256)
tile_cost_kernel(const int32_t* __restrict__ head_mode, PatternDev p, int B, int H_kv, uint32_t* __restrict__ hdr,
                 int* __restrict__ cost) {
  const int x = blockIdx.x * blockDim.x + threadIdx.x;
  if (x >= B * H_kv * p.n_qt) return;
  const int tl = x % p.n_qt, bh = x / p.n_qt, h = bh % H_kv, b = bh / H_kv;
  const int t = tl + p.q_tile0;   // global query tile
  uint32_t bad = 0;
  const int m = head_mode[b * H_kv + h];
  if (m != 0 && m != 1) bad |= kStatusBadMode;
  const int kind = head_kind(p, head_mode, H_kv, b, h);
  if (kind == EA_BLOCK_SPARSE) {   // the tile's CSR rows (1 at block 128, 2 at 64)
    const int per = kTile / p.block;
    for (int u = 0; u < per; ++u) {
      const int qb = t * per + u;
      if (qb >= p.n_qb) break;
      const long long r = ((long long)b * H_kv + h) * p.n_qb + qb;
      const long long a0 = p.row_ptr[r], a1 = p.row_ptr[r + 1];
      if (a0 < 0 || a1 < a0 || a1 > p.nnz || a1 == a0) {
        bad |= kStatusBadLayout;
      } else {
        int prev = -1;
        for (long long e = a0; e < a1; ++e) {
          const int c = p.cols[e];
          if (c <= prev || c > qb) bad |= kStatusBadLayout;
          prev = c;
        }
        if (prev != qb) bad |= kStatusBadLayout;
      }
    }
  }
  cost[x] = n_live_tiles(p, kind, H_kv, b, h, t);
  if (bad) atomicOr(hdr + kWsStatus / 4, bad);
}

__device__ __forceinline__ int item_cost(const int* cost, int n_qt, int H_kv, int G, int b, int h, int tl, int pr,
                                         int n_bins) {
  const int heads = min(2, G - 2 * pr);
  return min(cost[(b * H_kv + h) * n_qt + tl] * heads, n_bins - 1);
}

__global__ void __launch_bounds__(kSchedThreads)
schedule_kernel(const int* __restrict__ cost, PatternDev p, int H_kv, int G, int np, int n_items, int n_bins,
                uint32_t* __restrict__ hdr, int4* __restrict__ items) {
  __shared__ int bins[kMaxBins];
  __shared__ int part[kSchedThreads];
  const int tid = threadIdx.x;
  for (int i = tid; i < n_bins; i += kSchedThreads) bins[i] = 0;
  __syncthreads();
  for (int x = tid; x < n_items; x += kSchedThreads) {
    int b, h, tl, pr;
    decode_item(x, np, p.n_qt, H_kv, b, h, tl, pr);
    atomicAdd(&bins[item_cost(cost, p.n_qt, H_kv, G, b, h, tl, pr, n_bins)], 1);
  }
  // (items store the local query tile; the attention kernels add q_tile0)
  __syncthreads();
  // Exclusive scan of the bins in descending cost order: bins[c] <- items costing more than c.
  const int chunk = (n_bins + kSchedThreads - 1) / kSchedThreads;
  const int q0 = tid * chunk;  // descending position q <-> bin n_bins - 1 - q
  int local = 0;
  for (int q = q0; q < min(q0 + chunk, n_bins); ++q) local += bins[n_bins - 1 - q];
  part[tid] = local;
  __syncthreads();
  for (int off = 1; off < kSchedThreads; off <<= 1) {  // Hillis-Steele inclusive scan
    const int v = tid >= off ? part[tid - off] : 0;
    __syncthreads();
    part[tid] += v;
    __syncthreads();
  }
  int run = part[tid] - local;
  for (int q = q0; q < min(q0 + chunk, n_bins); ++q) {
    const int c = n_bins - 1 - q;
    const int cnt = bins[c];
    bins[c] = run;
    run += cnt;
  }
  __syncthreads();
  for (int x = tid; x < n_items; x += kSchedThreads) {
    int b, h, tl, pr;
    decode_item(x, np, p.n_qt, H_kv, b, h, tl, pr);
    const int pos = atomicAdd(&bins[item_cost(cost, p.n_qt, H_kv, G, b, h, tl, pr, n_bins)], 1);
    items[pos] = make_int4(b, h, tl, pr);
  }
  if (tid == 0) {
    hdr[kWsNItems / 4] = (uint32_t)n_items;
    hdr[kWsClaim / 4] = 0u;   // the attention launch claims items from 0
    hdr[kWsDone / 4] = 0u;
  }
}

// grid (n_qt, H_kv, B), 128 threads: thread = query row of tile t.
__global__ void __launch_bounds__(kTile)
sparsity_kernel(const int32_t* __restrict__ head_mode, PatternDev p, int S, int H_kv, int G,
                unsigned long long* __restrict__ counters, int* __restrict__ sparse_heads) {
  const int t = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int i = t * kTile + threadIdx.x;
  const int kind = head_kind(p, head_mode, H_kv, b, h);
  long long cnt = 0;
  if (i < S) {
    if (kind == EA_STREAMING) {
      cnt = min(i + 1, p.window) + max(0, min(p.n_sink, i - p.window + 1));
    } else if (kind == EA_STREAMING_BLOCKS) {
      const int B = p.block, qb = i / B;
      const long long local_start = (long long)max(0, qb - cdiv(p.window, B) + 1) * B;
      cnt = (i - local_start + 1) + max(0LL, min((long long)cdiv(p.n_sink, B) * B, local_start));
    } else if (kind == EA_BLOCK_SPARSE) {
      const int B = p.block, qb = i / B;
      long long a, e;
      csr_row(p, H_kv, b, h, qb, a, e);
      int below = 0;
      bool diag = false;
      for (long long x = a; x < e; ++x) {
        const int c = p.cols[x];
        below += (c >= 0 && c < qb);
        diag |= (c == qb);
      }
      cnt = (long long)below * B + (diag ? (i - qb * B + 1) : 0);
    } else {
      cnt = i + 1;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
  __shared__ long long red[kTile / 32];
  if (threadIdx.x % 32 == 0) red[threadIdx.x / 32] = cnt;
  __syncthreads();
  if (threadIdx.x == 0) {
    long long s = 0;
    for (int w = 0; w < kTile / 32; ++w) s += red[w];
    atomicAdd(counters + 0, (unsigned long long)(s * G));
    atomicAdd(counters + 1, (unsigned long long)n_live_tiles(p, kind, H_kv, b, h, t) * G);
    if (t == 0 && head_mode[b * H_kv + h] != 0) atomicAdd(sparse_heads + b, 1);
  }
}

}  // namespace

int n_pairs(int H_q, int H_kv) { return (H_q / H_kv + 1) / 2; }

static size_t items_offset(int B) { return kWsHeader + ((size_t)B * 4 + 255) / 256 * 256; }

// Workspace: header | per-sample sparse-head counts | int4 work items | int32 tile costs.
static size_t costs_offset(int B, int S, int H_q, int H_kv) {
  const size_t n_items = (size_t)B * H_kv * cdiv(S, kTile) * n_pairs(H_q, H_kv);
  return items_offset(B) + n_items * sizeof(int4);
}

size_t attn_costs_offset(int B, int S, int H_q, int H_kv) { return costs_offset(B, S, H_q, H_kv); }

size_t attn_workspace_bytes(int B, int S, int H_q, int H_kv) {
  return costs_offset(B, S, H_q, H_kv) + ((size_t)B * H_kv * cdiv(S, kTile) * 4 + 255) / 256 * 256;
}

ea_status launch_schedule(const int32_t* head_mode, const PatternDev& pat, int B, int S, int H_q, int H_kv,
                          void* workspace, cudaStream_t st) {
  const int G = H_q / H_kv, np = n_pairs(H_q, H_kv);
  const long long n_items = (long long)B * H_kv * pat.n_qt * np;
  if (n_items > (1LL << 30)) return EA_ERR_UNSUPPORTED;
  const int n_bins = min(kMaxBins, 2 * (pat.n_qt + pat.q_tile0) + 1);
  char* ws = static_cast<char*>(workspace);
  int* cost = reinterpret_cast<int*>(ws + costs_offset(B, S, H_q, H_kv));
  const int n_bt = B * H_kv * pat.n_qt;
  tile_cost_kernel<<<cdiv(n_bt, 256), 256, 0, st>>>(head_mode, pat, B, H_kv, reinterpret_cast<uint32_t*>(ws), cost);
  if (cudaGetLastError() != cudaSuccess) return EA_ERR_CUDA;
  schedule_kernel<<<1, kSchedThreads, 0, st>>>(cost, pat, H_kv, G, np, (int)n_items, n_bins,
                                               reinterpret_cast<uint32_t*>(ws),
                                               reinterpret_cast<int4*>(ws + items_offset(B)));
  return cudaGetLastError() == cudaSuccess ? EA_OK : EA_ERR_CUDA;
}

ea_status launch_sparsity(const int32_t* head_mode, const PatternDev& pat, int B, int S, int H_q, int H_kv,
                          void* workspace, cudaStream_t st, bool clear) {
  char* ws = static_cast<char*>(workspace);
  if (clear && cudaMemsetAsync(ws + kWsLivePairs, 0, 16, st) != cudaSuccess) return EA_ERR_CUDA;
  if (clear && cudaMemsetAsync(ws + kWsHeader, 0, (size_t)B * 4, st) != cudaSuccess) return EA_ERR_CUDA;
  dim3 grid(pat.n_qt, H_kv, B);
  sparsity_kernel<<<grid, kTile, 0, st>>>(head_mode, pat, S, H_kv, H_q / H_kv,
                                          reinterpret_cast<unsigned long long*>(ws + kWsLivePairs),
                                          reinterpret_cast<int*>(ws + kWsHeader));
  return cudaGetLastError() == cudaSuccess ? EA_OK : EA_ERR_CUDA;
}

}  // namespace ea
