// ea_abi.cu — the exported C ABI (include/ea.h): host-side argument checks,
// parameter packing and dispatch to the kernels.  No device memory is allocated
// here; every scratch byte comes from the caller's workspace.
#include <cuda_runtime.h>
#include <cmath>
#include <cstdint>
#include <cstring>
#include "ea_common.cuh"
#include "ea_internal.h"

using namespace ea;

namespace {

inline cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool any_kind(const ea_pattern_params* p, int H_kv, int kind) {
  for (int h = 0; h < H_kv; ++h)
    if (p->kind_if_dense[h] == kind || p->kind_if_sparse[h] == kind) return true;
  return false;
}

// Checks shared by every attention-side call; fills the device pattern block.  The call's
// S_q query rows are rows q_offset.. of a sequence whose keys are the S_k rows of k and v.
ea_status check_pattern(const int32_t* head_mode, const ea_pattern_params* p, int B, int S_q, int S_k,
                        int q_offset, int H_q, int H_kv, int d, PatternDev* out) {
  if (!head_mode || !p || !p->kind_if_dense || !p->kind_if_sparse) return EA_ERR_INVALID_ARG;
  if (B < 1 || S_q < 1 || H_kv < 1 || H_q < 1 || H_q % H_kv != 0) return EA_ERR_INVALID_ARG;
  if (q_offset < 0 || q_offset % kTile != 0 || (long long)q_offset + S_q > (long long)S_k) return EA_ERR_INVALID_ARG;
  const int S = S_k;
  if (H_kv > EA_MAX_KV_HEADS) return EA_ERR_UNSUPPORTED;
  if (d != 64 && d != 128) return EA_ERR_UNSUPPORTED;
  if (p->n_sink < 0 || p->window < 1 || p->block < 1) return EA_ERR_INVALID_ARG;
  if (!(p->softmax_scale >= 0.f) || std::isinf(p->softmax_scale)) return EA_ERR_INVALID_ARG;
  for (int h = 0; h < H_kv; ++h) {
    const int a = p->kind_if_dense[h], b = p->kind_if_sparse[h];
    if (a < EA_FULL || a > EA_STREAMING_BLOCKS || b < EA_FULL || b > EA_STREAMING_BLOCKS) return EA_ERR_INVALID_ARG;
  }
  const bool bsa = any_kind(p, H_kv, EA_BLOCK_SPARSE);
  if (bsa && (!p->bs_row_ptr || !p->bs_col || p->bs_nnz < 0)) return EA_ERR_INVALID_ARG;
  if ((bsa || any_kind(p, H_kv, EA_STREAMING_BLOCKS)) && p->block != kTile && p->block != 64)
    return EA_ERR_UNSUPPORTED;
  if ((long long)S > (1LL << 30) || (long long)B * S > (1LL << 31)) return EA_ERR_UNSUPPORTED;
  std::memset(out, 0, sizeof(*out));
  out->n_sink = p->n_sink;
  out->window = p->window;
  out->block = p->block;
  out->n_qt = cdiv(S_q, kTile);
  out->q_tile0 = q_offset / kTile;
  out->n_qb = cdiv(S_k, (bsa || any_kind(p, H_kv, EA_STREAMING_BLOCKS)) ? p->block : kTile);
  out->row_ptr = bsa ? p->bs_row_ptr : nullptr;
  out->cols = bsa ? p->bs_col : nullptr;
  out->nnz = bsa ? p->bs_nnz : 0;
  const double scale = p->softmax_scale > 0.f ? (double)p->softmax_scale : 1.0 / std::sqrt((double)d);
  out->scale = (float)scale;
  out->scale_log2 = (float)(scale * 1.4426950408889634);
  for (int h = 0; h < H_kv; ++h) {
    out->kind_dense[h] = p->kind_if_dense[h];
    out->kind_sparse[h] = p->kind_if_sparse[h];
  }
  return EA_OK;
}

ea_status check_attn_data(const void* q, const void* k, const void* v, const void* o, ea_dtype dtype, int d) {
  if (!q || !k || !v || !o) return EA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return EA_ERR_INVALID_ARG;
  if (dtype == EA_DT_BF16) return d == 128 ? EA_OK : EA_ERR_UNSUPPORTED;
  if (dtype == EA_DT_F32) return EA_OK;
  return EA_ERR_INVALID_ARG;
}

// The router reads its weight matrices with 16-byte loads.
bool router_weights_aligned(const ea_router_weights* w) {
  return aligned16(w->w_k) && aligned16(w->w_t1) && aligned16(w->w_t2) && aligned16(w->w_r1) && aligned16(w->w_o);
}

ea_status check_ws(const void* ws, size_t bytes, size_t need) {
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return EA_ERR_INVALID_ARG;
  return bytes >= need ? EA_OK : EA_ERR_INVALID_ARG;
}

}  // namespace

extern "C" {

size_t ea_router_workspace_size(int B, int S, int D, int H_kv, int d, int n_boundary) {
  if (B < 1 || S < 1 || D < 1 || H_kv < 1 || d < 1) return 0;
  return router_workspace_bytes(B, S, D, H_kv, d, n_boundary);
}

size_t ea_router_pool_workspace_size(int B, int S, int D, int n_boundary) {
  if (B < 1 || S < 1 || D < 1) return 0;
  return router_pool_workspace_bytes(B, S, D, n_boundary);
}

ea_status ea_router(const void* hidden, ea_dtype dtype, int B, int S, int D, int H_kv, int d,
                    const ea_router_weights* w, const ea_router_params* prm, int32_t* head_mode, float* logits,
                    void* workspace, size_t workspace_bytes, void* stream) {
  if (!hidden || !w || !prm || !head_mode) return EA_ERR_INVALID_ARG;
  if (!w->w_k || !w->w_t1 || !w->b_t1 || !w->w_t2 || !w->b_t2 || !w->w_r1 || !w->b_r1 || !w->w_o || !w->b_o)
    return EA_ERR_INVALID_ARG;
  if (B < 1 || S < 1 || D < 1 || H_kv < 1) return EA_ERR_INVALID_ARG;
  if (H_kv > EA_MAX_KV_HEADS) return EA_ERR_UNSUPPORTED;
  if (d != 64 && d != 128) return EA_ERR_UNSUPPORTED;
  if (dtype != EA_DT_BF16 && dtype != EA_DT_F32) return EA_ERR_INVALID_ARG;
  if (D % (dtype == EA_DT_BF16 ? 8 : 4) != 0 || !aligned16(hidden)) return EA_ERR_INVALID_ARG;
  if ((size_t)D * sizeof(float) + 12u * d * sizeof(float) > 200u * 1024u) return EA_ERR_UNSUPPORTED;
  if (!router_weights_aligned(w)) return EA_ERR_INVALID_ARG;
  if (ea_status s = check_ws(workspace, workspace_bytes, router_workspace_bytes(B, S, D, H_kv, d, prm->n_boundary)))
    return s;
  return launch_router(hidden, dtype, B, S, D, H_kv, d, w, prm, head_mode, logits, workspace, as_stream(stream));
}

ea_status ea_router_pool(const void* hidden, ea_dtype dtype, int B, int S, int D, int n_boundary, float* hbar,
                         void* workspace, size_t workspace_bytes, void* stream) {
  if (!hidden || !hbar) return EA_ERR_INVALID_ARG;
  if (B < 1 || S < 1 || D < 1) return EA_ERR_INVALID_ARG;
  if (dtype != EA_DT_BF16 && dtype != EA_DT_F32) return EA_ERR_INVALID_ARG;
  if (D % (dtype == EA_DT_BF16 ? 8 : 4) != 0 || !aligned16(hidden)) return EA_ERR_INVALID_ARG;
  if ((long long)B * D > (1LL << 31) - 256) return EA_ERR_UNSUPPORTED;
  if (ea_status s = check_ws(workspace, workspace_bytes, router_pool_workspace_bytes(B, S, D, n_boundary))) return s;
  return launch_router_pool(hidden, dtype, B, S, D, n_boundary, hbar, workspace, as_stream(stream));
}

size_t ea_attn_workspace_size(int B, int S, int H_q, int H_kv) {
  if (B < 1 || S < 1 || H_kv < 1 || H_q < H_kv || H_q % H_kv != 0) return 0;
  return attn_workspace_bytes(B, S, H_q, H_kv);
}

ea_status ea_build_schedule(const int32_t* head_mode, const ea_pattern_params* pattern, int B, int S, int H_q,
                            int H_kv, int d, void* workspace, size_t workspace_bytes, void* stream) {
  PatternDev pd;
  if (ea_status s = check_pattern(head_mode, pattern, B, S, S, 0, H_q, H_kv, d, &pd)) return s;
  if (ea_status s = check_ws(workspace, workspace_bytes, attn_workspace_bytes(B, S, H_q, H_kv))) return s;
  return launch_schedule(head_mode, pd, B, S, H_q, H_kv, workspace, as_stream(stream));
}

ea_status ea_attn_scheduled(const void* q, const void* k, const void* v, ea_dtype dtype, int B, int S, int H_q,
                            int H_kv, int d, const int32_t* head_mode, const ea_pattern_params* pattern, void* o,
                            void* workspace, size_t workspace_bytes, void* stream) {
  PatternDev pd;
  if (ea_status s = check_pattern(head_mode, pattern, B, S, S, 0, H_q, H_kv, d, &pd)) return s;
  if (ea_status s = check_attn_data(q, k, v, o, dtype, d)) return s;
  if (ea_status s = check_ws(workspace, workspace_bytes, attn_workspace_bytes(B, S, H_q, H_kv))) return s;
  if (dtype == EA_DT_F32)
    return launch_attn_simt(static_cast<const float*>(q), static_cast<const float*>(k),
                            static_cast<const float*>(v), static_cast<float*>(o), head_mode, pd, B, S, S, H_q, H_kv,
                            d, as_stream(stream));
  return launch_attn_tc(q, k, v, o, head_mode, pd, B, S, S, H_q, H_kv, workspace, as_stream(stream));
}

static ea_status attn_prefill(const void* q, const void* k, const void* v, ea_dtype dtype, int B, int S_q,
                              int q_offset, int S_k, int H_q, int H_kv, int d, const int32_t* head_mode,
                              const ea_pattern_params* pattern, void* o, void* workspace, size_t workspace_bytes,
                              void* stream) {
  PatternDev pd;
  if (ea_status s = check_pattern(head_mode, pattern, B, S_q, S_k, q_offset, H_q, H_kv, d, &pd)) return s;
  if (ea_status s = check_attn_data(q, k, v, o, dtype, d)) return s;
  if (ea_status s = check_ws(workspace, workspace_bytes, attn_workspace_bytes(B, S_q, H_q, H_kv))) return s;
  // The schedule kernel also checks head_mode and the block layout on the device.
  if (ea_status s = launch_schedule(head_mode, pd, B, S_q, H_q, H_kv, workspace, as_stream(stream))) return s;
  if (dtype == EA_DT_BF16)
    return launch_attn_tc(q, k, v, o, head_mode, pd, B, S_q, S_k, H_q, H_kv, workspace, as_stream(stream));
  return launch_attn_simt(static_cast<const float*>(q), static_cast<const float*>(k), static_cast<const float*>(v),
                          static_cast<float*>(o), head_mode, pd, B, S_q, S_k, H_q, H_kv, d, as_stream(stream));
}

ea_status ea_hybrid_attn_prefill(const void* q, const void* k, const void* v, ea_dtype dtype, int B, int S,
                                 int H_q, int H_kv, int d, const int32_t* head_mode,
                                 const ea_pattern_params* pattern, void* o, void* workspace,
                                 size_t workspace_bytes, void* stream) {
  return attn_prefill(q, k, v, dtype, B, S, 0, S, H_q, H_kv, d, head_mode, pattern, o, workspace, workspace_bytes,
                      stream);
}

ea_status ea_hybrid_attn_prefill_chunk(const void* q, const void* k, const void* v, ea_dtype dtype, int B,
                                       int S_q, int q_offset, int S_k, int H_q, int H_kv, int d,
                                       const int32_t* head_mode, const ea_pattern_params* pattern, void* o,
                                       void* workspace, size_t workspace_bytes, void* stream) {
  return attn_prefill(q, k, v, dtype, B, S_q, q_offset, S_k, H_q, H_kv, d, head_mode, pattern, o, workspace,
                      workspace_bytes, stream);
}

// Sparsity counts of L layers (head_mode [L, B, H_kv], one pattern) accumulated on the device.
static ea_status stack_sparsity(const int32_t* head_mode, const ea_pattern_params* pattern, int L, int B, int S,
                                int H_q, int H_kv, int d, float* omega_msr_per_sample, ea_sparsity_report* report,
                                void* workspace, size_t workspace_bytes, void* stream) {
  PatternDev pd;
  if (!report || L < 1) return EA_ERR_INVALID_ARG;
  if (ea_status s = check_pattern(head_mode, pattern, B, S, S, 0, H_q, H_kv, d, &pd)) return s;
  if (ea_status s = check_ws(workspace, workspace_bytes, attn_workspace_bytes(B, S, H_q, H_kv))) return s;
  cudaStream_t st = as_stream(stream);
  for (int l = 0; l < L; ++l)
    if (ea_status s = launch_sparsity(head_mode + (size_t)l * B * H_kv, pd, B, S, H_q, H_kv, workspace, st, l == 0))
      return s;
  char* ws = static_cast<char*>(workspace);
  unsigned long long counters[2] = {0, 0};
  uint32_t status = 0;
  if (cudaMemcpyAsync(counters, ws + kWsLivePairs, sizeof(counters), cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return EA_ERR_CUDA;
  if (cudaMemcpyAsync(&status, ws + kWsStatus, sizeof(status), cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return EA_ERR_CUDA;
  int* sparse = new int[B];
  if (cudaMemcpyAsync(sparse, ws + kWsHeader, sizeof(int) * B, cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess) {
    delete[] sparse;
    return EA_ERR_CUDA;
  }
  double mean = 0.0;
  for (int b = 0; b < B; ++b) {
    const double om = (double)sparse[b] / ((double)L * H_kv);
    if (omega_msr_per_sample) omega_msr_per_sample[b] = (float)om;
    mean += om / B;
  }
  delete[] sparse;
  const long long causal_pairs = (long long)L * B * H_q * ((long long)S * (S + 1) / 2);
  const long long nq = cdiv(S, kTile);
  report->omega_msr_mean = mean;
  report->live_pairs = (long long)counters[0];
  report->causal_pairs = causal_pairs;
  report->omega_esr = 1.0 - (double)counters[0] / (double)causal_pairs;
  report->live_tiles = (long long)counters[1];
  report->causal_tiles = (long long)L * B * H_q * (nq * (nq + 1) / 2);
  report->live_flops = 4.0 * d * kTile * kTile * (double)counters[1];
  if (status & kStatusTimeout) return EA_ERR_TIMEOUT;
  if (status & (kStatusBadLayout | kStatusBadMode)) return EA_ERR_BAD_LAYOUT;
  return EA_OK;
}

ea_status ea_effective_sparsity(const int32_t* head_mode, const ea_pattern_params* pattern, int B, int S, int H_q,
                                int H_kv, int d, float* omega_msr_per_sample, ea_sparsity_report* report,
                                void* workspace, size_t workspace_bytes, void* stream) {
  return stack_sparsity(head_mode, pattern, 1, B, S, H_q, H_kv, d, omega_msr_per_sample, report, workspace,
                        workspace_bytes, stream);
}

ea_status ea_model_sparsity(const int32_t* head_mode, const ea_pattern_params* pattern, int L, int B, int S, int H_q,
                            int H_kv, int d, float* omega_msr_per_sample, ea_sparsity_report* report,
                            void* workspace, size_t workspace_bytes, void* stream) {
  return stack_sparsity(head_mode, pattern, L, B, S, H_q, H_kv, d, omega_msr_per_sample, report, workspace,
                        workspace_bytes, stream);
}

size_t ea_retrieval_workspace_size(int B, int S, int H_q, int H_kv) {
  if (B < 1 || S < 1 || H_q < 1 || H_kv < 1 || H_q % H_kv != 0) return 0;
  return retrieval_workspace_bytes(B, S, H_q, H_kv);
}

ea_status ea_retrieval_scores(const void* q, const void* k, ea_dtype dtype, int B, int S, int H_q, int H_kv, int d,
                              int needle_begin, int needle_end, float softmax_scale, float* scores, void* workspace,
                              size_t workspace_bytes, void* stream) {
  if (!q || !k || !scores) return EA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k)) return EA_ERR_INVALID_ARG;
  if (B < 1 || S < 1 || H_q < 1 || H_kv < 1 || H_q % H_kv != 0) return EA_ERR_INVALID_ARG;
  if (needle_begin < 0 || needle_end < needle_begin || needle_end > S) return EA_ERR_INVALID_ARG;
  if (!(softmax_scale >= 0.f) || std::isinf(softmax_scale)) return EA_ERR_INVALID_ARG;
  if (dtype != EA_DT_BF16 && dtype != EA_DT_F32) return EA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return EA_ERR_UNSUPPORTED;
  if (H_q / H_kv > 64 || (long long)B * S * H_q * d > (1LL << 40)) return EA_ERR_UNSUPPORTED;
  if (ea_status s = check_ws(workspace, workspace_bytes, retrieval_workspace_bytes(B, S, H_q, H_kv))) return s;
  const double scale = softmax_scale > 0.f ? (double)softmax_scale : 1.0 / std::sqrt((double)d);
  return launch_retrieval(q, k, dtype, B, S, H_q, H_kv, d, needle_begin, needle_end,
                          (float)(scale * 1.4426950408889634), scores, workspace, as_stream(stream));
}

ea_status ea_static_head_assignment(const float* scores, int L, int B, int H_q, int H_kv, double omega_msr,
                                    int32_t* head_mode, void* stream) {
  if (!scores || !head_mode) return EA_ERR_INVALID_ARG;
  if (L < 1 || B < 1 || H_q < 1 || H_kv < 1 || H_q % H_kv != 0) return EA_ERR_INVALID_ARG;
  if (!(omega_msr >= 0.0 && omega_msr <= 1.0)) return EA_ERR_INVALID_ARG;
  if (!assignment_shape_ok(L, H_kv)) return EA_ERR_UNSUPPORTED;
  const int k_full = (int)std::floor((1.0 - omega_msr) * (double)(L * H_kv));
  return launch_assignment(scores, L, B, H_q, H_kv, k_full, head_mode, as_stream(stream));
}

size_t ea_xattn_workspace_size(int B, int S, int H_q, int H_kv, int stride, int block) {
  if (B < 1 || S < 1 || H_q < 1 || H_kv < 1 || H_q % H_kv != 0) return 0;
  if (!xattn_shape_ok(S, H_q, H_kv, stride, block)) return 0;
  return xattn_workspace_bytes(B, S, H_q, H_kv, stride, block);
}

ea_status ea_xattn_block_select(const void* q, const void* k, ea_dtype dtype, int B, int S, int H_q, int H_kv, int d,
                                const int32_t* head_mode, const ea_pattern_params* pattern, int stride, float tau,
                                int32_t* row_ptr, int32_t* cols, long long cols_capacity, float* block_scores,
                                void* workspace, size_t workspace_bytes, void* stream) {
  if (!q || !k || !row_ptr || !cols || !pattern) return EA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k)) return EA_ERR_INVALID_ARG;
  if (!(tau >= 0.f && tau <= 1.f)) return EA_ERR_INVALID_ARG;
  if (dtype != EA_DT_BF16 && dtype != EA_DT_F32) return EA_ERR_INVALID_ARG;
  if (dtype != EA_DT_BF16 || d != 128) return EA_ERR_UNSUPPORTED;
  // The layout being produced stands in for the pattern's own, so the usual checks apply.
  ea_pattern_params pp = *pattern;
  pp.bs_row_ptr = row_ptr;
  pp.bs_col = cols;
  pp.bs_nnz = cols_capacity;
  PatternDev pd;
  if (ea_status s = check_pattern(head_mode, &pp, B, S, S, 0, H_q, H_kv, d, &pd)) return s;
  if (!xattn_shape_ok(S, H_q, H_kv, stride, pp.block)) return EA_ERR_UNSUPPORTED;
  pd.n_qb = cdiv(S, pp.block);   // the layout is written at the pattern's block edge
  const long long n_qb = pd.n_qb;
  if (cols_capacity < (long long)B * H_kv * n_qb * (n_qb + 1) / 2) return EA_ERR_INVALID_ARG;
  if (ea_status s = check_ws(workspace, workspace_bytes, xattn_workspace_bytes(B, S, H_q, H_kv, stride, pp.block)))
    return s;
  return launch_xattn(q, k, head_mode, pd, B, S, H_q, H_kv, stride, tau, row_ptr, cols, block_scores, workspace,
                      as_stream(stream));
}

ea_status ea_workspace_status(void* workspace, void* stream) {
  if (!workspace) return EA_ERR_INVALID_ARG;
  cudaStream_t st = as_stream(stream);
  uint32_t status = 0;
  char* ws = static_cast<char*>(workspace);
  if (cudaMemcpyAsync(&status, ws + kWsStatus, sizeof(status), cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return EA_ERR_CUDA;
  if (cudaMemsetAsync(ws + kWsStatus, 0, sizeof(uint32_t), st) != cudaSuccess) return EA_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return EA_ERR_CUDA;
  if (status & kStatusTimeout) return EA_ERR_TIMEOUT;
  if (status & (kStatusBadLayout | kStatusBadMode)) return EA_ERR_BAD_LAYOUT;
  return EA_OK;
}

const char* ea_status_string(ea_status s) {
  switch (s) {
    case EA_OK: return "ok";
    case EA_ERR_INVALID_ARG: return "invalid argument";
    case EA_ERR_UNSUPPORTED: return "unsupported configuration";
    case EA_ERR_CUDA: return "CUDA error";
    case EA_ERR_TIMEOUT: return "device pipeline wait timed out";
    case EA_ERR_BAD_LAYOUT: return "malformed head_mode or block layout (device check)";
  }
  return "unknown status";
}

}  // extern "C"
