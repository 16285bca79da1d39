// ea_internal.h — launchers behind the C ABI (host side, not exported).
#pragma once
#include <cuda_runtime.h>
#include <cstddef>
#include <cstdint>
#include "../../include/ea.h"

namespace ea {
struct PatternDev;

size_t router_workspace_bytes(int B, int S, int D, int H_kv, int d, int n_boundary);
ea_status launch_router(const void* hidden, ea_dtype dtype, int B, int S, int D, int H_kv, int d,
                        const ea_router_weights* w, const ea_router_params* prm, int32_t* head_mode,
                        float* logits, void* workspace, cudaStream_t st);
size_t router_pool_workspace_bytes(int B, int S, int D, int n_boundary);
ea_status launch_router_pool(const void* hidden, ea_dtype dtype, int B, int S, int D, int n_boundary, float* hbar,
                             void* workspace, cudaStream_t st);

size_t attn_workspace_bytes(int B, int S, int H_q, int H_kv);
// Offset in the attention workspace of the schedule's live-tile counts: int32 per
// (b, h_kv, query tile of the call), index (b * H_kv + h) * n_qt + t.
size_t attn_costs_offset(int B, int S, int H_q, int H_kv);
int n_pairs(int H_q, int H_kv);
ea_status launch_schedule(const int32_t* head_mode, const PatternDev& pat, int B, int S, int H_q, int H_kv,
                          void* workspace, cudaStream_t st);
// clear: zero the counters first (otherwise the launch adds to them, e.g. layer after layer).
ea_status launch_sparsity(const int32_t* head_mode, const PatternDev& pat, int B, int S, int H_q, int H_kv,
                          void* workspace, cudaStream_t st, bool clear = true);
// S: query rows of this call (q and o); S_k: rows of k and v.  pat.q_tile0 * 128 is the
// position of the first query row in the sequence.
ea_status launch_attn_simt(const float* q, const float* k, const float* v, float* o, const int32_t* head_mode,
                           const PatternDev& pat, int B, int S, int S_k, int H_q, int H_kv, int d, cudaStream_t st);
ea_status launch_attn_tc(const void* q, const void* k, const void* v, void* o, const int32_t* head_mode,
                         const PatternDev& pat, int B, int S, int S_k, int H_q, int H_kv, void* workspace,
                         cudaStream_t st);
// Test hook (ea_debug_inject_stall): true for the next N launches of a kernel with bounded
// pipeline waits; that launch's first CTA then waits on a barrier nothing arrives on.
bool take_inject_stall();
// Block-64 layouts (ea_attn_tc64.cu); launch_attn_tc forwards to it.
ea_status launch_attn_tc64(const void* q, const void* k, const void* v, void* o, const int32_t* head_mode,
                           const PatternDev& pat, int B, int S, int S_k, int H_q, int H_kv, void* workspace,
                           cudaStream_t st);

// XAttention block selection (ea_xattn.cu).
bool xattn_shape_ok(int S, int H_q, int H_kv, int stride, int block);
size_t xattn_workspace_bytes(int B, int S, int H_q, int H_kv, int stride, int block);
ea_status launch_xattn(const void* q, const void* k, const int32_t* head_mode, const PatternDev& pd, int B, int S,
                       int H_q, int H_kv, int stride, float tau, int32_t* row_ptr, int32_t* cols, float* scores,
                       void* workspace, cudaStream_t st);

// Retrieval scores and static assignment (ea_assign.cu).
size_t retrieval_workspace_bytes(int B, int S, int H_q, int H_kv);
ea_status launch_retrieval(const void* q, const void* k, ea_dtype dtype, int B, int S, int H_q, int H_kv, int d,
                           int needle_begin, int needle_end, float scale_log2, float* scores, void* workspace,
                           cudaStream_t st);
bool assignment_shape_ok(int L, int H_kv);
ea_status launch_assignment(const float* scores, int L, int B, int H_q, int H_kv, int k_full, int32_t* head_mode,
                            cudaStream_t st);
}  // namespace ea
