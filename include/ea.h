/*
 * ea.h — C ABI of the Elastic Attention prefill path for NVIDIA B200 (sm_100a).
 *
 * The method: "Elastic Attention: Test-time Adaptive Sparsity Ratios for
 * Efficient Transformers" (arXiv 2601.17367; paperlayer.ai summary).  An
 * Attention Router reads a layer's hidden states and gives every GQA key-value
 * head a hard full / sparse decision (section 3 "Attention Router"); one
 * hybrid-head attention launch then computes full causal heads and sparse
 * heads (streaming sink + local window, or block-sparse) together and writes
 * every head's output side by side (section 2 "Hybrid Head Mechanism";
 * section 3 "Efficient Deployment"; appendix D.1 "Sparse Inference").
 *
 * Conventions for every call:
 *  - Device pointers are CUDA device addresses on the current device; host
 *    pointers are ordinary CPU memory.  The caller owns every buffer.  The
 *    library never allocates device memory: scratch space is the caller's
 *    `workspace`, sized by the matching *_workspace_size call, 256-byte
 *    aligned, and zero-filled once before its first use (it keeps a sticky
 *    device status word between calls).
 *  - Layouts are row-major: q, o [B, S, H_q, d]; k, v [B, S, H_kv, d];
 *    hidden [B, S, D].  Query head h_q reads KV head h_q / (H_q / H_kv).
 *    q, k, v, o and hidden must be 16-byte aligned.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream).  Calls enqueue work on it and return without waiting, except
 *    ea_effective_sparsity, ea_model_sparsity and ea_workspace_status, which
 *    synchronise it.
 *  - Errors: argument checks run on the host before any launch and return
 *    EA_ERR_INVALID_ARG or EA_ERR_UNSUPPORTED with nothing enqueued.  A
 *    failed launch returns EA_ERR_CUDA.  Problems only the device can see (a
 *    malformed block layout or head_mode value, a pipeline wait that ran past
 *    its time limit) set bits in the workspace status word; they surface on
 *    the next ea_workspace_status / ea_effective_sparsity call on that
 *    workspace as EA_ERR_BAD_LAYOUT or EA_ERR_TIMEOUT.
 *  - Thread safety: calls that share a workspace must be ordered on one
 *    stream.
 */
#ifndef EA_H_
#define EA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define EA_API __attribute__((visibility("default")))
#else
#define EA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  EA_OK = 0,
  EA_ERR_INVALID_ARG = 1,  /* a pointer, size or parameter is out of contract */
  EA_ERR_UNSUPPORTED = 2,  /* valid, but not built (e.g. bf16 with d != 128)   */
  EA_ERR_CUDA = 3,         /* a CUDA runtime or driver call failed             */
  EA_ERR_TIMEOUT = 4,      /* a device pipeline wait ran out (status word)     */
  EA_ERR_BAD_LAYOUT = 5    /* device-side check of head_mode / CSR failed      */
} ea_status;

typedef enum { EA_DT_F32 = 0, EA_DT_BF16 = 1 } ea_dtype;

/* Head kinds (attention patterns).  FULL: keys 0..i.  STREAMING: keys j <= i
 * with j < n_sink or i - j < window (sinks and the local window, united).
 * BLOCK_SPARSE: keys j <= i whose block floor(j/block) is listed for the
 * query block floor(i/block).  STREAMING_BLOCKS: streaming at block
 * granularity (appendix D.1 runs streaming through the block-sparse kernel):
 * keys j <= i whose block kb = floor(j/block) is a sink block
 * (kb < ceil(n_sink/block)) or one of the last ceil(window/block) blocks up to
 * the query's block. */
typedef enum { EA_FULL = 0, EA_STREAMING = 1, EA_BLOCK_SPARSE = 2, EA_STREAMING_BLOCKS = 3 } ea_kind;

/* Largest H_kv the calls accept (the per-head kind tables travel by value). */
#define EA_MAX_KV_HEADS 64

/* ------------------------------------------------------------------------
 * Attention Router (section 3 "Attention Router"; appendix H.4 "Router
 * Input Length"; section 5 "Attention Router" for the x4 MLP width).
 *   hbar    = mean of hidden[b, t, :] over the pooled tokens: the first and
 *             the last n_boundary tokens (every token once when
 *             S <= 2 * n_boundary; the whole sequence when n_boundary <= 0)
 *   p_h     = W_k[:, h*d:(h+1)*d]^T hbar                 (pooled key state)
 *   tau_h   = W_t2 relu(W_t1 p_h + b_t1) + b_t2          (task MLP d->4d->d)
 *   u_h     = relu(W_r1 [p_h; tau_h] + b_r1)              (router MLP 2d->4d)
 *   z_h     = w_o[h] . u_h + b_o[h];  head_mode = (z_h > 0) (1 = sparse)
 * ---------------------------------------------------------------------- */
typedef struct {
  int n_boundary; /* tokens pooled at each end; 100 by the pages; <= 0: all */
} ea_router_params;

typedef struct {          /* all device pointers, row-major                   */
  const void* w_k;        /* [D, H_kv*d] key projection, in the hidden dtype  */
  const float* w_t1;      /* [4d, d]   */
  const float* b_t1;      /* [4d]      */
  const float* w_t2;      /* [d, 4d]   */
  const float* b_t2;      /* [d]       */
  const float* w_r1;      /* [4d, 2d]  (input is [p; tau]) */
  const float* b_r1;      /* [4d]      */
  const float* w_o;       /* [H_kv, 4d] per-head output rows */
  const float* b_o;       /* [H_kv]    */
} ea_router_weights;

/* Bytes of workspace ea_router needs (pooling and key-projection partial sums). */
EA_API size_t ea_router_workspace_size(int B, int S, int D, int H_kv, int d, int n_boundary);

/* Router for one layer.  hidden: device [B, S, D] in `dtype`
 * (D % 8 == 0 for bf16, D % 4 == 0 for f32); d in {64, 128};
 * 1 <= H_kv <= EA_MAX_KV_HEADS; w_k, w_t1, w_t2, w_r1 and w_o 16-byte
 * aligned.  Writes head_mode [B, H_kv] (device int32, 0 dense / 1 sparse)
 * and, when `logits` is not NULL, z [B, H_kv] (device float).  Arithmetic is
 * fp32 in fixed summation orders (repeated calls give identical results).
 * The workspace needs no zero fill. */
EA_API ea_status ea_router(const void* hidden, ea_dtype dtype, int B, int S, int D, int H_kv, int d,
                    const ea_router_weights* weights, const ea_router_params* params,
                    int32_t* head_mode, float* logits,
                    void* workspace, size_t workspace_bytes, void* stream);

/* Router pooling alone (the first step above): hbar [B, D] (device float) =
 * mean of hidden[b, t, :] over the pooled tokens, with the same pooling rule,
 * alignment and dtype contract as ea_router.  Scratch: a workspace of
 * ea_router_pool_workspace_size bytes (256-byte aligned, no zero fill). */
EA_API size_t ea_router_pool_workspace_size(int B, int S, int D, int n_boundary);
EA_API ea_status ea_router_pool(const void* hidden, ea_dtype dtype, int B, int S, int D, int n_boundary,
                                float* hbar, void* workspace, size_t workspace_bytes, void* stream);

/* Router with library-owned scratch.  The paper has no counterpart: this is an
 * interface for callers that cannot allocate device memory, such as a runtime or
 * plugin host that owns every device allocation.  Same arguments and outputs as
 * ea_router, without the workspace: the scratch is a fixed EA_ROUTER_STATIC_SCRATCH_BYTES array
 * inside the library, held on every GPU that loads it until the process exits.
 * It allocates nothing (no cudaMalloc, cudaFree or allocating library call).
 * Problems whose scratch (ea_router_workspace_size) exceeds the array return
 * EA_ERR_INVALID_ARG before any launch.  The first call in each context (per
 * device; again after a device reset or in a caller's own context) looks up
 * the array's device address with a host-side runtime query.  All calls share
 * the array: calls that overlap on the GPU race, so order them on one stream.
 * Nothing in the array needs to start at zero. */
#define EA_ROUTER_STATIC_SCRATCH_BYTES ((size_t)8 << 20)
EA_API ea_status ea_router_static_scratch(const void* hidden, ea_dtype dtype, int B, int S, int D, int H_kv,
                                          int d, const ea_router_weights* weights,
                                          const ea_router_params* params, int32_t* head_mode, float* logits,
                                          void* stream);

/* ------------------------------------------------------------------------
 * Hybrid-head attention (section 2 "Hybrid Head Mechanism"; section 3
 * "Efficient Deployment"; appendix D.1 "Sparse Inference": the routing
 * metadata goes straight into one kernel launch).
 *   kind(b, h)  = head_mode[b, h] ? kind_if_sparse[h] : kind_if_dense[h]
 *   o[b,i,h_q]  = sum_{j in L(i)} softmax_j(scale * q_i . k_j) v_j
 * ---------------------------------------------------------------------- */
typedef struct {
  int n_sink;                   /* streaming sink tokens (>= 0); pages: 128        */
  int window;                   /* streaming local window incl. the query (>= 1)   */
  int block;                    /* block edge of BLOCK_SPARSE / STREAMING_BLOCKS: 64 (the pages') or 128 */
  const int32_t* bs_row_ptr;    /* device CSR [B*H_kv*ceil(S/block) + 1]; rows r = */
  const int32_t* bs_col;        /*   (b*H_kv + h)*n_qb + qb; cols sorted, with qb  */
  long long bs_nnz;             /* entries in bs_col (bounds every column read)    */
  const int8_t* kind_if_dense;  /* host [H_kv]: ea_kind of a dense decision        */
  const int8_t* kind_if_sparse; /* host [H_kv]: ea_kind of a sparse decision       */
  float softmax_scale;          /* 0 selects 1/sqrt(d)                             */
} ea_pattern_params;

/* Bytes of workspace the attention calls and ea_effective_sparsity need. */
EA_API size_t ea_attn_workspace_size(int B, int S, int H_q, int H_kv);

/* One call = schedule build + attention launch (below).  dtype bf16: d == 128,
 * tcgen05 tensor cores, fp32 softmax and accumulation, bf16 output.  dtype
 * f32: d in {64, 128}, fp32 CUDA-core kernel (exact fp32 arithmetic).
 * H_q % H_kv == 0, S >= 1.  head_mode: device int32 [B, H_kv]. */
EA_API ea_status ea_hybrid_attn_prefill(const void* q, const void* k, const void* v, ea_dtype dtype,
                                 int B, int S, int H_q, int H_kv, int d,
                                 const int32_t* head_mode, const ea_pattern_params* pattern,
                                 void* o, void* workspace, size_t workspace_bytes, void* stream);

/* Chunked prefill (appendix D.1 "Sparse Inference": long prompts are prefilled
 * in chunks, 16,384 tokens in the pages).  q and o [B, S_q, H_q, d] hold query
 * rows q_offset .. q_offset + S_q - 1 of the sequence; k and v [B, S_k, H_kv, d]
 * hold its keys from position 0 (a cache; rows past q_offset + S_q - 1 are not
 * read).  Head patterns use sequence positions, and the block layout has
 * ceil(S_k / block) query blocks per (sample, KV head).  q_offset % 128 == 0 and
 * q_offset + S_q <= S_k.  Workspace: ea_attn_workspace_size(B, S_q, H_q, H_kv).
 * Processing a sequence chunk by chunk gives the same result as one
 * ea_hybrid_attn_prefill over all of it (the same tiles, in the same order). */
EA_API ea_status ea_hybrid_attn_prefill_chunk(const void* q, const void* k, const void* v, ea_dtype dtype,
                                              int B, int S_q, int q_offset, int S_k, int H_q, int H_kv, int d,
                                              const int32_t* head_mode, const ea_pattern_params* pattern,
                                              void* o, void* workspace, size_t workspace_bytes, void* stream);

/* The two halves of ea_hybrid_attn_prefill, for callers that time or reuse
 * them.  ea_build_schedule reads head_mode and the pattern on the device and
 * writes the list of live (query tile, head group) work items, longest first,
 * into the workspace; ea_attn_scheduled runs the attention kernel over that
 * list and must receive the same head_mode, pattern and shapes. */
EA_API ea_status ea_build_schedule(const int32_t* head_mode, const ea_pattern_params* pattern,
                            int B, int S, int H_q, int H_kv, int d,
                            void* workspace, size_t workspace_bytes, void* stream);
EA_API ea_status ea_attn_scheduled(const void* q, const void* k, const void* v, ea_dtype dtype,
                            int B, int S, int H_q, int H_kv, int d,
                            const int32_t* head_mode, const ea_pattern_params* pattern,
                            void* o, void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * XAttention block selection for the BLOCK_SPARSE heads (section 4
 * "Evaluation Setting": the block-sparse pattern is XAttention at tau = 0.9;
 * appendix G.2 "Efficiency Results": FA-XA and XA-SSA pairings).  The pages
 * name the method; the steps are those of Xu et al., "XAttention: Block Sparse
 * Attention with Antidiagonal Scoring" (2025):
 *   R[i, j]   = sum_{m<st} q[i*st+m] . k[j*st+st-1-m]       (reduced i, j < S/st)
 *   P[i, :]   = softmax over j <= i of R[i, j] * scale / st  (scale as below)
 *   A[qb, kb] = mean over the G query heads of KV head h of the P mass of the
 *               block x block tile (qb, kb), block = pattern->block (64 or 128)
 *   row qb    = {qb} plus blocks in descending A (ties: lower index) while the
 *               kept mass < tau * sum_kb A[qb, kb]
 * Rows are computed for every (b, h) whose kind under head_mode is
 * BLOCK_SPARSE; the other rows are empty.  The output is the CSR the attention
 * calls read (bs_row_ptr / bs_col with bs_nnz = cols_capacity), written on
 * `stream` with no host round trip.
 * ---------------------------------------------------------------------- */

/* Bytes of workspace ea_xattn_block_select needs for layouts at block edge
 * `block` (64 or 128): per reduced row (S/stride of them per query head) one
 * float per key block and per 128-row reduced tile, plus O(B*H_kv*S/block)
 * for the counts and bitmaps. */
EA_API size_t ea_xattn_workspace_size(int B, int S, int H_q, int H_kv, int stride, int block);

/* q: device [B, S, H_q, 128] bf16, k: device [B, S, H_kv, 128] bf16 (16-byte
 * aligned).  stride in {4, 8, 16} with S % stride == 0; ceil(S/block) <= 2048;
 * (H_q / H_kv) * block / stride <= 1024; 0 <= tau <= 1.  pattern: kinds,
 * block (64 or 128) and softmax_scale are read; its bs_* fields are ignored.
 * row_ptr: device int32 [B*H_kv*n_qb + 1] (written), n_qb = ceil(S/block).
 * cols: device int32 with cols_capacity >= B*H_kv*n_qb*(n_qb+1)/2 entries
 * (the first row_ptr[last] are written, ascending within each row).
 * block_scores: NULL, or device float [B, H_kv, n_qb, n_qb] receiving A (zero
 * above the diagonal and on rows of other kinds).  Buffers are the caller's;
 * nothing is allocated.  Argument errors return before any launch; device-side
 * errors (bad head_mode values, a wait past ~2 s) are recorded in the
 * workspace status word (ea_workspace_status).  Calls on one workspace must not
 * overlap. */
EA_API ea_status ea_xattn_block_select(const void* q, const void* k, ea_dtype dtype, int B, int S, int H_q,
                                       int H_kv, int d, const int32_t* head_mode,
                                       const ea_pattern_params* pattern, int stride, float tau,
                                       int32_t* row_ptr, int32_t* cols, long long cols_capacity,
                                       float* block_scores, void* workspace, size_t workspace_bytes,
                                       void* stream);

/* ------------------------------------------------------------------------
 * Sparsity report (section 2 "Sparsity Ratio Computation"; appendix C.1).
 * Omega_MSR per sample = sparse KV heads / H_kv.  Omega_ESR = 1 - live
 * (query, key) pairs / causal pairs over all samples and query heads.  Tiles
 * are 128 x 128; live_flops = 4 * d * 128^2 per live tile per query head.
 * Counts run on the device; the call synchronises `stream` and fills the
 * host outputs.  omega_msr_per_sample: host float [B] (may be NULL).
 * ---------------------------------------------------------------------- */
typedef struct {
  double omega_msr_mean;
  double omega_esr;
  long long live_pairs, causal_pairs;
  long long live_tiles, causal_tiles;
  double live_flops;
} ea_sparsity_report;

EA_API ea_status ea_effective_sparsity(const int32_t* head_mode, const ea_pattern_params* pattern,
                                int B, int S, int H_q, int H_kv, int d,
                                float* omega_msr_per_sample, ea_sparsity_report* report,
                                void* workspace, size_t workspace_bytes, void* stream);

/* The same report over a stack of L layers that share `pattern`: head_mode is
 * device int32 [L, B, H_kv] (layer-major).  Pairs, tiles and FLOPs are summed
 * over the layers; Omega_ESR = 1 - live / causal pairs of all layers; Omega_MSR
 * per sample = its sparse KV heads over L * H_kv.  Workspace:
 * ea_attn_workspace_size(B, S, H_q, H_kv).  Synchronises `stream`. */
EA_API ea_status ea_model_sparsity(const int32_t* head_mode, const ea_pattern_params* pattern,
                                   int L, int B, int S, int H_q, int H_kv, int d,
                                   float* omega_msr_per_sample, ea_sparsity_report* report,
                                   void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Static retrieval-head assignment (appendix C.1 "Retrieval Score
 * Calculation" and "Sparsity Assignment").
 *   score[b, h_q] = sum_{needle_begin <= j < needle_end} softmax_j(scale q_{S-1} . k_j)
 * (the attention mass of the last token on the needle span), per layer; then
 *   kv_score[l, h] = mean over b and the G query heads of KV head h of score
 *   k = floor((1 - omega_msr) * L * H_kv)   (double precision)
 *   head_mode[l, b, h] = 0 (full) for the k best kv_scores (ties: lower
 *   l * H_kv + h first), 1 (sparse) for the others, the same for every b.
 * ---------------------------------------------------------------------- */

/* Bytes of workspace ea_retrieval_scores needs (per-slice partial sums). */
EA_API size_t ea_retrieval_workspace_size(int B, int S, int H_q, int H_kv);

/* One layer's retrieval scores.  q: device [B, S, H_q, d], k: device
 * [B, S, H_kv, d] (bf16 or f32, 16-byte aligned; only q row S-1 is read);
 * d in {64, 128}; H_q / H_kv <= 64; 0 <= needle_begin <= needle_end <= S; softmax_scale 0
 * selects 1/sqrt(d).  scores: device float [B, H_q] (written).  fp32
 * accumulation. */
EA_API ea_status ea_retrieval_scores(const void* q, const void* k, ea_dtype dtype, int B, int S, int H_q,
                                     int H_kv, int d, int needle_begin, int needle_end, float softmax_scale,
                                     float* scores, void* workspace, size_t workspace_bytes, void* stream);

/* scores: device float [L, B, H_q] (the layers' ea_retrieval_scores outputs
 * stacked); head_mode: device int32 [L, B, H_kv] (written).  L * H_kv <= 8192,
 * 0 <= omega_msr <= 1.  One kernel launch, no allocation. */
EA_API ea_status ea_static_head_assignment(const float* scores, int L, int B, int H_q, int H_kv,
                                           double omega_msr, int32_t* head_mode, void* stream);

/* Test hook for the failure path (no counterpart in the paper): the next
 * `launches` tensor-core attention launches of layouts other than block 64
 * (block-64 launches neither use nor consume it) make the MMA thread of their first
 * CTA wait on a barrier that nothing arrives on.  That bounded wait runs out
 * (about 2 s), the CTA drains its own copies and MMAs, frees TMEM and exits, and
 * the workspace status word reads EA_ERR_TIMEOUT; the output of that CTA's work
 * items is left unwritten.  0 disables the hook (the default). */
EA_API void ea_debug_inject_stall(int launches);

/* Synchronises `stream`, reads and clears the workspace's device status
 * word: EA_OK, EA_ERR_TIMEOUT or EA_ERR_BAD_LAYOUT. */
EA_API ea_status ea_workspace_status(void* workspace, void* stream);

/* Static text for a status code. */
EA_API const char* ea_status_string(ea_status status);

#ifdef __cplusplus
}
#endif
#endif /* EA_H_ */
