"""Oracle: hybrid-head GQA attention for prefill, fp64 — TEST INFRASTRUCTURE ONLY.

Source: "Elastic Attention: Test-time Adaptive Sparsity Ratios for Efficient
Transformers" (paperlayer.ai summary of arXiv 2601.17367v2):
  * section 2 "Hybrid Head Mechanism": every head runs full attention (FA)
    or sparse attention (SA); the head outputs are concatenated;
  * section 3 "Attention Router": the assignment is per key-value head, so
    every query head of a GQA group shares its KV head's mode;
    "Takeaways & Limitations": the evaluation uses the GQA definition;
  * section 1 / B.2 "Intra-layer Hybridization": SA is streaming sparse
    attention (attention sinks plus a local window) or block-sparse attention;
    appendix D.1 "Sparse Inference": 128 sink tokens, block size 64 (the
    block edge is a parameter here), streaming run through the block-sparse
    kernel, i.e. at block granularity;
  * section 1 "Introduction": full attention is the quadratic causal softmax
    attention.

Definition computed, for query row i of query head h_q (KV head
h_kv = h_q // G, G = H_q / H_kv, 0-indexed aligned prefill positions):
    L(i)   = live keys of the head's kind (below; causality j <= i always)
    s_ij   = scale * q_i . k_j            (scale = 1/sqrt(d) unless given)
    o_i    = sum_{j in L(i)} softmax_j(s_ij) v_j
  FULL:          L(i) = {0..i}
  STREAMING:     L(i) = {j <= i : j < n_sink or i - j < window}
  BLOCK_SPARSE:  L(i) = {j <= i : floor(j/block) listed for (b, h_kv, floor(i/block))}
  STREAMING_BLOCKS (streaming at block granularity, appendix D.1):
                 L(i) = {j <= i : floor(j/block) < ceil(n_sink/block)
                                  or floor(i/block) - floor(j/block) < ceil(window/block)}
Readings: token-exact sink and window (the window counts i itself), sink and
window sets are united, never added; the mode -> kind map is per KV head
(kind_if_dense[h] / kind_if_sparse[h]).
"""
from __future__ import annotations

import numpy as np

FULL, STREAMING, BLOCK_SPARSE, STREAMING_BLOCKS = 0, 1, 2, 3


def head_kind(head_mode, b: int, h_kv: int, kind_if_dense, kind_if_sparse) -> int:
    """Pattern of KV head h_kv of sample b: the router's sparse decision picks kind_if_sparse."""
    return int(kind_if_sparse[h_kv]) if int(head_mode[b][h_kv]) != 0 else int(kind_if_dense[h_kv])


def csr_row(pattern, b: int, h_kv: int, qb: int, H_kv: int, S: int) -> np.ndarray:
    n_qb = -(-S // pattern["block"])
    r = (b * H_kv + h_kv) * n_qb + qb
    rp = pattern["row_ptr"]
    return np.asarray(pattern["cols"][rp[r]:rp[r + 1]], dtype=np.int64)


def live_keys(i: int, kind: int, pattern, b: int = 0, h_kv: int = 0, H_kv: int = 1, S: int = 0):
    """L(i): the keys query row i attends to under the head's kind (sorted)."""
    j = np.arange(i + 1)
    if kind == FULL:
        return j
    if kind == STREAMING:
        return j[(j < pattern["n_sink"]) | (i - j < pattern["window"])]
    if kind == BLOCK_SPARSE:
        blk = pattern["block"]
        listed = csr_row(pattern, b, h_kv, i // blk, H_kv, S)
        return j[np.isin(j // blk, listed)]
    if kind == STREAMING_BLOCKS:
        blk = pattern["block"]
        sink_blocks = -(-pattern["n_sink"] // blk)
        local_blocks = -(-pattern["window"] // blk)
        kb, qb = j // blk, i // blk
        return j[(kb < sink_blocks) | (qb - kb < local_blocks)]
    raise ValueError(f"unknown head kind {kind}")


def softmax_scale(pattern, d: int) -> float:
    s = float(pattern.get("softmax_scale", 0.0) or 0.0)
    return s if s != 0.0 else 1.0 / np.sqrt(d)


def attend_row(q_i, K, V, live, scale):
    """One softmax attention row over the keys in ``live``.  Returns (o_i, weights)."""
    s = scale * (K[live] @ q_i)
    e = np.exp(s - s.max())
    wts = e / e.sum()
    return wts @ V[live], wts


def hybrid_attention_rows(q, k, v, head_mode, pattern, rows=None, q_row_index=None):
    """o[b, i, h_q, :] for the requested rows (all rows when ``rows`` is None), fp64.

    q: [B, Sq, H_q, d] holding query rows ``q_row_index`` (all S rows when
    None); k, v: [B, S, H_kv, d]; head_mode: [B, H_kv]; pattern: dict with
    n_sink, window, block, row_ptr, cols, kind_if_dense, kind_if_sparse and an
    optional softmax_scale.  Returns an array [B, len(rows), H_q, d]."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, S, H_kv, d = k.shape
    H_q = q.shape[2]
    G = H_q // H_kv
    assert H_q == G * H_kv
    rows = np.arange(S) if rows is None else np.asarray(rows, dtype=np.int64)
    qpos = {int(r): n for n, r in enumerate(np.arange(S) if q_row_index is None else q_row_index)}
    scale = softmax_scale(pattern, d)
    out = np.zeros((B, len(rows), H_q, d))
    for b in range(B):
        for h_q in range(H_q):
            h_kv = h_q // G
            kind = head_kind(head_mode, b, h_kv, pattern["kind_if_dense"], pattern["kind_if_sparse"])
            K, V = k[b, :, h_kv, :], v[b, :, h_kv, :]
            for n, i in enumerate(rows):
                live = live_keys(int(i), kind, pattern, b, h_kv, H_kv, S)
                out[b, n, h_q], _ = attend_row(q[b, qpos[int(i)], h_q], K, V, live, scale)
    return out


def hybrid_attention(q, k, v, head_mode, pattern):
    """Every row of every head: o [B, S, H_q, d] (the heads' outputs side by side)."""
    return hybrid_attention_rows(q, k, v, head_mode, pattern)
