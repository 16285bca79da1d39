"""Oracle: XAttention block selection for block-sparse heads, fp64 — TEST INFRASTRUCTURE ONLY.

Source: "Elastic Attention: Test-time Adaptive Sparsity Ratios for Efficient
Transformers" (paperlayer.ai summary of arXiv 2601.17367v2):
  * section 4 "Evaluation Setting": the block-sparse pattern is XAttention, run
    with its default settings except the threshold tau = 0.9;
  * section 5 / appendix G.2 "Efficiency Results": the FA-XA pairing (router
    "full" heads dense, "sparse" heads XAttention) and XA-SSA (router "full"
    heads XAttention, "sparse" heads streaming);
  * appendix D.1 "Sparse Inference": the selected blocks feed the block-sparse
    attention kernel.
The pages name XAttention but do not restate it; this module writes out the
published method (Xu et al., "XAttention: Block Sparse Attention with
Antidiagonal Scoring", 2025) as read here:

  1. Antidiagonal scoring at stride st.  Reduced query row i stands for query
     rows i*st .. i*st+st-1, reduced key column j for keys j*st .. j*st+st-1;
     the reduced score is the sum over the antidiagonal of that st x st
     sub-block of Q K^T:
         R[i, j] = sum_{m=0}^{st-1} q[i*st + m] . k[j*st + st-1 - m]
  2. Softmax of the reduced scores along each reduced row, over the causal
     reduced columns j <= i, at scale 1/(sqrt(d) * st) (the mean of the st
     antidiagonal products, at the attention's 1/sqrt(d)).
  3. Block importance: the softmax mass summed over each (block x block) tile
     of the original matrix, i.e. over the block/st reduced rows and columns
     it covers.  Every reduced row sums to 1, so a full query block's row of
     importances sums to block/st.
  4. Selection per query block qb (keys blocks 0..qb): the diagonal block is
     always kept (every query row keeps its own key); the other blocks are
     taken in descending importance (ties: lower block index first) while the
     kept mass is still below tau x the row's total.

Readings where the pages are silent (all stated, none pinned by the pages):
stride 8 and block 128 (XAttention's defaults; the block equals the attention
kernel's 128-key tile); the layout is per KV head as the router's assignment is
(section 3 "Attention Router"), so the G query heads of a group are merged by
taking the mean of their importances before step 4; S must be a multiple of st
for the CUDA path (the oracle pads with zero rows, which add nothing to R).
Parity with XAttention's own implementation is unpinned (the pages print none);
the written steps are pinned in tests/test_oracle_xattention.py against a
brute-force antidiagonal sum of the full score matrix, closed forms and
hand-computed selections.
"""
from __future__ import annotations

import numpy as np

from .attention import BLOCK_SPARSE, head_kind


def reduced_scores(q_h: np.ndarray, k_h: np.ndarray, stride: int) -> np.ndarray:
    """Step 1: R[i, j] for one query head and its KV head; q_h, k_h are [S, d]."""
    S, d = q_h.shape
    n = -(-S // stride)
    pad = n * stride - S
    q = np.concatenate([np.asarray(q_h, np.float64), np.zeros((pad, d))]).reshape(n, stride, d)
    k = np.concatenate([np.asarray(k_h, np.float64), np.zeros((pad, d))]).reshape(n, stride, d)
    R = np.zeros((n, n))
    for m in range(stride):
        R += q[:, m, :] @ k[:, stride - 1 - m, :].T
    return R


def reduced_softmax(R: np.ndarray, scale: float) -> np.ndarray:
    """Step 2: causal row softmax of scale * R (entries j > i are zero)."""
    n = R.shape[0]
    P = np.zeros_like(R)
    for i in range(n):
        s = scale * R[i, :i + 1]
        e = np.exp(s - s.max())
        P[i, :i + 1] = e / e.sum()
    return P


def block_importance(P: np.ndarray, stride: int, block: int) -> np.ndarray:
    """Step 3: A[qb, kb] = softmax mass of the (block x block) tile (qb, kb)."""
    if block % stride:
        raise ValueError("block must be a multiple of the stride")
    r = block // stride
    n = P.shape[0]
    nb = -(-n // r)
    A = np.zeros((nb, nb))
    for qb in range(nb):
        for kb in range(qb + 1):
            A[qb, kb] = P[qb * r:(qb + 1) * r, kb * r:(kb + 1) * r].sum()
    return A


def head_importance(q_h, k_h, stride: int, block: int, scale: float) -> np.ndarray:
    """Steps 1-3 for one query head."""
    return block_importance(reduced_softmax(reduced_scores(q_h, k_h, stride), scale / stride), stride, block)


def group_importance(q, k, b: int, h_kv: int, stride: int, block: int, scale: float | None = None) -> np.ndarray:
    """Mean of the G query heads' importances of KV head h_kv (q [B,S,H_q,d], k [B,S,H_kv,d])."""
    H_q, H_kv, d = q.shape[2], k.shape[2], q.shape[3]
    G = H_q // H_kv
    sc = 1.0 / np.sqrt(d) if scale is None else scale
    acc = None
    for g in range(G):
        a = head_importance(q[b, :, h_kv * G + g, :], k[b, :, h_kv, :], stride, block, sc)
        acc = a if acc is None else acc + a
    return acc / G


def row_importance(q, k, b: int, h_kv: int, qb: int, stride: int, block: int, scale: float | None = None,
                   q_first_row: int = 0):
    """A[qb, 0..qb] alone (steps 1-3 restricted to the reduced rows of query block qb, group
    mean over the G query heads); the same definition as group_importance, for sampled
    rows of long sequences.  q may hold only rows q_first_row.. of the sequence (it must
    include the rows of block qb); k holds rows 0.. (at least through block qb)."""
    H_q, d = q.shape[2], q.shape[3]
    S = k.shape[1]
    H_kv = k.shape[2]
    G = H_q // H_kv
    sc = (1.0 / np.sqrt(d) if scale is None else scale) / stride
    r = block // stride
    n = -(-S // stride)
    i_lo, i_hi = qb * r, min((qb + 1) * r, n)

    def reduced_rows(x, first, lo, hi):     # sequence rows lo*st .. hi*st-1 of x (row 0 = first), zero past S
        out = np.zeros(((hi - lo) * stride, d))
        top = min(hi * stride, S)
        out[:top - lo * stride] = x[lo * stride - first:top - first]
        return out.reshape(hi - lo, stride, d)

    A = np.zeros(qb + 1)
    kk = reduced_rows(np.asarray(k[b, :, h_kv, :], np.float64), 0, 0, i_hi)
    for g in range(G):
        qq = reduced_rows(np.asarray(q[b, :, h_kv * G + g, :], np.float64), q_first_row, i_lo, i_hi)
        R = np.zeros((i_hi - i_lo, i_hi))
        for m in range(stride):
            R += qq[:, m, :] @ kk[:, stride - 1 - m, :].T
        for t, i in enumerate(range(i_lo, i_hi)):
            s = sc * R[t, :i + 1]
            e = np.exp(s - s.max())
            p = e / e.sum()
            for kb in range(qb + 1):
                A[kb] += p[kb * r:(kb + 1) * r].sum()
    return A / G


def select_blocks(a_row: np.ndarray, qb: int, tau: float) -> np.ndarray:
    """Step 4 on one row of importances (entries 0..qb).  Returns the kept blocks, ascending."""
    a = np.asarray(a_row[:qb + 1], np.float64)
    need = tau * a.sum()
    kept = [qb]
    mass = a[qb]
    order = sorted(range(qb), key=lambda c: (-a[c], c))
    for c in order:
        if mass >= need:
            break
        kept.append(c)
        mass += a[c]
    return np.array(sorted(kept), dtype=np.int64)


def xattn_layout(q, k, head_mode, pattern, stride: int = 8, tau: float = 0.9, block: int = 128):
    """The CSR block layout for every (b, h_kv, query block): XAttention's selection where the
    head's kind under head_mode is BLOCK_SPARSE, an empty row elsewhere.

    Returns (row_ptr int64 [B*H_kv*n_qb + 1], cols int64, importance {(b, h_kv): A})."""
    B, S, H_q, d = q.shape
    H_kv = k.shape[2]
    n_qb = -(-S // block)
    sc = pattern.get("softmax_scale", 0.0) or None
    row_ptr = [0]
    cols = []
    imp = {}
    for b in range(B):
        for h in range(H_kv):
            kind = head_kind(head_mode, b, h, pattern["kind_if_dense"], pattern["kind_if_sparse"])
            if kind == BLOCK_SPARSE:
                A = group_importance(q, k, b, h, stride, block, sc)
                imp[(b, h)] = A
            for qb in range(n_qb):
                if kind == BLOCK_SPARSE:
                    cols.extend(select_blocks(A[qb], qb, tau).tolist())
                row_ptr.append(len(cols))
    return np.array(row_ptr, np.int64), np.array(cols, np.int64), imp
