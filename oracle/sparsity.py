"""Oracle: model and effective sparsity ratios — TEST INFRASTRUCTURE ONLY.

Source: "Elastic Attention: Test-time Adaptive Sparsity Ratios for Efficient
Transformers" (paperlayer.ai summary of arXiv 2601.17367v2):
  * section 2 "Sparsity Ratio Computation": Omega_MSR is the fraction of
    sparse heads; the effective sparsity Omega_ESR also accounts for the
    token pattern of those heads;
  * appendix C.1 "Sparsity Assignment": Omega_MSR is the proportion of heads
    switched to sparse attention.

Readings: Omega_MSR per sample = sparse KV heads / H_kv (every query head of
a group shares its KV head's decision, so the query-head fraction is the
same); Omega_ESR = 1 - (live query-key pairs) / (causal query-key pairs),
summed over all samples and query heads.  The tile counts use 128 x 128
tiles of (query rows, key columns): a tile is live when it holds at least one
live pair; live FLOPs = 4 * d * 128^2 per live tile per query head (the
QK^T and PV products a tensor-core kernel executes on it).
"""
from __future__ import annotations

import math

import numpy as np

from .attention import FULL, STREAMING, BLOCK_SPARSE, STREAMING_BLOCKS, head_kind, live_keys, csr_row

TILE = 128


def omega_msr(head_mode):
    """Per-sample fraction of sparse KV heads, and the batch mean."""
    m = (np.asarray(head_mode) != 0).astype(np.float64)
    per = m.mean(axis=1)
    return per, float(per.mean())


def row_live_counts_plain(S, kind, pattern, b=0, h_kv=0, H_kv=1):
    """|L(i)| for every row, straight from the live-key sets (O(S^2): small S only)."""
    return np.array([len(live_keys(i, kind, pattern, b, h_kv, H_kv, S)) for i in range(S)],
                    dtype=np.int64)


def row_live_counts(S, kind, pattern, b=0, h_kv=0, H_kv=1):
    """|L(i)| for every row, counted interval by interval (O(S + nnz)).

    FULL: i+1.  STREAMING: the window {max(0,i-W+1)..i} plus the sink keys
    below it.  BLOCK_SPARSE: whole listed blocks below the diagonal block,
    plus the causal part of the diagonal block."""
    i = np.arange(S, dtype=np.int64)
    if kind == FULL:
        return i + 1
    if kind == STREAMING:
        W, ns = int(pattern["window"]), int(pattern["n_sink"])
        return np.minimum(i + 1, W) + np.maximum(0, np.minimum(ns, i - W + 1))
    if kind == BLOCK_SPARSE:
        blk = int(pattern["block"])
        out = np.zeros(S, np.int64)
        for qb in range(-(-S // blk)):
            r0, r1 = qb * blk, min(S, (qb + 1) * blk)
            cols = csr_row(pattern, b, h_kv, qb, H_kv, S)
            below = int(np.sum(cols < qb)) * blk
            diag = (i[r0:r1] - r0 + 1) if np.any(cols == qb) else 0
            out[r0:r1] = below + diag
        return out
    if kind == STREAMING_BLOCKS:
        blk = int(pattern["block"])
        sb, lb = -(-int(pattern["n_sink"]) // blk), -(-int(pattern["window"]) // blk)
        local_start = np.maximum(0, i // blk - lb + 1) * blk        # first key of the local blocks
        return (i - local_start + 1) + np.maximum(0, np.minimum(sb * blk, local_start))
    raise ValueError(kind)


def tile_live_counts(S, kind, pattern, b=0, h_kv=0, H_kv=1):
    """Number of live 128-key tiles for every 128-row query tile."""
    n_qt = -(-S // TILE)
    out = np.zeros(n_qt, np.int64)
    for t in range(n_qt):
        r0, r1 = t * TILE, min(S, (t + 1) * TILE) - 1       # first and last row of the tile
        if kind == FULL:
            out[t] = t + 1
        elif kind == STREAMING:
            ns, W = int(pattern["n_sink"]), int(pattern["window"])
            sink = set(range(0, min(-(-ns // TILE), t + 1)))
            win = set(range(max(0, r0 - W + 1) // TILE, t + 1))
            out[t] = len(sink | win)
        elif kind == BLOCK_SPARSE:
            blk = int(pattern["block"])
            tiles = set()
            for qb in range(r0 // blk, r1 // blk + 1):
                hi_row = min(r1, (qb + 1) * blk - 1)
                for c in csr_row(pattern, b, h_kv, qb, H_kv, S):
                    k0, k1 = int(c) * blk, min(int(c) * blk + blk - 1, hi_row, S - 1)
                    if k0 <= k1:
                        tiles.update(range(k0 // TILE, k1 // TILE + 1))
            out[t] = len(tiles)
        elif kind == STREAMING_BLOCKS:
            tiles = set()
            for i in range(r0, r1 + 1):
                tiles.update(int(j) // TILE for j in live_keys(i, kind, pattern, b, h_kv, H_kv, S))
            out[t] = len(tiles)
        else:
            raise ValueError(kind)
    return out


def sparsity_report(head_mode, pattern, B, S, H_q, H_kv, d, plain=False):
    """Omega_MSR (per sample and mean), Omega_ESR and the live pair / tile / FLOP counts."""
    G = H_q // H_kv
    per, mean = omega_msr(head_mode)
    counts = row_live_counts_plain if plain else row_live_counts
    live_pairs = 0
    live_tiles = 0
    for b in range(B):
        for h in range(H_kv):
            kind = head_kind(head_mode, b, h, pattern["kind_if_dense"], pattern["kind_if_sparse"])
            live_pairs += G * int(counts(S, kind, pattern, b, h, H_kv).sum())
            live_tiles += G * int(tile_live_counts(S, kind, pattern, b, h, H_kv).sum())
    causal_pairs = B * H_q * S * (S + 1) // 2
    n_qt = math.ceil(S / TILE)
    causal_tiles = B * H_q * n_qt * (n_qt + 1) // 2
    return dict(omega_msr_per_sample=per, omega_msr_mean=mean,
                omega_esr=1.0 - live_pairs / causal_pairs,
                live_pairs=live_pairs, causal_pairs=causal_pairs,
                live_tiles=live_tiles, causal_tiles=causal_tiles,
                live_flops=4.0 * d * TILE * TILE * live_tiles)
