"""Oracle: static retrieval-head assignment over a layer stack, fp64 — TEST INFRASTRUCTURE ONLY.

Source: "Elastic Attention: Test-time Adaptive Sparsity Ratios for Efficient
Transformers" (paperlayer.ai summary of arXiv 2601.17367v2):
  * appendix C.1 "Retrieval Score Calculation": a needle is placed in a long
    haystack; the retrieval score S_{l,h} of head h in layer l is the
    attention mass that the last token puts on the needle positions;
  * appendix C.1 "Sparsity Assignment": heads are ranked by retrieval score;
    for a target Omega_MSR, the k = floor((1 - Omega_MSR) * L * H) highest
    scoring heads keep full attention and the others use streaming sparse
    attention;
  * section 2 "Sparsity Ratio Computation": Omega_MSR and Omega_ESR, here
    summed over every layer of the stack.

Readings (both sides take them): the needle is the contiguous span of key
positions [needle_begin, needle_end); the last token is row S-1 and attends
causally to every key; the assignment is per KV head (the unit the router
assigns, section 3 "Attention Router"), so a KV head's score is the mean of its
G query heads' scores over the probe samples; ties rank the lower flat index
(l * H_kv + h) first; k is computed in double precision exactly as written;
the whole-model Omega_ESR is 1 - (live pairs of all layers) / (causal pairs of
all layers), Omega_MSR per sample is its sparse KV heads over L * H_kv.
"""
from __future__ import annotations

import math

import numpy as np

from . import sparsity
from .attention import softmax_scale


def retrieval_score(q, k, b: int, h_q: int, needle_begin: int, needle_end: int, scale: float | None = None):
    """Attention mass of the last query row of head h_q (sample b) on keys [needle_begin, needle_end)."""
    S, H_q, d = q.shape[1], q.shape[2], q.shape[3]
    G = H_q // k.shape[2]
    sc = 1.0 / np.sqrt(d) if scale is None else scale
    s = sc * (np.asarray(k[b, :, h_q // G, :], np.float64) @ np.asarray(q[b, S - 1, h_q, :], np.float64))
    p = np.exp(s - s.max())
    p /= p.sum()
    return float(p[needle_begin:needle_end].sum())


def retrieval_scores(q, k, needle_begin: int, needle_end: int, scale: float | None = None) -> np.ndarray:
    """[B, H_q] retrieval scores of one layer."""
    B, H_q = q.shape[0], q.shape[2]
    return np.array([[retrieval_score(q, k, b, h, needle_begin, needle_end, scale) for h in range(H_q)]
                     for b in range(B)])


def kv_head_scores(scores: np.ndarray, H_kv: int) -> np.ndarray:
    """[L, B, H_q] per-query-head scores -> [L, H_kv]: mean over the samples and the G heads of a group."""
    L, B, H_q = scores.shape
    G = H_q // H_kv
    return np.asarray(scores, np.float64).reshape(L, B, H_kv, G).mean(axis=(1, 3))


def n_full_heads(L: int, H: int, omega_msr: float) -> int:
    """k = floor((1 - Omega_MSR) * L * H), in double precision as written."""
    return int(math.floor((1.0 - float(omega_msr)) * (L * H)))


def static_assignment(kv_scores: np.ndarray, omega_msr: float) -> np.ndarray:
    """[L, H_kv] head_mode: 0 (full) for the k best-scoring heads, 1 (sparse) for the rest."""
    L, H = kv_scores.shape
    k = n_full_heads(L, H, omega_msr)
    flat = np.asarray(kv_scores, np.float64).reshape(-1)
    order = sorted(range(L * H), key=lambda i: (-flat[i], i))
    mode = np.ones(L * H, np.int32)
    for i in order[:k]:
        mode[i] = 0
    return mode.reshape(L, H)


def model_sparsity(modes, pattern, B: int, S: int, H_q: int, H_kv: int, d: int) -> dict:
    """Whole-stack report for per-layer head_mode modes [L, B, H_kv] sharing one pattern."""
    modes = np.asarray(modes)
    L = modes.shape[0]
    reps = [sparsity.sparsity_report(modes[l], pattern, B, S, H_q, H_kv, d) for l in range(L)]
    live = sum(r["live_pairs"] for r in reps)
    causal = sum(r["causal_pairs"] for r in reps)
    tiles = sum(r["live_tiles"] for r in reps)
    per_sample = np.array([(modes[:, b, :] != 0).sum() / (L * H_kv) for b in range(B)])
    return {"omega_msr_per_sample": per_sample, "omega_msr_mean": float(per_sample.mean()),
            "omega_esr": 1.0 - live / causal, "live_pairs": int(live), "causal_pairs": int(causal),
            "live_tiles": int(tiles), "causal_tiles": int(sum(r["causal_tiles"] for r in reps)),
            "live_flops": float(sum(r["live_flops"] for r in reps))}


__all__ = ["retrieval_score", "retrieval_scores", "kv_head_scores", "n_full_heads", "static_assignment",
           "model_sparsity", "softmax_scale"]
