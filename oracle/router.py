"""Oracle: the Attention Router, fp64 — TEST INFRASTRUCTURE ONLY.

Source: "Elastic Attention: Test-time Adaptive Sparsity Ratios for Efficient
Transformers" (paperlayer.ai summary of arXiv 2601.17367v2):
  * section 3 "Attention Router": each key-value head gets a binary full /
    sparse assignment from head-wise logits computed from pooled key hidden
    states and task-aware representations; a task MLP infers the task, a
    router MLP picks FA or SA per head;
  * section 3 "Router Optimization" and appendix D.1 "Router Optimization":
    the forward pass is hard (straight-through), so inference thresholds the
    logit;
  * section 5 "Attention Router": MLP intermediate width x4 is the default;
  * section 1: the router adds 0.27M parameters per layer;
  * appendix H.4 "Router Input Length": the router pools the first and the
    last 100 tokens rather than the whole sequence.

Readings taken where the pages are silent (each pinned in
tests/test_oracle_router.py, except the last):
  * pooling is the mean over the pooling set; when S <= 2*n_boundary the set
    is every token once; n_boundary <= 0 selects the whole sequence;
  * the pooled key state of KV head h is p_h = W_k[:, h*d:(h+1)*d]^T hbar
    (pooling then projecting equals projecting then pooling, so both readings
    of "pooled key hidden states" agree; RoPE is not applied);
  * task MLP (shared by all heads): tau_h = W_t2 relu(W_t1 p_h + b_t1) + b_t2,
    d -> 4d -> d;
  * router MLP: u_h = relu(W_r1 [p_h; tau_h] + b_r1), 2d -> 4d (shared), then
    a per-head output row: z_h = w_o[h] . u_h + b_o[h];
  * z_h is the logit of "sparse": head_mode = 1 (sparse) iff z_h > 0;
  * parity unpinned: that this wiring is the paper's trained network.  With
    d = 128 and 8 KV heads it holds 267,400 parameters (the pages' 0.27M).
"""
from __future__ import annotations

import numpy as np


def pooling_rows(S: int, n_boundary: int) -> np.ndarray:
    """Token indices the router pools (appendix H.4: first and last n_boundary tokens)."""
    if n_boundary <= 0 or S <= 2 * n_boundary:
        return np.arange(S)
    return np.concatenate([np.arange(n_boundary), np.arange(S - n_boundary, S)])


def pool_hidden(hidden, n_boundary: int) -> np.ndarray:
    """hbar[b] = mean of hidden[b, t, :] over the pooling set, fp64 [B, D]."""
    hidden = np.asarray(hidden)
    rows = pooling_rows(hidden.shape[1], n_boundary)
    return hidden[:, rows, :].astype(np.float64).mean(axis=1)


def relu(x):
    return np.maximum(x, 0.0)


def router_param_count(d: int, H_kv: int) -> int:
    """Trainable parameters of the router as written here (the frozen W_k is not counted)."""
    task = 4 * d * d + 4 * d + d * 4 * d + d
    route = 4 * d * 2 * d + 4 * d
    out = H_kv * 4 * d + H_kv
    return task + route + out


def head_logits(hbar_b, w, H_kv: int, d: int) -> np.ndarray:
    """z[h] for one sample from its pooled hidden state hbar_b [D] (fp64)."""
    f = lambda a: np.asarray(a, dtype=np.float64)  # noqa: E731
    W_k = f(w["w_k"])
    assert W_k.shape == (hbar_b.shape[0], H_kv * d)
    z = np.empty(H_kv)
    for h in range(H_kv):
        p = W_k[:, h * d:(h + 1) * d].T @ hbar_b                       # pooled key state of head h
        tau = f(w["w_t2"]) @ relu(f(w["w_t1"]) @ p + f(w["b_t1"])) + f(w["b_t2"])   # task MLP
        u = relu(f(w["w_r1"]) @ np.concatenate([p, tau]) + f(w["b_r1"]))          # router MLP
        z[h] = f(w["w_o"])[h] @ u + f(w["b_o"])[h]                      # head-wise logit
    return z


def router_forward(hidden, w, H_kv: int, d: int, n_boundary: int = 100):
    """Router on hidden [B, S, D] (float values).  Returns (z [B, H_kv] fp64, head_mode int32)."""
    hbar = pool_hidden(hidden, n_boundary)
    z = np.stack([head_logits(hbar[b], w, H_kv, d) for b in range(hbar.shape[0])])
    return z, (z > 0).astype(np.int32)
