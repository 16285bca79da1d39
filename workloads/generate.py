"""Seeded input generators for the Elastic Attention prefill path.

Everything here is a random draw, a dtype conversion of a draw, a shape, or (for
the workloads that ask for it) a fixed positional component added to the q/k
draws so that attention concentrates on nearby keys and a few sink keys, as it
does in trained models.
The workloads take the shapes of the layers the pages evaluate (Llama-3.1-8B
and Qwen3 attention layers, 8K-128K contexts; "Elastic Attention:
Test-time Adaptive Sparsity Ratios for Efficient Transformers", paperlayer.ai
summary, sections 4 "Training Data" and 4 "Length Extrapolation").  No
benchmark data set, trained router or backbone weight is used: every value is
drawn from numpy's PCG64 (``numpy.random.default_rng``) with an explicit seed.

Conventions shared with the C ABI and the oracle (an interface, not code):
  * head kinds: 0 = full causal attention, 1 = streaming (sink + local
    window), 2 = block-sparse, 3 = streaming at block granularity;
  * head_mode[b, h_kv]: 0 = the router's dense decision, 1 = sparse;
  * q, o: [B, S, H_q, d]; k, v: [B, S, H_kv, d]; hidden: [B, S, D]; all
    row-major.  Query head h_q reads KV head h_q // (H_q // H_kv).
  * block-sparse layout: CSR over rows r = (b * H_kv + h_kv) * n_qb + qb,
    columns (key block indices) sorted ascending and always holding the
    diagonal block qb.
"""
from __future__ import annotations

import dataclasses
import json
import math
import os
from typing import Optional, Sequence

import numpy as np

FULL, STREAMING, BLOCK_SPARSE, STREAMING_BLOCKS = 0, 1, 2, 3

# Stream ids keep the draws of different tensors independent of each other.
_SID_Q, _SID_K, _SID_V, _SID_HIDDEN, _SID_WK = 11, 12, 13, 14, 15
_SID_MLP, _SID_ROUTE, _SID_LAYOUT, _SID_SINK, _SID_PROBE = 16, 17, 18, 19, 20
_ROW_CHUNK = 1024

_TUNING_PATH = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                            "tests", "golden", "router_tuning.json")


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    S: int
    D: int
    H_q: int
    H_kv: int
    d: int
    dtype: str                      # "f32" or "bf16"
    n_sink: int
    window: int
    block: int
    density: float                  # extra key blocks per query block, as a fraction of qb+1
    kind_if_dense: tuple
    kind_if_sparse: tuple
    routing: tuple                  # ("fixed", n_sparse) or ("per_sample", (k_0, .., k_{B-1}))
    n_boundary: int = 100
    seed: int = 0
    note: str = ""
    layout: str = "random"          # "random": block_layout(); "xattn": selected by XAttention
    stride: int = 8                 # XAttention antidiagonal stride
    tau: float = 0.9                # XAttention threshold
    pos_amp: float = 0.0            # amplitude of the positional component of q and k
    sink_amp: float = 0.0           # amplitude of the sink direction (all q rows, the first 4 k rows)
    layers: int = 1                 # > 1: a stack with static retrieval-head assignment
    needle: tuple = (0, 0)          # retrieval probe needle span [begin, end)
    omega_static: float = 0.5       # target Omega_MSR of the static assignment

    @property
    def G(self) -> int:
        return self.H_q // self.H_kv


def _w(name, B, S, D, H_q, H_kv, d, dtype, n_sink, window, kinds_sparse, routing,
       block=128, density=0.1, note="", kinds_dense=None, **extra):
    return Workload(name=name, B=B, S=S, D=D, H_q=H_q, H_kv=H_kv, d=d, dtype=dtype,
                    n_sink=n_sink, window=window, block=block, density=density,
                    kind_if_dense=(FULL,) * H_kv if kinds_dense is None else tuple(kinds_dense),
                    kind_if_sparse=tuple(kinds_sparse), routing=routing, note=note, **extra)


# Amplitudes: at S = 32k-64k XAttention (stride 8, tau 0.9) then keeps ~5-15 % of the causal blocks,
# most query blocks only their diagonal and some tens of blocks; the small parity cases use a
# weaker positional component so that their selections are not all diagonal.
_XA = dict(layout="xattn", sink_amp=10.0)


_ALT = lambda H: tuple(STREAMING if h % 2 == 0 else BLOCK_SPARSE for h in range(H))  # noqa: E731

WORKLOADS = {w.name: w for w in [
    # The five layer shapes the measurements are quoted on.
    _w("tiny-fp32-s512", 1, 512, 512, 8, 2, 64, "f32", 16, 128, (STREAMING,) * 2, ("fixed", 1),
       note="one KV head streaming (sink 16, window 128), one full"),
    _w("llama3-8b-s32k-streaming", 1, 32768, 4096, 32, 8, 128, "bf16", 128, 2048,
       (STREAMING,) * 8, ("fixed", 4), note="Llama-3.1-8B layer, Omega_MSR = 50%"),
    _w("qwen-g7-s64k-blocksparse", 1, 65536, 3584, 28, 4, 128, "bf16", 128, 2048,
       (BLOCK_SPARSE,) * 4, ("fixed", 2),
       note="Qwen-style GQA (G=7), 128x128 blocks: first + diagonal + 10% of causal blocks"),
    _w("llama3-8b-s128k-sweep", 1, 131072, 4096, 32, 8, 128, "bf16", 128, 4096,
       (STREAMING,) * 8, ("fixed", 4), note="Omega_MSR sweep; head_mode forced in the sweep"),
    _w("llama3-8b-b4-s16k-mixed", 4, 16384, 4096, 32, 8, 128, "bf16", 128, 2048,
       _ALT(8), ("per_sample", (2, 3, 5, 6)),
       note="per-sample routing 25-75%; even KV heads streaming, odd block-sparse"),
    # Small cases for element-wise parity against the oracle (several tiles, ragged tails).
    _w("small-mixed-g4-s1000", 2, 1000, 256, 8, 2, 128, "bf16", 64, 300,
       (STREAMING, BLOCK_SPARSE), ("per_sample", (1, 2)), density=0.3),
    _w("small-bsa-g7-s777", 1, 777, 384, 14, 2, 128, "bf16", 0, 1,
       (BLOCK_SPARSE,) * 2, ("fixed", 1), density=0.3),
    _w("small-stream-g1-s700", 1, 700, 256, 4, 4, 128, "bf16", 130, 257,
       (STREAMING,) * 4, ("per_sample", (2,))),
    _w("small-fp32-d128-s300", 2, 300, 256, 4, 2, 128, "f32", 5, 64,
       (STREAMING, BLOCK_SPARSE), ("per_sample", (1, 2)), density=0.5),
    # Streaming at block granularity (sink and local-window blocks of 128 keys).
    _w("small-blockstream-g4-s900", 2, 900, 256, 8, 2, 128, "bf16", 128, 256,
       (STREAMING_BLOCKS, BLOCK_SPARSE), ("per_sample", (1, 2)), density=0.3),
    _w("small-fp32-blockstream-s400", 1, 400, 256, 4, 2, 64, "f32", 100, 129,
       (STREAMING_BLOCKS, STREAMING), ("fixed", 1)),
    _w("llama3-8b-s32k-blockstream", 1, 32768, 4096, 32, 8, 128, "bf16", 128, 2048,
       (STREAMING_BLOCKS,) * 8, ("fixed", 4),
       note="the Llama layer with streaming heads at block granularity (1 sink block, 16 local blocks)"),
    # XAttention block selection feeding the block-sparse heads (q/k with local + sink structure).
    _w("qwen-g7-s64k-xattn", 1, 65536, 3584, 28, 4, 128, "bf16", 128, 2048, (BLOCK_SPARSE,) * 4,
       ("fixed", 2), note="FA-XA: dense heads full, sparse heads XAttention (stride 8, tau 0.9)", pos_amp=1.8,
       **_XA),
    _w("qwen-g7-s64k-xattn-b64", 1, 65536, 3584, 28, 4, 128, "bf16", 128, 2048, (BLOCK_SPARSE,) * 4,
       ("fixed", 2), block=64, pos_amp=1.8,
       note="FA-XA with XAttention selecting 64-key blocks (the pages' block edge)", **_XA),
    _w("llama3-8b-s32k-xassa", 1, 32768, 4096, 32, 8, 128, "bf16", 128, 2048, (STREAMING,) * 8,
       ("fixed", 4), kinds_dense=(BLOCK_SPARSE,) * 8,
       note="XA-SSA: dense heads XAttention (stride 8, tau 0.9), sparse heads streaming", pos_amp=1.7, **_XA),
    # The pages' block edge, 64 (appendix D.1): block-sparse and block-granular streaming heads.
    _w("small-b64-g4-s1000", 2, 1000, 256, 8, 2, 128, "bf16", 128, 300, (STREAMING_BLOCKS, BLOCK_SPARSE),
       ("per_sample", (1, 2)), block=64, density=0.3),
    _w("small-b64-g7-s777", 1, 777, 384, 14, 2, 128, "bf16", 0, 1, (BLOCK_SPARSE,) * 2, ("fixed", 1),
       block=64, density=0.3),
    _w("small-fp32-b64-s700", 2, 700, 256, 4, 2, 64, "f32", 100, 129, (BLOCK_SPARSE, STREAMING_BLOCKS),
       ("per_sample", (1, 2)), block=64, density=0.4),
    _w("qwen-g7-s64k-blocksparse-b64", 1, 65536, 3584, 28, 4, 128, "bf16", 128, 2048, (BLOCK_SPARSE,) * 4,
       ("fixed", 2), block=64, note="config 3 at the pages' block edge 64: first + diagonal + 10% of causal blocks"),
    _w("llama3-8b-s32k-blockstream-b64", 1, 32768, 4096, 32, 8, 128, "bf16", 128, 2048,
       (STREAMING_BLOCKS,) * 8, ("fixed", 4), block=64,
       note="the Llama layer with streaming heads at 64-key blocks (2 sink blocks, 32 local blocks)"),
    # Static retrieval-head assignment over a stack of layers (probe q/k per layer, shared v).
    _w("llama3-8b-s32k-stack8", 1, 32768, 4096, 32, 8, 128, "bf16", 128, 2048, (STREAMING,) * 8,
       ("fixed", 4), layers=8, needle=(16384, 16448), omega_static=0.5,
       note="8 layers; k = floor(0.5 * 8 * 8) = 32 KV heads keep full attention, 32 stream"),
    _w("small-stack3-s1000", 1, 1000, 256, 8, 2, 128, "bf16", 64, 300, (STREAMING,) * 2, ("fixed", 1),
       layers=3, needle=(400, 432), omega_static=0.5, note="3 small layers with static assignment"),
    _w("small-xattn-g4-s2560", 2, 2560, 256, 8, 2, 128, "bf16", 64, 300, (BLOCK_SPARSE,) * 2,
       ("per_sample", (1, 2)), pos_amp=1.5, **_XA),
    _w("small-xattn-g7-s1000", 1, 1000, 384, 14, 2, 128, "bf16", 0, 1, (BLOCK_SPARSE,) * 2,
       ("fixed", 1), pos_amp=1.5, **_XA),
    _w("small-xassa-g4-s1536", 1, 1536, 256, 8, 2, 128, "bf16", 128, 256, (STREAMING,) * 2,
       ("fixed", 1), kinds_dense=(BLOCK_SPARSE,) * 2, pos_amp=1.5, **_XA),
]}


@dataclasses.dataclass
class Pattern:
    """Per-head sparse patterns, in the form the ABI's ea_pattern_params takes."""
    n_sink: int
    window: int
    block: int
    row_ptr: np.ndarray         # int32 [B*H_kv*n_qb + 1]
    cols: np.ndarray            # int32 [nnz]
    kind_if_dense: np.ndarray   # int8 [H_kv]
    kind_if_sparse: np.ndarray  # int8 [H_kv]
    softmax_scale: float = 0.0  # 0 means 1/sqrt(d)


# ---------------------------------------------------------------------------
# dtype helpers (conversions of draws; no arithmetic of the method)
# ---------------------------------------------------------------------------

def bf16_bits_from_f32(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (round to nearest even); return the bits as uint16."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def f32_from_bf16_bits(u: np.ndarray) -> np.ndarray:
    """Widen bfloat16 bits (uint16) to float32 exactly."""
    return (np.asarray(u, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _storage(x32: np.ndarray, dtype: str) -> np.ndarray:
    return bf16_bits_from_f32(x32) if dtype == "bf16" else np.ascontiguousarray(x32, np.float32)


def _rng(*parts) -> np.random.Generator:
    return np.random.default_rng([int(p) for p in parts])


def _row_chunked_normal(seed, sid, b, S, row_shape, rows: Optional[np.ndarray] = None) -> np.ndarray:
    """N(0,1) float32 of shape [S, *row_shape] (or only the given rows), drawn in 1024-row chunks."""
    if rows is None:
        out = np.empty((S,) + tuple(row_shape), np.float32)
        for c0 in range(0, S, _ROW_CHUNK):
            n = min(_ROW_CHUNK, S - c0)
            out[c0:c0 + n] = _rng(seed, sid, b, c0 // _ROW_CHUNK).standard_normal(
                (n,) + tuple(row_shape), dtype=np.float32)
        return out
    rows = np.asarray(rows, dtype=np.int64)
    out = np.empty((len(rows),) + tuple(row_shape), np.float32)
    for c in np.unique(rows // _ROW_CHUNK):
        c0 = int(c) * _ROW_CHUNK
        n = min(_ROW_CHUNK, S - c0)
        chunk = _rng(seed, sid, b, c).standard_normal((n,) + tuple(row_shape), dtype=np.float32)
        sel = np.nonzero(rows // _ROW_CHUNK == c)[0]
        out[sel] = chunk[rows[sel] - c0]
    return out


# ---------------------------------------------------------------------------
# attention inputs
# ---------------------------------------------------------------------------

def positional_component(rows: np.ndarray, d: int) -> np.ndarray:
    """[len(rows), d] float32: (cos, sin) pairs of the row index at d/2 frequencies whose
    periods run geometrically from 8 to 1024 positions.  Added to q and k with the same
    amplitude, it raises q_i . k_j when |i - j| is small (within a few hundred positions)."""
    rows = np.asarray(rows, np.float64)
    f = np.arange(d // 2, dtype=np.float64)
    period = 8.0 * (128.0 ** (f / max(d // 2 - 1, 1)))
    ang = rows[:, None] * (2.0 * np.pi / period)[None, :]
    out = np.empty((len(rows), d), np.float64)
    out[:, 0::2] = np.cos(ang)
    out[:, 1::2] = np.sin(ang)
    return out.astype(np.float32)


def _sink_direction(w: Workload) -> np.ndarray:
    v = _rng(w.seed, _SID_SINK).standard_normal(w.d)
    return (v / np.linalg.norm(v)).astype(np.float32)


def _structured(x: np.ndarray, rows: np.ndarray, w: Workload, is_key: bool) -> np.ndarray:
    """x [n, H, d] plus the positional component (both q and k) and the sink direction (every q
    row; k rows 0..3)."""
    if w.pos_amp == 0.0 and w.sink_amp == 0.0:
        return x
    out = x + np.float32(w.pos_amp) * positional_component(rows, w.d)[:, None, :]
    if w.sink_amp != 0.0:
        s = np.float32(w.sink_amp) * _sink_direction(w)
        if is_key:
            out[np.asarray(rows) < 4] += s
        else:
            out += s
    return out


def attention_inputs(w: Workload, batches: Optional[Sequence[int]] = None, q_rows=None):
    """q, k, v ~ N(0,1) in storage form (uint16 bf16 bits, or float32); workloads with
    pos_amp / sink_amp add the structured components of ``_structured`` to q and k.

    ``batches`` restricts the draw to some samples (the arrays then hold only
    those); ``q_rows`` restricts q to some rows (k and v stay whole)."""
    bs = list(range(w.B)) if batches is None else list(batches)
    all_rows = np.arange(w.S)
    qr = all_rows if q_rows is None else np.asarray(q_rows, np.int64)
    qs, ks, vs = [], [], []
    for b in bs:
        q = _structured(_row_chunked_normal(w.seed, _SID_Q, b, w.S, (w.H_q, w.d), q_rows), qr, w, False)
        k = _structured(_row_chunked_normal(w.seed, _SID_K, b, w.S, (w.H_kv, w.d)), all_rows, w, True)
        qs.append(_storage(q, w.dtype))
        ks.append(_storage(k, w.dtype))
        vs.append(_storage(_row_chunked_normal(w.seed, _SID_V, b, w.S, (w.H_kv, w.d)), w.dtype))
    return np.stack(qs), np.stack(ks), np.stack(vs)


# ---------------------------------------------------------------------------
# routing targets, router weights and hidden states
# ---------------------------------------------------------------------------

def routing_targets(w: Workload):
    """Per-sample hidden-state scales alpha[b] and per-head thresholds t[h].

    With the tuned router the logit of head h on sample b is alpha[b] - t[h]
    (up to the bf16 rounding of the scaled hidden states), so the intended
    decision is alpha[b] > t[h].  Returns (alpha [B], t [H_kv], intended
    head_mode [B, H_kv] int32)."""
    H = w.H_kv
    perm = _rng(w.seed, _SID_ROUTE).permutation(H)
    kind, arg = w.routing
    if kind == "fixed":
        sparse = set(int(h) for h in perm[:arg])
        t = np.array([0.5 if h in sparse else 1.5 for h in range(H)], np.float64)
        alpha = np.ones(w.B, np.float64)
    elif kind == "per_sample":
        ks = list(arg)
        assert len(ks) == w.B
        steps = np.array([0.5 + 1.5 * r / max(H - 1, 1) for r in range(H)])  # thresholds by rank
        t = np.empty(H)
        t[perm] = steps
        alpha = np.empty(w.B)
        for b, k in enumerate(ks):
            if k <= 0:
                alpha[b] = steps[0] / 2
            elif k >= H:
                alpha[b] = steps[-1] + 0.5
            else:
                alpha[b] = 0.5 * (steps[k - 1] + steps[k])
    else:
        raise ValueError(kind)
    mode = (alpha[:, None] > t[None, :]).astype(np.int32)
    return alpha, t, mode


def load_router_tuning():
    """The per-head raw router scores g_ref[h] that tests/golden/make_router_tuning.py
    computed with the oracle; the tuning below divides each output row by its score."""
    with open(_TUNING_PATH) as f:
        return json.load(f)


def router_weights(w: Workload, tuned: bool = True, tuning=None):
    """Router weights in the ABI's layouts.

    W_k [D, H_kv*d] (frozen key projection, storage dtype of the hidden
    states); task MLP w_t1 [4d, d], b_t1 [4d], w_t2 [d, 4d], b_t2 [d]; router
    MLP w_r1 [4d, 2d], b_r1 [4d]; per-head output w_o [H_kv, 4d], b_o [H_kv];
    all MLP weights float32, drawn N(0, 0.02) with zero inner biases.  The
    output rows are drawn as |N(0, 0.02)|.  ``tuned`` rescales output row h by
    1/g_ref[h] and sets b_o[h] = -t[h] (see ``routing_targets``)."""
    D, H, d = w.D, w.H_kv, w.d
    r = _rng(w.seed, _SID_WK)
    wk = _storage(0.02 * r.standard_normal((D, H * d), dtype=np.float32), w.dtype)
    r = _rng(w.seed, _SID_MLP)
    out = dict(
        w_k=wk,
        w_t1=(0.02 * r.standard_normal((4 * d, d))).astype(np.float32),
        b_t1=np.zeros(4 * d, np.float32),
        w_t2=(0.02 * r.standard_normal((d, 4 * d))).astype(np.float32),
        b_t2=np.zeros(d, np.float32),
        w_r1=(0.02 * r.standard_normal((4 * d, 2 * d))).astype(np.float32),
        b_r1=np.zeros(4 * d, np.float32),
        w_o=np.abs(0.02 * r.standard_normal((H, 4 * d))).astype(np.float32),
        b_o=np.zeros(H, np.float32),
    )
    if tuned:
        tuning = load_router_tuning() if tuning is None else tuning
        g_ref = np.asarray(tuning[w.name]["g_ref"], np.float64)
        _, t, _ = routing_targets(w)
        out["w_o"] = (out["w_o"].astype(np.float64) / g_ref[:, None]).astype(np.float32)
        out["b_o"] = (-t).astype(np.float32)
    return out


def hidden_states(w: Workload, tuned: bool = True, rows=None):
    """hidden[b] = alpha[b] * base with base ~ N(0,1) [S, D], in storage dtype.

    All samples share one base draw, so a tuned router's logits move with
    alpha[b] alone.  ``rows`` restricts the draw to some rows."""
    alpha = routing_targets(w)[0] if tuned else np.ones(w.B)
    base = _row_chunked_normal(w.seed, _SID_HIDDEN, 0, w.S, (w.D,), rows)
    out = [_storage((np.float32(a) * base) if a != 1.0 else base, w.dtype) for a in alpha]
    return np.stack(out)


# ---------------------------------------------------------------------------
# block-sparse layout and pattern
# ---------------------------------------------------------------------------

def block_layout(w: Workload):
    """Seeded block layout: for query block qb keep block 0, block qb and
    floor(density*(qb+1)) further blocks drawn without replacement from
    1..qb-1.  Returns (row_ptr int32, cols int32)."""
    n_qb = math.ceil(w.S / w.block)
    rows = []
    for b in range(w.B):
        for h in range(w.H_kv):
            r = _rng(w.seed, _SID_LAYOUT, b, h)
            for qb in range(n_qb):
                extra = min(int(math.floor(w.density * (qb + 1))), max(qb - 1, 0))
                picked = r.choice(np.arange(1, qb), size=extra, replace=False) if extra > 0 else []
                rows.append(np.unique(np.concatenate([[0, qb], np.asarray(picked, np.int64)])))
    lens = np.array([len(x) for x in rows], np.int64)
    row_ptr = np.zeros(len(rows) + 1, np.int64)
    np.cumsum(lens, out=row_ptr[1:])
    assert row_ptr[-1] < 2**31
    cols = np.concatenate(rows).astype(np.int32) if rows else np.zeros(0, np.int32)
    return row_ptr.astype(np.int32), cols


def pattern_for(w: Workload, layout=None) -> Pattern:
    row_ptr, cols = block_layout(w) if layout is None else layout
    return Pattern(n_sink=w.n_sink, window=w.window, block=w.block, row_ptr=row_ptr, cols=cols,
                   kind_if_dense=np.asarray(w.kind_if_dense, np.int8),
                   kind_if_sparse=np.asarray(w.kind_if_sparse, np.int8))


def probe_layer_inputs(w: Workload, layer: int, needle=(0, 0), amp: float = 6.0):
    """q, k of one layer of a retrieval probe (appendix C.1 "Retrieval Score Calculation"): the
    workload's q/k draws for seed (w.seed, layer), plus, for each KV head h, a unit direction u
    added with amplitude amp to the keys of the needle span and with amplitude amp * a[h] to the
    last query row of every query head of the group; the per-head affinities a[h] ~ U(0, 1.5) make
    the heads' needle masses differ.  Storage form like attention_inputs."""
    import dataclasses as _dc
    wl_ = _dc.replace(w, seed=w.seed * 1000 + layer + 1)
    q, k, _ = attention_inputs(wl_)
    q = f32_from_bf16_bits(q) if q.dtype == np.uint16 else q.copy()
    k = f32_from_bf16_bits(k) if k.dtype == np.uint16 else k.copy()
    r = _rng(w.seed, _SID_PROBE, layer)
    aff = r.uniform(0.0, 1.5, w.H_kv)
    G = w.H_q // w.H_kv
    n0, n1 = needle
    for h in range(w.H_kv):
        u = r.standard_normal(w.d)
        u = (u / np.linalg.norm(u)).astype(np.float32)
        k[:, n0:n1, h, :] += np.float32(amp) * u
        q[:, w.S - 1, h * G:(h + 1) * G, :] += np.float32(amp * aff[h]) * u
    return _storage(q, w.dtype), _storage(k, w.dtype)


def forced_head_mode(w: Workload, n_sparse: int) -> np.ndarray:
    """head_mode with the first n_sparse KV heads sparse in every sample."""
    m = np.zeros((w.B, w.H_kv), np.int32)
    m[:, :n_sparse] = 1
    return m
