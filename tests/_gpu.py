"""Helpers for the GPU parity tests: device copies of the seeded inputs, calls
through the C ABI, and the oracle on the same inputs (sampled rows for the
full-size workloads)."""
import functools

import numpy as np
import torch

import oracle
import workloads as wl
from sparse_gqa_attention_b200 import abi

BF16_MAX_ABS, BF16_MEAN_ABS, F32_MAX_ABS = 2e-2, 2e-3, 1e-4


@functools.lru_cache(maxsize=1)
def cached_inputs(name: str):
    """(q, k, v, hidden, router weights) of a named workload, drawn once per process."""
    w = wl.WORKLOADS[name]
    q, k, v = wl.attention_inputs(w)
    return q, k, v, wl.hidden_states(w), wl.router_weights(w)


def to_dev(x: np.ndarray, dtype: str):
    if dtype == "bf16" and x.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def to_f64(x: np.ndarray):
    return (wl.f32_from_bf16_bits(x) if x.dtype == np.uint16 else x).astype(np.float64)


def pattern_dict(pat: wl.Pattern):
    return dict(n_sink=pat.n_sink, window=pat.window, block=pat.block, row_ptr=pat.row_ptr, cols=pat.cols,
                kind_if_dense=pat.kind_if_dense, kind_if_sparse=pat.kind_if_sparse,
                softmax_scale=pat.softmax_scale)


def sample_rows(w: wl.Workload, n_random=24, seed=7):
    S, ns, W = w.S, w.n_sink, w.window
    fixed = [0, 1, ns - 1, ns, W - 1, W, W + ns, S // 2, S - 1]
    fixed += [e for t in (0, 1) for e in (128 * t, 128 * t + 63, 128 * t + 64, 128 * t + 127)]
    rnd = np.random.default_rng([seed, S]).integers(0, S, n_random)
    return np.unique(np.clip(np.concatenate([fixed, rnd]), 0, S - 1))


def run_router(w, hidden_storage, weights, n_boundary=None):
    nb = w.n_boundary if n_boundary is None else n_boundary
    hm = torch.zeros(w.B, w.H_kv, dtype=torch.int32, device="cuda")
    z = torch.zeros(w.B, w.H_kv, dtype=torch.float32, device="cuda")
    ws = torch.zeros(abi.ea_router_workspace_size(w.B, w.S, w.D, w.H_kv, w.d, nb), dtype=torch.uint8, device="cuda")
    abi.ea_router(to_dev(hidden_storage, w.dtype), {k: to_dev(v, w.dtype) for k, v in weights.items()}, hm, ws,
                  nb, logits=z)
    torch.cuda.synchronize()
    return hm.cpu().numpy(), z.cpu().numpy()


def oracle_router(w, hidden_storage, weights, n_boundary=None):
    nb = w.n_boundary if n_boundary is None else n_boundary
    hw = dict(weights)
    hw["w_k"] = to_f64(weights["w_k"])
    h32 = wl.f32_from_bf16_bits(hidden_storage) if hidden_storage.dtype == np.uint16 else hidden_storage
    return oracle.router.router_forward(h32, hw, w.H_kv, w.d, nb)


def run_attention(w, q, k, v, head_mode: np.ndarray, pat: wl.Pattern, split=False, rows=None, check_finite=True):
    """Output rows (all, or ``rows``) as float64 numpy, and the workspace status."""
    dq, dk, dv = to_dev(q, w.dtype), to_dev(k, w.dtype), to_dev(v, w.dtype)
    o = torch.full_like(dq, float("nan"))
    ws = torch.zeros(abi.ea_attn_workspace_size(w.B, w.S, w.H_q, w.H_kv), dtype=torch.uint8, device="cuda")
    hm = torch.from_numpy(np.ascontiguousarray(head_mode, np.int32)).cuda()
    dpat = abi.Pattern.from_workloads(pat)
    if split:
        abi.ea_build_schedule(hm, dpat, w.B, w.S, w.H_q, w.H_kv, w.d, ws)
        abi.ea_attn_scheduled(dq, dk, dv, hm, dpat, o, ws)
    else:
        abi.ea_hybrid_attn_prefill(dq, dk, dv, hm, dpat, o, ws)
    torch.cuda.synchronize()
    status = abi.ea_workspace_status(ws)
    if check_finite:
        assert bool(torch.isfinite(o).all()), "non-finite attention output"
    sel = o if rows is None else o[:, torch.as_tensor(rows, device=o.device)]
    return sel.float().cpu().numpy().astype(np.float64), status


def oracle_attention(w, q, k, v, head_mode, pat, rows=None):
    pd = pattern_dict(pat)
    if rows is None:
        return oracle.attention.hybrid_attention(to_f64(q), to_f64(k), to_f64(v), head_mode, pd)
    return oracle.attention.hybrid_attention_rows(to_f64(q[:, rows]), to_f64(k), to_f64(v), head_mode, pd, rows,
                                                  q_row_index=rows)


def assert_close(got, ref, dtype, what=""):
    err = np.abs(got - ref)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    if dtype == "bf16":
        assert err.max() <= BF16_MAX_ABS and err.mean() <= BF16_MEAN_ABS, \
            f"{what}: max-abs {err.max():.3g} mean-abs {err.mean():.3g}"
    else:
        assert err.max() <= F32_MAX_ABS, f"{what}: max-abs {err.max():.3g}"
    return float(err.max()), float(err.mean())
