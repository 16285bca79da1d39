"""GPU parity of XAttention block selection (ea_xattn_block_select) against the oracle.

Block masses are compared element by element (fp32 on the GPU, fp64 in the oracle).
Block selection is a threshold decision taken on those masses, so where a row's
selection differs from the oracle's (masses within rounding of each other or of the
threshold) the test checks that the GPU's row is still a valid selection of the
oracle's masses: it keeps the diagonal, covers tau x the row total, takes blocks in
descending mass and is minimal, each within a tolerance of 1e-4 x the row total.
The selected layout is then fed to the attention kernel and its output compared with
the attention oracle on that same layout.
"""
import numpy as np
import pytest
import torch

import oracle.xattention as ox
import workloads as wl
from sparse_gqa_attention_b200 import abi
from tests import _gpu

pytestmark = pytest.mark.gpu

SMALL = ["small-xattn-g4-s2560", "small-xattn-g7-s1000", "small-xassa-g4-s1536"]
FULL_SIZE = ["qwen-g7-s64k-xattn", "llama3-8b-s32k-xassa", "qwen-g7-s64k-xattn-b64"]
SEL_TOL = 1e-4


def _mode(w):
    return wl.routing_targets(w)[2]


def run_xattn(w, q, k, head_mode, stride=None, tau=None, scores=True):
    st = w.stride if stride is None else stride
    ta = w.tau if tau is None else tau
    dq, dk = _gpu.to_dev(q, w.dtype), _gpu.to_dev(k, w.dtype)
    hm = torch.from_numpy(np.ascontiguousarray(head_mode, np.int32)).cuda()
    pat = abi.Pattern.for_xattn(w.B, w.S, w.H_kv, w.n_sink, w.window, w.kind_if_dense, w.kind_if_sparse,
                                block=w.block)
    ws = torch.zeros(abi.ea_xattn_workspace_size(w.B, w.S, w.H_q, w.H_kv, st, w.block), dtype=torch.uint8,
                     device="cuda")
    n_qb = -(-w.S // w.block)
    sc = torch.full((w.B, w.H_kv, n_qb, n_qb), float("nan"), device="cuda") if scores else None
    abi.ea_xattn_block_select(dq, dk, hm, pat, ws, st, ta, sc)
    torch.cuda.synchronize()
    status = abi.ea_workspace_status(ws)
    rp = pat.row_ptr.cpu().numpy().astype(np.int64)
    cols = pat.cols.cpu().numpy()[:rp[-1]].astype(np.int64)
    return rp, cols, (None if sc is None else sc.cpu().numpy().astype(np.float64)), status, pat


def _kinds(w, mode, b, h):
    return int(w.kind_if_sparse[h]) if mode[b, h] else int(w.kind_if_dense[h])


def check_row(got, a, qb, tau):
    """True if got equals the oracle's selection; else asserts that it is valid within SEL_TOL."""
    want = ox.select_blocks(a, qb, tau)
    if len(got) == len(want) and np.all(got == want):
        return True
    a = np.asarray(a[:qb + 1])
    tol = SEL_TOL * max(a.sum(), 1e-30)
    assert got[-1] == qb and np.all(np.diff(got) > 0) and got[0] >= 0, got
    need = tau * a.sum()
    mass = a[got].sum()
    assert mass >= need - tol, (qb, mass, need)
    nondiag = got[got != qb]
    if len(nondiag):
        assert mass - a[nondiag].min() < need + tol, (qb, mass, need)
        rest = np.setdiff1d(np.arange(qb), nondiag)
        if len(rest):
            assert a[rest].max() <= a[nondiag].min() + tol
    return False


def check_layout_shape(w, mode, rp, cols):
    n_qb = -(-w.S // w.block)
    assert rp[0] == 0 and np.all(np.diff(rp) >= 0)
    for b in range(w.B):
        for h in range(w.H_kv):
            for qb in range(n_qb):
                r = (b * w.H_kv + h) * n_qb + qb
                row = cols[rp[r]:rp[r + 1]]
                if _kinds(w, mode, b, h) == wl.BLOCK_SPARSE:
                    assert len(row) >= 1 and row[-1] == qb and np.all(np.diff(row) > 0) and row[0] >= 0
                else:
                    assert len(row) == 0


def _w(name, block=128):
    import dataclasses
    w = wl.WORKLOADS[name]
    return w if block == w.block else dataclasses.replace(w, block=block)


@pytest.mark.parametrize("name,block", [(n, 128) for n in SMALL] + [(n, 64) for n in SMALL])
def test_small_scores_and_selection(name, block):
    w = _w(name, block)
    q, k, v, _, _ = _gpu.cached_inputs(name)
    mode = _mode(w)
    rp, cols, sc, status, _ = run_xattn(w, q, k, mode)
    assert status == abi.EA_OK
    check_layout_shape(w, mode, rp, cols)
    qf, kf = _gpu.to_f64(q), _gpu.to_f64(k)
    n_qb = -(-w.S // w.block)
    exact = total = 0
    for b in range(w.B):
        for h in range(w.H_kv):
            if _kinds(w, mode, b, h) != wl.BLOCK_SPARSE:
                assert np.all(sc[b, h] == 0)
                continue
            A = ox.group_importance(qf, kf, b, h, w.stride, w.block)
            np.testing.assert_allclose(sc[b, h], A, rtol=1e-3, atol=2e-5 * w.block / w.stride)
            for qb in range(n_qb):
                r = (b * w.H_kv + h) * n_qb + qb
                exact += check_row(cols[rp[r]:rp[r + 1]], A[qb], qb, w.tau)
                total += 1
    assert total > 0 and exact >= 0.9 * total, (exact, total)


@pytest.mark.parametrize("stride", [4, 16])
def test_other_strides(stride):
    w = wl.WORKLOADS["small-xattn-g4-s2560"]
    q, k, v, _, _ = _gpu.cached_inputs(w.name)
    mode = _mode(w)
    rp, cols, sc, status, _ = run_xattn(w, q, k, mode, stride=stride)
    assert status == abi.EA_OK
    qf, kf = _gpu.to_f64(q), _gpu.to_f64(k)
    n_qb = -(-w.S // w.block)
    for b in range(w.B):
        for h in range(w.H_kv):
            if _kinds(w, mode, b, h) != wl.BLOCK_SPARSE:
                continue
            A = ox.group_importance(qf, kf, b, h, stride, w.block)
            np.testing.assert_allclose(sc[b, h], A, rtol=1e-3, atol=2e-5 * w.block / stride)
            for qb in range(n_qb):
                r = (b * w.H_kv + h) * n_qb + qb
                check_row(cols[rp[r]:rp[r + 1]], A[qb], qb, w.tau)


def test_tau_zero_keeps_only_the_diagonal():
    w = wl.WORKLOADS["small-xattn-g4-s2560"]
    q, k, _, _, _ = _gpu.cached_inputs(w.name)
    mode = _mode(w)
    rp, cols, _, status, _ = run_xattn(w, q, k, mode, tau=0.0, scores=False)
    assert status == abi.EA_OK
    n_qb = -(-w.S // w.block)
    for b in range(w.B):
        for h in range(w.H_kv):
            for qb in range(n_qb):
                r = (b * w.H_kv + h) * n_qb + qb
                row = cols[rp[r]:rp[r + 1]].tolist()
                assert row == ([qb] if _kinds(w, mode, b, h) == wl.BLOCK_SPARSE else [])


def test_tau_one_is_a_valid_full_cover():
    w = wl.WORKLOADS["small-xattn-g7-s1000"]
    q, k, _, _, _ = _gpu.cached_inputs(w.name)
    mode = _mode(w)
    rp, cols, sc, status, _ = run_xattn(w, q, k, mode, tau=1.0)
    assert status == abi.EA_OK
    qf, kf = _gpu.to_f64(q), _gpu.to_f64(k)
    n_qb = -(-w.S // w.block)
    for h in range(w.H_kv):
        if _kinds(w, mode, 0, h) != wl.BLOCK_SPARSE:
            continue
        A = ox.group_importance(qf, kf, 0, h, w.stride, w.block)
        for qb in range(n_qb):
            r = h * n_qb + qb
            check_row(cols[rp[r]:rp[r + 1]], A[qb], qb, 1.0)


def test_no_block_sparse_heads_gives_an_empty_layout():
    w = wl.WORKLOADS["small-xattn-g4-s2560"]
    q, k, _, _, _ = _gpu.cached_inputs(w.name)
    mode = np.zeros((w.B, w.H_kv), np.int32)           # every head takes its dense kind (FULL)
    rp, cols, sc, status, _ = run_xattn(w, q, k, mode)
    assert status == abi.EA_OK
    assert np.all(rp == 0) and len(cols) == 0 and np.all(sc == 0)


def test_bad_head_mode_is_reported():
    w = wl.WORKLOADS["small-xattn-g4-s2560"]
    q, k, _, _, _ = _gpu.cached_inputs(w.name)
    mode = _mode(w).copy()
    mode[0, 0] = 3
    _, _, _, status, _ = run_xattn(w, q, k, mode, scores=False)
    assert status == abi.EA_ERR_BAD_LAYOUT


@pytest.mark.parametrize("name,block", [(n, 128) for n in SMALL] + [(SMALL[0], 64), (SMALL[2], 64)])
def test_attention_over_the_selected_layout(name, block):
    """The device layout goes straight into the attention call (no host round trip); the
    output matches the attention oracle on that layout."""
    w = _w(name, block)
    q, k, v, _, _ = _gpu.cached_inputs(name)
    mode = _mode(w)
    rp, cols, _, status, dpat = run_xattn(w, q, k, mode, scores=False)
    assert status == abi.EA_OK
    dq, dk, dv = (_gpu.to_dev(x, w.dtype) for x in (q, k, v))
    o = torch.full_like(dq, float("nan"))
    ws = torch.zeros(abi.ea_attn_workspace_size(w.B, w.S, w.H_q, w.H_kv), dtype=torch.uint8, device="cuda")
    hm = torch.from_numpy(np.ascontiguousarray(mode, np.int32)).cuda()
    abi.ea_hybrid_attn_prefill(dq, dk, dv, hm, dpat, o, ws)
    torch.cuda.synchronize()
    assert abi.ea_workspace_status(ws) == abi.EA_OK
    pat = wl.pattern_for(w, layout=(rp.astype(np.int32), cols.astype(np.int32)))
    ref = _gpu.oracle_attention(w, q, k, v, mode, pat)
    _gpu.assert_close(o.float().cpu().numpy().astype(np.float64), ref, w.dtype, name)


@pytest.mark.slow
@pytest.mark.parametrize("name", FULL_SIZE)
def test_full_size_sampled(name):
    """The bench's configuration: sampled query blocks of every block-sparse head against the
    oracle's row masses, and sampled attention rows over the device layout."""
    w = wl.WORKLOADS[name]
    q, k, v, _, _ = _gpu.cached_inputs(name)
    mode = _mode(w)
    rp, cols, sc, status, dpat = run_xattn(w, q, k, mode)
    assert status == abi.EA_OK
    n_qb = -(-w.S // w.block)
    assert rp[0] == 0 and np.all(np.diff(rp) >= 0)
    rng = np.random.default_rng(3)
    qbs = np.unique(np.concatenate([[0, 1, n_qb // 2, n_qb - 1], rng.integers(0, n_qb, 4)]))
    for b in range(w.B):
        for h in range(w.H_kv):
            if _kinds(w, mode, b, h) != wl.BLOCK_SPARSE:
                continue
            for qb in qbs:
                lo, hi = qb * w.block, min((qb + 1) * w.block, w.S)
                kb_hi = hi
                qs = _gpu.to_f64(q[b:b + 1, :hi])
                ks = _gpu.to_f64(k[b:b + 1, :kb_hi])
                a = ox.row_importance(qs, ks, 0, h, qb, w.stride, w.block)
                np.testing.assert_allclose(sc[b, h, qb, :qb + 1], a, rtol=1e-3, atol=2e-5 * w.block / w.stride)
                r = (b * w.H_kv + h) * n_qb + qb
                check_row(cols[rp[r]:rp[r + 1]], a, qb, w.tau)
    # attention over the device layout, sampled rows
    dq, dk, dv = (_gpu.to_dev(x, w.dtype) for x in (q, k, v))
    o = torch.empty_like(dq)
    ws = torch.zeros(abi.ea_attn_workspace_size(w.B, w.S, w.H_q, w.H_kv), dtype=torch.uint8, device="cuda")
    hm = torch.from_numpy(np.ascontiguousarray(mode, np.int32)).cuda()
    abi.ea_hybrid_attn_prefill(dq, dk, dv, hm, dpat, o, ws)
    torch.cuda.synchronize()
    assert abi.ea_workspace_status(ws) == abi.EA_OK
    rows = _gpu.sample_rows(w, n_random=8)
    got = o[:, torch.as_tensor(rows, device=o.device)].float().cpu().numpy().astype(np.float64)
    del o, dq, dk, dv
    pat = wl.pattern_for(w, layout=(rp.astype(np.int32), cols.astype(np.int32)))
    ref = _gpu.oracle_attention(w, q, k, v, mode, pat, rows=rows)
    _gpu.assert_close(got, ref, w.dtype, name)
