"""Pins for the XAttention block-selection oracle (CPU, fp64).

The oracle's steps are tied to things other than itself: a brute-force sum over
the antidiagonals of the full score matrix Q K^T (entry by entry), the stride-1
special case (plain Q K^T), a hand-derived fixture (uniform scores), brute-force
minimum-cardinality selection over all subsets, and the attention oracle's
full-causal case reached at tau = 1.  Sources: "Elastic Attention: Test-time
Adaptive Sparsity Ratios for Efficient Transformers" (paperlayer.ai) section 4
"Evaluation Setting" (XAttention, tau = 0.9), appendix D.1 "Sparse Inference";
the method restated from Xu et al., "XAttention: Block Sparse Attention with
Antidiagonal Scoring" (2025).
"""
import itertools
import json
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle.attention as oa
import oracle.xattention as ox
from tests import _ref

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _brute_reduced(q_h, k_h, st):
    """R[i, j] = sum of F[a, c] over the st x st sub-block (i, j) with (a - i*st) + (c - j*st) = st - 1,
    F = Q K^T over the real rows (rows past S count as zero)."""
    S = q_h.shape[0]
    F = q_h @ k_h.T
    n = -(-S // st)
    R = np.zeros((n, n))
    for i in range(n):
        for j in range(n):
            for a in range(st):
                c = st - 1 - a
                ra, rc = i * st + a, j * st + c
                if ra < S and rc < S:
                    R[i, j] += F[ra, rc]
    return R


@pytest.mark.parametrize("S,st", [(16, 2), (40, 8), (37, 4), (24, 1), (64, 16)])
def test_reduced_scores_are_antidiagonal_sums(rng, S, st):
    q = rng.standard_normal((S, 6))
    k = rng.standard_normal((S, 6))
    np.testing.assert_allclose(ox.reduced_scores(q, k, st), _brute_reduced(q, k, st), rtol=0, atol=1e-12)


def test_stride_one_is_plain_scores(rng):
    q, k = rng.standard_normal((20, 5)), rng.standard_normal((20, 5))
    np.testing.assert_allclose(ox.reduced_scores(q, k, 1), q @ k.T, atol=1e-12)


def test_reduced_softmax_is_causal_and_normalised(rng):
    R = rng.standard_normal((30, 30)) * 5
    P = ox.reduced_softmax(R, 0.7)
    assert np.all(np.triu(P, 1) == 0)
    np.testing.assert_allclose(P.sum(axis=1), 1.0, atol=1e-13)
    # each row is torch's softmax of its causal prefix
    import torch
    for i in (0, 7, 29):
        ref = torch.softmax(torch.tensor(0.7 * R[i, :i + 1], dtype=torch.float64), 0).numpy()
        np.testing.assert_allclose(P[i, :i + 1], ref, atol=1e-14)


def test_uniform_scores_golden():
    g = json.load(open(os.path.join(GOLDEN, "xattn_uniform.json")))
    S, st, blk = g["S"], g["stride"], g["block"]
    q = np.zeros((1, S, 1, 4))
    k = np.random.default_rng(5).standard_normal((1, S, 1, 4))
    A = ox.group_importance(q, k, 0, 0, st, blk)
    for qb, row in enumerate(g["importance_num_den"]):
        for kb, (num, den) in enumerate(row):
            assert abs(A[qb, kb] - num / den) < 1e-13
        assert sum(Fraction(n, d) for n, d in row) == Fraction(blk // st)
    for tau, rows in g["selected"].items():
        for qb, want in enumerate(rows):
            assert ox.select_blocks(A[qb], qb, float(tau)).tolist() == want, (tau, qb)


def test_block_rows_sum_to_reduced_rows(rng):
    S, st, blk = 96, 4, 16
    q, k = rng.standard_normal((1, S, 2, 8)), rng.standard_normal((1, S, 1, 8))
    A = ox.group_importance(q, k, 0, 0, st, blk)
    np.testing.assert_allclose(A.sum(axis=1), blk // st, atol=1e-12)
    assert np.all(np.triu(A, 1) == 0)


@pytest.mark.parametrize("row,qb,tau,want", [
    ([0.5, 0.05, 0.3, 0.15], 3, 0.9, [0, 2, 3]),
    ([0.5, 0.05, 0.3, 0.15], 3, 0.0, [3]),
    ([0.5, 0.05, 0.3, 0.15], 3, 1.0, [0, 1, 2, 3]),
    ([0.2, 0.2, 0.2, 0.4], 3, 0.7, [0, 1, 3]),
    ([0.9, 0.1], 1, 0.9, [0, 1]),
    ([0.1, 0.9], 1, 0.9, [1]),
    ([1.0], 0, 0.9, [0]),
])
def test_selection_hand_cases(row, qb, tau, want):
    assert ox.select_blocks(np.array(row), qb, tau).tolist() == want


def test_selection_is_a_minimum_covering_set(rng):
    for _ in range(300):
        n = int(rng.integers(1, 8))
        a = rng.random(n) ** 3
        tau = float(rng.random())
        qb = n - 1
        got = set(ox.select_blocks(a, qb, tau).tolist())
        need = tau * a.sum()
        # brute force: the fewest blocks (diagonal included) whose mass reaches tau x total
        best = None
        for r in range(0, qb + 1):
            for extra in itertools.combinations(range(qb), r):
                if a[qb] + a[list(extra)].sum() >= need:
                    best = r + 1
                    break
            if best is not None:
                break
        assert qb in got and len(got) == best
        assert a[list(got)].sum() >= need - 1e-15
        rest = [c for c in range(qb) if c not in got]
        kept = [c for c in got if c != qb]
        if rest and kept:
            assert max(a[rest]) <= min(a[kept])


def test_group_mean_and_head_order(rng):
    S, st, blk = 64, 8, 16
    q = rng.standard_normal((1, S, 3, 8))
    k = rng.standard_normal((1, S, 1, 8))
    per = [ox.head_importance(q[0, :, g], k[0, :, 0], st, blk, 1 / np.sqrt(8)) for g in range(3)]
    np.testing.assert_allclose(ox.group_importance(q, k, 0, 0, st, blk), sum(per) / 3, atol=1e-14)
    np.testing.assert_allclose(ox.group_importance(q[:, :, ::-1], k, 0, 0, st, blk),
                               ox.group_importance(q, k, 0, 0, st, blk), atol=1e-14)
    same = np.repeat(q[:, :, :1], 3, axis=2)
    np.testing.assert_allclose(ox.group_importance(same, k, 0, 0, st, blk), per[0], atol=1e-14)


def _pattern(H_kv, ks):
    return dict(n_sink=0, window=1, block=16, row_ptr=np.zeros(1, np.int32), cols=np.zeros(0, np.int32),
                kind_if_dense=[oa.FULL] * H_kv, kind_if_sparse=[ks] * H_kv)


def test_layout_rows_and_empty_rows(rng):
    B, S, H_kv, G, d = 2, 80, 2, 2, 8
    q = rng.standard_normal((B, S, H_kv * G, d))
    k = rng.standard_normal((B, S, H_kv, d))
    mode = np.array([[1, 0], [0, 1]], np.int32)
    rp, cols, imp = ox.xattn_layout(q, k, mode, _pattern(H_kv, oa.BLOCK_SPARSE), stride=4, tau=0.9, block=16)
    n_qb = 5
    assert set(imp) == {(0, 0), (1, 1)}
    for b in range(B):
        for h in range(H_kv):
            rows = _ref.csr_rows(rp, cols, b, h, H_kv, n_qb)
            for qb, r in enumerate(rows):
                if mode[b, h]:
                    assert r[-1] == qb and np.all(np.diff(r) > 0) and r[0] >= 0
                    assert r.tolist() == ox.select_blocks(imp[(b, h)][qb], qb, 0.9).tolist()
                else:
                    assert len(r) == 0


def test_tau_one_layout_gives_full_causal_attention(rng):
    """tau = 1 keeps every block of positive mass, i.e. all of them: attention over that layout is
    plain causal attention (torch fp64 SDPA)."""
    B, S, H_kv, G, d = 1, 48, 1, 2, 8
    q = rng.standard_normal((B, S, H_kv * G, d))
    k = rng.standard_normal((B, S, H_kv, d))
    v = rng.standard_normal((B, S, H_kv, d))
    p = _pattern(H_kv, oa.BLOCK_SPARSE)
    mode = np.ones((B, H_kv), np.int32)
    rp, cols, _ = ox.xattn_layout(q, k, mode, p, stride=4, tau=1.0, block=16)
    assert len(cols) == 3 * 4 // 2
    p.update(row_ptr=rp, cols=cols)
    o = oa.hybrid_attention(q, k, v, mode, p)
    np.testing.assert_allclose(o, _ref.sdpa(q, k, v, causal=True), atol=1e-12)


@pytest.mark.parametrize("S,st,blk,G", [(96, 4, 16, 2), (100, 4, 16, 3), (64, 8, 32, 1)])
def test_row_importance_matches_full_matrix(rng, S, st, blk, G):
    q = rng.standard_normal((1, S, 2 * G, 8))
    k = rng.standard_normal((1, S, 2, 8))
    full = ox.group_importance(q, k, 0, 1, st, blk)
    for qb in range(full.shape[0]):
        np.testing.assert_allclose(ox.row_importance(q, k, 0, 1, qb, st, blk), full[qb, :qb + 1], atol=1e-13)
        lo = qb * blk       # q given as the block's rows only
        np.testing.assert_allclose(ox.row_importance(q[:, lo:lo + blk], k, 0, 1, qb, st, blk, q_first_row=lo),
                                   full[qb, :qb + 1], atol=1e-13)


# --- planted mistakes must fail a pin -------------------------------------------------------

def _antidiag_pin_holds(rng):
    q, k = rng.standard_normal((32, 4)), rng.standard_normal((32, 4))
    return np.allclose(ox.reduced_scores(q, k, 4), _brute_reduced(q, k, 4), atol=1e-12)


def test_unreversed_key_rows_are_caught(rng, monkeypatch):
    def bad(q_h, k_h, stride):
        S, d = q_h.shape
        n = S // stride
        qq, kk = q_h.reshape(n, stride, d), k_h.reshape(n, stride, d)
        return sum(qq[:, m] @ kk[:, m].T for m in range(stride))   # main diagonal, not antidiagonal
    monkeypatch.setattr(ox, "reduced_scores", bad)
    assert not _antidiag_pin_holds(rng)


def test_dropped_stride_in_scale_is_caught(monkeypatch):
    g = json.load(open(os.path.join(GOLDEN, "xattn_uniform.json")))
    rng = np.random.default_rng(9)
    q = rng.standard_normal((1, 16, 1, 4))
    k = rng.standard_normal((1, 16, 1, 4))
    good = ox.group_importance(q, k, 0, 0, 2, 4)
    monkeypatch.setattr(ox, "head_importance",
                        lambda q_h, k_h, st, blk, sc: ox.block_importance(
                            ox.reduced_softmax(ox.reduced_scores(q_h, k_h, st), sc), st, blk))
    assert not np.allclose(ox.group_importance(q, k, 0, 0, 2, 4), good)
    # ... and with q = 0 the scale cannot matter: the golden values still hold
    A = ox.group_importance(np.zeros((1, 16, 1, 4)), k, 0, 0, 2, 4)
    assert abs(A[1, 0] - 7 / 6) < 1e-13 and len(g["selected"]) == 3


def test_selection_without_forced_diagonal_is_caught(monkeypatch):
    def bad(a_row, qb, tau):
        a = np.asarray(a_row[:qb + 1])
        need, kept, mass = tau * a.sum(), [], 0.0
        for c in sorted(range(qb + 1), key=lambda c: (-a[c], c)):
            if mass >= need:
                break
            kept.append(c)
            mass += a[c]
        return np.array(sorted(kept))
    monkeypatch.setattr(ox, "select_blocks", bad)
    g = json.load(open(os.path.join(GOLDEN, "xattn_uniform.json")))
    A = ox.group_importance(np.zeros((1, 16, 1, 4)), np.ones((1, 16, 1, 4)), 0, 0, 2, 4)
    got = [ox.select_blocks(A[qb], qb, 0.2).tolist() for qb in range(4)]
    assert got != g["selected"]["0.2"]
