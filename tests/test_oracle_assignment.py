"""Pins for the static retrieval-head assignment oracle (CPU, fp64).

The retrieval score is checked against torch's fp64 SDPA with an indicator value
vector (the last row's output is then the needle mass), closed forms (uniform
attention, a needle covering everything); the assignment against hand cases,
a brute-force ranking and its floor rule; the whole-stack sparsity against
brute-force counts of explicit masks.  Sources: "Elastic Attention:
Test-time Adaptive Sparsity Ratios for Efficient Transformers" (paperlayer.ai)
appendix C.1 "Retrieval Score Calculation" and "Sparsity Assignment",
section 2 "Sparsity Ratio Computation".
"""
import numpy as np
import pytest
import torch

import oracle.assignment as oas
from oracle.attention import FULL, STREAMING
from tests import _ref


def _sdpa_needle_mass(q, k, n0, n1):
    """Last-row output of SDPA (GQA) with v_j = 1 on the needle, 0 elsewhere."""
    B, S, H_q, d = q.shape
    H_kv = k.shape[2]
    v = np.zeros((B, S, H_kv, 1))
    v[:, n0:n1] = 1.0
    Q = torch.from_numpy(q[:, S - 1:S]).permute(0, 2, 1, 3)
    K = torch.from_numpy(k).permute(0, 2, 1, 3)
    V = torch.from_numpy(v).permute(0, 2, 1, 3)
    o = torch.nn.functional.scaled_dot_product_attention(Q, K, V, enable_gqa=H_q != H_kv)
    return o[:, :, 0, 0].numpy()           # [B, H_q]


@pytest.mark.parametrize("G,n0,n1", [(1, 10, 20), (4, 0, 1), (3, 57, 64), (2, 30, 31)])
def test_retrieval_score_is_the_sdpa_needle_mass(rng, G, n0, n1):
    B, S, H_kv, d = 2, 64, 2, 16
    q = rng.standard_normal((B, S, H_kv * G, d)) * 2
    k = rng.standard_normal((B, S, H_kv, d))
    np.testing.assert_allclose(oas.retrieval_scores(q, k, n0, n1), _sdpa_needle_mass(q, k, n0, n1), atol=1e-14)


def test_retrieval_score_closed_forms(rng):
    S, d = 50, 8
    q = np.zeros((1, S, 2, d))
    k = rng.standard_normal((1, S, 1, d))
    assert abs(oas.retrieval_score(q, k, 0, 1, 10, 17) - 7 / 50) < 1e-15      # uniform attention
    q = rng.standard_normal((1, S, 2, d))
    assert abs(oas.retrieval_score(q, k, 0, 0, 0, S) - 1.0) < 1e-14           # needle = everything
    assert oas.retrieval_score(q, k, 0, 0, 5, 5) == 0.0                        # empty needle
    # a key aligned with the last query row dominates
    k2 = k.copy()
    k2[0, 33, 0] = 40 * q[0, S - 1, 1] / np.linalg.norm(q[0, S - 1, 1])
    assert oas.retrieval_score(q, k2, 0, 1, 33, 34) > 0.999


def test_kv_head_scores_mean_over_samples_and_group():
    s = np.arange(3 * 4, dtype=np.float64).reshape(1, 3, 4)                   # L=1, B=3, H_q=4
    s = np.concatenate([s, 2 * s])                                            # L=2
    got = oas.kv_head_scores(s, 2)
    want0 = [np.mean([s[0, b, g] for b in range(3) for g in (0, 1)]), np.mean([s[0, b, g] for b in range(3) for g in (2, 3)])]
    np.testing.assert_allclose(got[0], want0)
    np.testing.assert_allclose(got[1], 2 * np.array(want0))


@pytest.mark.parametrize("L,H,omega,k", [(2, 5, 0.7, 3), (1, 7, 0.5, 3), (32, 8, 0.0, 256), (32, 8, 1.0, 0),
                                         (4, 8, 0.25, 24), (3, 3, 1 / 3, 6), (32, 8, 0.65, 89)])
def test_number_of_full_heads(L, H, omega, k):
    assert oas.n_full_heads(L, H, omega) == k


def test_assignment_hand_case_with_ties():
    sc = np.array([[0.9, 0.1, 0.5], [0.5, 0.05, 0.95]])       # flat: 0.9 0.1 0.5 0.5 0.05 0.95
    m = oas.static_assignment(sc, 0.5)                         # k = 3: 0.95, 0.9, then the first 0.5
    np.testing.assert_array_equal(m, [[0, 1, 0], [1, 1, 0]])


def test_assignment_against_brute_force_ranking(rng):
    for _ in range(200):
        L, H = int(rng.integers(1, 5)), int(rng.integers(1, 5))
        sc = np.round(rng.random((L, H)), 1)                   # many ties
        om = float(rng.random())
        m = oas.static_assignment(sc, om)
        k = int(np.floor((1 - om) * L * H))
        assert int((m == 0).sum()) == k
        flat, mf = sc.reshape(-1), m.reshape(-1)
        full = [i for i in range(L * H) if mf[i] == 0]
        rest = [i for i in range(L * H) if mf[i] == 1]
        for i in full:
            for j in rest:
                assert flat[i] > flat[j] or (flat[i] == flat[j] and i < j)


def _pattern(H_kv):
    return dict(n_sink=4, window=16, block=16, row_ptr=np.zeros(1, np.int32), cols=np.zeros(0, np.int32),
                kind_if_dense=[FULL] * H_kv, kind_if_sparse=[STREAMING] * H_kv)


def test_model_sparsity_against_mask_counts():
    L, B, S, H_kv, G, d = 3, 2, 100, 2, 2, 8
    modes = np.array([[[0, 1], [1, 1]], [[0, 0], [0, 0]], [[1, 0], [1, 1]]], np.int32)
    r = oas.model_sparsity(modes, _pattern(H_kv), B, S, H_kv * G, H_kv, d)
    full = int(_ref.causal_mask(S).sum())
    stream = int(_ref.streaming_mask(S, 4, 16).sum())
    live = sum(G * (stream if modes[l, b, h] else full) for l in range(L) for b in range(B) for h in range(H_kv))
    causal = L * B * H_kv * G * full
    assert r["live_pairs"] == live and r["causal_pairs"] == causal
    assert abs(r["omega_esr"] - (1 - live / causal)) < 1e-15
    np.testing.assert_allclose(r["omega_msr_per_sample"], [2 / 6, 4 / 6])


def test_identical_layers_match_one_layer():
    modes = np.array([[[0, 1, 1, 0]]] * 4, np.int32)
    one = oas.model_sparsity(modes[:1], _pattern(4), 1, 300, 8, 4, 64)
    four = oas.model_sparsity(modes, _pattern(4), 1, 300, 8, 4, 64)
    assert abs(one["omega_esr"] - four["omega_esr"]) < 1e-15 and four["live_pairs"] == 4 * one["live_pairs"]
    assert one["omega_msr_mean"] == four["omega_msr_mean"] == 0.5


# --- planted mistakes -------------------------------------------------------------------------

def test_ceil_instead_of_floor_is_caught(monkeypatch):
    import math
    monkeypatch.setattr(oas, "n_full_heads", lambda L, H, om: int(math.ceil((1.0 - om) * (L * H))))
    assert oas.n_full_heads(1, 7, 0.5) != 3


def test_ascending_rank_is_caught(monkeypatch):
    def bad(kv, om):
        L, H = kv.shape
        k = oas.n_full_heads(L, H, om)
        flat = kv.reshape(-1)
        order = sorted(range(L * H), key=lambda i: (flat[i], i))
        m = np.ones(L * H, np.int32)
        m[order[:k]] = 0
        return m.reshape(L, H)
    monkeypatch.setattr(oas, "static_assignment", bad)
    m = oas.static_assignment(np.array([[0.9, 0.1, 0.5], [0.5, 0.05, 0.95]]), 0.5)
    assert not np.array_equal(m, [[0, 1, 0], [1, 1, 0]])


def test_inclusive_needle_end_is_caught(rng, monkeypatch):
    q = rng.standard_normal((1, 40, 2, 8))
    k = rng.standard_normal((1, 40, 1, 8))
    orig = oas.retrieval_score
    monkeypatch.setattr(oas, "retrieval_score",
                        lambda q, k, b, h, n0, n1, scale=None: orig(q, k, b, h, n0, n1 + 1, scale))
    assert not np.allclose(oas.retrieval_scores(q, k, 5, 9), _sdpa_needle_mass(q, k, 5, 9), atol=1e-12)
