"""Pins for the router oracle (CPU, fp64).

Sources: "Elastic Attention: Test-time Adaptive Sparsity Ratios for Efficient
Transformers" (paperlayer.ai) section 1 (0.27M router parameters per layer),
section 3 "Attention Router", section 5 "Attention Router" (x4 width),
appendix H.4 "Router Input Length" (first and last 100 tokens).
"""
import json
import os

import numpy as np
import pytest

import oracle.router as orr
import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_parameter_count_matches_pages_budget():
    n = orr.router_param_count(128, 8)
    assert n == 267_400
    assert round(n / 1e6, 2) == 0.27
    w = wl.WORKLOADS["llama3-8b-s32k-streaming"]
    arrays = wl.router_weights(w, tuned=False)
    assert sum(a.size for key, a in arrays.items() if key != "w_k") == n


def test_pooling_rows_boundary_and_full():
    r = orr.pooling_rows(1000, 100)
    assert list(r) == list(range(100)) + list(range(900, 1000))
    assert list(orr.pooling_rows(200, 100)) == list(range(200))
    assert list(orr.pooling_rows(150, 100)) == list(range(150))
    assert list(orr.pooling_rows(1000, 0)) == list(range(1000))
    assert list(orr.pooling_rows(7, -1)) == list(range(7))


@pytest.mark.parametrize("S,nb", [(7, 2), (4, 2), (9, 0), (30, 3)])
def test_pooling_brute_force(rng, S, nb):
    h = rng.standard_normal((2, S, 5))
    got = orr.pool_hidden(h, nb)
    for b in range(2):
        acc, cnt = np.zeros(5), 0
        for t in range(S):
            if nb <= 0 or S <= 2 * nb or t < nb or t >= S - nb:
                acc += h[b, t]
                cnt += 1
        np.testing.assert_allclose(got[b], acc / cnt, rtol=0, atol=1e-14)


def test_pooling_constant_and_linear(rng):
    c = rng.standard_normal(6)
    h = np.broadcast_to(c, (1, 500, 6))
    np.testing.assert_allclose(orr.pool_hidden(h, 100)[0], c, atol=1e-14)
    a, b = rng.standard_normal((1, 500, 6)), rng.standard_normal((1, 500, 6))
    np.testing.assert_allclose(orr.pool_hidden(2 * a - 3 * b, 100),
                               2 * orr.pool_hidden(a, 100) - 3 * orr.pool_hidden(b, 100), atol=1e-13)


def test_hand_derived_router():
    g = json.load(open(os.path.join(GOLDEN, "router_tiny.json")))
    w = {k: np.array(g[k]) for k in ["w_k", "w_t1", "b_t1", "w_t2", "b_t2", "w_r1", "b_r1", "w_o", "b_o"]}
    z, mode = orr.router_forward(np.array(g["hidden"]), w, H_kv=2, d=1, n_boundary=100)
    np.testing.assert_allclose(z, np.array(g["z"]), rtol=0, atol=1e-14)
    np.testing.assert_array_equal(mode, np.array(g["head_mode"]))


def test_positive_homogeneity_with_zero_biases(rng):
    """Pooling, projection, ReLU MLPs and the output row are positively homogeneous."""
    w = wl.WORKLOADS["small-mixed-g4-s1000"]
    weights = wl.router_weights(w, tuned=False)
    weights["w_k"] = wl.f32_from_bf16_bits(weights["w_k"])
    weights["w_o"] = rng.standard_normal(weights["w_o"].shape)
    h = rng.standard_normal((1, 300, w.D))
    z1, _ = orr.router_forward(h, weights, w.H_kv, w.d)
    for a in [0.25, 3.0]:
        z2, _ = orr.router_forward(a * h, weights, w.H_kv, w.d)
        np.testing.assert_allclose(z2, a * z1, rtol=1e-12, atol=1e-15)


def test_head_mode_is_sign_of_logit_and_omega_counts(rng):
    w = wl.WORKLOADS["small-stream-g1-s700"]
    weights = wl.router_weights(w, tuned=False)
    weights["w_k"] = wl.f32_from_bf16_bits(weights["w_k"])
    weights["w_o"] = rng.standard_normal(weights["w_o"].shape)
    z, mode = orr.router_forward(rng.standard_normal((3, 250, w.D)), weights, w.H_kv, w.d)
    np.testing.assert_array_equal(mode, (z > 0).astype(np.int32))


def _tuned_logits(w):
    weights = wl.router_weights(w)
    if w.dtype == "bf16":
        weights["w_k"] = wl.f32_from_bf16_bits(weights["w_k"])
    rows = orr.pooling_rows(w.S, w.n_boundary)
    h = wl.hidden_states(w, rows=rows)
    if w.dtype == "bf16":
        h = wl.f32_from_bf16_bits(h)
    return orr.router_forward(h, weights, w.H_kv, w.d, w.n_boundary)


@pytest.mark.parametrize("name", sorted(wl.WORKLOADS))
def test_tuned_workloads_route_as_intended_with_margin(name):
    """The stored tuning gives each workload its intended decisions, far from the threshold."""
    w = wl.WORKLOADS[name]
    z, mode = _tuned_logits(w)
    alpha, t, intended = wl.routing_targets(w)
    np.testing.assert_array_equal(mode, intended)
    assert np.min(np.abs(z)) > 0.03
    np.testing.assert_allclose(z, alpha[:, None] - t[None, :], atol=0.02)
