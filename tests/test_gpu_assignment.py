"""GPU parity of the static retrieval-head assignment path against the oracle.

ea_retrieval_scores (fp32 accumulation) against the oracle's fp64 needle masses; the
assignment kernel bit-exact on given scores (values whose group means are exact in
fp32); a stack of layers end to end (probe -> assignment -> per-layer attention ->
whole-stack sparsity) against the oracle run on the same seeded inputs.
"""
import numpy as np
import pytest
import torch

import oracle
import oracle.assignment as oas
import workloads as wl
from sparse_gqa_attention_b200 import abi
from tests import _gpu

pytestmark = pytest.mark.gpu

NEEDLE = (400, 432)


def gpu_scores(w, q, k, needle):
    dq, dk = _gpu.to_dev(q, w.dtype), _gpu.to_dev(k, w.dtype)
    sc = torch.full((w.B, w.H_q), float("nan"), device="cuda")
    ws = torch.zeros(abi.ea_retrieval_workspace_size(w.B, w.S, w.H_q, w.H_kv), dtype=torch.uint8, device="cuda")
    abi.ea_retrieval_scores(dq, dk, needle[0], needle[1], sc, ws)
    torch.cuda.synchronize()
    return sc


@pytest.mark.parametrize("name,needle", [("small-mixed-g4-s1000", NEEDLE), ("small-fp32-d128-s300", (0, 5)),
                                         ("small-bsa-g7-s777", (700, 777)), ("tiny-fp32-s512", (100, 101))])
def test_retrieval_scores_match_oracle(name, needle):
    w = wl.WORKLOADS[name]
    for layer in range(2):
        q, k = wl.probe_layer_inputs(w, layer, needle=needle)
        got = gpu_scores(w, q, k, needle).cpu().numpy().astype(np.float64)
        ref = oas.retrieval_scores(_gpu.to_f64(q), _gpu.to_f64(k), *needle)
        np.testing.assert_allclose(got, ref, rtol=1e-3, atol=1e-5)


@pytest.mark.parametrize("L,B,H_q,H_kv,omega", [(6, 1, 8, 8, 0.5), (5, 2, 8, 4, 0.3), (32, 1, 32, 8, 0.65),
                                                (3, 3, 14, 2, 1.0), (4, 2, 4, 4, 0.0)])
def test_assignment_bit_exact_on_given_scores(L, B, H_q, H_kv, omega):
    rng = np.random.default_rng([L, B, H_q])
    scores = (rng.integers(0, 16, (L, B, H_q)) / 64.0).astype(np.float32)   # means exact in fp32, many ties
    hm = torch.full((L, B, H_kv), -1, dtype=torch.int32, device="cuda")
    abi.ea_static_head_assignment(torch.from_numpy(scores).cuda(), H_kv, omega, hm)
    torch.cuda.synchronize()
    want = oas.static_assignment(oas.kv_head_scores(scores.astype(np.float64), H_kv), omega)
    got = hm.cpu().numpy()
    for b in range(B):
        np.testing.assert_array_equal(got[:, b, :], want)


def test_model_sparsity_given_modes():
    w = wl.WORKLOADS["small-mixed-g4-s1000"]
    L = 5
    modes = np.random.default_rng(11).integers(0, 2, (L, w.B, w.H_kv)).astype(np.int32)
    pat = wl.pattern_for(w)
    dpat = abi.Pattern.from_workloads(pat)
    ws = torch.zeros(abi.ea_attn_workspace_size(w.B, w.S, w.H_q, w.H_kv), dtype=torch.uint8, device="cuda")
    per, rep = abi.ea_model_sparsity(torch.from_numpy(modes).cuda(), dpat, L, w.B, w.S, w.H_q, w.H_kv, w.d, ws)
    ref = oas.model_sparsity(modes, _gpu.pattern_dict(pat), w.B, w.S, w.H_q, w.H_kv, w.d)
    assert rep["live_pairs"] == ref["live_pairs"] and rep["causal_pairs"] == ref["causal_pairs"]
    assert rep["live_tiles"] == ref["live_tiles"] and rep["causal_tiles"] == ref["causal_tiles"]
    assert abs(rep["omega_esr"] - ref["omega_esr"]) < 1e-12
    np.testing.assert_allclose(per, ref["omega_msr_per_sample"], atol=1e-7)


def test_stack_end_to_end():
    """Probe -> assignment -> per-layer hybrid attention -> whole-stack report, four layers."""
    w = wl.WORKLOADS["small-mixed-g4-s1000"]
    L, omega = 4, 0.5
    pat = wl.pattern_for(w)
    dpat = abi.Pattern.from_workloads(pat)
    layers = [wl.probe_layer_inputs(w, l, needle=NEEDLE) for l in range(L)]
    _, _, v = wl.attention_inputs(w)
    scores = torch.empty((L, w.B, w.H_q), device="cuda")
    for l, (q, k) in enumerate(layers):
        scores[l] = gpu_scores(w, q, k, NEEDLE)
    hm = torch.empty((L, w.B, w.H_kv), dtype=torch.int32, device="cuda")
    abi.ea_static_head_assignment(scores, w.H_kv, omega, hm)
    torch.cuda.synchronize()
    got_modes = hm.cpu().numpy()

    ref_scores = np.stack([oas.retrieval_scores(_gpu.to_f64(q), _gpu.to_f64(k), *NEEDLE) for q, k in layers])
    kv = oas.kv_head_scores(ref_scores, w.H_kv)
    ref_mode = oas.static_assignment(kv, omega)
    k_full = oas.n_full_heads(L, w.H_kv, omega)
    srt = np.sort(kv.reshape(-1))[::-1]
    assert srt[k_full - 1] - srt[k_full] > 1e-3, "inputs must leave a margin at the cut"
    for b in range(w.B):
        np.testing.assert_array_equal(got_modes[:, b, :], ref_mode)

    ws = torch.zeros(abi.ea_attn_workspace_size(w.B, w.S, w.H_q, w.H_kv), dtype=torch.uint8, device="cuda")
    dv = _gpu.to_dev(v, w.dtype)
    for l, (q, k) in enumerate(layers):
        dq, dk = _gpu.to_dev(q, w.dtype), _gpu.to_dev(k, w.dtype)
        o = torch.full_like(dq, float("nan"))
        abi.ea_hybrid_attn_prefill(dq, dk, dv, hm[l].contiguous(), dpat, o, ws)
        torch.cuda.synchronize()
        assert abi.ea_workspace_status(ws) == abi.EA_OK
        mode_l = np.repeat(ref_mode[l][None, :], w.B, axis=0)
        ref = oracle.attention.hybrid_attention(_gpu.to_f64(q), _gpu.to_f64(k), _gpu.to_f64(v), mode_l,
                                                _gpu.pattern_dict(pat))
        _gpu.assert_close(o.float().cpu().numpy().astype(np.float64), ref, w.dtype, f"layer {l}")

    per, rep = abi.ea_model_sparsity(hm, dpat, L, w.B, w.S, w.H_q, w.H_kv, w.d, ws)
    ref_rep = oas.model_sparsity(np.repeat(ref_mode[:, None, :], w.B, axis=1), _gpu.pattern_dict(pat), w.B, w.S,
                                 w.H_q, w.H_kv, w.d)
    assert rep["live_pairs"] == ref_rep["live_pairs"] and rep["live_tiles"] == ref_rep["live_tiles"]
    assert abs(rep["omega_msr_mean"] - omega) < 1e-12 and abs(rep["omega_esr"] - ref_rep["omega_esr"]) < 1e-12
