"""CUDA path vs the CPU oracle, through the C ABI, on seeded inputs.

Tolerances (stated for the path in its contract): routing decisions bit-exact
(generators keep |logit| > 1e-3); bf16 attention max-abs <= 2e-2 and
mean-abs <= 2e-3; fp32 attention max-abs <= 1e-4.  Small workloads are
compared on every row; the full-size workloads (the layer shapes the bench
runs) on sampled rows of every query head.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from sparse_gqa_attention_b200 import abi
from tests import _gpu

pytestmark = pytest.mark.gpu

SMALL = ["tiny-fp32-s512", "small-mixed-g4-s1000", "small-bsa-g7-s777", "small-stream-g1-s700",
         "small-fp32-d128-s300", "small-blockstream-g4-s900", "small-fp32-blockstream-s400",
         "small-b64-g4-s1000", "small-b64-g7-s777", "small-fp32-b64-s700"]
FULL = ["llama3-8b-s32k-streaming", "qwen-g7-s64k-blocksparse", "llama3-8b-b4-s16k-mixed",
        "llama3-8b-s128k-sweep", "llama3-8b-s32k-blockstream", "qwen-g7-s64k-blocksparse-b64",
        "llama3-8b-s32k-blockstream-b64"]


@pytest.fixture(scope="module", autouse=True)
def _built():
    import __graft_entry__
    __graft_entry__.build()
    assert torch.cuda.is_available()


# ---------------------------------------------------------------------------- router

@pytest.mark.parametrize("name", SMALL + FULL)
def test_router_decisions_bit_exact(name):
    w = wl.WORKLOADS[name]
    _, _, _, hidden, weights = _gpu.cached_inputs(name)
    hm, z = _gpu.run_router(w, hidden, weights)
    z_ref, m_ref = _gpu.oracle_router(w, hidden, weights)
    np.testing.assert_array_equal(hm, m_ref)
    np.testing.assert_array_equal(m_ref, wl.routing_targets(w)[2])
    np.testing.assert_allclose(z, z_ref, rtol=1e-4, atol=1e-5)


@pytest.mark.parametrize("name", SMALL + ["llama3-8b-s32k-streaming"])
def test_router_full_sequence_pooling(name):
    w = wl.WORKLOADS[name]
    weights, hidden = wl.router_weights(w), wl.hidden_states(w)
    hm, z = _gpu.run_router(w, hidden, weights, n_boundary=0)
    z_ref, m_ref = _gpu.oracle_router(w, hidden, weights, n_boundary=0)
    np.testing.assert_allclose(z, z_ref, rtol=1e-4, atol=1e-5)
    sure = np.abs(z_ref) > 1e-3
    np.testing.assert_array_equal(hm[sure], m_ref[sure])


@pytest.mark.parametrize("name,n_boundary", [(n, nb) for n in SMALL[:4] + ["llama3-8b-b4-s16k-mixed"] for nb in (100, 0)]
                         + [("llama3-8b-s32k-streaming", 100), ("llama3-8b-s32k-streaming", 0)])
def test_router_pooling_matches_oracle(name, n_boundary):
    """ea_router_pool (the pooling step alone) against the oracle's pooled mean."""
    w = wl.WORKLOADS[name]
    hidden = wl.hidden_states(w)
    hb = torch.full((w.B, w.D), float("nan"), dtype=torch.float32, device="cuda")
    ws = torch.empty(abi.ea_router_pool_workspace_size(w.B, w.S, w.D, n_boundary), dtype=torch.uint8, device="cuda")
    abi.ea_router_pool(_gpu.to_dev(hidden, w.dtype), hb, ws, n_boundary)
    torch.cuda.synchronize()
    ref = oracle.router.pool_hidden(_gpu.to_f64(hidden), n_boundary)
    np.testing.assert_allclose(hb.cpu().numpy(), ref, rtol=1e-4, atol=1e-5)


@pytest.mark.parametrize("name", ["small-mixed-g4-s1000", "llama3-8b-b4-s16k-mixed"])
def test_router_repeats_bit_for_bit(name):
    """Fixed summation orders: the same inputs give the same logits on every call, also
    with a workspace that was not zero-filled."""
    w = wl.WORKLOADS[name]
    _, _, _, hidden, weights = _gpu.cached_inputs(name)
    hid = _gpu.to_dev(hidden, w.dtype)
    wd = {k: _gpu.to_dev(v, w.dtype) for k, v in weights.items()}
    zs = []
    for fill in (0, 255):
        ws = torch.full((abi.ea_router_workspace_size(w.B, w.S, w.D, w.H_kv, w.d, w.n_boundary),), fill,
                        dtype=torch.uint8, device="cuda")
        hm = torch.full((w.B, w.H_kv), -1, dtype=torch.int32, device="cuda")
        z = torch.full((w.B, w.H_kv), float("nan"), dtype=torch.float32, device="cuda")
        for _ in range(2):
            abi.ea_router(hid, wd, hm, ws, w.n_boundary, logits=z)
            zs.append(z.clone())
    torch.cuda.synchronize()
    for z in zs[1:]:
        assert torch.equal(z, zs[0])


# ---------------------------------------------------------------------------- attention

@pytest.mark.parametrize("name", SMALL)
def test_attention_every_row(name):
    w = wl.WORKLOADS[name]
    q, k, v = wl.attention_inputs(w)
    mode = wl.routing_targets(w)[2]
    pat = wl.pattern_for(w)
    got, status = _gpu.run_attention(w, q, k, v, mode, pat)
    assert status == abi.EA_OK
    _gpu.assert_close(got, _gpu.oracle_attention(w, q, k, v, mode, pat), w.dtype, name)


@pytest.mark.parametrize("mode", [[[0, 0], [0, 0]], [[1, 1], [1, 1]], [[0, 1], [1, 0]]])
def test_attention_forced_modes(mode):
    w = wl.WORKLOADS["small-mixed-g4-s1000"]
    q, k, v = wl.attention_inputs(w)
    pat = wl.pattern_for(w)
    m = np.array(mode, np.int32)
    got, status = _gpu.run_attention(w, q, k, v, m, pat)
    assert status == abi.EA_OK
    _gpu.assert_close(got, _gpu.oracle_attention(w, q, k, v, m, pat), w.dtype, str(mode))


EDGE = [  # (S, H_q, H_kv, n_sink, window, sparse kinds, dtype)
    (1, 4, 2, 0, 1, (1, 2), "bf16"),
    (2, 2, 2, 1, 1, (1, 1), "bf16"),
    (127, 8, 1, 3, 10, (1,), "bf16"),
    (128, 6, 2, 128, 128, (1, 2), "bf16"),
    (129, 7, 7, 0, 1, (1, 1, 1, 2, 2, 2, 0), "bf16"),
    (256, 14, 2, 200, 5, (1, 2), "bf16"),
    (300, 4, 4, 1000, 1, (1, 1, 2, 2), "bf16"),
    (385, 8, 2, 0, 1000, (1, 2), "bf16"),
    (1, 4, 2, 0, 1, (1, 2), "f32"),
    (129, 3, 1, 2, 70, (1,), "f32"),
    (200, 4, 2, 64, 1, (1, 2), "f32"),
    (700, 4, 2, 0, 1, (3, 2), "bf16"),
    (513, 6, 3, 129, 300, (3, 3, 1), "bf16"),
    (260, 4, 2, 1, 128, (3, 0), "f32"),
]


@pytest.mark.parametrize("S,H_q,H_kv,n_sink,window,kinds,dtype", EDGE)
def test_attention_edge_shapes(S, H_q, H_kv, n_sink, window, kinds, dtype):
    base = wl.WORKLOADS["small-mixed-g4-s1000"]
    w = dataclasses.replace(base, name=f"edge-{S}", B=2, S=S, H_q=H_q, H_kv=H_kv, n_sink=n_sink, window=window,
                            kind_if_dense=(0,) * H_kv, kind_if_sparse=tuple(kinds), dtype=dtype,
                            d=128, density=0.4)
    q, k, v = wl.attention_inputs(w)
    pat = wl.pattern_for(w)
    mode = np.array([[1] * H_kv, [h % 2 for h in range(H_kv)]], np.int32)
    got, status = _gpu.run_attention(w, q, k, v, mode, pat)
    assert status == abi.EA_OK
    _gpu.assert_close(got, _gpu.oracle_attention(w, q, k, v, mode, pat), dtype, w.name)


EDGE64 = [  # block 64: (S, n_sink, window, sparse kinds, dtype)
    (1, 0, 1, (2, 3), "bf16"),
    (63, 1, 1, (2, 3), "bf16"),
    (64, 64, 64, (3, 2), "bf16"),
    (65, 0, 65, (2, 3), "bf16"),
    (127, 130, 1, (3, 2), "bf16"),
    (129, 0, 1, (2, 2), "bf16"),
    (300, 64, 128, (3, 3), "bf16"),
    (383, 200, 1000, (2, 3), "bf16"),
    (65, 1, 64, (2, 3), "f32"),
    (300, 65, 129, (3, 2), "f32"),
]


@pytest.mark.parametrize("S,n_sink,window,kinds,dtype", EDGE64)
def test_attention_block64_edges(S, n_sink, window, kinds, dtype):
    """The pages' block edge 64 (appendix D.1): every 128x128 tile holds 2x2 blocks, so
    ragged block rows, half-live tiles and the diagonal block halves are all exercised."""
    base = wl.WORKLOADS["small-b64-g4-s1000"]
    w = dataclasses.replace(base, name=f"edge64-{S}", B=2, S=S, n_sink=n_sink, window=window,
                            kind_if_dense=(0, 0), kind_if_sparse=tuple(kinds), dtype=dtype, density=0.4)
    q, k, v = wl.attention_inputs(w)
    pat = wl.pattern_for(w)
    mode = np.array([[1, 1], [0, 1]], np.int32)
    got, status = _gpu.run_attention(w, q, k, v, mode, pat)
    assert status == abi.EA_OK
    _gpu.assert_close(got, _gpu.oracle_attention(w, q, k, v, mode, pat), dtype, w.name)


def test_split_calls_equal_one_call_and_are_deterministic():
    w = wl.WORKLOADS["small-bsa-g7-s777"]
    q, k, v = wl.attention_inputs(w)
    mode, pat = wl.routing_targets(w)[2], wl.pattern_for(w)
    a, _ = _gpu.run_attention(w, q, k, v, mode, pat)
    b, _ = _gpu.run_attention(w, q, k, v, mode, pat, split=True)
    c, _ = _gpu.run_attention(w, q, k, v, mode, pat)
    np.testing.assert_array_equal(a, b)
    np.testing.assert_array_equal(a, c)


@pytest.mark.parametrize("name", FULL)
def test_full_size_sampled_rows(name):
    w = wl.WORKLOADS[name]
    q, k, v, _, _ = _gpu.cached_inputs(name)
    mode, pat = wl.routing_targets(w)[2], wl.pattern_for(w)
    rows = _gpu.sample_rows(w)
    got, status = _gpu.run_attention(w, q, k, v, mode, pat, rows=rows)
    assert status == abi.EA_OK
    ref = _gpu.oracle_attention(w, q, k, v, mode, pat, rows)
    _gpu.assert_close(got, ref, w.dtype, name)


@pytest.mark.parametrize("n_sparse", [0, 2, 4, 6, 8])
def test_omega_sweep_sampled_rows(n_sparse):
    w = wl.WORKLOADS["llama3-8b-s128k-sweep"]
    q, k, v, _, _ = _gpu.cached_inputs(w.name)
    pat = wl.pattern_for(w)
    mode = wl.forced_head_mode(w, n_sparse)
    rows = _gpu.sample_rows(w, n_random=6)
    got, status = _gpu.run_attention(w, q, k, v, mode, pat, rows=rows)
    assert status == abi.EA_OK
    _gpu.assert_close(got, _gpu.oracle_attention(w, q, k, v, mode, pat, rows), w.dtype, str(n_sparse))


# ---------------------------------------------------------------------------- sparsity report

@pytest.mark.parametrize("name", SMALL + FULL)
def test_sparsity_report_matches_oracle(name):
    w = wl.WORKLOADS[name]
    mode, pat = wl.routing_targets(w)[2], wl.pattern_for(w)
    ws = torch.zeros(abi.ea_attn_workspace_size(w.B, w.S, w.H_q, w.H_kv), dtype=torch.uint8, device="cuda")
    per, rep = abi.ea_effective_sparsity(torch.from_numpy(mode).cuda(), abi.Pattern.from_workloads(pat), w.B, w.S,
                                         w.H_q, w.H_kv, w.d, ws)
    ref = oracle.sparsity.sparsity_report(mode, _gpu.pattern_dict(pat), w.B, w.S, w.H_q, w.H_kv, w.d)
    for key in ["live_pairs", "causal_pairs", "live_tiles", "causal_tiles"]:
        assert rep[key] == ref[key], key
    assert rep["omega_esr"] == pytest.approx(ref["omega_esr"], abs=1e-12)
    assert rep["live_flops"] == ref["live_flops"]
    np.testing.assert_allclose(per, ref["omega_msr_per_sample"], atol=1e-7)


# ---------------------------------------------------------------------------- device-side checks

def test_malformed_layout_and_mode_are_reported():
    w = wl.WORKLOADS["small-mixed-g4-s1000"]
    q, k, v = wl.attention_inputs(w)
    pat = wl.pattern_for(w)
    bad = dataclasses.replace(pat, cols=pat.cols.copy())
    n_qb = -(-w.S // w.block)
    r = (0 * w.H_kv + 1) * n_qb + 2             # KV head 1 is block-sparse when routed sparse
    assert w.kind_if_sparse[1] == wl.BLOCK_SPARSE
    bad.cols[pat.row_ptr[r + 1] - 1] = 0        # its query block 2 loses the diagonal block
    mode = np.ones((w.B, w.H_kv), np.int32)
    _, status = _gpu.run_attention(w, q, k, v, mode, bad)
    assert status == abi.EA_ERR_BAD_LAYOUT
    mode[0, 0] = 3
    _, status = _gpu.run_attention(w, q, k, v, mode, pat)
    assert status == abi.EA_ERR_BAD_LAYOUT
    _, status = _gpu.run_attention(w, q, k, v, np.ones((w.B, w.H_kv), np.int32), pat)
    assert status == abi.EA_OK
