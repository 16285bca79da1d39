"""Pins for the attention oracle (CPU, fp64).

Each test ties the oracle to something other than itself: torch's fp64 SDPA
on masks built by whole-matrix band / Kronecker operations, closed forms
(o_i = v_i, means of values), invariants (row sums, shift invariance, GQA
grouping) and a hand-derived fixture.  Sources: "Elastic Attention:
Test-time Adaptive Sparsity Ratios for Efficient Transformers" (paperlayer.ai)
section 2 "Hybrid Head Mechanism", section 3 "Attention Router", appendix D.1
"Sparse Inference".
"""
import json
import os

import numpy as np
import pytest

import oracle.attention as oa
from tests import _ref

FULL, STREAMING, BLOCK_SPARSE = oa.FULL, oa.STREAMING, oa.BLOCK_SPARSE
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _qkv(rng, B, S, H_q, H_kv, d):
    return (rng.standard_normal((B, S, H_q, d)), rng.standard_normal((B, S, H_kv, d)),
            rng.standard_normal((B, S, H_kv, d)))


def _pattern(H_kv, kind_sparse, n_sink=0, window=1, block=16, row_ptr=None, cols=None, scale=0.0):
    return dict(n_sink=n_sink, window=window, block=block,
                row_ptr=np.zeros(1, np.int32) if row_ptr is None else row_ptr,
                cols=np.zeros(0, np.int32) if cols is None else cols,
                kind_if_dense=[FULL] * H_kv, kind_if_sparse=[kind_sparse] * H_kv, softmax_scale=scale)


@pytest.mark.parametrize("G", [1, 2, 4, 7])
def test_all_full_equals_causal_sdpa_with_gqa(rng, G):
    B, S, H_kv, d = 2, 37, 2, 8
    q, k, v = _qkv(rng, B, S, G * H_kv, H_kv, d)
    o = oa.hybrid_attention(q, k, v, np.zeros((B, H_kv), np.int32), _pattern(H_kv, STREAMING))
    np.testing.assert_allclose(o, _ref.sdpa(q, k, v, causal=True), rtol=0, atol=1e-12)


@pytest.mark.parametrize("n_sink,window", [(0, 1), (0, 5), (3, 4), (4, 1), (1, 10), (50, 3), (2, 36)])
def test_streaming_equals_band_mask_sdpa(rng, n_sink, window):
    B, S, H_kv, G, d = 1, 37, 2, 2, 8
    q, k, v = _qkv(rng, B, S, G * H_kv, H_kv, d)
    o = oa.hybrid_attention(q, k, v, np.ones((B, H_kv), np.int32), _pattern(H_kv, STREAMING, n_sink, window))
    ref = _ref.sdpa(q, k, v, mask=_ref.streaming_mask(S, n_sink, window))
    np.testing.assert_allclose(o, ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("window", [37, 38, 1000])
def test_streaming_window_at_least_S_is_full(rng, window):
    B, S, H_kv, d = 1, 37, 1, 8
    q, k, v = _qkv(rng, B, S, 3, H_kv, d)
    p = _pattern(H_kv, STREAMING, n_sink=0, window=window)
    o_s = oa.hybrid_attention(q, k, v, np.ones((B, H_kv), np.int32), p)
    o_f = oa.hybrid_attention(q, k, v, np.zeros((B, H_kv), np.int32), p)
    np.testing.assert_allclose(o_s, o_f, rtol=0, atol=1e-13)


def test_streaming_window_one_no_sink_returns_own_value(rng):
    B, S, H_kv, d = 2, 23, 2, 4
    q, k, v = _qkv(rng, B, S, 4, H_kv, d)
    o = oa.hybrid_attention(q, k, v, np.ones((B, H_kv), np.int32), _pattern(H_kv, STREAMING, 0, 1))
    np.testing.assert_array_equal(o, np.repeat(v, 2, axis=2))


@pytest.mark.parametrize("block,S", [(16, 64), (16, 61), (8, 45), (128, 300)])
def test_block_sparse_equals_kron_mask_sdpa(rng, block, S):
    B, H_kv, G, d = 2, 2, 2, 8
    q, k, v = _qkv(rng, B, S, G * H_kv, H_kv, d)
    rp, cols = _ref.random_csr(rng, B, H_kv, S, block)
    p = _pattern(H_kv, BLOCK_SPARSE, block=block, row_ptr=rp, cols=cols)
    o = oa.hybrid_attention(q, k, v, np.ones((B, H_kv), np.int32), p)
    n_qb = -(-S // block)
    mask = np.zeros((B, G * H_kv, S, S), dtype=bool)
    for b in range(B):
        for h_q in range(G * H_kv):
            mask[b, h_q] = _ref.block_mask(S, block, _ref.csr_rows(rp, cols, b, h_q // G, H_kv, n_qb))
    np.testing.assert_allclose(o, _ref.sdpa(q, k, v, mask=mask), rtol=0, atol=1e-12)


def test_block_sparse_all_blocks_is_full(rng):
    B, S, H_kv, block, d = 1, 50, 2, 16, 8
    q, k, v = _qkv(rng, B, S, 4, H_kv, d)
    rp, cols = _ref.random_csr(rng, B, H_kv, S, block, full=True)
    o = oa.hybrid_attention(q, k, v, np.ones((B, H_kv), np.int32),
                            _pattern(H_kv, BLOCK_SPARSE, block=block, row_ptr=rp, cols=cols))
    np.testing.assert_allclose(o, _ref.sdpa(q, k, v, causal=True), rtol=0, atol=1e-12)


def test_block_sparse_diagonal_only_is_blockwise_causal(rng):
    B, S, H_kv, block, d = 1, 50, 1, 16, 8
    q, k, v = _qkv(rng, B, S, 2, H_kv, d)
    rp, cols = _ref.random_csr(rng, B, H_kv, S, block, diag_only=True)
    o = oa.hybrid_attention(q, k, v, np.ones((B, H_kv), np.int32),
                            _pattern(H_kv, BLOCK_SPARSE, block=block, row_ptr=rp, cols=cols))
    for r0 in range(0, S, block):
        r1 = min(S, r0 + block)
        ref = _ref.sdpa(q[:, r0:r1], k[:, r0:r1], v[:, r0:r1], causal=True)
        np.testing.assert_allclose(o[:, r0:r1], ref, rtol=0, atol=1e-12)


def test_zero_query_averages_live_values(rng):
    B, S, H_kv, d = 1, 40, 1, 4
    _, k, v = _qkv(rng, B, S, 1, H_kv, d)
    q = np.zeros((B, S, 1, d))
    n_sink, W = 3, 5
    o = oa.hybrid_attention(q, k, v, np.ones((B, H_kv), np.int32), _pattern(H_kv, STREAMING, n_sink, W))
    m = _ref.streaming_mask(S, n_sink, W)
    expect = (m.astype(np.float64) @ v[0, :, 0, :]) / m.sum(axis=1, keepdims=True)
    np.testing.assert_allclose(o[0, :, 0, :], expect, rtol=0, atol=1e-13)


def test_row_weights_sum_to_one(rng):
    S, d = 200, 16
    K, V = rng.standard_normal((S, d)) * 3, rng.standard_normal((S, d))
    for i in [0, 1, 57, 199]:
        live = np.arange(i + 1)
        _, w = oa.attend_row(rng.standard_normal(d) * 3, K, V, live, 0.5)
        assert abs(w.sum() - 1.0) < 1e-12 and np.all(w >= 0)


def test_shift_of_keys_does_not_change_output(rng):
    B, S, H_kv, d = 1, 30, 1, 8
    q, k, v = _qkv(rng, B, S, 2, H_kv, d)
    p = _pattern(H_kv, STREAMING, 2, 7)
    o1 = oa.hybrid_attention(q, k, v, np.ones((B, H_kv), np.int32), p)
    o2 = oa.hybrid_attention(q, k + rng.standard_normal(d), v, np.ones((B, H_kv), np.int32), p)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-11)


def test_softmax_scale_parameter(rng):
    B, S, H_kv, d = 1, 20, 1, 8
    q, k, v = _qkv(rng, B, S, 1, H_kv, d)
    p = _pattern(H_kv, STREAMING, scale=0.3)
    o = oa.hybrid_attention(q, k, v, np.zeros((B, H_kv), np.int32), p)
    np.testing.assert_allclose(o, _ref.sdpa(q, k, v, causal=True, scale=0.3), rtol=0, atol=1e-12)


def test_mixed_heads_are_the_per_head_results_side_by_side(rng):
    """Per-sample, per-KV-head modes in one call equal each head computed alone."""
    B, S, H_kv, G, d, blk = 2, 33, 3, 2, 8, 8
    q, k, v = _qkv(rng, B, S, G * H_kv, H_kv, d)
    rp, cols = _ref.random_csr(rng, B, H_kv, S, blk)
    p = dict(n_sink=2, window=5, block=blk, row_ptr=rp, cols=cols,
             kind_if_dense=[FULL, FULL, STREAMING], kind_if_sparse=[STREAMING, BLOCK_SPARSE, BLOCK_SPARSE])
    mode = np.array([[1, 0, 1], [0, 1, 0]], np.int32)
    o = oa.hybrid_attention(q, k, v, mode, p)
    n_qb = -(-S // blk)
    for b in range(B):
        for h_q in range(G * H_kv):
            h = h_q // G
            kind = p["kind_if_sparse"][h] if mode[b, h] else p["kind_if_dense"][h]
            if kind == FULL:
                m = _ref.causal_mask(S)
            elif kind == STREAMING:
                m = _ref.streaming_mask(S, 2, 5)
            else:
                m = _ref.block_mask(S, blk, _ref.csr_rows(rp, cols, b, h, H_kv, n_qb))
            ref = _ref.sdpa(q[b:b + 1, :, h_q:h_q + 1], k[b:b + 1, :, h:h + 1], v[b:b + 1, :, h:h + 1], mask=m)
            np.testing.assert_allclose(o[b, :, h_q], ref[0, :, 0], rtol=0, atol=1e-12)


def test_gqa_query_heads_read_their_group_kv_head(rng):
    """Query heads 0..G-1 read KV head 0; with V of KV head 1 zero their outputs stay nonzero."""
    B, S, H_kv, G, d = 1, 16, 2, 3, 4
    q, k, v = _qkv(rng, B, S, G * H_kv, H_kv, d)
    v[:, :, 1, :] = 0.0
    o = oa.hybrid_attention(q, k, v, np.zeros((B, H_kv), np.int32), _pattern(H_kv, STREAMING))
    assert np.all(np.abs(o[:, :, :G]).sum(axis=-1) > 0)
    assert np.all(o[:, :, G:] == 0)


def test_hand_derived_streaming_example():
    g = json.load(open(os.path.join(GOLDEN, "attention_tiny.json")))
    S, d = g["S"], g["d"]
    p = _pattern(1, STREAMING, g["n_sink"], g["window"], scale=g["softmax_scale"])
    for i in range(S):
        assert list(oa.live_keys(i, STREAMING, p)) == g["live"][i]
    q = np.array(g["q"]).reshape(1, S, 1, d)
    k = np.array(g["k"]).reshape(1, S, 1, d)
    v = np.array(g["v"]).reshape(1, S, 1, d)
    o = oa.hybrid_attention(q, k, v, np.ones((1, 1), np.int32), p)
    np.testing.assert_allclose(o[0, :, 0, :], np.array(g["o"]), rtol=0, atol=1e-12)


def test_sampled_rows_match_all_rows(rng):
    B, S, H_kv, d = 1, 40, 2, 8
    q, k, v = _qkv(rng, B, S, 4, H_kv, d)
    p = _pattern(H_kv, STREAMING, 3, 9)
    mode = np.array([[1, 0]], np.int32)
    full = oa.hybrid_attention(q, k, v, mode, p)
    rows = np.array([0, 5, 17, 39])
    np.testing.assert_array_equal(oa.hybrid_attention_rows(q, k, v, mode, p, rows), full[:, rows])
    sub = oa.hybrid_attention_rows(q[:, rows], k, v, mode, p, rows, q_row_index=rows)
    np.testing.assert_array_equal(sub, full[:, rows])


@pytest.mark.parametrize("n_sink,window,block,S", [(128, 256, 64, 300), (1, 1, 16, 77), (0, 1, 8, 50),
                                                   (20, 40, 16, 100), (0, 10_000, 32, 90)])
def test_block_streaming_equals_kron_mask_sdpa(rng, n_sink, window, block, S):
    """Block-granular streaming: sink blocks and local blocks of the block bitmap, made causal."""
    B, H_kv, G, d = 1, 2, 2, 8
    q, k, v = _qkv(rng, B, S, G * H_kv, H_kv, d)
    p = _pattern(H_kv, oa.STREAMING_BLOCKS, n_sink, window, block=block)
    o = oa.hybrid_attention(q, k, v, np.ones((B, H_kv), np.int32), p)
    n_qb = -(-S // block)
    sb, lb = -(-n_sink // block), -(-window // block)
    rows = [[c for c in range(qb + 1) if c < sb or qb - c < lb] for qb in range(n_qb)]
    np.testing.assert_allclose(o, _ref.sdpa(q, k, v, mask=_ref.block_mask(S, block, rows)), rtol=0, atol=1e-12)


def test_block_streaming_special_cases(rng):
    B, S, H_kv, d, blk = 1, 70, 1, 8, 16
    q, k, v = _qkv(rng, B, S, 2, H_kv, d)
    # no sinks, one local block: block-wise causal attention
    o = oa.hybrid_attention(q, k, v, np.ones((B, H_kv), np.int32), _pattern(H_kv, oa.STREAMING_BLOCKS, 0, 1, blk))
    for r0 in range(0, S, blk):
        r1 = min(S, r0 + blk)
        np.testing.assert_allclose(o[:, r0:r1], _ref.sdpa(q[:, r0:r1], k[:, r0:r1], v[:, r0:r1], causal=True),
                                   rtol=0, atol=1e-12)
    # a window of whole blocks covering the sequence: full causal attention
    o = oa.hybrid_attention(q, k, v, np.ones((B, H_kv), np.int32), _pattern(H_kv, oa.STREAMING_BLOCKS, 0, S, blk))
    np.testing.assert_allclose(o, _ref.sdpa(q, k, v, causal=True), rtol=0, atol=1e-12)
