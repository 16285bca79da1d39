"""Pins for the sparsity oracle (CPU).

Counts are checked against brute-force counts of explicit masks (band and
Kronecker constructions) and against closed forms.  Sources: "Elastic
Attention: Test-time Adaptive Sparsity Ratios for Efficient Transformers"
(paperlayer.ai) section 2 "Sparsity Ratio Computation", appendix C.1.
"""
import numpy as np
import pytest

import oracle.sparsity as osp
from oracle.attention import FULL, STREAMING, BLOCK_SPARSE
from tests import _ref


def _p(n_sink=0, window=1, block=16, rp=None, cols=None, H_kv=1, ks=STREAMING):
    return dict(n_sink=n_sink, window=window, block=block,
                row_ptr=np.zeros(1, np.int32) if rp is None else rp,
                cols=np.zeros(0, np.int32) if cols is None else cols,
                kind_if_dense=[FULL] * H_kv, kind_if_sparse=[ks] * H_kv)


def _mask_tiles_live(m, tile=128):
    S = m.shape[0]
    n = -(-S // tile)
    out = np.zeros(n, np.int64)
    for t in range(n):
        blk = m[t * tile:(t + 1) * tile]
        out[t] = sum(1 for c in range(n) if blk[:, c * tile:(c + 1) * tile].any())
    return out


@pytest.mark.parametrize("S,ns,W", [(300, 0, 1), (300, 16, 128), (700, 130, 257), (513, 128, 128),
                                    (1000, 64, 300), (260, 300, 5), (129, 1, 1000)])
def test_streaming_counts_match_band_mask(S, ns, W):
    p = _p(ns, W)
    m = _ref.streaming_mask(S, ns, W)
    np.testing.assert_array_equal(osp.row_live_counts(S, STREAMING, p), m.sum(axis=1))
    np.testing.assert_array_equal(osp.row_live_counts_plain(S, STREAMING, p), m.sum(axis=1))
    np.testing.assert_array_equal(osp.tile_live_counts(S, STREAMING, p), _mask_tiles_live(m))


@pytest.mark.parametrize("S,block", [(300, 128), (777, 128), (500, 64), (333, 32)])
def test_block_sparse_counts_match_kron_mask(rng, S, block):
    rp, cols = _ref.random_csr(rng, 1, 1, S, block, p_extra=0.25)
    p = _p(block=block, rp=rp, cols=cols, ks=BLOCK_SPARSE)
    m = _ref.block_mask(S, block, _ref.csr_rows(rp, cols, 0, 0, 1, -(-S // block)))
    np.testing.assert_array_equal(osp.row_live_counts(S, BLOCK_SPARSE, p), m.sum(axis=1))
    np.testing.assert_array_equal(osp.tile_live_counts(S, BLOCK_SPARSE, p), _mask_tiles_live(m))


@pytest.mark.parametrize("S", [1, 127, 128, 129, 300])
def test_full_counts_closed_form(S):
    p = _p()
    np.testing.assert_array_equal(osp.row_live_counts(S, FULL, p), np.arange(1, S + 1))
    n = -(-S // 128)
    np.testing.assert_array_equal(osp.tile_live_counts(S, FULL, p), np.arange(1, n + 1))


def test_report_all_full_has_zero_effective_sparsity():
    r = osp.sparsity_report(np.zeros((2, 4), np.int32), _p(H_kv=4), 2, 300, 8, 4, 128)
    assert r["omega_esr"] == 0.0 and r["omega_msr_mean"] == 0.0
    assert r["live_pairs"] == r["causal_pairs"] == 2 * 8 * 300 * 301 // 2
    assert r["live_tiles"] == r["causal_tiles"] == 2 * 8 * 3 * 4 // 2
    assert r["live_flops"] == 4 * 128 * 128 * 128 * r["live_tiles"]


def test_report_streaming_closed_form_and_omega_msr():
    S, W, H_kv, G = 500, 64, 4, 2
    mode = np.array([[1, 0, 1, 1]], np.int32)
    r = osp.sparsity_report(mode, _p(0, W, H_kv=H_kv), 1, S, H_kv * G, H_kv, 64)
    i = np.arange(S)
    pairs_stream = int(np.minimum(i + 1, W).sum())
    pairs_full = S * (S + 1) // 2
    assert r["live_pairs"] == G * (3 * pairs_stream + pairs_full)
    assert np.isclose(r["omega_esr"], 1 - r["live_pairs"] / (G * H_kv * pairs_full))
    np.testing.assert_allclose(r["omega_msr_per_sample"], [0.75])


def test_report_plain_and_interval_counts_agree(rng):
    S, H_kv, block = 400, 2, 128
    rp, cols = _ref.random_csr(rng, 2, H_kv, S, block)
    p = dict(n_sink=20, window=100, block=block, row_ptr=rp, cols=cols,
             kind_if_dense=[FULL, FULL], kind_if_sparse=[STREAMING, BLOCK_SPARSE])
    mode = np.array([[1, 1], [0, 1]], np.int32)
    a = osp.sparsity_report(mode, p, 2, S, 4, H_kv, 128, plain=True)
    b = osp.sparsity_report(mode, p, 2, S, 4, H_kv, 128)
    for key in ["live_pairs", "live_tiles", "omega_esr"]:
        assert a[key] == b[key]


@pytest.mark.parametrize("S,ns,W,block", [(300, 128, 256, 128), (777, 1, 1, 128), (500, 0, 300, 64),
                                          (260, 300, 5, 32), (1000, 128, 2048, 128)])
def test_block_streaming_counts_match_kron_mask(S, ns, W, block):
    from oracle.attention import STREAMING_BLOCKS
    p = _p(ns, W, block=block, ks=STREAMING_BLOCKS)
    sb, lb = -(-ns // block), -(-W // block)
    n_qb = -(-S // block)
    m = _ref.block_mask(S, block, [[c for c in range(qb + 1) if c < sb or qb - c < lb] for qb in range(n_qb)])
    np.testing.assert_array_equal(osp.row_live_counts(S, STREAMING_BLOCKS, p), m.sum(axis=1))
    np.testing.assert_array_equal(osp.tile_live_counts(S, STREAMING_BLOCKS, p), _mask_tiles_live(m))
