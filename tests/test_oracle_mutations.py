"""Planted mistakes in the oracle must fail its pins (CPU only).

Each case patches one plausible error into the oracle (a dropped sink term,
an off-by-one window, a transposed GQA grouping, a wrong softmax scale, a
swapped router concatenation, a pooling over the wrong rows) and checks that
at least one independent reference disagrees with it.
"""
import json
import os

import numpy as np
import pytest

import oracle.attention as oa
import oracle.router as orr
from tests import _ref

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _stream_case(rng):
    B, S, H_kv, G, d = 1, 40, 2, 2, 8
    q = rng.standard_normal((B, S, G * H_kv, d))
    k = rng.standard_normal((B, S, H_kv, d))
    v = rng.standard_normal((B, S, H_kv, d))
    p = dict(n_sink=3, window=6, block=16, row_ptr=np.zeros(1, np.int32), cols=np.zeros(0, np.int32),
             kind_if_dense=[0, 0], kind_if_sparse=[1, 1])
    return q, k, v, p


def _streaming_pin_holds(rng):
    q, k, v, p = _stream_case(rng)
    o = oa.hybrid_attention(q, k, v, np.ones((1, 2), np.int32), p)
    return np.allclose(o, _ref.sdpa(q, k, v, mask=_ref.streaming_mask(40, 3, 6)), atol=1e-12)


def _full_gqa_pin_holds(rng):
    q, k, v, p = _stream_case(rng)
    o = oa.hybrid_attention(q, k, v, np.zeros((1, 2), np.int32), p)
    return np.allclose(o, _ref.sdpa(q, k, v, causal=True), atol=1e-12)


def test_unpatched_pins_hold(rng):
    assert _streaming_pin_holds(rng) and _full_gqa_pin_holds(rng)


def test_dropped_sink_term_is_caught(rng, monkeypatch):
    orig = oa.live_keys

    def bad(i, kind, pattern, *a, **kw):
        if kind == oa.STREAMING:
            j = np.arange(i + 1)
            return j[i - j < pattern["window"]]
        return orig(i, kind, pattern, *a, **kw)
    monkeypatch.setattr(oa, "live_keys", bad)
    assert not _streaming_pin_holds(rng)


def test_off_by_one_window_is_caught(rng, monkeypatch):
    orig = oa.live_keys

    def bad(i, kind, pattern, *a, **kw):
        if kind == oa.STREAMING:
            j = np.arange(i + 1)
            return j[(j < pattern["n_sink"]) | (i - j <= pattern["window"])]
        return orig(i, kind, pattern, *a, **kw)
    monkeypatch.setattr(oa, "live_keys", bad)
    assert not _streaming_pin_holds(rng)


def test_wrong_softmax_scale_is_caught(rng, monkeypatch):
    monkeypatch.setattr(oa, "softmax_scale", lambda pattern, d: 1.0 / d)
    assert not _full_gqa_pin_holds(rng)


def test_interleaved_gqa_grouping_is_caught(rng, monkeypatch):
    q, k, v, p = _stream_case(rng)
    ref = _ref.sdpa(q, k, v, causal=True)
    # Query head h reading KV head h % H_kv instead of h // G: swap heads 1 and 2 of q.
    qs = q[:, :, [0, 2, 1, 3]]
    o = oa.hybrid_attention(qs, k, v, np.zeros((1, 2), np.int32), p)[:, :, [0, 2, 1, 3]]
    assert not np.allclose(o, ref, atol=1e-6)


def test_swapped_router_concat_is_caught(monkeypatch):
    g = json.load(open(os.path.join(GOLDEN, "router_tiny.json")))
    w = {k: np.array(g[k]) for k in ["w_k", "w_t1", "b_t1", "w_t2", "b_t2", "w_r1", "b_r1", "w_o", "b_o"]}
    real_concat = np.concatenate

    def swapped(arrs, *a, **kw):
        if len(arrs) == 2 and np.ndim(arrs[0]) == 1 and np.ndim(arrs[1]) == 1:
            return real_concat([arrs[1], arrs[0]], *a, **kw)
        return real_concat(arrs, *a, **kw)
    monkeypatch.setattr(orr.np, "concatenate", swapped)
    z, _ = orr.router_forward(np.array(g["hidden"]), w, 2, 1)
    assert not np.allclose(z, np.array(g["z"]))


@pytest.mark.parametrize("bad_rows", [lambda S, nb: np.arange(nb), lambda S, nb: np.arange(S)])
def test_wrong_pooling_set_is_caught(rng, monkeypatch, bad_rows):
    h = rng.standard_normal((1, 500, 4))
    expect = np.concatenate([h[0, :100], h[0, 400:]]).mean(axis=0)
    monkeypatch.setattr(orr, "pooling_rows", bad_rows)
    assert not np.allclose(orr.pool_hidden(h, 100)[0], expect)
