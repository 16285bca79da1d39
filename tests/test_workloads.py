"""The seeded input generators (CPU): determinism, bf16 rounding, layout rules."""
import numpy as np

import workloads as wl


def test_bf16_rounding_is_round_to_nearest_even():
    # 1 + 2^-8 is halfway between 1 and 1 + 2^-7: ties go to the even mantissa (1.0).
    x = np.array([1.0, 1 + 2**-8, 1 + 3 * 2**-8, -2.5, 3.140625], np.float32)
    got = wl.f32_from_bf16_bits(wl.bf16_bits_from_f32(x))
    np.testing.assert_array_equal(got, np.array([1.0, 1.0, 1 + 2**-6, -2.5, 3.140625], np.float32))


def test_row_chunked_draw_is_consistent():
    w = wl.WORKLOADS["small-mixed-g4-s1000"]
    q, k, v = wl.attention_inputs(w)
    rows = np.array([0, 5, 999, 1000 - 1, 512])
    q2, k2, _ = wl.attention_inputs(w, q_rows=rows)
    np.testing.assert_array_equal(q2, q[:, rows])
    np.testing.assert_array_equal(k2, k)
    q3, _, _ = wl.attention_inputs(w, batches=[1])
    np.testing.assert_array_equal(q3[0], q[1])
    h = wl.hidden_states(w)
    np.testing.assert_array_equal(wl.hidden_states(w, rows=rows), h[:, rows])


def test_block_layout_rules():
    w = wl.WORKLOADS["small-mixed-g4-s1000"]
    rp, cols = wl.block_layout(w)
    n_qb = -(-w.S // w.block)
    assert len(rp) == w.B * w.H_kv * n_qb + 1
    for r in range(len(rp) - 1):
        c = cols[rp[r]:rp[r + 1]]
        qb = r % n_qb
        assert np.all(np.diff(c) > 0) and c[0] == 0 and c[-1] == qb
        assert len(c) == len(set([0, qb])) + min(int(np.floor(w.density * (qb + 1))), max(qb - 1, 0))


def test_routing_targets_span_intended_omegas():
    w = wl.WORKLOADS["llama3-8b-b4-s16k-mixed"]
    _, _, mode = wl.routing_targets(w)
    assert list(mode.sum(axis=1)) == [2, 3, 5, 6]
    w = wl.WORKLOADS["llama3-8b-s32k-streaming"]
    assert wl.routing_targets(w)[2].sum() == 4


def test_positional_component_peaks_on_the_diagonal():
    import numpy as np
    import workloads as wl
    rows = np.arange(2048)
    u = wl.positional_component(rows, 128).astype(np.float64)
    gram = u[1000] @ u.T                      # q_1000 . k_j for the positional parts alone
    assert np.argmax(gram) == 1000 and abs(gram[1000] - 64.0) < 1e-3       # sum of cos^2 + sin^2 = d/2
    assert np.abs(gram[:500]).max() < 0.5 * gram[1000]                      # far keys well below the peak


def test_structured_inputs_leave_unstructured_workloads_unchanged():
    import numpy as np
    import dataclasses
    import workloads as wl
    w = wl.WORKLOADS["small-xattn-g7-s1000"]
    plain = dataclasses.replace(w, pos_amp=0.0, sink_amp=0.0)
    q, k, v = wl.attention_inputs(w)
    q0, k0, v0 = wl.attention_inputs(plain)
    assert np.array_equal(v, v0) and not np.array_equal(q, q0) and not np.array_equal(k, k0)
    # the q_rows restriction draws the same rows as the full draw
    rows = np.array([0, 5, 511, 999])
    qr, _, _ = wl.attention_inputs(w, q_rows=rows)
    assert np.array_equal(qr, q[:, rows])


def test_probe_inputs_touch_only_the_needle_and_the_last_query_row():
    import numpy as np
    import dataclasses
    import workloads as wl
    w = wl.WORKLOADS["small-mixed-g4-s1000"]
    q, k = wl.probe_layer_inputs(w, 2, needle=(400, 432))
    base = dataclasses.replace(w, seed=w.seed * 1000 + 3)
    q0, k0, _ = wl.attention_inputs(base)
    dk = np.any(k != k0, axis=(0, 2, 3))
    dq = np.any(q != q0, axis=(0, 2, 3))
    assert set(np.nonzero(dk)[0]) <= set(range(400, 432)) and dk[400:432].all()
    assert set(np.nonzero(dq)[0]) == {w.S - 1}
    q2, k2 = wl.probe_layer_inputs(w, 2, needle=(400, 432))
    assert np.array_equal(q, q2) and np.array_equal(k, k2)                 # seeded
