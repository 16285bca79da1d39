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
