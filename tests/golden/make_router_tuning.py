"""Write tests/golden/router_tuning.json: per-head raw router scores from the oracle.

For every workload, the untuned router (output rows |N(0, 0.02)|, zero
biases) is evaluated by the CPU oracle on the workload's base hidden states
(scale 1).  Its logit for head h is g_ref[h] > 0 (the output row and the
ReLU features are non-negative).  The generators divide output row h by
g_ref[h] and set b_o[h] = -t[h], so the tuned logit is alpha[b] - t[h]
(workloads.routing_targets); the tests check the resulting decisions and
margins with the oracle.

Run from the repository root:  python tests/golden/make_router_tuning.py
The only computation is the oracle's router; the inputs are the seeded draws.
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle.router as orouter  # noqa: E402
import workloads as wl  # noqa: E402


def raw_scores(w):
    weights = wl.router_weights(w, tuned=False)
    if w.dtype == "bf16":
        weights["w_k"] = wl.f32_from_bf16_bits(weights["w_k"])
    rows = orouter.pooling_rows(w.S, w.n_boundary)
    # The router reads only the pooled rows; drawing just those rows gives the same values.
    h = wl.hidden_states(w, tuned=False, rows=rows)[:1]
    if w.dtype == "bf16":
        h = wl.f32_from_bf16_bits(h)
    # Passing the pooled rows alone is exact: the oracle pools every row of an
    # input of at most 2 * n_boundary rows, which is this set.
    z, _ = orouter.router_forward(h, weights, w.H_kv, w.d, w.n_boundary)
    g = z[0]
    assert np.all(g > 0), (w.name, g)
    return g


def main():
    out = {}
    for name, w in wl.WORKLOADS.items():
        g = raw_scores(w)
        out[name] = {"g_ref": [float(x) for x in g], "n_boundary": w.n_boundary, "seed": w.seed}
        print(name, np.round(g, 8))
    path = os.path.join(ROOT, "tests", "golden", "router_tuning.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=1)
        f.write("\n")


if __name__ == "__main__":
    main()
