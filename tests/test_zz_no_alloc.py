"""The router entry point that allocates nothing (GPU).

ea_router_static_scratch serves callers that cannot call cudaMalloc (such as a
runtime that owns every device allocation): it
keeps its scratch in a fixed array inside the library instead of a caller
workspace.  Its decisions and logits must match ea_router's on the same inputs,
on two calls in a row (the second call reuses the array the first one left
behind), and a problem whose scratch exceeds the array must be refused before
any launch.  This file is collected last so a failure here never hides another.
"""
import numpy as np
import pytest
import torch

import workloads as wl
from sparse_gqa_attention_b200 import abi
from tests import _gpu
from tests._static_scratch import REFUSED, refusal_without_a_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    import __graft_entry__
    __graft_entry__.build()
    assert torch.cuda.is_available()


@pytest.mark.parametrize("name,n_boundary", [("small-mixed-g4-s1000", 100), ("tiny-fp32-s512", 100),
                                             ("llama3-8b-b4-s16k-mixed", 100), ("small-stream-g1-s700", 0)])
def test_matches_workspace_router_twice(name, n_boundary):
    w = wl.WORKLOADS[name]
    hidden = _gpu.to_dev(wl.hidden_states(w), w.dtype)
    weights = {k: _gpu.to_dev(v, w.dtype) for k, v in wl.router_weights(w).items()}
    ws = torch.zeros(abi.ea_router_workspace_size(w.B, w.S, w.D, w.H_kv, w.d, n_boundary), dtype=torch.uint8, device="cuda")
    hm_ref = torch.zeros(w.B, w.H_kv, dtype=torch.int32, device="cuda")
    z_ref = torch.zeros(w.B, w.H_kv, dtype=torch.float32, device="cuda")
    abi.ea_router(hidden, weights, hm_ref, ws, n_boundary, logits=z_ref)
    for _ in range(2):
        hm = torch.full((w.B, w.H_kv), -1, dtype=torch.int32, device="cuda")
        z = torch.full((w.B, w.H_kv), float("nan"), dtype=torch.float32, device="cuda")
        abi.ea_router_static_scratch(hidden, weights, hm, n_boundary, logits=z)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(hm.cpu().numpy(), hm_ref.cpu().numpy())
        np.testing.assert_allclose(z.cpu().numpy(), z_ref.cpu().numpy(), rtol=1e-4, atol=1e-5)


def test_refuses_problems_beyond_the_scratch_array():
    r = REFUSED
    assert abi.ea_router_workspace_size(r["B"], r["S"], r["D"], r["H_kv"], r["d"], 100) > abi.ROUTER_STATIC_SCRATCH_BYTES
    # First on a process without a GPU, where nothing can be launched ...
    assert refusal_without_a_gpu() == abi.EA_ERR_INVALID_ARG
    # ... then here, with real device buffers of the refused problem's sizes (hidden 4 MB,
    # W_k 64 MB), so that every input pointer is valid memory.
    B, S, D, H_kv, d = r["B"], r["S"], r["D"], r["H_kv"], r["d"]
    hidden = torch.zeros(B, S, D, dtype=torch.bfloat16, device="cuda")
    weights = {"w_k": torch.zeros(D, H_kv * d, dtype=torch.bfloat16, device="cuda"),
               "w_t1": torch.zeros(4 * d, d, device="cuda"), "b_t1": torch.zeros(4 * d, device="cuda"),
               "w_t2": torch.zeros(d, 4 * d, device="cuda"), "b_t2": torch.zeros(d, device="cuda"),
               "w_r1": torch.zeros(4 * d, 2 * d, device="cuda"), "b_r1": torch.zeros(4 * d, device="cuda"),
               "w_o": torch.zeros(H_kv, 4 * d, device="cuda"), "b_o": torch.zeros(H_kv, device="cuda")}
    hm = torch.full((B, H_kv), -1, dtype=torch.int32, device="cuda")
    with pytest.raises(abi.EAError) as e:
        abi.ea_router_static_scratch(hidden, weights, hm, 100)
    assert e.value.status == abi.EA_ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert (hm == -1).all()            # nothing was written
