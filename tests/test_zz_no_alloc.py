"""The router entry point that allocates nothing (GPU).

ea_router_static_scratch serves callers that cannot call cudaMalloc (a runtime
that owns every device allocation, or code running under stream capture): it
keeps its scratch in a fixed array inside the library instead of a caller
workspace.  Its decisions and logits must match ea_router's on the same inputs,
on two calls in a row (the second call reuses the array the first one left
behind), and a problem whose scratch exceeds the array must be refused before
any launch.  This file is collected last so a failure here never hides another.
"""
import ctypes

import numpy as np
import pytest
import torch

import workloads as wl
from sparse_gqa_attention_b200 import abi
from tests import _gpu

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
    lib = abi._lib()
    fake = ctypes.c_void_p(0x10000)   # never dereferenced: the size check fails on the host first
    w = abi.RouterWeights(*([fake] * 9))
    prm = abi.RouterParams(100)
    # 64 samples x D = 32768: the pooled states alone need 8 MiB plus partial sums.
    assert abi.ea_router_workspace_size(64, 1000, 32768, 8, 128, 100) > (8 << 20)
    st = lib.ea_router_static_scratch(fake, abi.EA_DT_BF16, 64, 1000, 32768, 8, 128, ctypes.byref(w),
                                      ctypes.byref(prm), fake, None, None)
    assert st == abi.EA_ERR_INVALID_ARG
