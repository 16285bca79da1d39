"""Failure detection without a GPU fault: a pipeline wait that nothing completes.

The tensor-core attention kernel bounds every mbarrier wait (about 2 s).  The
test hook ea_debug_inject_stall makes one CTA wait on a barrier that nothing
arrives on; the kernel must report EA_ERR_TIMEOUT through the workspace status
word instead of hanging, and the CUDA context must stay usable: the next call
returns correct results."""
import time

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


def test_stalled_wait_reports_timeout_and_context_recovers():
    w = wl.WORKLOADS["small-mixed-g4-s1000"]
    q, k, v = wl.attention_inputs(w)
    mode, pat = wl.routing_targets(w)[2], wl.pattern_for(w)
    abi.ea_debug_inject_stall(1)
    t0 = time.time()
    try:
        _, status = _gpu.run_attention(w, q, k, v, mode, pat, check_finite=False)
    finally:
        abi.ea_debug_inject_stall(0)
    assert status == abi.EA_ERR_TIMEOUT
    assert time.time() - t0 < 30
    got, status = _gpu.run_attention(w, q, k, v, mode, pat)
    assert status == abi.EA_OK
    _gpu.assert_close(got, _gpu.oracle_attention(w, q, k, v, mode, pat), w.dtype, "after timeout")
