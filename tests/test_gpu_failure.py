"""Failure detection without a GPU fault: a pipeline wait that nothing completes.

Every kernel with an mbarrier pipeline (the block-128 and block-64 tensor-core
attention kernels, the XAttention scoring kernel) bounds every wait (about 2 s).
The test hook ea_debug_inject_stall makes one CTA of the next such launch wait on
a barrier that nothing arrives on; the kernel must report EA_ERR_TIMEOUT through
the workspace status word instead of hanging, and the CUDA context must stay
usable: the next call returns correct results."""
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


def test_stalled_wait_block64_kernel():
    """The block-64 tensor-core kernel (the pages' block edge) honours the same bounded waits."""
    w = wl.WORKLOADS["small-b64-g4-s1000"]
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
    _gpu.assert_close(got, _gpu.oracle_attention(w, q, k, v, mode, pat), w.dtype, "block 64 after timeout")


def test_stalled_wait_xattention_score_kernel():
    """The XAttention scoring kernel (tcgen05, bounded waits) reports a stalled wait as
    EA_ERR_TIMEOUT in its workspace status; the next selection is correct."""
    from tests import test_gpu_xattn as tx
    w = wl.WORKLOADS["small-xattn-g4-s2560"]
    q, k, _ = wl.attention_inputs(w)
    mode = wl.routing_targets(w)[2]
    abi.ea_debug_inject_stall(1)
    t0 = time.time()
    try:
        _, _, _, status, _ = tx.run_xattn(w, q, k, mode, scores=False)
    finally:
        abi.ea_debug_inject_stall(0)
    assert status == abi.EA_ERR_TIMEOUT
    assert time.time() - t0 < 30
    rp, cols, sc, status, _ = tx.run_xattn(w, q, k, mode)
    assert status == abi.EA_OK
    tx.check_layout_shape(w, mode, rp, cols)
    exact = rows = 0
    for b in range(w.B):
        for h in range(w.H_kv):
            if tx._kinds(w, mode, b, h) != wl.BLOCK_SPARSE:
                continue
            for qb in range(-(-w.S // w.block)):
                r = (b * w.H_kv + h) * (-(-w.S // w.block)) + qb
                a = tx.ox.row_importance(_gpu.to_f64(q[b:b + 1, qb * w.block:(qb + 1) * w.block]),
                                         _gpu.to_f64(k[b:b + 1, :(qb + 1) * w.block]), 0, h, qb, w.stride, w.block,
                                         q_first_row=qb * w.block)
                exact += tx.check_row(cols[rp[r]:rp[r + 1]], a, qb, w.tau)
                rows += 1
    assert rows > 0 and exact >= 0.9 * rows
