"""Chunked prefill (GPU): a sequence prefilled chunk by chunk through
ea_hybrid_attn_prefill_chunk equals one ea_hybrid_attn_prefill over all of it,
bit for bit, and matches the oracle on sampled rows of a chunk."""
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


def _chunked(w, q, k, v, mode, pat, chunk):
    dq, dk, dv = _gpu.to_dev(q, w.dtype), _gpu.to_dev(k, w.dtype), _gpu.to_dev(v, w.dtype)
    hm = torch.from_numpy(np.ascontiguousarray(mode, np.int32)).cuda()
    dpat = abi.Pattern.from_workloads(pat)
    full = torch.full_like(dq, float("nan"))
    ws = torch.zeros(abi.ea_attn_workspace_size(w.B, w.S, w.H_q, w.H_kv), dtype=torch.uint8, device="cuda")
    abi.ea_hybrid_attn_prefill(dq, dk, dv, hm, dpat, full, ws)
    parts = []
    for q0 in range(0, w.S, chunk):
        qc = dq[:, q0:q0 + chunk].contiguous()
        oc = torch.full_like(qc, float("nan"))
        wsc = torch.zeros(abi.ea_attn_workspace_size(w.B, qc.shape[1], w.H_q, w.H_kv), dtype=torch.uint8,
                          device="cuda")
        abi.ea_hybrid_attn_prefill_chunk(qc, dk, dv, hm, dpat, oc, wsc, q0)
        assert abi.ea_workspace_status(wsc) == abi.EA_OK
        parts.append(oc)
    torch.cuda.synchronize()
    assert abi.ea_workspace_status(ws) == abi.EA_OK
    return full, torch.cat(parts, dim=1)


@pytest.mark.parametrize("name,chunk", [("small-mixed-g4-s1000", 256), ("small-blockstream-g4-s900", 384),
                                        ("small-b64-g4-s1000", 256), ("small-fp32-b64-s700", 128),
                                        ("small-bsa-g7-s777", 128), ("small-fp32-d128-s300", 128),
                                        ("tiny-fp32-s512", 256)])
def test_chunks_equal_one_call(name, chunk):
    w = wl.WORKLOADS[name]
    q, k, v = wl.attention_inputs(w)
    mode, pat = wl.routing_targets(w)[2], wl.pattern_for(w)
    full, chunked = _chunked(w, q, k, v, mode, pat, chunk)
    assert torch.equal(full, chunked)


def test_chunk_rows_match_oracle():
    w = wl.WORKLOADS["small-mixed-g4-s1000"]
    q, k, v = wl.attention_inputs(w)
    mode, pat = wl.routing_targets(w)[2], wl.pattern_for(w)
    q0, S_q = 512, 300
    dq = _gpu.to_dev(q[:, q0:q0 + S_q], w.dtype)
    oc = torch.full_like(dq, float("nan"))
    ws = torch.zeros(abi.ea_attn_workspace_size(w.B, S_q, w.H_q, w.H_kv), dtype=torch.uint8, device="cuda")
    abi.ea_hybrid_attn_prefill_chunk(dq, _gpu.to_dev(k, w.dtype), _gpu.to_dev(v, w.dtype),
                                     torch.from_numpy(mode).cuda(), abi.Pattern.from_workloads(pat), oc, ws, q0)
    torch.cuda.synchronize()
    rows = np.arange(q0, q0 + S_q)
    ref = _gpu.oracle_attention(w, q, k, v, mode, pat, rows)
    _gpu.assert_close(oc.float().cpu().numpy().astype(np.float64), ref, w.dtype, "chunk")


def test_32k_layer_in_two_chunks_equals_one_call():
    w = wl.WORKLOADS["llama3-8b-s32k-streaming"]
    q, k, v, _, _ = _gpu.cached_inputs(w.name)
    mode, pat = wl.routing_targets(w)[2], wl.pattern_for(w)
    full, chunked = _chunked(w, q, k, v, mode, pat, 16384)
    assert torch.equal(full, chunked)
