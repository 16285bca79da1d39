"""The C-ABI library without a GPU: it loads, exports every symbol include/ea.h
declares, sizes workspaces, and rejects out-of-contract arguments on the host
(before any CUDA call, so these run on CPU-only machines too)."""
import ctypes

import numpy as np
import pytest

import __graft_entry__
from sparse_gqa_attention_b200 import abi


@pytest.fixture(scope="module")
def lib():
    __graft_entry__.build()
    return abi._lib()


def test_every_declared_symbol_is_exported(lib):
    names = abi.declared_symbols()
    assert len(names) == 12
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings(lib):
    for s in range(6):
        assert abi.ea_status_string(s)
    assert "unknown" in abi.ea_status_string(99)


def test_workspace_sizes(lib):
    # 2 pairs x 8 KV heads x 256 query tiles of 16-byte items, after a 256 + 256 byte header.
    assert abi.ea_attn_workspace_size(1, 32768, 32, 8) == 512 + 8 * 256 * 2 * 16
    assert abi.ea_attn_workspace_size(1, 100, 7, 2) == 0          # H_q not a multiple of H_kv
    assert abi.ea_attn_workspace_size(1, 65536, 28, 4) == 512 + 4 * 512 * 4 * 16
    n = abi.ea_router_workspace_size(1, 32768, 4096, 8, 128, 100)
    assert n > 4096 * 4 and n % 256 == 0


def _pattern(H_kv, kinds=(0, 1), block=128, window=16):
    dense = np.zeros(H_kv, np.int8)
    sparse = np.array([kinds[1]] * H_kv, np.int8)
    return abi.PatternParams(4, window, block, None, None, 0, dense.ctypes.data_as(ctypes.c_void_p),
                             sparse.ctypes.data_as(ctypes.c_void_p), 0.0), (dense, sparse)


FAKE = ctypes.c_void_p(0x10000)   # never dereferenced: every case fails a host check first


@pytest.mark.parametrize("case,expect", [
    (dict(H_q=7, H_kv=2), abi.EA_ERR_INVALID_ARG),        # H_q % H_kv != 0
    (dict(S=0), abi.EA_ERR_INVALID_ARG),
    (dict(d=96), abi.EA_ERR_UNSUPPORTED),
    (dict(d=64, dtype=abi.EA_DT_BF16), abi.EA_ERR_UNSUPPORTED),   # tensor-core path is d = 128
    (dict(window=0), abi.EA_ERR_INVALID_ARG),
    (dict(kinds=(0, 2)), abi.EA_ERR_INVALID_ARG),          # block-sparse without a layout
    (dict(kinds=(0, 5)), abi.EA_ERR_INVALID_ARG),          # unknown kind
    (dict(H_kv=65, H_q=65), abi.EA_ERR_UNSUPPORTED),
    (dict(ws_bytes=16), abi.EA_ERR_INVALID_ARG),
    (dict(null_q=True), abi.EA_ERR_INVALID_ARG),
])
def test_host_argument_checks(lib, case, expect):
    B, S, H_q, H_kv, d = 1, case.get("S", 256), case.get("H_q", 8), case.get("H_kv", 2), case.get("d", 128)
    pp, keep = _pattern(H_kv, case.get("kinds", (0, 1)), window=case.get("window", 16))
    dtype = case.get("dtype", abi.EA_DT_BF16 if d == 128 else abi.EA_DT_F32)
    q = ctypes.c_void_p(0) if case.get("null_q") else FAKE
    st = lib.ea_hybrid_attn_prefill(q, FAKE, FAKE, dtype, B, S, H_q, H_kv, d, FAKE, ctypes.byref(pp), FAKE,
                                    ctypes.c_void_p(0x100000), case.get("ws_bytes", 1 << 30), None)
    assert st == expect


def test_router_argument_checks(lib):
    w = abi.RouterWeights(*([FAKE] * 9))
    prm = abi.RouterParams(100)
    ws = ctypes.c_void_p(0x100000)
    assert lib.ea_router(FAKE, abi.EA_DT_BF16, 1, 300, 100, 2, 128, ctypes.byref(w), ctypes.byref(prm), FAKE,
                         None, ws, 1 << 30, None) == abi.EA_ERR_INVALID_ARG      # D % 8 != 0 for bf16
    assert lib.ea_router(FAKE, abi.EA_DT_F32, 1, 300, 256, 2, 96, ctypes.byref(w), ctypes.byref(prm), FAKE,
                         None, ws, 1 << 30, None) == abi.EA_ERR_UNSUPPORTED      # d not in {64, 128}
    assert lib.ea_router(FAKE, abi.EA_DT_F32, 1, 300, 256, 2, 128, ctypes.byref(w), ctypes.byref(prm), FAKE,
                         None, ws, 8, None) == abi.EA_ERR_INVALID_ARG            # workspace too small


@pytest.mark.parametrize("q_offset,S_q,S_k,expect", [
    (64, 100, 1000, abi.EA_ERR_INVALID_ARG),     # chunks start on a multiple of 128
    (896, 200, 1000, abi.EA_ERR_INVALID_ARG),    # rows past the keys
    (-128, 100, 1000, abi.EA_ERR_INVALID_ARG),
])
def test_chunk_argument_checks(lib, q_offset, S_q, S_k, expect):
    pp, keep = _pattern(2)
    st = lib.ea_hybrid_attn_prefill_chunk(FAKE, FAKE, FAKE, abi.EA_DT_BF16, 1, S_q, q_offset, S_k, 8, 2, 128, FAKE,
                                          ctypes.byref(pp), FAKE, ctypes.c_void_p(0x100000), 1 << 30, None)
    assert st == expect
