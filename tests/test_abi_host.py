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
    assert len(names) == 20
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings(lib):
    for s in range(6):
        assert abi.ea_status_string(s)
    assert "unknown" in abi.ea_status_string(99)


def test_workspace_sizes(lib):
    # 2 pairs x 8 KV heads x 256 query tiles of 16-byte items, after a 256 + 256 byte header,
    # then one int32 live-tile count per (KV head, query tile).
    assert abi.ea_attn_workspace_size(1, 32768, 32, 8) == 512 + 8 * 256 * 2 * 16 + 8 * 256 * 4
    assert abi.ea_attn_workspace_size(1, 100, 7, 2) == 0          # H_q not a multiple of H_kv
    assert abi.ea_attn_workspace_size(1, 65536, 28, 4) == 512 + 4 * 512 * 4 * 16 + 4 * 512 * 4
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


def test_router_weight_alignment_is_checked(lib):
    """The router stages W_k and the MLP weights with 16-byte asynchronous copies, so each
    weight matrix must start on a 16-byte boundary; a misaligned one is refused on the host."""
    ws = ctypes.c_void_p(0x100000)
    prm = abi.RouterParams(100)
    for i in (0, 1, 3, 5, 7):   # w_k, w_t1, w_t2, w_r1, w_o
        ptrs = [FAKE] * 9
        ptrs[i] = ctypes.c_void_p(0x10004)
        w = abi.RouterWeights(*ptrs)
        assert lib.ea_router(FAKE, abi.EA_DT_F32, 1, 300, 256, 2, 128, ctypes.byref(w), ctypes.byref(prm), FAKE,
                             None, ws, 1 << 30, None) == abi.EA_ERR_INVALID_ARG, i


@pytest.mark.parametrize("case", [
    dict(hidden=None),                       # no input
    dict(hbar=None),                         # no output
    dict(B=0), dict(S=0), dict(D=0),
    dict(D=100),                             # D % 8 != 0 for bf16
    dict(hidden=ctypes.c_void_p(0x10008)),   # not 16-byte aligned
    dict(dtype=7),                           # unknown dtype
    dict(ws_bytes=8),                        # workspace too small
    dict(ws=ctypes.c_void_p(0x100010)),      # workspace not 256-byte aligned
])
def test_router_pool_argument_checks(lib, case):
    c = dict(hidden=FAKE, dtype=abi.EA_DT_BF16, B=1, S=300, D=256, n=100, hbar=FAKE, ws=ctypes.c_void_p(0x100000),
             ws_bytes=1 << 30)
    c.update(case)
    assert lib.ea_router_pool(c["hidden"], c["dtype"], c["B"], c["S"], c["D"], c["n"], c["hbar"], c["ws"],
                              c["ws_bytes"], None) == abi.EA_ERR_INVALID_ARG


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


def _xattn_call(lib, S=1024, H_q=8, H_kv=2, d=128, dtype=None, stride=8, tau=0.9, block=128, cap=None,
                ws_bytes=1 << 30, kinds=(0, 2)):
    dense = np.zeros(H_kv, np.int8)
    sparse = np.array([kinds[1]] * H_kv, np.int8)
    pp = abi.PatternParams(128, 2048, block, None, None, 0, dense.ctypes.data_as(ctypes.c_void_p),
                           sparse.ctypes.data_as(ctypes.c_void_p), 0.0)
    n_qb = -(-S // 128)
    cap = 1 * H_kv * n_qb * (n_qb + 1) // 2 if cap is None else cap
    dtype = abi.EA_DT_BF16 if dtype is None else dtype
    return lib.ea_xattn_block_select(FAKE, FAKE, dtype, 1, S, H_q, H_kv, d, FAKE, ctypes.byref(pp), stride, tau,
                                     FAKE, FAKE, cap, None, ctypes.c_void_p(0x100000), ws_bytes, None)


@pytest.mark.parametrize("case,expect", [
    (dict(stride=6), abi.EA_ERR_UNSUPPORTED),
    (dict(stride=32), abi.EA_ERR_UNSUPPORTED),
    (dict(S=1001), abi.EA_ERR_UNSUPPORTED),               # S % stride != 0
    (dict(S=262144 + 128), abi.EA_ERR_UNSUPPORTED),       # more than 2048 query blocks
    (dict(tau=1.5), abi.EA_ERR_INVALID_ARG),
    (dict(tau=-0.1), abi.EA_ERR_INVALID_ARG),
    (dict(dtype=abi.EA_DT_F32), abi.EA_ERR_UNSUPPORTED),
    (dict(d=64), abi.EA_ERR_UNSUPPORTED),
    (dict(block=32), abi.EA_ERR_UNSUPPORTED),
    (dict(cap=10), abi.EA_ERR_INVALID_ARG),
    (dict(ws_bytes=1024), abi.EA_ERR_INVALID_ARG),
    (dict(H_q=7), abi.EA_ERR_INVALID_ARG),
    (dict(H_q=66, H_kv=2, stride=4), abi.EA_ERR_UNSUPPORTED),   # 33 heads x 32 reduced rows per block
])
def test_xattn_argument_checks(lib, case, expect):
    assert _xattn_call(lib, **case) == expect


def test_xattn_workspace_size(lib):
    B, S, H_q, H_kv, st = 1, 65536, 28, 4, 8
    n_red, n_rt, n_qb = S // st, S // st // 128, S // 128
    n = abi.ea_xattn_workspace_size(B, S, H_q, H_kv, st, 128)
    parts = B * H_q * n_red * n_rt * 4 * (1 + st)          # tile maxima + per-block partial sums
    assert parts < n < parts + 1024 + B * H_kv * n_qb * 4 * (1 + n_qb // 32 + 1) + 1024
    assert n % 256 == 0
    assert abi.ea_xattn_workspace_size(B, S, H_q, H_kv, 6, 128) == 0
    assert abi.ea_xattn_workspace_size(B, 1001, H_q, H_kv, 8, 128) == 0
    assert abi.ea_xattn_workspace_size(B, S, H_q, H_kv, 8, 96) == 0
    # block 64: twice the per-block partial sums of block 128
    n64 = abi.ea_xattn_workspace_size(B, S, H_q, H_kv, st, 64)
    assert n64 > n + B * H_q * n_red * n_rt * 4 * st - 4096
    assert abi.ea_xattn_workspace_size(1, 262144, 8, 8, 8, 64) == 0      # 4096 blocks of 64
    assert abi.xattn_cols_capacity(2, 300, 3) == 2 * 3 * 3 * 4 // 2
    assert abi.xattn_cols_capacity(1, 300, 1, 64) == 5 * 6 // 2


@pytest.mark.parametrize("case,expect", [
    (dict(n1=300), abi.EA_ERR_INVALID_ARG),            # needle past S
    (dict(n0=20, n1=10), abi.EA_ERR_INVALID_ARG),
    (dict(d=96), abi.EA_ERR_UNSUPPORTED),
    (dict(H_q=7), abi.EA_ERR_INVALID_ARG),
    (dict(ws=8), abi.EA_ERR_INVALID_ARG),
    (dict(scale=-1.0), abi.EA_ERR_INVALID_ARG),
])
def test_retrieval_argument_checks(lib, case, expect):
    S, H_q, d = 256, case.get("H_q", 8), case.get("d", 128)
    st = lib.ea_retrieval_scores(FAKE, FAKE, abi.EA_DT_BF16, 1, S, H_q, 2, d, case.get("n0", 10), case.get("n1", 20),
                                 case.get("scale", 0.0), FAKE, ctypes.c_void_p(0x100000), case.get("ws", 1 << 30), None)
    assert st == expect


def test_assignment_and_stack_argument_checks(lib):
    assert lib.ea_static_head_assignment(FAKE, 4, 1, 8, 2, 1.5, FAKE, None) == abi.EA_ERR_INVALID_ARG
    assert lib.ea_static_head_assignment(FAKE, 4, 1, 8, 3, 0.5, FAKE, None) == abi.EA_ERR_INVALID_ARG
    assert lib.ea_static_head_assignment(FAKE, 2000, 1, 8, 8, 0.5, FAKE, None) == abi.EA_ERR_UNSUPPORTED
    assert lib.ea_static_head_assignment(None, 4, 1, 8, 2, 0.5, FAKE, None) == abi.EA_ERR_INVALID_ARG
    pp, keep = _pattern(2)
    rep = abi.SparsityReport()
    assert lib.ea_model_sparsity(FAKE, ctypes.byref(pp), 0, 1, 256, 8, 2, 128, None, ctypes.byref(rep),
                                 ctypes.c_void_p(0x100000), 1 << 30, None) == abi.EA_ERR_INVALID_ARG
    assert abi.ea_retrieval_workspace_size(1, 32768, 32, 8) % 256 == 0
    assert abi.ea_retrieval_workspace_size(1, 32768, 30, 8) == 0


def _declared_arity():
    """name -> number of parameters, parsed from include/ea.h."""
    import re
    text = open(abi.HEADER_PATH).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    out = {}
    for m in re.finditer(r"EA_API\s+[\w\s\*]+?\b(ea_\w+)\s*\(([^)]*)\)", text):
        params = m.group(2).strip()
        out[m.group(1)] = 0 if params in ("", "void") else params.count(",") + 1
    return out


def test_binding_signatures_match_the_header(lib):
    """Every ctypes signature the binding sets has the parameter count the header declares."""
    arity = _declared_arity()
    assert len(arity) == len(abi.declared_symbols())
    checked = 0
    for name, n in arity.items():
        fn = getattr(lib, name)
        if fn.argtypes is not None:
            assert len(fn.argtypes) == n, (name, len(fn.argtypes), n)
            checked += 1
    assert checked == len(arity)


def test_no_fallback_without_the_library(monkeypatch, tmp_path):
    """The binding never computes on the host: without libea.so every call raises."""
    monkeypatch.setattr(abi, "_LIB", None)
    monkeypatch.setattr(abi, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="not built"):
        abi.ea_attn_workspace_size(1, 128, 8, 2)
    with pytest.raises(RuntimeError, match="not built"):
        abi.ea_router_workspace_size(1, 128, 256, 2, 128, 100)


def test_host_tensors_are_refused(lib):
    """Device pointers only: a CPU tensor is rejected before any call into the library."""
    import torch
    q = torch.zeros(1, 128, 8, 128, dtype=torch.bfloat16)
    k = torch.zeros(1, 128, 2, 128, dtype=torch.bfloat16)
    with pytest.raises(TypeError, match="CUDA tensor"):
        abi._dev(q, "q")
    with pytest.raises(TypeError):
        abi.ea_retrieval_scores(q, k, 0, 1, torch.zeros(1, 8), torch.zeros(1024, dtype=torch.uint8))


def test_static_scratch_refusal_needs_no_gpu(lib):
    """ea_router_static_scratch refuses a problem beyond its fixed array on the host, before
    any CUDA call (checked in a child process that sees no GPU, so nothing can launch)."""
    from tests._static_scratch import REFUSED, refusal_without_a_gpu
    import re
    text = open(abi.HEADER_PATH).read()
    m = re.search(r"#define EA_ROUTER_STATIC_SCRATCH_BYTES \(\(size_t\)(\d+) << (\d+)\)", text)
    assert m and int(m.group(1)) << int(m.group(2)) == abi.ROUTER_STATIC_SCRATCH_BYTES
    r = REFUSED
    assert abi.ea_router_workspace_size(r["B"], r["S"], r["D"], r["H_kv"], r["d"], 100) > abi.ROUTER_STATIC_SCRATCH_BYTES
    assert refusal_without_a_gpu() == abi.EA_ERR_INVALID_ARG
