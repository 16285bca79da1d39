"""Python binding of the C ABI in include/ea.h (argument marshalling only).

Every function here has the name of the C entry point it calls and does no
arithmetic of its own: it checks that tensors live on the GPU with the
expected dtype and layout, passes their device pointers and the current CUDA
stream to libea.so, and turns a non-zero ea_status into an ``EAError``.  There
is no fallback: without the built library (or without a GPU) the calls raise.
"""
from __future__ import annotations

import ctypes
import os
import re
from ctypes import POINTER, Structure, c_double, c_float, c_int, c_longlong, c_size_t, c_void_p

import numpy as np
import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libea.so")
HEADER_PATH = os.path.join(os.path.dirname(_PKG), "include", "ea.h")

EA_OK, EA_ERR_INVALID_ARG, EA_ERR_UNSUPPORTED, EA_ERR_CUDA, EA_ERR_TIMEOUT, EA_ERR_BAD_LAYOUT = range(6)
EA_DT_F32, EA_DT_BF16 = 0, 1
EA_FULL, EA_STREAMING, EA_BLOCK_SPARSE = 0, 1, 2
MAX_KV_HEADS = 64
ROUTER_STATIC_SCRATCH_BYTES = 8 << 20   # EA_ROUTER_STATIC_SCRATCH_BYTES


class EAError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {_lib().ea_status_string(status).decode()} (ea_status {status})")


class RouterParams(Structure):
    _fields_ = [("n_boundary", c_int)]


class RouterWeights(Structure):
    _fields_ = [(n, c_void_p) for n in ("w_k", "w_t1", "b_t1", "w_t2", "b_t2", "w_r1", "b_r1", "w_o", "b_o")]


class PatternParams(Structure):
    _fields_ = [("n_sink", c_int), ("window", c_int), ("block", c_int),
                ("bs_row_ptr", c_void_p), ("bs_col", c_void_p), ("bs_nnz", c_longlong),
                ("kind_if_dense", c_void_p), ("kind_if_sparse", c_void_p), ("softmax_scale", c_float)]


class SparsityReport(Structure):
    _fields_ = [("omega_msr_mean", c_double), ("omega_esr", c_double),
                ("live_pairs", c_longlong), ("causal_pairs", c_longlong),
                ("live_tiles", c_longlong), ("causal_tiles", c_longlong), ("live_flops", c_double)]


_LIB = None


def _lib():
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is not built; run __graft_entry__.build() or "
                               "python -m sparse_gqa_attention_b200.build")
        lib = ctypes.CDLL(LIB_PATH)
        st = c_int
        lib.ea_status_string.restype = ctypes.c_char_p
        lib.ea_status_string.argtypes = [c_int]
        lib.ea_router_workspace_size.restype = c_size_t
        lib.ea_router_workspace_size.argtypes = [c_int, c_int, c_int, c_int, c_int, c_int]
        lib.ea_attn_workspace_size.restype = c_size_t
        lib.ea_attn_workspace_size.argtypes = [c_int, c_int, c_int, c_int]
        lib.ea_router_pool_workspace_size.restype = c_size_t
        lib.ea_router_pool_workspace_size.argtypes = [c_int, c_int, c_int, c_int]
        lib.ea_router_pool.restype = st
        lib.ea_router_pool.argtypes = [c_void_p, c_int, c_int, c_int, c_int, c_int, c_void_p, c_void_p, c_size_t,
                                       c_void_p]
        lib.ea_router.restype = st
        lib.ea_router.argtypes = [c_void_p, c_int, c_int, c_int, c_int, c_int, c_int,
                                  POINTER(RouterWeights), POINTER(RouterParams), c_void_p, c_void_p,
                                  c_void_p, c_size_t, c_void_p]
        attn = [c_void_p, c_void_p, c_void_p, c_int, c_int, c_int, c_int, c_int, c_int,
                c_void_p, POINTER(PatternParams), c_void_p, c_void_p, c_size_t, c_void_p]
        lib.ea_hybrid_attn_prefill.restype = st
        lib.ea_hybrid_attn_prefill.argtypes = attn
        lib.ea_hybrid_attn_prefill_chunk.restype = st
        lib.ea_hybrid_attn_prefill_chunk.argtypes = [c_void_p, c_void_p, c_void_p, c_int, c_int, c_int, c_int, c_int,
                                                     c_int, c_int, c_int, c_void_p, POINTER(PatternParams), c_void_p,
                                                     c_void_p, c_size_t, c_void_p]
        lib.ea_attn_scheduled.restype = st
        lib.ea_attn_scheduled.argtypes = attn
        lib.ea_build_schedule.restype = st
        lib.ea_build_schedule.argtypes = [c_void_p, POINTER(PatternParams), c_int, c_int, c_int, c_int, c_int,
                                          c_void_p, c_size_t, c_void_p]
        lib.ea_effective_sparsity.restype = st
        lib.ea_effective_sparsity.argtypes = [c_void_p, POINTER(PatternParams), c_int, c_int, c_int, c_int, c_int,
                                              c_void_p, POINTER(SparsityReport), c_void_p, c_size_t, c_void_p]
        lib.ea_router_static_scratch.restype = st
        lib.ea_router_static_scratch.argtypes = [c_void_p, c_int, c_int, c_int, c_int, c_int, c_int,
                                                 POINTER(RouterWeights), POINTER(RouterParams), c_void_p,
                                                 c_void_p, c_void_p]
        lib.ea_xattn_workspace_size.restype = c_size_t
        lib.ea_xattn_workspace_size.argtypes = [c_int, c_int, c_int, c_int, c_int, c_int]
        lib.ea_xattn_block_select.restype = st
        lib.ea_xattn_block_select.argtypes = [c_void_p, c_void_p, c_int, c_int, c_int, c_int, c_int, c_int, c_void_p,
                                              POINTER(PatternParams), c_int, c_float, c_void_p, c_void_p,
                                              c_longlong, c_void_p, c_void_p, c_size_t, c_void_p]
        lib.ea_model_sparsity.restype = st
        lib.ea_model_sparsity.argtypes = [c_void_p, POINTER(PatternParams), c_int, c_int, c_int, c_int, c_int, c_int,
                                          c_void_p, POINTER(SparsityReport), c_void_p, c_size_t, c_void_p]
        lib.ea_retrieval_workspace_size.restype = c_size_t
        lib.ea_retrieval_workspace_size.argtypes = [c_int, c_int, c_int, c_int]
        lib.ea_retrieval_scores.restype = st
        lib.ea_retrieval_scores.argtypes = [c_void_p, c_void_p, c_int, c_int, c_int, c_int, c_int, c_int, c_int,
                                            c_int, c_float, c_void_p, c_void_p, c_size_t, c_void_p]
        lib.ea_static_head_assignment.restype = st
        lib.ea_static_head_assignment.argtypes = [c_void_p, c_int, c_int, c_int, c_int, c_double, c_void_p,
                                                  c_void_p]
        lib.ea_debug_inject_stall.restype = None
        lib.ea_debug_inject_stall.argtypes = [c_int]
        lib.ea_workspace_status.restype = st
        lib.ea_workspace_status.argtypes = [c_void_p, c_void_p]
        _LIB = lib
    return _LIB


def declared_symbols():
    """Names of the functions include/ea.h exports."""
    text = open(HEADER_PATH).read()
    return sorted(set(re.findall(r"EA_API\s+[\w\s\*]+?\b(ea_\w+)\s*\(", text)))


def _check(status: int, where: str):
    if status != EA_OK:
        raise EAError(status, where)


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return c_void_p(s.cuda_stream)


def _dev(t: torch.Tensor, name: str, dtype=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous (row-major)")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    return c_void_p(t.data_ptr())


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return EA_DT_BF16
    if t.dtype == torch.float32:
        return EA_DT_F32
    raise TypeError(f"unsupported dtype {t.dtype}; bfloat16 or float32")


class Pattern:
    """Device-side block layout plus host kind tables, kept alive for the C struct."""

    def __init__(self, n_sink, window, block, row_ptr, cols, kind_if_dense, kind_if_sparse,
                 softmax_scale=0.0, device="cuda"):
        self.n_sink, self.window, self.block = int(n_sink), int(window), int(block)
        self.row_ptr = torch.as_tensor(np.asarray(row_ptr, np.int32)).to(device)
        self.cols = torch.as_tensor(np.asarray(cols, np.int32)).to(device)
        self.kind_if_dense = np.ascontiguousarray(kind_if_dense, dtype=np.int8)
        self.kind_if_sparse = np.ascontiguousarray(kind_if_sparse, dtype=np.int8)
        self.softmax_scale = float(softmax_scale)

    @classmethod
    def for_xattn(cls, B, S, H_kv, n_sink, window, kind_if_dense, kind_if_sparse, softmax_scale=0.0,
                  device="cuda", block=128):
        """A pattern whose block layout ea_xattn_block_select fills: row_ptr and cols are
        device buffers of the sizes that call needs (cols at its worst-case capacity)."""
        n_qb = -(-S // block)
        return cls(n_sink, window, block, np.zeros(B * H_kv * n_qb + 1, np.int32),
                   np.zeros(xattn_cols_capacity(B, S, H_kv, block), np.int32), kind_if_dense, kind_if_sparse,
                   softmax_scale, device)

    @classmethod
    def from_workloads(cls, p, device="cuda"):
        return cls(p.n_sink, p.window, p.block, p.row_ptr, p.cols, p.kind_if_dense, p.kind_if_sparse,
                   p.softmax_scale, device)

    def c_struct(self) -> PatternParams:
        return PatternParams(self.n_sink, self.window, self.block,
                             c_void_p(self.row_ptr.data_ptr() if self.cols.numel() else 0),
                             c_void_p(self.cols.data_ptr() if self.cols.numel() else 0),
                             self.cols.numel(),
                             self.kind_if_dense.ctypes.data_as(c_void_p),
                             self.kind_if_sparse.ctypes.data_as(c_void_p),
                             self.softmax_scale)


# ---------------------------------------------------------------------------
# Router
# ---------------------------------------------------------------------------

def ea_router_workspace_size(B: int, S: int, D: int, H_kv: int, d: int, n_boundary: int = 100) -> int:
    """Bytes of scratch ea_router needs (pooling and projection partial sums, MLP vectors)."""
    return int(_lib().ea_router_workspace_size(B, S, D, H_kv, d, n_boundary))


def ea_router(hidden: torch.Tensor, weights: dict, head_mode: torch.Tensor, workspace: torch.Tensor,
              n_boundary: int = 100, logits: torch.Tensor | None = None, stream=None):
    """head_mode[B, H_kv] (int32, device) <- router(hidden[B, S, D]); optional logits (float32)."""
    B, S, D = hidden.shape
    H_kv = weights["w_o"].shape[0]
    d = weights["w_t1"].shape[1]
    w = RouterWeights(*[_dev(weights[n], n) for n in
                        ("w_k", "w_t1", "b_t1", "w_t2", "b_t2", "w_r1", "b_r1", "w_o", "b_o")])
    prm = RouterParams(n_boundary)
    status = _lib().ea_router(_dev(hidden, "hidden"), _dtype_code(hidden), B, S, D, H_kv, d, ctypes.byref(w),
                              ctypes.byref(prm), _dev(head_mode, "head_mode", torch.int32),
                              _dev(logits, "logits", torch.float32) if logits is not None else None,
                              _dev(workspace, "workspace"), workspace.numel() * workspace.element_size(),
                              _stream(stream))
    _check(status, "ea_router")


def ea_router_pool_workspace_size(B: int, S: int, D: int, n_boundary: int = 100) -> int:
    """Bytes of scratch ea_router_pool needs (pooling partial sums)."""
    return int(_lib().ea_router_pool_workspace_size(B, S, D, n_boundary))


def ea_router_pool(hidden: torch.Tensor, hbar: torch.Tensor, workspace: torch.Tensor, n_boundary: int = 100,
                   stream=None):
    """hbar[B, D] (float32, device) <- mean of hidden[B, S, D] over the pooled tokens."""
    B, S, D = hidden.shape
    status = _lib().ea_router_pool(_dev(hidden, "hidden"), _dtype_code(hidden), B, S, D, n_boundary,
                                   _dev(hbar, "hbar", torch.float32), _dev(workspace, "workspace"),
                                   workspace.numel() * workspace.element_size(), _stream(stream))
    _check(status, "ea_router_pool")


def ea_router_static_scratch(hidden: torch.Tensor, weights: dict, head_mode: torch.Tensor, n_boundary: int = 100,
                             logits: torch.Tensor | None = None, stream=None):
    """ea_router without a workspace: the library's fixed scratch array is used instead
    (for callers that cannot allocate device memory; see include/ea.h)."""
    B, S, D = hidden.shape
    H_kv = weights["w_o"].shape[0]
    d = weights["w_t1"].shape[1]
    w = RouterWeights(*[_dev(weights[n], n) for n in
                        ("w_k", "w_t1", "b_t1", "w_t2", "b_t2", "w_r1", "b_r1", "w_o", "b_o")])
    prm = RouterParams(n_boundary)
    status = _lib().ea_router_static_scratch(_dev(hidden, "hidden"), _dtype_code(hidden), B, S, D, H_kv, d,
                                             ctypes.byref(w), ctypes.byref(prm),
                                             _dev(head_mode, "head_mode", torch.int32),
                                             _dev(logits, "logits", torch.float32) if logits is not None else None,
                                             _stream(stream))
    _check(status, "ea_router_static_scratch")


# ---------------------------------------------------------------------------
# Hybrid attention
# ---------------------------------------------------------------------------

def ea_attn_workspace_size(B: int, S: int, H_q: int, H_kv: int) -> int:
    """Bytes of workspace the attention calls and the sparsity reports need."""
    return int(_lib().ea_attn_workspace_size(B, S, H_q, H_kv))


def _attn_args(q, k, v, head_mode, pattern: Pattern, o, workspace, stream):
    B, S, H_q, d = q.shape
    H_kv = k.shape[2]
    p = pattern.c_struct()
    return (_dev(q, "q"), _dev(k, "k", q.dtype), _dev(v, "v", q.dtype), _dtype_code(q), B, S, H_q, H_kv, d,
            _dev(head_mode, "head_mode", torch.int32), ctypes.byref(p), _dev(o, "o", q.dtype),
            _dev(workspace, "workspace"), workspace.numel() * workspace.element_size(), _stream(stream)), p


def ea_hybrid_attn_prefill(q, k, v, head_mode, pattern: Pattern, o, workspace, stream=None):
    """o[B, S, H_q, d] <- hybrid-head attention of q, k, v under head_mode and pattern."""
    args, keep = _attn_args(q, k, v, head_mode, pattern, o, workspace, stream)
    _check(_lib().ea_hybrid_attn_prefill(*args), "ea_hybrid_attn_prefill")


def ea_hybrid_attn_prefill_chunk(q, k, v, head_mode, pattern: Pattern, o, workspace, q_offset: int, stream=None):
    """Chunked prefill: q, o [B, S_q, H_q, d] are rows q_offset.. of the sequence whose keys
    are the rows of k, v [B, S_k, H_kv, d] (q_offset % 128 == 0, q_offset + S_q <= S_k)."""
    B, S_q, H_q, d = q.shape
    S_k, H_kv = k.shape[1], k.shape[2]
    p = pattern.c_struct()
    _check(_lib().ea_hybrid_attn_prefill_chunk(
        _dev(q, "q"), _dev(k, "k", q.dtype), _dev(v, "v", q.dtype), _dtype_code(q), B, S_q, int(q_offset), S_k, H_q,
        H_kv, d, _dev(head_mode, "head_mode", torch.int32), ctypes.byref(p), _dev(o, "o", q.dtype),
        _dev(workspace, "workspace"), workspace.numel() * workspace.element_size(), _stream(stream)),
        "ea_hybrid_attn_prefill_chunk")


def ea_build_schedule(head_mode, pattern: Pattern, B, S, H_q, H_kv, d, workspace, stream=None):
    """Device work list of live (query tile, head pair) items, longest first, into the workspace."""
    p = pattern.c_struct()
    _check(_lib().ea_build_schedule(_dev(head_mode, "head_mode", torch.int32), ctypes.byref(p), B, S, H_q, H_kv,
                                    d, _dev(workspace, "workspace"), workspace.numel() * workspace.element_size(),
                                    _stream(stream)), "ea_build_schedule")


def ea_attn_scheduled(q, k, v, head_mode, pattern: Pattern, o, workspace, stream=None):
    """The attention launch over the work list ea_build_schedule wrote (same head_mode and pattern)."""
    args, keep = _attn_args(q, k, v, head_mode, pattern, o, workspace, stream)
    _check(_lib().ea_attn_scheduled(*args), "ea_attn_scheduled")


def xattn_cols_capacity(B: int, S: int, H_kv: int, block: int = 128) -> int:
    """Entries ea_xattn_block_select may write into cols: every causal block of every row."""
    n_qb = -(-S // block)
    return B * H_kv * n_qb * (n_qb + 1) // 2


def ea_xattn_workspace_size(B: int, S: int, H_q: int, H_kv: int, stride: int = 8, block: int = 128) -> int:
    """Bytes of workspace ea_xattn_block_select needs at this stride and block edge."""
    return int(_lib().ea_xattn_workspace_size(B, S, H_q, H_kv, stride, block))


def ea_xattn_block_select(q, k, head_mode, pattern: Pattern, workspace, stride: int = 8, tau: float = 0.9,
                          block_scores=None, stream=None):
    """XAttention's block layout for the BLOCK_SPARSE heads, written into pattern.row_ptr and
    pattern.cols (a Pattern.for_xattn), with block_scores (float [B, H_kv, n_qb, n_qb]) if given."""
    B, S, H_q, d = q.shape
    H_kv = k.shape[2]
    p = pattern.c_struct()
    sc = c_void_p(0) if block_scores is None else _dev(block_scores, "block_scores", torch.float32)
    _check(_lib().ea_xattn_block_select(
        _dev(q, "q"), _dev(k, "k", q.dtype), _dtype_code(q), B, S, H_q, H_kv, d,
        _dev(head_mode, "head_mode", torch.int32), ctypes.byref(p), int(stride), float(tau),
        _dev(pattern.row_ptr, "row_ptr", torch.int32), _dev(pattern.cols, "cols", torch.int32),
        pattern.cols.numel(), sc, _dev(workspace, "workspace"), workspace.numel() * workspace.element_size(),
        _stream(stream)), "ea_xattn_block_select")


def ea_effective_sparsity(head_mode, pattern: Pattern, B, S, H_q, H_kv, d, workspace, stream=None):
    """(Omega_MSR per sample [B] numpy, report dict); synchronises the stream."""
    p = pattern.c_struct()
    per = np.zeros(B, np.float32)
    rep = SparsityReport()
    status = _lib().ea_effective_sparsity(_dev(head_mode, "head_mode", torch.int32), ctypes.byref(p), B, S, H_q,
                                          H_kv, d, per.ctypes.data_as(c_void_p), ctypes.byref(rep),
                                          _dev(workspace, "workspace"),
                                          workspace.numel() * workspace.element_size(), _stream(stream))
    _check(status, "ea_effective_sparsity")
    return per, {f: getattr(rep, f) for f, _ in SparsityReport._fields_}



def ea_model_sparsity(head_mode, pattern: Pattern, L, B, S, H_q, H_kv, d, workspace, stream=None):
    """Whole-stack report for head_mode [L, B, H_kv] (synchronises the stream)."""
    p = pattern.c_struct()
    per = (c_float * B)()
    rep = SparsityReport()
    _check(_lib().ea_model_sparsity(_dev(head_mode, "head_mode", torch.int32), ctypes.byref(p), L, B, S, H_q, H_kv,
                                    d, per, ctypes.byref(rep), _dev(workspace, "workspace"),
                                    workspace.numel() * workspace.element_size(), _stream(stream)),
           "ea_model_sparsity")
    return np.array(per[:], np.float64), {f: getattr(rep, f) for f, _ in SparsityReport._fields_}


def ea_retrieval_workspace_size(B: int, S: int, H_q: int, H_kv: int) -> int:
    """Bytes of workspace ea_retrieval_scores needs (per-slice partial sums)."""
    return int(_lib().ea_retrieval_workspace_size(B, S, H_q, H_kv))


def ea_retrieval_scores(q, k, needle_begin: int, needle_end: int, scores, workspace, softmax_scale: float = 0.0,
                        stream=None):
    """scores [B, H_q] (float32, device) <- attention mass of the last token on the needle span."""
    B, S, H_q, d = q.shape
    H_kv = k.shape[2]
    _check(_lib().ea_retrieval_scores(_dev(q, "q"), _dev(k, "k", q.dtype), _dtype_code(q), B, S, H_q, H_kv, d,
                                      int(needle_begin), int(needle_end), float(softmax_scale),
                                      _dev(scores, "scores", torch.float32), _dev(workspace, "workspace"),
                                      workspace.numel() * workspace.element_size(), _stream(stream)),
           "ea_retrieval_scores")


def ea_static_head_assignment(scores, H_kv: int, omega_msr: float, head_mode, stream=None):
    """head_mode [L, B, H_kv] (int32, device) <- static assignment from scores [L, B, H_q]."""
    L, B, H_q = scores.shape
    _check(_lib().ea_static_head_assignment(_dev(scores, "scores", torch.float32), L, B, H_q, H_kv,
                                            float(omega_msr), _dev(head_mode, "head_mode", torch.int32),
                                            _stream(stream)), "ea_static_head_assignment")

def ea_workspace_status(workspace, stream=None) -> int:
    """Reads and clears the workspace status word; returns the ea_status it maps to."""
    return int(_lib().ea_workspace_status(_dev(workspace, "workspace"), _stream(stream)))


def ea_debug_inject_stall(launches: int):
    """Test hook: the next `launches` tensor-core attention launches stall one CTA until
    its bounded wait runs out, so the timeout path can be exercised (see include/ea.h)."""
    _lib().ea_debug_inject_stall(int(launches))


def ea_status_string(status: int) -> str:
    """Static text for an ea_status code."""
    return _lib().ea_status_string(status).decode()
