"""Python binding of the C ABI in include/dsa.h (argument marshalling only).

Every function here forwards to the same-named entry point of
``libdsa_b200.so``; tensors are passed as raw device pointers.  Nothing is
computed in Python and there is no fallback: if the library is missing or a
call fails, a ``DsaError`` is raised.
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libdsa_b200.so")

DSA_OK = 0
DSA_ERR_INVALID_ARG = -1
DSA_ERR_UNSUPPORTED = -2
DSA_ERR_CUDA = -3
DSA_ERR_WORKSPACE = -4
DSA_ERR_TIMEOUT = -5
DSA_ERR_DEVICE_CHECK = -6

OP_INDEXER_SCORES = 0
OP_TOPK = 1
OP_INDEXER_TOPK = 2
OP_SPARSE_MLA_DECODE = 3
OP_SPARSE_MLA_PREFILL = 4
OP_FORWARD = 5
OP_INDEX_KL_SPARSE = 6
OP_INDEX_KL_DENSE = 7
OP_MASKED_MHA = 8

# Entry points declared in include/dsa.h.
ENTRY_POINTS = (
    "dsa_workspace_size", "dsa_indexer_scores", "dsa_topk", "dsa_indexer_topk",
    "dsa_sparse_mla_decode", "dsa_sparse_mla_prefill", "dsa_forward", "dsa_forward_paged",
    "dsa_indexer_topk_static", "dsa_project_workspace_size", "dsa_indexer_project",
    "dsa_index_kl", "dsa_masked_mha_prefill", "dsa_sparse_mla_decode_fp8",
    "dsa_check_status", "dsa_last_error",
)


class DsaError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__("%s (status %d)" % (msg, code))
        self.code = code


class Params(ctypes.Structure):
    _fields_ = [("nq", ctypes.c_int32), ("h_idx", ctypes.c_int32), ("d_idx", ctypes.c_int32),
                ("h", ctypes.c_int32), ("d_qk", ctypes.c_int32), ("d_v", ctypes.c_int32),
                ("topk", ctypes.c_int32), ("max_n", ctypes.c_int32),
                ("q_per_seq", ctypes.c_int32), ("scale", ctypes.c_float)]


class ProjectParams(ctypes.Structure):
    _fields_ = [("nt", ctypes.c_int32), ("hidden", ctypes.c_int32), ("q_lora_rank", ctypes.c_int32),
                ("h_idx", ctypes.c_int32), ("d_idx", ctypes.c_int32), ("rope_dim", ctypes.c_int32),
                ("ln_eps", ctypes.c_float), ("rope_theta", ctypes.c_float)]


class KV(ctypes.Structure):
    _fields_ = [("q_seq", ctypes.c_void_p), ("q_n", ctypes.c_void_p),
                ("seq_row0", ctypes.c_void_p), ("page_table", ctypes.c_void_p),
                ("max_pages", ctypes.c_int32), ("page_size", ctypes.c_int32),
                ("cache_rows", ctypes.c_int64)]


_lock = threading.Lock()
_lib: Optional[ctypes.CDLL] = None
_P = ctypes.c_void_p


def lib() -> ctypes.CDLL:
    """Load libdsa_b200.so (raises if it was not built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise DsaError(DSA_ERR_CUDA, "libdsa_b200.so not built (run "
                               "python -m long_context_decode_indexer_b200.build)")
            L = ctypes.CDLL(LIB_PATH)
            pp, kp = ctypes.POINTER(Params), ctypes.POINTER(KV)
            L.dsa_workspace_size.argtypes = [pp, kp, ctypes.c_int, ctypes.POINTER(ctypes.c_size_t)]
            L.dsa_indexer_scores.argtypes = [pp, kp, _P, _P, _P, _P, _P, ctypes.c_int64, _P,
                                             ctypes.c_size_t, _P]
            L.dsa_topk.argtypes = [pp, _P, ctypes.c_int64, _P, _P, _P, _P, ctypes.c_size_t, _P]
            L.dsa_indexer_topk.argtypes = [pp, kp, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]
            for name in ("dsa_sparse_mla_decode", "dsa_sparse_mla_prefill"):
                getattr(L, name).argtypes = [pp, kp, _P, _P, ctypes.c_int64, _P, _P, _P, _P,
                                             ctypes.c_size_t, _P]
            for name in ("dsa_forward", "dsa_forward_paged"):
                getattr(L, name).argtypes = [pp, kp, _P, _P, _P, _P, _P, _P, ctypes.c_int64, _P,
                                             _P, _P, _P, ctypes.c_size_t, _P]
            L.dsa_indexer_topk_static.argtypes = [pp, kp, _P, _P, _P, _P, _P, _P, _P, _P]
            jp = ctypes.POINTER(ProjectParams)
            L.dsa_project_workspace_size.argtypes = [jp, ctypes.POINTER(ctypes.c_size_t)]
            L.dsa_indexer_project.argtypes = [jp, kp] + [_P] * 17 + [ctypes.c_size_t, _P]
            L.dsa_index_kl.argtypes = [pp, kp, _P, _P, ctypes.c_int64, _P, ctypes.c_int64, _P, _P, _P,
                                       _P, ctypes.c_size_t, _P]
            L.dsa_masked_mha_prefill.argtypes = [pp, kp, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]
            L.dsa_sparse_mla_decode_fp8.argtypes = [pp, kp, _P, _P, ctypes.c_int64, _P, _P, _P, _P, _P,
                                                    ctypes.c_size_t, _P]
            L.dsa_check_status.argtypes = [_P, _P]
            L.dsa_last_error.restype = ctypes.c_char_p
            for name in ENTRY_POINTS[:-1]:
                getattr(L, name).restype = ctypes.c_int
            _lib = L
    return _lib


def last_error() -> str:
    return lib().dsa_last_error().decode()


def _check(rc: int, what: str):
    if rc != DSA_OK:
        raise DsaError(rc, "%s: %s" % (what, last_error()))


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return stream if isinstance(stream, int) else stream.cuda_stream


def make_params(*, nq, h_idx, d_idx, h, topk, max_n, q_per_seq=1, scale, d_qk=576, d_v=512) -> Params:
    return Params(int(nq), int(h_idx), int(d_idx), int(h), int(d_qk), int(d_v), int(topk),
                  int(max_n), int(q_per_seq), float(scale))


def make_kv(*, q_seq, q_n, seq_row0=None, page_table=None, page_size=0, cache_rows) -> KV:
    max_pages = int(page_table.shape[1]) if page_table is not None else 0
    return KV(_ptr(q_seq), _ptr(q_n), _ptr(seq_row0), _ptr(page_table), max_pages,
              int(page_size) if page_table is not None else 0, int(cache_rows))


def workspace_size(p: Params, kv: Optional[KV], op: int) -> int:
    out = ctypes.c_size_t(0)
    _check(lib().dsa_workspace_size(ctypes.byref(p), ctypes.byref(kv) if kv is not None else None,
                                    int(op), ctypes.byref(out)), "dsa_workspace_size")
    return int(out.value)


def indexer_scores(p, kv, q_idx, w, kidx_cache, k_scale, scores, ld_scores, ws, stream=None):
    _check(lib().dsa_indexer_scores(ctypes.byref(p), ctypes.byref(kv), _ptr(q_idx), _ptr(w),
                                    _ptr(kidx_cache), _ptr(k_scale), _ptr(scores), int(ld_scores),
                                    _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "dsa_indexer_scores")


def topk(p, scores, ld_scores, q_n, idx, nsel, ws, stream=None):
    _check(lib().dsa_topk(ctypes.byref(p), _ptr(scores), int(ld_scores), _ptr(q_n), _ptr(idx),
                          _ptr(nsel), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "dsa_topk")


def indexer_topk(p, kv, q_idx, w, kidx_cache, k_scale, idx, nsel, ws, stream=None):
    _check(lib().dsa_indexer_topk(ctypes.byref(p), ctypes.byref(kv), _ptr(q_idx), _ptr(w),
                                  _ptr(kidx_cache), _ptr(k_scale), _ptr(idx), _ptr(nsel), _ptr(ws),
                                  ws.numel() * ws.element_size(), _stream(stream)),
           "dsa_indexer_topk")


def indexer_topk_static(p, kv, q_idx, w, kidx_cache, k_scale, idx, nsel, status, stream=None):
    """dsa_indexer_topk with the library's fixed scratch array (no workspace)."""
    _check(lib().dsa_indexer_topk_static(ctypes.byref(p), ctypes.byref(kv), _ptr(q_idx), _ptr(w),
                                         _ptr(kidx_cache), _ptr(k_scale), _ptr(idx), _ptr(nsel),
                                         _ptr(status), _stream(stream)),
           "dsa_indexer_topk_static")


def sparse_mla_decode(p, kv, q, kv_cache, kv_row_stride, idx, out, lse, ws, stream=None):
    _check(lib().dsa_sparse_mla_decode(ctypes.byref(p), ctypes.byref(kv), _ptr(q), _ptr(kv_cache),
                                       int(kv_row_stride), _ptr(idx), _ptr(out), _ptr(lse), _ptr(ws),
                                       ws.numel() * ws.element_size(), _stream(stream)),
           "dsa_sparse_mla_decode")


def sparse_mla_decode_fp8(p, kv, q, kv8_cache, kv8_row_bytes, kv_scale, idx, out, lse, ws, stream=None):
    """Sparse attention over an FP8 latent cache (e4m3 codes, power-of-two row scales)."""
    _check(lib().dsa_sparse_mla_decode_fp8(ctypes.byref(p), ctypes.byref(kv), _ptr(q), _ptr(kv8_cache),
                                           int(kv8_row_bytes), _ptr(kv_scale), _ptr(idx), _ptr(out),
                                           _ptr(lse), _ptr(ws), ws.numel() * ws.element_size(),
                                           _stream(stream)),
           "dsa_sparse_mla_decode_fp8")


def sparse_mla_prefill(p, kv, q, kv_cache, kv_row_stride, idx, out, lse, ws, stream=None):
    _check(lib().dsa_sparse_mla_prefill(ctypes.byref(p), ctypes.byref(kv), _ptr(q), _ptr(kv_cache),
                                        int(kv_row_stride), _ptr(idx), _ptr(out), _ptr(lse), _ptr(ws),
                                        ws.numel() * ws.element_size(), _stream(stream)),
           "dsa_sparse_mla_prefill")


def index_kl(p, kv, q, kv_cache, kv_row_stride, index_scores, ld_scores, idx, kl, p_out, ws,
             stream=None):
    """Indexer distillation loss per query; idx None selects the dense stage
    (every visible position), else the sparse stage over idx's entries."""
    _check(lib().dsa_index_kl(ctypes.byref(p), ctypes.byref(kv), _ptr(q), _ptr(kv_cache),
                              int(kv_row_stride), _ptr(index_scores), int(ld_scores), _ptr(idx),
                              _ptr(kl), _ptr(p_out), _ptr(ws), ws.numel() * ws.element_size(),
                              _stream(stream)),
           "dsa_index_kl")


def masked_mha_prefill(p, kv, q, k, v, idx, out, lse, ws, stream=None):
    """Dense MHA under the index set's mask (idx None: causal only)."""
    _check(lib().dsa_masked_mha_prefill(ctypes.byref(p), ctypes.byref(kv), _ptr(q), _ptr(k), _ptr(v),
                                        _ptr(idx), _ptr(out), _ptr(lse), _ptr(ws),
                                        ws.numel() * ws.element_size(), _stream(stream)),
           "dsa_masked_mha_prefill")


def forward(p, kv, q_idx, w, kidx_cache, k_scale, q, kv_cache, kv_row_stride, out, lse, idx_out,
            ws, stream=None, paged=False):
    fn = lib().dsa_forward_paged if paged else lib().dsa_forward
    _check(fn(ctypes.byref(p), ctypes.byref(kv), _ptr(q_idx), _ptr(w), _ptr(kidx_cache),
              _ptr(k_scale), _ptr(q), _ptr(kv_cache), int(kv_row_stride), _ptr(out), _ptr(lse),
              _ptr(idx_out), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "dsa_forward_paged" if paged else "dsa_forward")


def make_project_params(*, nt, hidden, q_lora_rank, h_idx, d_idx, rope_dim=64, ln_eps=1e-6,
                        rope_theta=10000.0) -> ProjectParams:
    return ProjectParams(int(nt), int(hidden), int(q_lora_rank), int(h_idx), int(d_idx),
                         int(rope_dim), float(ln_eps), float(rope_theta))


def project_workspace_size(pp: ProjectParams) -> int:
    out = ctypes.c_size_t(0)
    _check(lib().dsa_project_workspace_size(ctypes.byref(pp), ctypes.byref(out)),
           "dsa_project_workspace_size")
    return int(out.value)


def indexer_project(pp, kv, x, q_lora, w_qb, w_k, w_proj, ln_gamma, ln_beta, positions, q_idx,
                    q_scale, w, kidx_cache, k_scale, ws, q_f32=None, k_f32=None, w_f32=None,
                    stream=None):
    _check(lib().dsa_indexer_project(
        ctypes.byref(pp), ctypes.byref(kv), _ptr(x), _ptr(q_lora), _ptr(w_qb), _ptr(w_k),
        _ptr(w_proj), _ptr(ln_gamma), _ptr(ln_beta), _ptr(positions), _ptr(q_idx), _ptr(q_scale),
        _ptr(w), _ptr(kidx_cache), _ptr(k_scale), _ptr(q_f32), _ptr(k_f32), _ptr(w_f32), _ptr(ws),
        ws.numel() * ws.element_size(), _stream(stream)), "dsa_indexer_project")


def check_status(ws, stream=None) -> int:
    """Synchronise the stream and return (then clear) the device status word."""
    return int(lib().dsa_check_status(_ptr(ws), _stream(stream)))
