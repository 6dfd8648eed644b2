"""fp64 CPU oracle for the DSA decode path -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` leg of
``bench.py`` may import this package.  The GPU library never imports it, and
this package imports nothing from the GPU library.

The arithmetic lives in ``dsa_oracle.c`` (plain C, fp64).  This module only
compiles it with gcc and marshals numpy arrays into its entry points.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dsa_oracle.c")
_LIB = os.path.join(_HERE, "libdsa_oracle.so")
_lock = threading.Lock()
_lib = None

_P = ctypes.c_void_p
_I32 = ctypes.c_int32
_I64 = ctypes.c_int64
_F64 = ctypes.c_double


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/libdsa_oracle.so`` (gcc, OpenMP).

    -ffp-contract=off keeps every multiply and add separately rounded, so the
    fp64 sums follow the order written in the C source.
    """
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        cmd = ["gcc", "-std=c11", "-O2", "-ffp-contract=off", "-fno-fast-math",
               "-fopenmp", "-fPIC", "-shared", _SRC, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            lib.dsa_oracle_e4m3_to_f64.restype = _F64
            lib.dsa_oracle_e4m3_to_f64.argtypes = [ctypes.c_uint8]
            lib.dsa_oracle_bf16_to_f64.restype = _F64
            lib.dsa_oracle_bf16_to_f64.argtypes = [ctypes.c_uint16]
            lib.dsa_oracle_max_threads.restype = _I32
            lib.dsa_oracle_indexer_scores.restype = ctypes.c_int
            lib.dsa_oracle_indexer_scores.argtypes = [
                _I32, _I32, _I32, _P, _P, _P, _P, _P, _P, _P, _P, _I32, _I32,
                _P, _P, _I64, _I32]
            lib.dsa_oracle_topk.restype = ctypes.c_int
            lib.dsa_oracle_topk.argtypes = [_I64, _P, _I32, _P, _P]
            lib.dsa_oracle_sparse_mla.restype = ctypes.c_int
            lib.dsa_oracle_sparse_mla.argtypes = [
                _I32, _I32, _I32, _I32, _F64, _P, _P, _I64, _P, _P, _P, _P,
                _I32, _I32, _P, _I32, _P, _P, _I32]
            lib.dsa_oracle_sparse_mla_fp8.restype = ctypes.c_int
            lib.dsa_oracle_sparse_mla_fp8.argtypes = [
                _I32, _I32, _I32, _I32, _F64, _P, _P, _I64, _P, _P, _P, _P, _P,
                _I32, _I32, _P, _I32, _P, _P, _I32]
            lib.dsa_oracle_dense_mla.restype = ctypes.c_int
            lib.dsa_oracle_dense_mla.argtypes = [
                _I32, _I32, _I32, _I32, _F64, _P, _P, _I64, _P, _P, _P, _P,
                _I32, _I32, _P, _P, _I32]
            lib.dsa_oracle_forward.restype = ctypes.c_int
            lib.dsa_oracle_forward.argtypes = [
                _I32, _I32, _I32, _I32, _I32, _I32, _I32, _F64, _P, _P, _P, _P,
                _P, _P, _I64, _P, _P, _P, _P, _I32, _I32, _P, _P, _P, _I32]
            lib.dsa_oracle_f64_to_e4m3.restype = ctypes.c_uint8
            lib.dsa_oracle_f64_to_e4m3.argtypes = [_F64]
            lib.dsa_oracle_masked_mha.restype = ctypes.c_int
            lib.dsa_oracle_masked_mha.argtypes = [
                _I32, _I32, _I32, _I32, _F64, _P, _P, _P, _P, _P, _P, _P, _I32, _P, _P, _I32]
            lib.dsa_oracle_index_kl.restype = ctypes.c_int
            lib.dsa_oracle_index_kl.argtypes = [
                _I32, _I32, _I32, _F64, _P, _P, _I64, _P, _P, _P, _P, _I32, _I32, _P, _I64, _P,
                _I32, _P, _P, _I32]
            lib.dsa_oracle_pow2_scale.restype = _F64
            lib.dsa_oracle_pow2_scale.argtypes = [_F64]
            lib.dsa_oracle_f64_to_bf16.restype = ctypes.c_uint16
            lib.dsa_oracle_f64_to_bf16.argtypes = [_F64]
            lib.dsa_oracle_quantize_rows.restype = ctypes.c_int
            lib.dsa_oracle_quantize_rows.argtypes = [_I64, _I32, _P, _P, _P]
            lib.dsa_oracle_fold_weights.restype = ctypes.c_int
            lib.dsa_oracle_fold_weights.argtypes = [_I64, _I32, _I32, _P, _P, _P, _P]
            lib.dsa_oracle_indexer_project.restype = ctypes.c_int
            lib.dsa_oracle_indexer_project.argtypes = [
                _I32, _I32, _I32, _I32, _I32, _I32, _P, _P, _P, _P, _P, _P, _P, _F64,
                _P, _F64, _P, _P, _P, _P, _P, _P, _P, _P, _I32]
            _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    """Contiguous array of the given dtype (None passes through)."""
    if a is None:
        return None
    return np.ascontiguousarray(a, dtype=dtype)


def max_threads() -> int:
    return int(_load().dsa_oracle_max_threads())


def e4m3_to_f64(code: int) -> float:
    return float(_load().dsa_oracle_e4m3_to_f64(int(code)))


def bf16_to_f64(bits: int) -> float:
    return float(_load().dsa_oracle_bf16_to_f64(int(bits)))


def _kv_args(q_seq, q_n, seq_row0, page_table, page_size):
    q_seq = _c(q_seq, np.int32)
    q_n = _c(q_n, np.int32)
    if page_table is not None:
        page_table = _c(page_table, np.int32)
        if page_table.ndim != 2:
            raise ValueError("page_table must be [nseq, max_pages]")
        return q_seq, q_n, None, page_table, page_table.shape[1], int(page_size)
    return q_seq, q_n, _c(seq_row0, np.int64), None, 0, 0


def indexer_scores(q_idx, w, kidx, q_seq, q_n, *, seq_row0=None, page_table=None,
                   page_size=0, k_scale=None, ld=None, with_abs=False, nthreads=0):
    """I[q, s] for s < q_n[q] (fp64); -inf beyond.  Shapes:
    q_idx [nq, H_I, d_I] uint8 (e4m3 codes), w [nq, H_I] uint16 (bf16 bits),
    kidx [rows, d_I] uint8, k_scale [rows] float32 or None."""
    q_idx = _c(q_idx, np.uint8)
    nq, h_idx, d_idx = q_idx.shape
    w = _c(w, np.uint16)
    kidx = _c(kidx, np.uint8)
    k_scale = _c(k_scale, np.float32)
    q_seq, q_n, seq_row0, page_table, max_pages, page_size = _kv_args(
        q_seq, q_n, seq_row0, page_table, page_size)
    if ld is None:
        ld = int(q_n.max()) if nq else 0
    scores = np.empty((nq, ld), np.float64)
    absv = np.empty((nq, ld), np.float64) if with_abs else None
    rc = _load().dsa_oracle_indexer_scores(
        nq, h_idx, d_idx, _ptr(q_idx), _ptr(w), _ptr(kidx), _ptr(k_scale),
        _ptr(q_seq), _ptr(q_n), _ptr(seq_row0), _ptr(page_table), max_pages,
        page_size, _ptr(scores), _ptr(absv), ld, nthreads)
    if rc != 0:
        raise RuntimeError("dsa_oracle_indexer_scores failed: %d" % rc)
    return (scores, absv) if with_abs else scores


def topk(scores, k, n=None):
    """Selected positions (rank order) padded with -1 to length k, and nsel."""
    scores = _c(scores, np.float64)
    if n is None:
        n = scores.shape[0]
    idx = np.empty(k, np.int32)
    nsel = np.zeros(1, np.int32)
    rc = _load().dsa_oracle_topk(int(n), _ptr(scores), int(k), _ptr(idx), _ptr(nsel))
    if rc != 0:
        raise RuntimeError("dsa_oracle_topk failed: %d" % rc)
    return idx, int(nsel[0])


def sparse_mla(q, kv, idx, q_seq, q_n, *, scale, d_v=512, seq_row0=None,
               page_table=None, page_size=0, nthreads=0):
    """out [nq, H, d_v] fp64, lse [nq, H] fp64.  q [nq, H, d_qk] uint16,
    kv [rows, d_qk] uint16 (bf16 bits), idx [nq, k] int32."""
    q = _c(q, np.uint16)
    nq, h, d_qk = q.shape
    kv = _c(kv, np.uint16)
    idx = _c(idx, np.int32)
    k = idx.shape[1] if idx.ndim == 2 else 0
    q_seq, q_n, seq_row0, page_table, max_pages, page_size = _kv_args(
        q_seq, q_n, seq_row0, page_table, page_size)
    out = np.empty((nq, h, d_v), np.float64)
    lse = np.empty((nq, h), np.float64)
    rc = _load().dsa_oracle_sparse_mla(
        nq, h, d_qk, d_v, float(scale), _ptr(q), _ptr(kv), kv.shape[1],
        _ptr(q_seq), _ptr(q_n), _ptr(seq_row0), _ptr(page_table), max_pages,
        page_size, _ptr(idx), k, _ptr(out), _ptr(lse), nthreads)
    if rc != 0:
        raise RuntimeError("dsa_oracle_sparse_mla failed: %d" % rc)
    return out, lse


def sparse_mla_fp8(q, kv8, kv_scale, idx, q_seq, q_n, *, scale, d_v=512, seq_row0=None,
                   page_table=None, page_size=0, nthreads=0):
    """Sparse attention over an FP8 latent cache: kv8 [rows, row_bytes] uint8
    e4m3 codes (the first d_qk used), kv_scale [rows] fp32.  Returns out
    [nq, H, d_v], lse [nq, H] (fp64)."""
    q = _c(q, np.uint16)
    nq, h, d_qk = q.shape
    kv8 = _c(kv8, np.uint8)
    kv_scale = _c(kv_scale, np.float32)
    idx = _c(idx, np.int32)
    k = idx.shape[1] if idx.ndim == 2 else 0
    q_seq, q_n, seq_row0, page_table, max_pages, page_size = _kv_args(
        q_seq, q_n, seq_row0, page_table, page_size)
    out = np.empty((nq, h, d_v), np.float64)
    lse = np.empty((nq, h), np.float64)
    rc = _load().dsa_oracle_sparse_mla_fp8(
        nq, h, d_qk, d_v, float(scale), _ptr(q), _ptr(kv8), kv8.shape[1], _ptr(kv_scale),
        _ptr(q_seq), _ptr(q_n), _ptr(seq_row0), _ptr(page_table), max_pages,
        page_size, _ptr(idx), k, _ptr(out), _ptr(lse), nthreads)
    if rc != 0:
        raise RuntimeError("dsa_oracle_sparse_mla_fp8 failed: %d" % rc)
    return out, lse


def dense_mla(q, kv, q_seq, q_n, *, scale, d_v=512, seq_row0=None,
              page_table=None, page_size=0, nthreads=0):
    """Textbook attention over all visible positions (no index list)."""
    q = _c(q, np.uint16)
    nq, h, d_qk = q.shape
    kv = _c(kv, np.uint16)
    q_seq, q_n, seq_row0, page_table, max_pages, page_size = _kv_args(
        q_seq, q_n, seq_row0, page_table, page_size)
    out = np.empty((nq, h, d_v), np.float64)
    lse = np.empty((nq, h), np.float64)
    rc = _load().dsa_oracle_dense_mla(
        nq, h, d_qk, d_v, float(scale), _ptr(q), _ptr(kv), kv.shape[1],
        _ptr(q_seq), _ptr(q_n), _ptr(seq_row0), _ptr(page_table), max_pages,
        page_size, _ptr(out), _ptr(lse), nthreads)
    if rc != 0:
        raise RuntimeError("dsa_oracle_dense_mla failed: %d" % rc)
    return out, lse


def forward(q_idx, w, kidx, q, kv, q_seq, q_n, *, k, scale, d_v=512,
            seq_row0=None, page_table=None, page_size=0, k_scale=None,
            nthreads=0):
    """Score -> TopK -> sparse attention.  Returns (idx [nq,k], out, lse)."""
    q_idx = _c(q_idx, np.uint8)
    nq, h_idx, d_idx = q_idx.shape
    w = _c(w, np.uint16)
    kidx = _c(kidx, np.uint8)
    k_scale = _c(k_scale, np.float32)
    q = _c(q, np.uint16)
    _, h, d_qk = q.shape
    kv = _c(kv, np.uint16)
    q_seq, q_n, seq_row0, page_table, max_pages, page_size = _kv_args(
        q_seq, q_n, seq_row0, page_table, page_size)
    idx = np.empty((nq, k), np.int32)
    out = np.empty((nq, h, d_v), np.float64)
    lse = np.empty((nq, h), np.float64)
    rc = _load().dsa_oracle_forward(
        nq, h_idx, d_idx, h, d_qk, d_v, int(k), float(scale), _ptr(q_idx),
        _ptr(w), _ptr(kidx), _ptr(k_scale), _ptr(q), _ptr(kv), kv.shape[1],
        _ptr(q_seq), _ptr(q_n), _ptr(seq_row0), _ptr(page_table), max_pages,
        page_size, _ptr(idx), _ptr(out), _ptr(lse), nthreads)
    if rc != 0:
        raise RuntimeError("dsa_oracle_forward failed: %d" % rc)
    return idx, out, lse


def f64_to_e4m3(x: float) -> int:
    """E4M3 code nearest to x after clamping to [-448, 448] (ties to even)."""
    return int(_load().dsa_oracle_f64_to_e4m3(float(x)))


def indexer_project(x, q_lora, w_qb, w_k, w_proj, ln_gamma, ln_beta, positions, *,
                    h_idx, d_idx, rope_dim=64, ln_eps=1e-6, rope_theta=10000.0, nthreads=0):
    """The indexer's q^I / k^I / w producer for nt tokens (see the C source).

    x [nt, hidden] and q_lora [nt, q_lora_rank] bf16 bits; w_qb
    [h_idx*d_idx, q_lora_rank], w_k [d_idx, hidden], w_proj [h_idx, hidden]
    bf16 bits ([out, in]); ln_gamma / ln_beta [d_idx] float32; positions [nt]
    int32.  Returns a dict: q_f, k_f, w_f (fp64 before quantisation), q_code,
    q_scale, k_code, k_scale (FP8 codes and power-of-two scales), w_bf16.
    """
    x = _c(x, np.uint16)
    nt, hidden = x.shape
    q_lora = _c(q_lora, np.uint16)
    rank = q_lora.shape[1]
    w_qb, w_k, w_proj = _c(w_qb, np.uint16), _c(w_k, np.uint16), _c(w_proj, np.uint16)
    ln_gamma, ln_beta = _c(ln_gamma, np.float32), _c(ln_beta, np.float32)
    positions = _c(positions, np.int32)
    out = dict(q_f=np.empty((nt, h_idx, d_idx)), k_f=np.empty((nt, d_idx)), w_f=np.empty((nt, h_idx)),
               q_code=np.empty((nt, h_idx, d_idx), np.uint8), q_scale=np.empty((nt, h_idx), np.float32),
               k_code=np.empty((nt, d_idx), np.uint8), k_scale=np.empty(nt, np.float32),
               w_bf16=np.empty((nt, h_idx), np.uint16))
    rc = _load().dsa_oracle_indexer_project(
        nt, hidden, rank, int(h_idx), int(d_idx), int(rope_dim), _ptr(x), _ptr(q_lora), _ptr(w_qb),
        _ptr(w_k), _ptr(w_proj), _ptr(ln_gamma), _ptr(ln_beta), float(ln_eps), _ptr(positions),
        float(rope_theta), _ptr(out["q_f"]), _ptr(out["k_f"]), _ptr(out["w_f"]), _ptr(out["q_code"]),
        _ptr(out["q_scale"]), _ptr(out["k_code"]), _ptr(out["k_scale"]), _ptr(out["w_bf16"]), nthreads)
    if rc != 0:
        raise RuntimeError("dsa_oracle_indexer_project failed: %d" % rc)
    return out


def pow2_scale(amax: float) -> float:
    """Smallest power of two 2^e with amax / 2^e <= 448 (1 for amax = 0)."""
    return float(_load().dsa_oracle_pow2_scale(float(amax)))


def f64_to_bf16(x: float) -> int:
    """bf16 bits nearest to x (ties to even), rounded once from fp64."""
    return int(_load().dsa_oracle_f64_to_bf16(float(x)))


def quantize_rows(v):
    """Per-row power-of-two scale and E4M3 codes of v [rows, d] (fp64 in)."""
    v = _c(v, np.float64)
    rows, d = v.shape
    codes = np.empty((rows, d), np.uint8)
    scales = np.empty(rows, np.float32)
    if _load().dsa_oracle_quantize_rows(rows, d, _ptr(v), _ptr(codes), _ptr(scales)) != 0:
        raise RuntimeError("dsa_oracle_quantize_rows failed")
    return codes, scales


def fold_weights(wp, q_scale, d_idx):
    """w = wp / sqrt(H_I) / sqrt(d_I) * q_scale (fp64) and its bf16 bits;
    wp [n, H_I] fp64, q_scale [n, H_I] float32."""
    wp = _c(wp, np.float64)
    q_scale = _c(q_scale, np.float32)
    n, h = wp.shape
    w_f = np.empty((n, h), np.float64)
    w_b = np.empty((n, h), np.uint16)
    if _load().dsa_oracle_fold_weights(n, h, int(d_idx), _ptr(wp), _ptr(q_scale), _ptr(w_f),
                                       _ptr(w_b)) != 0:
        raise RuntimeError("dsa_oracle_fold_weights failed")
    return w_f, w_b


def masked_mha(q, k, v, q_seq, q_n, seq_row0, *, scale, idx=None, nthreads=0):
    """Dense MHA attention over every visible position under the index set's
    mask (idx None: no mask beyond s < q_n).  q [nq, H, d_qk], k [rows, H, d_qk],
    v [rows, H, d_v] uint16 (bf16 bits).  Returns out [nq, H, d_v], lse [nq, H]
    (fp64)."""
    q = _c(q, np.uint16)
    nq, h, d_qk = q.shape
    k = _c(k, np.uint16)
    v = _c(v, np.uint16)
    d_v = v.shape[2]
    assert k.shape[1] == h and v.shape[1] == h and k.shape[2] == d_qk and k.shape[0] == v.shape[0]
    q_seq = _c(q_seq, np.int32)
    q_n = _c(q_n, np.int32)
    seq_row0 = _c(seq_row0, np.int64)
    idx = _c(idx, np.int32)
    topk = idx.shape[1] if idx is not None else 0
    out = np.empty((nq, h, d_v), np.float64)
    lse = np.empty((nq, h), np.float64)
    rc = _load().dsa_oracle_masked_mha(nq, h, d_qk, d_v, float(scale), _ptr(q), _ptr(k), _ptr(v),
                                       _ptr(q_seq), _ptr(q_n), _ptr(seq_row0), _ptr(idx), topk,
                                       _ptr(out), _ptr(lse), nthreads)
    if rc != 0:
        raise RuntimeError("dsa_oracle_masked_mha failed: %d" % rc)
    return out, lse


def index_kl(q, kv, q_seq, q_n, index_scores, *, scale, idx=None, seq_row0=None, page_table=None,
             page_size=0, with_p=False, nthreads=0):
    """Indexer distillation loss per query (fp64): KL(p || softmax(I)) over every
    visible position (idx None: the dense stage) or over idx's valid entries
    (the sparse stage); p = the heads' attention distributions summed over
    heads and L1-normalised.  index_scores [nq, ld] fp64.  Returns kl [nq]
    (and p [nq, ld] with with_p)."""
    q = _c(q, np.uint16)
    nq, h, d_qk = q.shape
    kv = _c(kv, np.uint16)
    index_scores = _c(index_scores, np.float64)
    ld = index_scores.shape[1]
    q_seq, q_n, seq_row0, page_table, max_pages, page_size = _kv_args(
        q_seq, q_n, seq_row0, page_table, page_size)
    idx = _c(idx, np.int32)
    k = idx.shape[1] if idx is not None else 0
    kl = np.empty(nq, np.float64)
    p = np.empty((nq, ld), np.float64) if with_p else None
    rc = _load().dsa_oracle_index_kl(nq, h, d_qk, float(scale), _ptr(q), _ptr(kv), kv.shape[1],
                                     _ptr(q_seq), _ptr(q_n), _ptr(seq_row0), _ptr(page_table),
                                     max_pages, page_size, _ptr(index_scores), ld, _ptr(idx), k,
                                     _ptr(kl), _ptr(p), nthreads)
    if rc != 0:
        raise RuntimeError("dsa_oracle_index_kl failed: %d" % rc)
    return (kl, p) if with_p else kl
