"""C-ABI checks that need no GPU: the library builds and loads, exports every
entry point include/dsa.h declares, sizes workspaces, and rejects invalid
arguments on the host before launching anything."""
import ctypes
import os
import re

import pytest

from conftest import ROOT

from long_context_decode_indexer_b200 import build as dsa_build
from long_context_decode_indexer_b200 import dsa
from long_context_decode_indexer_b200.synth import CONFIGS


@pytest.fixture(scope="module")
def L():
    dsa_build.build()
    return dsa.lib()


def declared_functions():
    text = open(os.path.join(ROOT, "include", "dsa.h")).read()
    return set(re.findall(r"^(?:int|const char \*)\s*(dsa_\w+)\s*\(", text, re.M))


def test_header_declares_the_entry_points():
    assert declared_functions() == set(dsa.ENTRY_POINTS)


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), name


def test_bindings_pass_every_declared_parameter(L):
    """Each ctypes binding types as many arguments as its C declaration has
    parameters: an argument past the typed ones would go through as a
    32-bit int (the stream handle of the producer once did)."""
    text = open(os.path.join(ROOT, "include", "dsa.h")).read()
    decls = dict(re.findall(r"\n(?:int|const char \*)\s*(dsa_\w+)\(([^;]*?)\);", text, re.S))
    assert set(decls) == set(dsa.ENTRY_POINTS)
    for name, params in decls.items():
        n = 0 if params.strip() in ("", "void") else params.count(",") + 1
        types = getattr(L, name).argtypes
        assert len(types or []) == n, "%s: %d parameters, %d argtypes" % (name, n, len(types or []))


def _params(cfg=3, **kw):
    c = CONFIGS[cfg]
    base = dict(nq=c["nseq"], h_idx=c["h_idx"], d_idx=c["d_idx"], h=c["h"], topk=c["topk"],
                max_n=c["L"], q_per_seq=1, scale=576 ** -0.5)
    base.update(kw)
    return dsa.make_params(**base)


def _kv(paged=False, **kw):
    base = dict(q_seq=0x1000, q_n=0x2000, cache_rows=1 << 21)
    if paged:
        base.update(page_table=None)
    base.update(kw)
    kv = dsa.make_kv(**{k: v for k, v in base.items() if k in ("q_seq", "q_n", "seq_row0", "cache_rows")},
                     page_table=None)
    if paged:
        kv.page_table = 0x3000
        kv.max_pages = kw.get("max_pages", 4096)
        kv.page_size = kw.get("page_size", 64)
    else:
        kv.seq_row0 = 0x4000
    return kv


@pytest.mark.parametrize("cfg", [1, 2, 3, 4, 5])
@pytest.mark.parametrize("op", [dsa.OP_INDEXER_SCORES, dsa.OP_TOPK, dsa.OP_INDEXER_TOPK,
                                dsa.OP_SPARSE_MLA_DECODE, dsa.OP_SPARSE_MLA_PREFILL, dsa.OP_FORWARD])
def test_workspace_size_for_every_workload(L, cfg, op):
    c = CONFIGS[cfg]
    nq = c["nseq"] * (2 if c["kind"] == "paged2" else 1)
    if c["kind"] == "prefill":
        nq = c["L"]
    p = _params(cfg, nq=nq, max_n=min(c["L"] + 1, 131073),
                q_per_seq=nq if c["kind"] == "prefill" else (2 if c["kind"] == "paged2" else 1))
    n = dsa.workspace_size(p, _kv(paged=c["kind"] == "paged2", max_pages=2049), op)
    assert n >= 256
    assert n < (8 << 30)


def test_forward_workspace_holds_indices_and_partials(L):
    p = _params(3)
    n_fwd = dsa.workspace_size(p, _kv(), dsa.OP_FORWARD)
    n_idx = dsa.workspace_size(p, _kv(), dsa.OP_INDEXER_TOPK)
    n_mla = dsa.workspace_size(p, _kv(), dsa.OP_SPARSE_MLA_DECODE)
    assert n_fwd >= n_idx + 16 * 2048 * 4 + n_mla - 2 * 256


@pytest.mark.parametrize("field,value", [("h_idx", 0), ("h_idx", 65), ("d_idx", 96), ("topk", 0),
                                         ("topk", 4096), ("h", 0), ("h", 129), ("nq", -1),
                                         ("max_n", -5), ("q_per_seq", 0)])
def test_invalid_shapes_are_rejected_on_the_host(L, field, value):
    p = _params(3)
    setattr(p, field, value)
    out = ctypes.c_size_t(0)
    rc = L.dsa_workspace_size(ctypes.byref(p), ctypes.byref(_kv()), dsa.OP_FORWARD, ctypes.byref(out))
    assert rc == dsa.DSA_ERR_INVALID_ARG
    assert dsa.last_error() != ""


def test_unsupported_head_width_is_reported(L):
    p = _params(3, d_qk=512)
    out = ctypes.c_size_t(0)
    assert L.dsa_workspace_size(ctypes.byref(p), ctypes.byref(_kv()), dsa.OP_FORWARD,
                                ctypes.byref(out)) == dsa.DSA_ERR_UNSUPPORTED


def test_kv_layout_must_be_exactly_one_of_contiguous_or_paged(L):
    kv = _kv()
    kv.page_table = 0x3000
    kv.page_size = 64
    kv.max_pages = 4096
    out = ctypes.c_size_t(0)
    p = _params(3)
    assert L.dsa_workspace_size(ctypes.byref(p), ctypes.byref(kv), dsa.OP_FORWARD,
                                ctypes.byref(out)) == dsa.DSA_ERR_INVALID_ARG
    kv2 = _kv(paged=True, page_size=32)
    assert L.dsa_workspace_size(ctypes.byref(p), ctypes.byref(kv2), dsa.OP_FORWARD,
                                ctypes.byref(out)) == dsa.DSA_ERR_UNSUPPORTED
    kv3 = _kv(paged=True, max_pages=10)   # 10 * 64 < max_n
    assert L.dsa_workspace_size(ctypes.byref(p), ctypes.byref(kv3), dsa.OP_FORWARD,
                                ctypes.byref(out)) == dsa.DSA_ERR_INVALID_ARG


def test_small_or_misaligned_workspace_is_rejected_before_any_launch(L):
    p = _params(3)
    kv = _kv()
    need = dsa.workspace_size(p, kv, dsa.OP_INDEXER_TOPK)
    fake = 1 << 40  # never dereferenced: validation fails first
    rc = L.dsa_indexer_topk(ctypes.byref(p), ctypes.byref(kv), fake, fake, fake, None, fake, None,
                            fake, need - 256, None)
    assert rc == dsa.DSA_ERR_WORKSPACE
    rc = L.dsa_indexer_topk(ctypes.byref(p), ctypes.byref(kv), fake, fake, fake, None, fake, None,
                            fake + 64, need, None)
    assert rc == dsa.DSA_ERR_WORKSPACE
    rc = L.dsa_indexer_topk(ctypes.byref(p), ctypes.byref(kv), fake, fake, fake, None, fake, None,
                            None, need, None)
    assert rc == dsa.DSA_ERR_WORKSPACE


def test_null_and_misaligned_tensors_are_rejected(L):
    p = _params(3)
    kv = _kv()
    fake = 1 << 40
    rc = L.dsa_forward(ctypes.byref(p), ctypes.byref(kv), None, fake, fake, None, fake, fake, 576,
                       fake, fake, None, fake, 1 << 40, None)
    assert rc == dsa.DSA_ERR_INVALID_ARG
    rc = L.dsa_forward(ctypes.byref(p), ctypes.byref(kv), fake + 8, fake, fake, None, fake, fake, 576,
                       fake, fake, None, fake, 1 << 40, None)
    assert rc == dsa.DSA_ERR_INVALID_ARG
    rc = L.dsa_forward(ctypes.byref(p), ctypes.byref(kv), fake, fake, fake, None, fake, fake, 570,
                       fake, fake, None, fake, 1 << 40, None)
    assert rc == dsa.DSA_ERR_INVALID_ARG
    rc = L.dsa_forward_paged(ctypes.byref(p), ctypes.byref(kv), fake, fake, fake, None, fake, fake, 576,
                             fake, fake, None, fake, 1 << 40, None)
    assert rc == dsa.DSA_ERR_INVALID_ARG


def test_binding_fails_loudly_without_the_library(monkeypatch, tmp_path):
    monkeypatch.setattr(dsa, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(dsa, "_lib", None)
    with pytest.raises(dsa.DsaError):
        dsa.lib()


def test_host_fault_hook_fails_a_step_before_any_launch(L, monkeypatch):
    """DSA_TEST_INJECT_HOST_ERROR=<step> makes that step return DSA_ERR_CUDA
    after its arguments were validated and before anything is enqueued (no
    GPU needed: the failure comes first); other steps are unaffected."""
    p = _params(3)
    kv = _kv()
    fake = 1 << 40  # never dereferenced
    need_idx = dsa.workspace_size(p, kv, dsa.OP_INDEXER_TOPK)
    need_att = dsa.workspace_size(p, kv, dsa.OP_SPARSE_MLA_DECODE)
    monkeypatch.setenv("DSA_TEST_INJECT_HOST_ERROR", "indexer")
    rc = L.dsa_indexer_topk(ctypes.byref(p), ctypes.byref(kv), fake, fake, fake, None, fake, None,
                            fake, need_idx, None)
    assert rc == dsa.DSA_ERR_CUDA and "injected host failure in indexer" in dsa.last_error()
    monkeypatch.setenv("DSA_TEST_INJECT_HOST_ERROR", "all")
    rc = L.dsa_sparse_mla_decode(ctypes.byref(p), ctypes.byref(kv), fake, fake, 576, fake, fake, fake,
                                 fake, need_att, None)
    assert rc == dsa.DSA_ERR_CUDA and "injected host failure in attention" in dsa.last_error()
    # validation still comes first: a bad workspace is reported as such
    rc = L.dsa_indexer_topk(ctypes.byref(p), ctypes.byref(kv), fake, fake, fake, None, fake, None,
                            fake, need_idx - 256, None)
    assert rc == dsa.DSA_ERR_WORKSPACE
