"""Helpers shared by the GPU parity tests: run the C-ABI entry points on a
device batch and compare against the fp64 oracle with the tolerances of the
spec contract."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from long_context_decode_indexer_b200 import dsa
from long_context_decode_indexer_b200.batch import DeviceBatch, upload, workspace

# tolerances
SCORE_REL = 1e-3      # |dI| <= 1e-3 |I_ref| ...
SCORE_ABS_REL = 1e-5  # ... or |dI| <= 1e-5 * sum_j |w_j| ReLU(q_j.k)|k_s|
RECALL_BATCH = 0.999
RECALL_QUERY = 0.99
SWAP_GAP = 1e-3       # a swapped position's score is within 1e-3 (relative) of the k-th
OUT_MAX_ABS = 1e-2
OUT_REL_L2 = 2e-3
LSE_ABS = 1e-3


def ok_status(ws):
    st = dsa.check_status(ws)
    assert st == dsa.DSA_OK, "device status %d: %s" % (st, dsa.last_error())


def gpu_scores(db: DeviceBatch, ld=None, max_n=None):
    i = db.inp
    ld = i.max_n if ld is None else ld
    p = db.params(max_n=max_n)
    kv = db.kvdesc()
    ws = workspace(dsa.workspace_size(p, kv, dsa.OP_INDEXER_SCORES))
    scores = torch.full((i.nq, max(ld, 1)), float("nan"), dtype=torch.float32, device="cuda")
    dsa.indexer_scores(p, kv, db.q_idx, db.w, db.kidx, db.k_scale, scores, ld, ws)
    ok_status(ws)
    return scores[:, :ld]


def gpu_topk_from_scores(scores: torch.Tensor, q_n: torch.Tensor, *, topk: int, max_n: int):
    nq = scores.shape[0]
    p = dsa.make_params(nq=nq, h_idx=64, d_idx=128, h=128, topk=topk, max_n=max_n, scale=1.0)
    ws = workspace(dsa.workspace_size(p, None, dsa.OP_TOPK))
    idx = torch.full((nq, topk), -7, dtype=torch.int32, device="cuda")
    nsel = torch.full((nq,), -7, dtype=torch.int32, device="cuda")
    dsa.topk(p, scores, scores.stride(0), q_n, idx, nsel, ws)
    ok_status(ws)
    return idx.cpu().numpy(), nsel.cpu().numpy()


def gpu_indexer_topk(db: DeviceBatch, max_n=None):
    i = db.inp
    p = db.params(max_n=max_n)
    kv = db.kvdesc()
    ws = workspace(dsa.workspace_size(p, kv, dsa.OP_INDEXER_TOPK))
    idx = torch.full((i.nq, i.topk), -7, dtype=torch.int32, device="cuda")
    nsel = torch.full((i.nq,), -7, dtype=torch.int32, device="cuda")
    dsa.indexer_topk(p, kv, db.q_idx, db.w, db.kidx, db.k_scale, idx, nsel, ws)
    ok_status(ws)
    return idx.cpu().numpy(), nsel.cpu().numpy()


def gpu_mla(db: DeviceBatch, idx: np.ndarray, prefill=False):
    i = db.inp
    p = db.params(topk=idx.shape[1])
    kv = db.kvdesc()
    op = dsa.OP_SPARSE_MLA_PREFILL if prefill else dsa.OP_SPARSE_MLA_DECODE
    ws = workspace(dsa.workspace_size(p, kv, op))
    idx_d = torch.from_numpy(np.ascontiguousarray(idx, np.int32)).cuda()
    out = torch.full((i.nq, i.h, i.d_v), 12345, dtype=torch.int16, device="cuda")
    lse = torch.full((i.nq, i.h), float("nan"), dtype=torch.float32, device="cuda")
    fn = dsa.sparse_mla_prefill if prefill else dsa.sparse_mla_decode
    fn(p, kv, db.q, db.kv, db.kv_row_stride, idx_d, out, lse, ws)
    ok_status(ws)
    return out.view(torch.bfloat16).double().cpu().numpy(), lse.double().cpu().numpy()


def gpu_forward(db: DeviceBatch):
    i = db.inp
    p = db.params()
    kv = db.kvdesc()
    ws = workspace(dsa.workspace_size(p, kv, dsa.OP_FORWARD))
    idx = torch.full((i.nq, i.topk), -7, dtype=torch.int32, device="cuda")
    out = torch.full((i.nq, i.h, i.d_v), 12345, dtype=torch.int16, device="cuda")
    lse = torch.full((i.nq, i.h), float("nan"), dtype=torch.float32, device="cuda")
    dsa.forward(p, kv, db.q_idx, db.w, db.kidx, db.k_scale, db.q, db.kv, db.kv_row_stride, out,
                lse, idx, ws, paged=db.page_table is not None)
    ok_status(ws)
    return (idx.cpu().numpy(), out.view(torch.bfloat16).double().cpu().numpy(),
            lse.double().cpu().numpy())


def oracle_kw(inp):
    return dict(seq_row0=inp.seq_row0, page_table=inp.page_table, page_size=inp.page_size)


def oracle_scores(inp, with_abs=True, ld=None):
    return oracle.indexer_scores(inp.q_idx, inp.w, inp.kidx, inp.q_seq, inp.q_n,
                                 k_scale=inp.k_scale, ld=ld, with_abs=with_abs, **oracle_kw(inp))


def check_scores(gpu: np.ndarray, ref: np.ndarray, absref: np.ndarray, q_n: np.ndarray):
    for qi in range(gpu.shape[0]):
        n = int(q_n[qi])
        g, r, a = gpu[qi, :n].astype(np.float64), ref[qi, :n], absref[qi, :n]
        err = np.abs(g - r)
        bad = (err > SCORE_REL * np.abs(r)) & (err > SCORE_ABS_REL * a)
        assert not bad.any(), "query %d: %d bad scores, worst err %g at %d (ref %g, abs %g)" % (
            qi, bad.sum(), err.max(), int(err.argmax()), r[err.argmax()], a[err.argmax()])
        assert np.all(np.isneginf(gpu[qi, n:])), "query %d: entries beyond n are not -inf" % qi


def check_index_set_exact(gpu_idx: np.ndarray, ref_idx: np.ndarray, n: int, k: int):
    m = min(n, k)
    assert np.all(np.diff(gpu_idx[:m]) > 0), "selected positions are not in ascending order"
    g = np.sort(gpu_idx[:m])
    r = np.sort(ref_idx[:m])
    assert np.all(gpu_idx[m:] == -1), "padding is not -1"
    assert np.array_equal(g, r), "index sets differ: %d GPU-only, %d oracle-only" % (
        len(np.setdiff1d(g, r)), len(np.setdiff1d(r, g)))


def check_recall(gpu_idx: np.ndarray, ref_scores: np.ndarray, q_n: np.ndarray, k: int):
    """Recall against the oracle's own scores, with swaps only near the k-th."""
    hit = tot = 0
    for qi in range(gpu_idx.shape[0]):
        n = int(q_n[qi])
        m = min(n, k)
        gi = gpu_idx[qi, :m]
        assert np.all(gi >= 0) and np.all(gi < n), "query %d: index out of range" % qi
        assert np.all(np.diff(gi) > 0), "query %d: positions not in ascending order" % qi
        assert len(np.unique(gi)) == m, "query %d: duplicate indices" % qi
        assert np.all(gpu_idx[qi, m:] == -1), "query %d: padding is not -1" % qi
        ref_idx, _ = oracle.topk(ref_scores[qi, :n], k)
        rs = set(ref_idx[:m].tolist())
        got = sum(1 for s in gi.tolist() if s in rs)
        if n > k:
            tau = ref_scores[qi, ref_idx[m - 1]]
            for s in gi.tolist():
                if s not in rs:
                    assert ref_scores[qi, s] >= tau - SWAP_GAP * max(1.0, abs(tau)), (
                        "query %d: position %d (score %g) swapped in far below the k-th %g"
                        % (qi, s, ref_scores[qi, s], tau))
        assert got >= RECALL_QUERY * m, "query %d recall %d/%d" % (qi, got, m)
        hit += got
        tot += m
    assert hit >= RECALL_BATCH * tot, "batch recall %d/%d" % (hit, tot)


def check_attention(out: np.ndarray, lse: np.ndarray, ref_out: np.ndarray, ref_lse: np.ndarray,
                    magnitude: float = 1.0):
    """Attention output within max-abs 1e-2 (times `magnitude`, the scale of
    the latent values when a test scales them) and rel-L2 2e-3, over the batch
    and for every query on its own; LSE within 1e-3."""
    d = np.abs(out - ref_out)
    assert d.max() <= OUT_MAX_ABS * magnitude, "out max-abs error %g" % d.max()
    rel = np.linalg.norm(out - ref_out) / max(np.linalg.norm(ref_out), 1e-300)
    assert rel <= OUT_REL_L2, "out rel-L2 error %g" % rel
    for qi in range(out.shape[0]):
        nrm = np.linalg.norm(ref_out[qi])
        if nrm > 0:
            rq = np.linalg.norm(out[qi] - ref_out[qi]) / nrm
            assert rq <= OUT_REL_L2, "query %d: out rel-L2 error %g" % (qi, rq)
        else:
            assert not np.any(out[qi]), "query %d: output should be 0" % qi
    both_inf = np.isneginf(lse) & np.isneginf(ref_lse)
    assert np.array_equal(np.isneginf(lse), np.isneginf(ref_lse)), "lse -inf pattern differs"
    dl = np.abs(lse[~both_inf] - ref_lse[~both_inf])
    if dl.size:
        assert dl.max() <= LSE_ABS, "lse error %g" % dl.max()


def oracle_attention(inp, idx, sel=None):
    """Oracle attention for the queries `sel` (all when None) over `idx`."""
    if sel is None:
        sel = np.arange(inp.nq)
    return oracle.sparse_mla(inp.q[sel], inp.kv, idx[sel], inp.q_seq[sel], inp.q_n[sel],
                             scale=inp.scale, d_v=inp.d_v, **oracle_kw(inp))
