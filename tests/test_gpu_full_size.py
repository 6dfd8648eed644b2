"""Parity at the full workload sizes, in the launch configuration the benchmark
times (one dsa_forward over the whole batch).

The oracle cannot score every query of a full-size batch in a test's time,
so a seeded sample of queries is checked one by one: the TopK of each against
the oracle's fp64 scores of that query (recall and near-tie swaps), its
attention output and LSE against the oracle's attention over the GPU's
selection, and dsa_topk on the oracle's scores (rounded to fp32) against the
oracle's TopK of the same array, bit for bit.  The sample always holds the
extremes of the batch: the longest history, the shortest, and the
short-history boundary (n = k and n = k + 1) where the batch has one.
"""
import numpy as np
import pytest
import torch

import oracle
from conftest import cuda_ok
from gpu_util import (check_attention, check_index_set_exact, check_recall, gpu_topk_from_scores,
                      ok_status, oracle_kw)
from long_context_decode_indexer_b200 import dsa
from long_context_decode_indexer_b200.batch import upload, workspace
from long_context_decode_indexer_b200.synth import CONFIGS, make_inputs

pytestmark = [pytest.mark.gpu, pytest.mark.skipif(not cuda_ok(), reason="needs a CUDA GPU")]

WORKLOADS = {c["name"]: cid for cid, c in CONFIGS.items() if cid != 1}
WORKLOADS["long_decode_16x128k_ragged"] = 3   # L ~ U[1024, 131072], sequences 0/1 at 2048/2049


def _forward(db):
    i = db.inp
    p, kv = db.params(), db.kvdesc()
    ws = workspace(dsa.workspace_size(p, kv, dsa.OP_FORWARD))
    idx = torch.full((i.nq, i.topk), -7, dtype=torch.int32, device="cuda")
    out = torch.full((i.nq, i.h, i.d_v), 12345, dtype=torch.int16, device="cuda")
    lse = torch.full((i.nq, i.h), float("nan"), dtype=torch.float32, device="cuda")
    dsa.forward(p, kv, db.q_idx, db.w, db.kidx, db.k_scale, db.q, db.kv, db.kv_row_stride, out,
                lse, idx, ws, paged=db.page_table is not None)
    ok_status(ws)
    return idx, out, lse


def _sample(inp, cid, count=4):
    n = inp.q_n.astype(np.int64)
    k = inp.topk
    pick = {int(np.argmax(n)), int(np.argmin(n))}
    for target in (k, k + 1):
        hit = np.flatnonzero(n == target)
        if hit.size:
            pick.add(int(hit[0]))
    rng = np.random.default_rng(1234 + cid)
    pick.update(int(x) for x in rng.choice(inp.nq, size=min(count, inp.nq), replace=False))
    return np.array(sorted(pick))


def test_indexer_scores_at_full_context_element_by_element():
    """dsa_indexer_scores over two 131072-position histories (the long-decode
    shapes, heavy tail included), every score against the oracle."""
    from gpu_util import check_scores, gpu_scores, oracle_scores
    inp = make_inputs(3, nseq=2, with_attention=False)
    db = upload(inp)
    g = gpu_scores(db, ld=inp.max_n + 64).cpu().numpy()
    ref, absref = oracle_scores(inp, ld=inp.max_n + 64)
    check_scores(g, ref, absref, inp.q_n)


def test_indexer_scores_beyond_a_million_positions():
    """160 queries (more groups than SMs: one chunk per query, capped at 2^20
    positions, so the 1,100,000-position history takes two chunks) over one
    shared sequence; sampled windows, the chunk seam and the last tile are
    checked against the oracle, position by position."""
    import dataclasses
    from gpu_util import check_scores, gpu_scores
    from long_context_decode_indexer_b200.synth import encode_bf16, encode_e4m3
    n = 1_100_000
    base = make_inputs(3, lengths=[n], with_attention=False)
    nq = 160
    rng = np.random.default_rng(77)
    q_idx = encode_e4m3(rng.standard_normal((nq, base.h_idx, base.d_idx), dtype=np.float32))
    w = encode_bf16(rng.standard_normal((nq, base.h_idx), dtype=np.float32) * np.float32(0.125))
    q_n = np.full(nq, n, np.int32)
    q_n[1::7] = n - 12345                                   # some shorter histories
    inp = dataclasses.replace(base, q_idx=q_idx, w=w, q_seq=np.zeros(nq, np.int32), q_n=q_n,
                              q=np.zeros((nq, base.h, base.d_qk), np.uint16))
    db = upload(inp)
    g = gpu_scores(db, ld=n)
    sel = np.array([0, 1, 57, 159])
    windows = [(0, 3000), (n // 2 - 1500, 3000), ((1 << 20) - 1500, 3000), (n - 12345 - 700, 1400),
               (n - 3000, 3000)]
    for a, wlen in windows:
        view = dataclasses.replace(inp, q_idx=q_idx[sel], w=w[sel], q_seq=np.zeros(len(sel), np.int32),
                                   q_n=np.clip(q_n[sel].astype(np.int64) - a, 0, wlen).astype(np.int32),
                                   seq_row0=np.array([a], np.int64))
        ref, absref = oracle.indexer_scores(view.q_idx, view.w, view.kidx, view.q_seq, view.q_n,
                                            seq_row0=view.seq_row0, ld=wlen, with_abs=True)
        got = g[torch.from_numpy(sel).cuda(), a:a + wlen].cpu().numpy()
        got = np.where(np.arange(wlen)[None, :] < view.q_n[:, None], got, -np.inf)
        check_scores(got, ref, absref, view.q_n)
    tail = g[:, n - 12345:].cpu().numpy()                    # beyond n for the shorter queries
    assert np.all(np.isneginf(tail[1::7]))


@pytest.mark.parametrize("workload", sorted(WORKLOADS))
def test_full_size_forward_on_sampled_queries(workload):
    cid = WORKLOADS[workload]
    inp = make_inputs(cid, ragged=workload.endswith("_ragged"))
    db = upload(inp)
    idx, out, lse = _forward(db)
    sel = _sample(inp, cid)
    k = inp.topk
    idx_s = idx[torch.from_numpy(sel).cuda()].cpu().numpy()
    out_s = out[torch.from_numpy(sel).cuda()].view(torch.bfloat16).double().cpu().numpy()
    lse_s = lse[torch.from_numpy(sel).cuda()].double().cpu().numpy()
    del idx, out, lse
    q_n = inp.q_n[sel]
    ld = max(int(q_n.max()), 1)
    ref = oracle.indexer_scores(inp.q_idx[sel], inp.w[sel], inp.kidx, inp.q_seq[sel], q_n,
                                k_scale=inp.k_scale, ld=ld, **oracle_kw(inp))
    # TopK of the fused path against the oracle's own scores
    check_recall(idx_s, ref, q_n, k)
    # attention over the GPU's selection
    ref_out, ref_lse = oracle.sparse_mla(inp.q[sel], inp.kv, idx_s, inp.q_seq[sel], q_n,
                                         scale=inp.scale, d_v=inp.d_v, **oracle_kw(inp))
    check_attention(out_s, lse_s, ref_out, ref_lse)
    # dsa_topk on identical (fp32) scores is bit-exact
    s32 = np.where(np.isfinite(ref), ref, -np.inf).astype(np.float32)
    g_idx, g_nsel = gpu_topk_from_scores(torch.from_numpy(s32).cuda(),
                                         torch.from_numpy(q_n.astype(np.int32)).cuda(),
                                         topk=k, max_n=ld)
    for r in range(len(sel)):
        n = int(q_n[r])
        o_idx, o_nsel = oracle.topk(s32[r, :n].astype(np.float64), k)
        assert g_nsel[r] == o_nsel
        check_index_set_exact(g_idx[r], o_idx, n, k)
