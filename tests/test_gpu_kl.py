"""GPU parity of the indexer distillation loss (forward only; DSA blog by
marsggbo, sections 5.1 and 5.2) against the fp64 oracle.

Both sides take the same index scores (the GPU indexer's fp32 output, read
by the oracle as fp64) and, in the sparse stage, the same index set (the
GPU TopK's).  Tolerance, from the arithmetic: the GPU's scaled scores carry
fp32 accumulation error (576 bf16 products; the products are exact in fp32),
about 1e-6 of their magnitude on these workloads, and exp / log-sum-exp in
fp32 add a few ulp; every p[s] is therefore within a relative 1e-4 of the
oracle's.  A relative error eps in every p[s] moves the loss by at most
eps * (1 + sum_s p[s] |ln p[s] - ln r[s]|) (the KL's derivative in p), so
|kl_gpu - kl_ref| <= 1e-4 * (1 + sum_s p[s] |ln p[s] - ln r[s]|)."""
import numpy as np
import pytest
import torch

import oracle
from conftest import cuda_ok
from gpu_util import gpu_indexer_topk, gpu_scores, ok_status
from long_context_decode_indexer_b200 import dsa
from long_context_decode_indexer_b200.batch import upload, workspace
from long_context_decode_indexer_b200.synth import make_inputs

pytestmark = [pytest.mark.gpu, pytest.mark.skipif(not cuda_ok(), reason="needs a CUDA GPU")]

P_REL = 1e-4
KL_REL = 1e-4


def gpu_kl(db, scores, idx=None, with_p=True):
    i = db.inp
    topk = idx.shape[1] if idx is not None else i.topk
    p = db.params(topk=topk)
    kv = db.kvdesc()
    op = dsa.OP_INDEX_KL_DENSE if idx is None else dsa.OP_INDEX_KL_SPARSE
    ws = workspace(dsa.workspace_size(p, kv, op))
    kl = torch.full((i.nq,), float("nan"), dtype=torch.float32, device="cuda")
    ld = scores.shape[1]
    p_out = torch.full((i.nq, ld), float("nan"), dtype=torch.float32, device="cuda") if with_p else None
    idx_d = torch.from_numpy(np.ascontiguousarray(idx, np.int32)).cuda() if idx is not None else None
    dsa.index_kl(p, kv, db.q, db.kv, db.kv_row_stride, scores, scores.stride(0), idx_d, kl, p_out, ws)
    ok_status(ws)
    return kl.double().cpu().numpy(), (p_out.double().cpu().numpy() if with_p else None)


def oracle_kl(inp, scores_np, idx=None):
    kl, p = oracle.index_kl(inp.q, inp.kv, inp.q_seq, inp.q_n, scores_np, scale=inp.scale, idx=idx,
                            seq_row0=inp.seq_row0, page_table=inp.page_table,
                            page_size=inp.page_size, with_p=True)
    return kl, p


def kl_bound(p_ref, scores_np, inp, idx):
    """1 + sum_s p|ln p - ln r| per query, from the oracle's p and the scores."""
    out = np.ones(inp.nq)
    for qi in range(inp.nq):
        n = int(inp.q_n[qi])
        if idx is None:
            pos = np.arange(n)
        else:
            pos = idx[qi][(idx[qi] >= 0) & (idx[qi] < n)]
        if len(pos) == 0:
            continue
        I = scores_np[qi, pos]
        lr = I - (I.max() + np.log(np.exp(I - I.max()).sum()))
        pp = p_ref[qi, pos]
        # a position listed twice holds the sum of its shares in p_out
        _, inv, counts = np.unique(pos, return_inverse=True, return_counts=True)
        pe = pp / counts[inv]
        m = pe > 0
        out[qi] += np.sum(pe[m] * np.abs(np.log(pe[m]) - lr[m]))
    return out


def check(inp, scores, idx=None):
    db = upload(inp)
    kl, p = gpu_kl(db, scores, idx)
    s64 = scores.double().cpu().numpy()
    kl_ref, p_ref = oracle_kl(inp, s64, idx)
    assert np.all(np.isfinite(kl)), "non-finite loss"
    bound = KL_REL * kl_bound(p_ref, s64, inp, idx)
    err = np.abs(kl - kl_ref)
    assert np.all(err <= bound), "kl: worst err %g (bound %g) at query %d, kl_ref %g" % (
        err.max(), bound[err.argmax()], int(err.argmax()), kl_ref[err.argmax()])
    perr = np.abs(p - p_ref)
    pbad = perr > P_REL * p_ref + 1e-12
    assert not pbad.any(), "p: %d entries off, worst %g at %s (ref %g)" % (
        pbad.sum(), perr.max(), np.unravel_index(perr.argmax(), perr.shape), p_ref.flat[perr.argmax()])
    # p sums to 1 over a non-empty set; empty sets give kl = 0
    for qi in range(inp.nq):
        tot = p[qi].sum()
        if kl_ref[qi] == 0.0 and p_ref[qi].sum() == 0.0:
            assert kl[qi] == 0.0 and tot == 0.0
        else:
            assert abs(tot - 1.0) < 1e-4
    return kl, kl_ref


@pytest.mark.parametrize("case", ["v32_ragged", "padded_heads", "paged"])
def test_sparse_stage_matches_oracle(case):
    """The sparse stage over the GPU TopK's set (S_t of section 5.2)."""
    if case == "v32_ragged":
        inp = make_inputs(2, lengths=[5000, 3001, 129, 1])
    elif case == "padded_heads":
        inp = make_inputs(2, lengths=[2600, 700], h=64)
    else:
        inp = make_inputs(5, lengths=[2500, 900])
    db = upload(inp)
    scores = gpu_scores(db)
    idx, _ = gpu_indexer_topk(db)
    check(inp, scores, idx)


def test_sparse_stage_with_padding_and_a_duplicate():
    """Entries of -1 interleaved and a position listed twice (it counts twice)."""
    inp = make_inputs(2, lengths=[3000, 400], topk=512)
    rng = np.random.default_rng(17)
    idx = np.full((inp.nq, 512), -1, np.int32)
    for qi in range(inp.nq):
        n = int(inp.q_n[qi])
        m = min(n, 400)
        idx[qi, :m] = rng.choice(n, size=m, replace=False)
        idx[qi, m // 2] = idx[qi, 0]
        idx[qi] = idx[qi, rng.permutation(512)]
    db = upload(inp)
    check(inp, gpu_scores(db), idx)


@pytest.mark.parametrize("case", ["decode_ragged", "prefill"])
def test_dense_stage_matches_oracle(case):
    """The dense warm-up over every visible position (section 5.1): several
    splits of 256 rows with a ragged tail; the prefill's first query sees no
    position at all (kl = 0)."""
    if case == "decode_ragged":
        inp = make_inputs(2, lengths=[5000, 700, 1, 2049])
    else:
        inp = make_inputs(4, L=300, topk=256)
    db = upload(inp)
    check(inp, gpu_scores(db), None)


def test_loss_is_zero_when_the_indexer_matches_the_attention():
    """A property at any size: with index scores equal to ln p the KL is 0
    (up to rounding); the GPU's own p, fed back as scores, gives ~0."""
    inp = make_inputs(2, lengths=[3000, 1200])
    db = upload(inp)
    scores = gpu_scores(db)
    idx, _ = gpu_indexer_topk(db)
    _, p = gpu_kl(db, scores, idx)
    lp = torch.from_numpy(np.where(p > 0, np.log(np.maximum(p, 1e-300)), -1e30)).float().cuda()
    kl, _ = gpu_kl(db, lp.contiguous(), idx, with_p=False)
    assert np.all(np.abs(kl) < 1e-5), kl
