"""Failure detection on the GPU: a bounded wait that runs out.

Every mbarrier and inter-CTA wait in the kernels has a budget; when it runs
out the kernel records DSA_ERR_TIMEOUT in the status word, lets its other
waits run out the same way, waits for its own copies in flight, frees its
tensor memory and returns, so the context stays usable.  The library's test
hook (environment variable DSA_TEST_INJECT_TIMEOUT=indexer or =attention)
runs that kernel with a ~50 us budget and leaves out one arrival that the
first CTA's MMA issuer waits for: nothing faults, traps or spins forever,
the wait simply expires.  The next call without the hook must succeed and
give the right answer on the same workspace.
"""
import time

import numpy as np
import pytest
import torch

from conftest import cuda_ok
from gpu_util import check_attention, check_recall, oracle_attention, oracle_scores
from long_context_decode_indexer_b200 import dsa
from long_context_decode_indexer_b200.batch import upload, workspace
from long_context_decode_indexer_b200.synth import make_inputs

pytestmark = [pytest.mark.gpu, pytest.mark.skipif(not cuda_ok(), reason="needs a CUDA GPU")]


def _forward(db, ws, idx, out, lse):
    dsa.forward(db.params(), db.kvdesc(), db.q_idx, db.w, db.kidx, db.k_scale, db.q, db.kv,
                db.kv_row_stride, out, lse, idx, ws)


@pytest.mark.parametrize("kernel", ["indexer", "attention"])
def test_expired_wait_is_reported_and_the_next_call_succeeds(kernel, monkeypatch):
    # three queries: several chunks each (the parallel selection's waits),
    # one on the short-history boundary
    inp = make_inputs(2, lengths=[20000, 9000, 2049])
    db = upload(inp)
    p, kv = db.params(), db.kvdesc()
    ws = workspace(dsa.workspace_size(p, kv, dsa.OP_FORWARD))
    idx = torch.full((inp.nq, inp.topk), -7, dtype=torch.int32, device="cuda")
    out = torch.zeros((inp.nq, inp.h, inp.d_v), dtype=torch.int16, device="cuda")
    lse = torch.zeros((inp.nq, inp.h), dtype=torch.float32, device="cuda")

    monkeypatch.setenv("DSA_TEST_INJECT_TIMEOUT", kernel)
    torch.cuda.synchronize()
    t0 = time.time()
    _forward(db, ws, idx, out, lse)
    assert dsa.check_status(ws) == dsa.DSA_ERR_TIMEOUT
    assert time.time() - t0 < 0.5          # the short budget ran out, not the ~1 s one
    assert dsa.check_status(ws) == dsa.DSA_OK   # read once, then cleared

    monkeypatch.delenv("DSA_TEST_INJECT_TIMEOUT")
    _forward(db, ws, idx, out, lse)
    assert dsa.check_status(ws) == dsa.DSA_OK
    g_idx = idx.cpu().numpy()
    ref = oracle_scores(inp, with_abs=False, ld=inp.max_n)
    check_recall(g_idx, ref, inp.q_n, inp.topk)
    ref_out, ref_lse = oracle_attention(inp, g_idx)
    check_attention(out.view(torch.bfloat16).double().cpu().numpy(), lse.double().cpu().numpy(),
                    ref_out, ref_lse)


def test_expired_wait_in_the_score_pass(monkeypatch):
    inp = make_inputs(2, lengths=[9000, 3000])
    db = upload(inp)
    p, kv = db.params(), db.kvdesc()
    ws = workspace(dsa.workspace_size(p, kv, dsa.OP_INDEXER_SCORES))
    scores = torch.zeros((inp.nq, inp.max_n), dtype=torch.float32, device="cuda")
    monkeypatch.setenv("DSA_TEST_INJECT_TIMEOUT", "indexer")
    dsa.indexer_scores(p, kv, db.q_idx, db.w, db.kidx, db.k_scale, scores, inp.max_n, ws)
    assert dsa.check_status(ws) == dsa.DSA_ERR_TIMEOUT
    monkeypatch.delenv("DSA_TEST_INJECT_TIMEOUT")
    dsa.indexer_scores(p, kv, db.q_idx, db.w, db.kidx, db.k_scale, scores, inp.max_n, ws)
    assert dsa.check_status(ws) == dsa.DSA_OK
    from gpu_util import check_scores
    ref, absref = oracle_scores(inp, ld=inp.max_n)
    check_scores(scores.cpu().numpy(), ref, absref, inp.q_n)
