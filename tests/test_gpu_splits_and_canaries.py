"""Split-count sweep and canary-guarded outputs.

The attention cuts each query's selected rows into splits according to the
batch size (one split per query when the batch fills the SMs, up to 32 when
it does not); every split count must give the oracle's result.  Every
output buffer is allocated with a guard region after it, filled with a
canary value, and no call may write into it."""
import numpy as np
import pytest
import torch

from conftest import cuda_ok
from gpu_util import check_attention, ok_status, oracle_attention
from long_context_decode_indexer_b200 import dsa
from long_context_decode_indexer_b200.batch import upload, workspace
from long_context_decode_indexer_b200.synth import make_inputs

pytestmark = [pytest.mark.gpu, pytest.mark.skipif(not cuda_ok(), reason="needs a CUDA GPU")]

GUARD = 4096  # elements after each output


def guarded(shape, dtype, fill):
    n = int(np.prod(shape))
    buf = torch.full((n + GUARD,), fill, dtype=dtype, device="cuda")
    return buf, buf[:n].view(*shape)


def guard_intact(buf, fill):
    return bool(torch.all(buf[-GUARD:] == fill))


@pytest.mark.parametrize("nseq,topk", [(1, 2048), (3, 2048), (16, 2048), (40, 2048), (148, 256)])
def test_attention_every_split_count(nseq, topk):
    """32, 32, 9, 8 and 1 split(s) per query."""
    inp = make_inputs(2, nseq=nseq, L=4096, topk=topk)
    rng = np.random.default_rng(nseq)
    idx = np.stack([np.sort(rng.choice(int(n), size=inp.topk, replace=False)) for n in inp.q_n]).astype(np.int32)
    db = upload(inp)
    p = db.params(topk=inp.topk)
    kv = db.kvdesc()
    ws = workspace(dsa.workspace_size(p, kv, dsa.OP_SPARSE_MLA_DECODE))
    obuf, out = guarded((inp.nq, inp.h, inp.d_v), torch.int16, 12345)
    lbuf, lse = guarded((inp.nq, inp.h), torch.float32, -7.0)
    dsa.sparse_mla_decode(p, kv, db.q, db.kv, db.kv_row_stride, torch.from_numpy(idx).cuda(), out, lse, ws)
    ok_status(ws)
    assert guard_intact(obuf, 12345) and guard_intact(lbuf, -7.0)
    sel = np.arange(inp.nq) if inp.nq <= 16 else np.unique(np.r_[0, 1, inp.nq // 2, inp.nq - 1])
    ref_out, ref_lse = oracle_attention(inp, idx, sel)
    check_attention(out.view(torch.bfloat16).double().cpu().numpy()[sel], lse.double().cpu().numpy()[sel],
                    ref_out, ref_lse)


def test_forward_outputs_stay_in_bounds():
    """dsa_forward over a ragged batch (scored and short-history queries)
    writes nothing past out, lse and idx."""
    inp = make_inputs(2, lengths=[5000, 100, 2049, 2048])
    db = upload(inp)
    p, kv = db.params(), db.kvdesc()
    ws = workspace(dsa.workspace_size(p, kv, dsa.OP_FORWARD))
    obuf, out = guarded((inp.nq, inp.h, inp.d_v), torch.int16, 12345)
    lbuf, lse = guarded((inp.nq, inp.h), torch.float32, -7.0)
    ibuf, idx = guarded((inp.nq, inp.topk), torch.int32, -99)
    dsa.forward(p, kv, db.q_idx, db.w, db.kidx, db.k_scale, db.q, db.kv, db.kv_row_stride, out, lse, idx, ws)
    ok_status(ws)
    assert guard_intact(obuf, 12345) and guard_intact(lbuf, -7.0) and guard_intact(ibuf, -99)
    assert not torch.any(idx == -99)  # every index slot written (a position or -1)
