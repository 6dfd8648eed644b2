"""The allocation-free fused indexer + TopK entry point.

dsa_indexer_topk_static serves callers that cannot allocate device memory
(their framework's allocator owns the device, or they run under a fixed
memory budget): its scratch is a fixed array inside the library instead of a
caller workspace.  It must return exactly what dsa_indexer_topk returns, on
every call, although all calls share (and leave behind) the same scratch.
This file is collected last so that a failure here leaves the rest of a
stop-at-first-failure run already done.
"""
import numpy as np
import pytest
import torch

from conftest import cuda_ok
from gpu_util import gpu_indexer_topk
from long_context_decode_indexer_b200 import dsa
from long_context_decode_indexer_b200.batch import upload
from long_context_decode_indexer_b200.synth import make_inputs

pytestmark = [pytest.mark.gpu, pytest.mark.skipif(not cuda_ok(), reason="needs a CUDA GPU")]


def _static_call(db):
    i = db.inp
    idx = torch.full((i.nq, i.topk), -7, dtype=torch.int32, device="cuda")
    nsel = torch.full((i.nq,), -7, dtype=torch.int32, device="cuda")
    status = torch.full((1,), 12345, dtype=torch.int32, device="cuda")
    dsa.indexer_topk_static(db.params(), db.kvdesc(), db.q_idx, db.w, db.kidx, db.k_scale,
                            idx, nsel, status)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), nsel.cpu().numpy(), int(status.item())


@pytest.mark.parametrize("case", ["multichunk", "pairs_and_fallback"])
def test_static_scratch_matches_workspace_entry_point_twice(case):
    if case == "multichunk":
        # several chunks per query: histograms, candidate lists and the merge
        # all live in the scratch
        inp = make_inputs(2, lengths=[20000, 2049, 9000])
    else:
        inp = make_inputs(5, lengths=[3000, 2047, 700])
    db = upload(inp)
    ref_idx, ref_nsel = gpu_indexer_topk(db)
    for _ in range(2):  # the second call starts from the first call's leftovers
        idx, nsel, status = _static_call(db)
        assert status == dsa.DSA_OK
        assert np.array_equal(nsel, ref_nsel)
        assert np.array_equal(idx, ref_idx)   # same positions, same (ascending) order


def test_static_scratch_rejects_shapes_that_do_not_fit():
    inp = make_inputs(2, lengths=[2100, 2100])
    db = upload(inp)
    p = db.params(max_n=131072)        # 256 queries at 128K: about 25 MB of scratch
    p.nq = 256
    with pytest.raises(dsa.DsaError) as e:
        dsa.indexer_topk_static(p, db.kvdesc(), db.q_idx, db.w, db.kidx, None, 0x1000, None, None)
    assert e.value.code == dsa.DSA_ERR_UNSUPPORTED
