"""GPU parity: every C-ABI entry point against the fp64 oracle on seeded inputs.

Sizes span several 128-row tiles with a ragged tail, the multi-chunk TopK
merge and the single-chunk path, contiguous and paged caches, and the edge
cases of the method (empty history, n = k, n = k + 1, ties)."""
import numpy as np
import pytest
import torch

import oracle
from conftest import cuda_ok
from gpu_util import (check_attention, check_index_set_exact, check_recall, check_scores,
                      gpu_forward, gpu_indexer_topk, gpu_mla, gpu_scores, gpu_topk_from_scores,
                      oracle_attention, oracle_scores)
from long_context_decode_indexer_b200.batch import upload
from long_context_decode_indexer_b200.synth import make_inputs, to_paged

pytestmark = [pytest.mark.gpu, pytest.mark.skipif(not cuda_ok(), reason="needs a CUDA GPU")]


# --------------------------------------------------------------- indexer
@pytest.mark.parametrize("case", ["tiny", "v32_ragged", "v32_kscale", "paged_mtp"])
def test_indexer_scores_match_oracle(case):
    if case == "tiny":
        inp = make_inputs(1)
    elif case == "v32_ragged":
        inp = make_inputs(2, lengths=[5000, 3001, 129, 1])
    elif case == "v32_kscale":
        inp = make_inputs(3, lengths=[2500, 700], with_k_scale=True)
    else:
        inp = make_inputs(5, lengths=[1000, 3000, 520])
    db = upload(inp)
    ld = inp.max_n + 37
    g = gpu_scores(db, ld=ld).cpu().numpy()
    ref, absref = oracle_scores(inp, ld=ld)
    check_scores(g, ref, absref, inp.q_n)


# ------------------------------------------------------------------ TopK
def _topk_case(name):
    rng = np.random.default_rng(11)
    if name == "toy":
        s = np.array([[0.1, 0.2, 0.8, 0.1, 0.1, 0.7, 0.1, 0.1]], np.float32)
        return s, np.array([8]), 2
    if name == "ties":
        s = rng.choice(np.array([-1.0, -0.0, 0.0, 0.5, 2.0], np.float32), size=(3, 9000))
        return s, np.array([9000, 4097, 2000]), 2048
    if name == "boundary":
        s = rng.standard_normal((4, 3000)).astype(np.float32)
        return s, np.array([2048, 2049, 0, 1]), 2048
    if name == "long":
        s = rng.standard_normal((2, 131072)).astype(np.float32)
        return s, np.array([131072, 100000]), 2048
    if name == "small_k":
        s = (rng.standard_normal((3, 5000)) * 3).round().astype(np.float32)   # heavy ties
        return s, np.array([5000, 37, 4999]), 7
    raise ValueError(name)


@pytest.mark.parametrize("name", ["toy", "ties", "boundary", "long", "small_k"])
def test_topk_is_bit_exact_on_identical_scores(name):
    s, n, k = _topk_case(name)
    scores = torch.from_numpy(s).cuda()
    q_n = torch.from_numpy(n.astype(np.int32)).cuda()
    idx, nsel = gpu_topk_from_scores(scores, q_n, topk=k, max_n=int(n.max()))
    for qi in range(s.shape[0]):
        ref, rn = oracle.topk(s[qi, :n[qi]].astype(np.float64), k)
        assert nsel[qi] == rn
        check_index_set_exact(idx[qi], ref, int(n[qi]), k)


@pytest.mark.parametrize("case", ["tiny", "v32_multichunk", "mtp_pairs"])
def test_fused_indexer_topk_equals_scores_then_topk(case):
    if case == "tiny":
        inp = make_inputs(1)
    elif case == "v32_multichunk":
        inp = make_inputs(2, lengths=[20000, 2049, 2048, 7000])
    else:
        inp = make_inputs(5, lengths=[3000, 2047, 9000])
    db = upload(inp)
    idx_f, nsel_f = gpu_indexer_topk(db)
    sc = gpu_scores(db)
    idx_u, nsel_u = gpu_topk_from_scores(sc, db.q_n, topk=inp.topk, max_n=inp.max_n)
    assert np.array_equal(nsel_f, np.minimum(inp.q_n, inp.topk))
    assert np.array_equal(nsel_f, nsel_u)
    for qi in range(inp.nq):
        check_index_set_exact(idx_f[qi], idx_u[qi], int(inp.q_n[qi]), inp.topk)


@pytest.mark.parametrize("case", ["tiny", "v32_multichunk", "prefill_pairs", "heads64_dim64",
                                  "heads16_dim128", "key_scale"])
def test_fused_indexer_topk_recall_against_oracle(case):
    if case == "tiny":
        inp = make_inputs(1)
    elif case == "v32_multichunk":
        inp = make_inputs(2, lengths=[20000, 2049, 9000])
    elif case == "heads64_dim64":      # H_I = 64 with d_I = 64 (64-byte swizzle, N = 64)
        inp = make_inputs(2, lengths=[9000, 3000], d_idx=64)
    elif case == "heads16_dim128":     # H_I = 16 with d_I = 128 (N = 16)
        inp = make_inputs(2, lengths=[9000, 3000], h_idx=16)
    elif case == "key_scale":          # per-row key scales in the fused path
        inp = make_inputs(2, lengths=[12000, 2500], with_k_scale=True)
    else:
        inp = make_inputs(4, L=2600)   # queries t = 0..2599: fallback and scored
    db = upload(inp)
    idx, nsel = gpu_indexer_topk(db)
    if case == "prefill_pairs":
        sel = np.r_[0:3, 2046:2052, 2590:2600]
    else:
        sel = np.arange(inp.nq)
    ref = oracle.indexer_scores(inp.q_idx[sel], inp.w[sel], inp.kidx, inp.q_seq[sel], inp.q_n[sel],
                                seq_row0=inp.seq_row0, ld=inp.max_n, k_scale=inp.k_scale)
    check_recall(idx[sel], ref, inp.q_n[sel], inp.topk)


# -------------------------------------------------------- sparse MLA
@pytest.mark.parametrize("case", ["tiny", "v32", "padded_dups", "paged"])
def test_sparse_mla_matches_oracle(case):
    rng = np.random.default_rng(5)
    if case == "tiny":
        inp = make_inputs(1)
    elif case == "v32":
        inp = make_inputs(2, lengths=[5000, 3001])
    elif case == "padded_dups":
        inp = make_inputs(2, lengths=[600, 40, 3000], h=64)
    else:
        inp = make_inputs(5, lengths=[2500, 900])
    k = inp.topk
    idx = np.full((inp.nq, k), -1, np.int32)
    for qi in range(inp.nq):
        n = int(inp.q_n[qi])
        m = min(n, k)
        idx[qi, :m] = rng.choice(n, size=m, replace=False)
        if case == "padded_dups" and m > 10:
            idx[qi, m // 2] = idx[qi, 0]                          # a duplicate
            idx[qi] = idx[qi, rng.permutation(k)]                 # -1 interleaved
    db = upload(inp)
    out, lse = gpu_mla(db, idx)
    ref_out, ref_lse = oracle_attention(inp, idx)
    check_attention(out, lse, ref_out, ref_lse)


@pytest.mark.parametrize("magnitude", [1e9, 1e5, 1e-6])
def test_sparse_mla_split_partials_keep_the_bf16_range(magnitude):
    """Latents far outside fp16's range (|c| ~ 1e5 and 1e9: outputs beyond
    fp16's 65504) or deep in its subnormals (|c| ~ 1e-6), with the query scaled inversely so that the scores stay
    those of the standard workload: two queries give 32 splits each, so every
    output goes through the split partials and the combine."""
    import dataclasses
    from long_context_decode_indexer_b200.synth import encode_bf16
    inp = make_inputs(2, lengths=[3000, 2500])

    def scaled(bits, f):
        x = (bits.astype(np.uint32) << 16).view(np.float32) * np.float32(f)
        return encode_bf16(x)

    inp = dataclasses.replace(inp, kv=scaled(inp.kv, magnitude), q=scaled(inp.q, 1.0 / magnitude))
    rng = np.random.default_rng(21)
    idx = np.stack([rng.choice(int(n), size=inp.topk, replace=False) for n in inp.q_n]).astype(np.int32)
    db = upload(inp)
    out, lse = gpu_mla(db, idx)
    ref_out, ref_lse = oracle_attention(inp, idx)
    assert np.all(np.isfinite(out))
    check_attention(out, lse, ref_out, ref_lse, magnitude=magnitude)


def test_sparse_mla_prefill_entry_matches_oracle():
    inp = make_inputs(4, L=600, topk=256)
    rng = np.random.default_rng(9)
    idx = np.full((inp.nq, 256), -1, np.int32)
    for t in range(inp.nq):                      # token t sees positions s < t
        m = min(t, 256)
        idx[t, :m] = rng.choice(t, size=m, replace=False) if t else []
    db = upload(inp)
    out, lse = gpu_mla(db, idx, prefill=True)
    sel = np.r_[0:3, 255:259, 590:600]
    ref_out, ref_lse = oracle_attention(inp, idx, sel)
    check_attention(out[sel], lse[sel], ref_out, ref_lse)


# ------------------------------------------------------------ end to end
@pytest.mark.parametrize("case", ["tiny", "long_ragged_small", "paged_mtp", "prefill"])
def test_forward_matches_oracle(case):
    if case == "tiny":
        inp = make_inputs(1)
    elif case == "long_ragged_small":
        inp = make_inputs(3, lengths=[2048, 2049, 0, 9000, 3])
    elif case == "paged_mtp":
        inp = make_inputs(5, lengths=[600, 5000, 2047])
    else:
        inp = make_inputs(4, L=2200)
    db = upload(inp)
    idx, out, lse = gpu_forward(db)
    sel = np.arange(inp.nq) if case != "prefill" else np.r_[0:2, 2040:2060, 2190:2200]
    ref = oracle.indexer_scores(inp.q_idx[sel], inp.w[sel], inp.kidx, inp.q_seq[sel], inp.q_n[sel],
                                seq_row0=inp.seq_row0, page_table=inp.page_table,
                                page_size=inp.page_size, ld=max(inp.max_n, 1))
    check_recall(idx[sel], ref, inp.q_n[sel], inp.topk)
    # attention judged on the GPU's own index set
    ref_out, ref_lse = oracle_attention(inp, idx, sel)
    check_attention(out[sel], lse[sel], ref_out, ref_lse)


@pytest.mark.parametrize("page_size", [64, 128])
def test_paged_forward_equals_contiguous_bit_for_bit(page_size):
    inp = make_inputs(3, lengths=[3000, 2049, 700])
    pg = to_paged(inp, page_size=page_size)
    a = gpu_forward(upload(inp))
    b = gpu_forward(upload(pg))
    for qi in range(inp.nq):
        assert np.array_equal(np.sort(a[0][qi]), np.sort(b[0][qi]))
    assert np.array_equal(a[1], b[1]) and np.array_equal(a[2], b[2])


def test_index_beyond_history_is_flagged_and_skipped():
    from gpu_util import workspace
    from long_context_decode_indexer_b200 import dsa
    inp = make_inputs(1, L=500)
    db = upload(inp)
    idx = np.full((1, inp.topk), -1, np.int32)
    idx[0, :3] = [5, 600, 7]          # 600 >= n = 500
    p = db.params()
    kv = db.kvdesc()
    ws = workspace(dsa.workspace_size(p, kv, dsa.OP_SPARSE_MLA_DECODE))
    out = torch.zeros((1, inp.h, inp.d_v), dtype=torch.int16, device="cuda")
    lse = torch.zeros((1, inp.h), dtype=torch.float32, device="cuda")
    dsa.sparse_mla_decode(p, kv, db.q, db.kv, db.kv_row_stride, torch.from_numpy(idx).cuda(), out, lse, ws)
    assert dsa.check_status(ws) == dsa.DSA_ERR_DEVICE_CHECK
    assert dsa.check_status(ws) == dsa.DSA_OK          # cleared after reading
    ref_out, ref_lse = oracle_attention(inp, idx)       # the oracle skips it too
    check_attention(out.view(torch.bfloat16).double().cpu().numpy(), lse.double().cpu().numpy(),
                    ref_out, ref_lse)
