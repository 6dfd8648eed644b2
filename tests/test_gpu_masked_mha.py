"""GPU parity of the masked-MHA short-prefill path (DSA blog by marsggbo,
sections 4 and 6; aicoding.csdn.net DSA article, section 4.3) against the
fp64 oracle: per-head MHA attention over every visible position under the
index set's mask.  Tolerances as for the decode attention (same arithmetic:
bf16 products, fp32 accumulation, P as a bf16 hi/lo pair)."""
import numpy as np
import pytest
import torch

import oracle
from conftest import cuda_ok
from gpu_util import check_attention, gpu_indexer_topk, ok_status
from long_context_decode_indexer_b200 import dsa
from long_context_decode_indexer_b200.batch import upload, workspace
from long_context_decode_indexer_b200.synth import make_inputs, make_mha_inputs

pytestmark = [pytest.mark.gpu, pytest.mark.skipif(not cuda_ok(), reason="needs a CUDA GPU")]


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def gpu_mha(m, idx, *, q_per_seq, topk=None, max_n=None):
    nq, h, d_qk = m.q.shape
    d_v = m.v.shape[2]
    topk = idx.shape[1] if idx is not None else (topk or 1)
    max_n = int(m.q_n.max()) if max_n is None else max_n
    p = dsa.make_params(nq=nq, h_idx=1, d_idx=64, h=h, topk=topk, max_n=max_n, q_per_seq=q_per_seq,
                        scale=m.scale, d_qk=d_qk, d_v=d_v)
    q_seq, q_n, row0 = dev(m.q_seq), dev(m.q_n), dev(m.seq_row0)
    kv = dsa.make_kv(q_seq=q_seq, q_n=q_n, seq_row0=row0, cache_rows=m.k.shape[0])
    ws = workspace(dsa.workspace_size(p, kv, dsa.OP_MASKED_MHA))
    out = torch.full((nq, h, d_v), 12345, dtype=torch.int16, device="cuda")
    lse = torch.full((nq, h), float("nan"), dtype=torch.float32, device="cuda")
    idx_d = dev(idx.astype(np.int32)) if idx is not None else None
    q, k, v = dev(m.q), dev(m.k), dev(m.v)
    dsa.masked_mha_prefill(p, kv, q, k, v, idx_d, out, lse, ws)
    ok_status(ws)
    return out.view(torch.bfloat16).double().cpu().numpy(), lse.double().cpu().numpy()


def oracle_mha(m, idx, sel=None):
    sel = np.arange(len(m.q_n)) if sel is None else sel
    return oracle.masked_mha(m.q[sel], m.k, m.v, m.q_seq[sel], m.q_n[sel], m.seq_row0, scale=m.scale,
                             idx=None if idx is None else idx[sel])


def test_prefill_under_the_indexer_mask():
    """600 tokens, the GPU indexer's TopK (k = 256) as the mask: the first
    257 tokens see everything before them, the rest a sparse set; several
    128-query and 128-key tiles with ragged tails."""
    L = 600
    inp = make_inputs(4, L=L, topk=256, with_attention=False)
    idx, _ = gpu_indexer_topk(upload(inp))
    m = make_mha_inputs(L, h=16)
    out, lse = gpu_mha(m, idx, q_per_seq=L)
    ro, rl = oracle_mha(m, idx)
    check_attention(out, lse, ro, rl)


def test_causal_without_index_list_other_widths():
    """No index list (the mask is causal only), d_qk = 128, d_v = 64."""
    m = make_mha_inputs(300, h=8, d_qk=128, d_v=64)
    out, lse = gpu_mha(m, None, q_per_seq=300)
    ro, rl = oracle_mha(m, None)
    check_attention(out, lse, ro, rl)


def test_two_sequences_padding_and_duplicates():
    """Two sequences of 200 tokens (query blocks of 200: a tile never crosses
    into the other sequence), d_qk = 64; index lists with -1 entries and a
    position listed twice (kept once)."""
    import dataclasses
    m = make_mha_inputs(400, h=4, d_qk=64, d_v=128)
    m = dataclasses.replace(m, q_seq=np.repeat(np.arange(2, dtype=np.int32), 200),
                            q_n=np.tile(np.arange(200, dtype=np.int32), 2),
                            seq_row0=np.array([0, 200], np.int64))
    rng = np.random.default_rng(8)
    k = 64
    idx = np.full((400, k), -1, np.int32)
    for t in range(400):
        n = int(m.q_n[t])
        c = min(n, 40)
        if c:
            idx[t, :c] = rng.choice(n, size=c, replace=False)
            idx[t, c] = idx[t, 0]
        idx[t] = idx[t, rng.permutation(k)]
    out, lse = gpu_mha(m, idx, q_per_seq=200, max_n=200)
    ro, rl = oracle_mha(m, idx)
    check_attention(out, lse, ro, rl)


def test_full_size_short_prefill_sampled():
    """4096 tokens, 128 heads, d_qk = 192, d_v = 128, the indexer's k = 2048
    (the short-prefill workload): every output on the GPU, sampled queries
    (tile and k boundaries) against the oracle."""
    L = 4096
    inp = make_inputs(4, L=L, with_attention=False)
    idx, _ = gpu_indexer_topk(upload(inp))
    m = make_mha_inputs(L)
    out, lse = gpu_mha(m, idx, q_per_seq=L)
    sel = np.array([0, 1, 127, 128, 129, 2047, 2048, 2049, 2050, 3000, 4094, 4095])
    ro, rl = oracle_mha(m, idx, sel)
    check_attention(out[sel], lse[sel], ro, rl)
    assert np.all(np.isfinite(out))
