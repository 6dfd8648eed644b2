"""Pins of the masked-MHA short-prefill oracle (DSA blog by marsggbo,
sections 4 and 6; aicoding.csdn.net DSA article, section 4.3) to things
other than itself: torch's scaled-dot-product attention with a boolean mask
(fp64), the MQA sparse-attention oracle (pinned on its own) when every head
reads the same latent row, and closed forms."""
import numpy as np
import pytest
import torch

import oracle
from long_context_decode_indexer_b200.synth import encode_bf16

pytestmark = pytest.mark.filterwarnings("ignore::UserWarning")


def bf16(x):
    return encode_bf16(np.asarray(x, np.float32))


def f64(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def draw(seed, nq, h, d_qk, d_v, rows, sigma=1.0):
    rng = np.random.default_rng(seed)
    q = bf16(rng.standard_normal((nq, h, d_qk)) * sigma)
    k = bf16(rng.standard_normal((rows, h, d_qk)))
    v = bf16(rng.standard_normal((rows, h, d_v)))
    return q, k, v


def sdpa_ref(q, k, v, keep, scale, row0=0):
    """torch SDPA (fp64) per query with the boolean mask `keep` [nq, n]."""
    nq, h, _ = q.shape
    n = keep.shape[1]
    qt = torch.from_numpy(f64(q)).permute(1, 0, 2)              # [h, nq, d]
    kt = torch.from_numpy(f64(k[row0:row0 + n])).permute(1, 0, 2)  # [h, n, d]
    vt = torch.from_numpy(f64(v[row0:row0 + n])).permute(1, 0, 2)
    m = torch.from_numpy(keep)[None].expand(h, nq, n)
    out = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=m, scale=scale)
    s = torch.einsum("hqd,hnd->hqn", qt, kt) * scale
    lse = torch.logsumexp(s.masked_fill(~m, float("-inf")), dim=-1)
    return out.permute(1, 0, 2).numpy(), lse.permute(1, 0).numpy()


def test_masked_equals_sdpa_with_the_index_mask():
    nq, h, d_qk, d_v, L = 6, 3, 40, 24, 50
    q, k, v = draw(1, nq, h, d_qk, d_v, L)
    rng = np.random.default_rng(2)
    q_n = np.array([50, 37, 20, 9, 50, 44], np.int32)
    idx = np.full((nq, 12), -1, np.int32)
    keep = np.zeros((nq, L), bool)
    for t in range(nq):
        sel = rng.choice(int(q_n[t]), size=min(10, int(q_n[t])), replace=False)
        idx[t, :len(sel)] = sel
        keep[t, sel] = True
    idx[0, 11] = idx[0, 0]             # a duplicate: kept once
    idx[1, 10] = 45                    # >= q_n[1]: ignored
    scale = 0.17
    out, lse = oracle.masked_mha(q, k, v, np.zeros(nq, np.int32), q_n, np.array([0], np.int64),
                                 scale=scale, idx=idx)
    ro, rl = sdpa_ref(q, k, v, keep, scale)
    np.testing.assert_allclose(out, ro, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse, rl, rtol=1e-12, atol=1e-12)


def test_no_index_list_is_causal_attention():
    """idx None keeps every visible position: a prefill's causal attention."""
    L, h, d_qk, d_v = 33, 2, 16, 8
    q, k, v = draw(3, L, h, d_qk, d_v, L + 5)
    q_n = np.arange(1, L + 1, dtype=np.int32)       # query t sees s <= t
    out, lse = oracle.masked_mha(q, k, v, np.zeros(L, np.int32), q_n, np.array([5], np.int64),
                                 scale=0.3)
    keep = np.tril(np.ones((L, L), bool))
    ro, rl = sdpa_ref(q, k, v, keep, 0.3, row0=5)
    np.testing.assert_allclose(out, ro, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse, rl, rtol=1e-12, atol=1e-12)


def test_shared_latent_rows_reduce_to_the_mqa_sparse_oracle():
    """With every head's key = the whole latent row and value = its first d_v
    columns (the MQA form) and distinct indices, masked MHA is the sparse
    MQA attention over the same set."""
    nq, h, d_qk, d_v, L = 3, 4, 576, 512, 300
    rng = np.random.default_rng(4)
    c = bf16(rng.standard_normal((L, d_qk)))
    q = bf16(rng.standard_normal((nq, h, d_qk)) * 0.05)
    k = np.repeat(c[:, None, :], h, axis=1)
    v = np.repeat(c[:, None, :d_v], h, axis=1)
    q_n = np.array([300, 150, 64], np.int32)
    idx = np.full((nq, 64), -1, np.int32)
    for t in range(nq):
        idx[t] = np.sort(rng.choice(int(q_n[t]), size=64, replace=False))
    idx[2, 5:] = -1
    q_seq = np.zeros(nq, np.int32)
    row0 = np.array([0], np.int64)
    scale = 576 ** -0.5
    out, lse = oracle.masked_mha(q, k, v, q_seq, q_n, row0, scale=scale, idx=idx)
    ro, rl = oracle.sparse_mla(q, c, idx, q_seq, q_n, scale=scale, d_v=d_v, seq_row0=row0)
    np.testing.assert_allclose(out, ro, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(lse, rl, rtol=1e-12, atol=1e-12)


def test_closed_forms():
    """Zero scale: the mean of the kept values and lse = ln(#kept); an empty
    mask gives out = 0 and lse = -inf; a single kept position returns its value."""
    nq, h, d_qk, d_v, L = 3, 2, 8, 4, 20
    q, k, v = draw(5, nq, h, d_qk, d_v, L)
    q_n = np.array([20, 0, 20], np.int32)
    idx = np.array([[3, 7, 7, 11, -1], [0, 1, 2, -1, -1], [5, -1, -1, -1, -1]], np.int32)
    out, lse = oracle.masked_mha(q, k, v, np.zeros(nq, np.int32), q_n, np.array([0], np.int64),
                                 scale=0.0, idx=idx)
    vv = f64(v)
    np.testing.assert_allclose(out[0], vv[[3, 7, 11]].mean(axis=0), rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(lse[0], np.log(3.0), rtol=1e-14)
    assert np.all(out[1] == 0.0) and np.all(np.isneginf(lse[1]))
    out2, _ = oracle.masked_mha(q, k, v, np.zeros(nq, np.int32), q_n, np.array([0], np.int64),
                                scale=1.3, idx=idx)
    np.testing.assert_allclose(out2[2], vv[5], rtol=1e-14, atol=1e-15)
