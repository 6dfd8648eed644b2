"""Pins of the FP8-latent attention oracle: the cache read as e4m3 codes times
a power-of-two row scale (the pages' FP8 format for the indexer's keys,
applied to the latent rows).  Pinned to the bf16 sparse-attention oracle
(pinned on its own) on a bf16 cache holding the same values, decoded by
torch's float8 cast, and to a closed-form scaling property."""
import numpy as np
import torch

import oracle
from long_context_decode_indexer_b200.synth import encode_bf16, make_fp8_latent


def decode_rows(codes, scale):
    f = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float32).numpy()
    return f * scale[:, None]


def case(seed, rows=700, nq=3, h=4):
    rng = np.random.default_rng(seed)
    codes, scale = make_fp8_latent(rows, seed_offset=seed)
    q = encode_bf16(rng.standard_normal((nq, h, 576)).astype(np.float32) * 0.05)
    q_n = np.array([700, 300, 50], np.int32)[:nq]
    idx = np.full((nq, 64), -1, np.int32)
    for t in range(nq):
        idx[t, :40] = rng.choice(int(q_n[t]), size=40, replace=False)
    idx[0, 40] = idx[0, 0]  # a duplicate counts twice, as in the bf16 attention
    return codes, scale, q, q_n, idx


def test_fp8_cache_equals_the_bf16_oracle_on_the_decoded_values():
    codes, scale, q, q_n, idx = case(1)
    vals = decode_rows(codes, scale)
    bf = encode_bf16(vals)
    # the decoded values are exact in bf16 (4 significant bits, power-of-two scale)
    assert np.array_equal((bf.astype(np.uint32) << 16).view(np.float32), vals)
    kw = dict(scale=576 ** -0.5, seq_row0=np.array([0], np.int64))
    q_seq = np.zeros(len(q_n), np.int32)
    o8, l8 = oracle.sparse_mla_fp8(q, codes, scale, idx, q_seq, q_n, **kw)
    ob, lb = oracle.sparse_mla(q, bf, idx, q_seq, q_n, **kw)
    assert np.array_equal(o8, ob) and np.array_equal(l8, lb)


def test_doubling_every_row_scale_doubles_the_output():
    """S is unchanged when q is halved and every scale doubled; the values double."""
    codes, scale, q, q_n, idx = case(2)
    qh = encode_bf16((q.astype(np.uint32) << 16).view(np.float32) * 0.5)
    kw = dict(scale=576 ** -0.5, seq_row0=np.array([0], np.int64))
    q_seq = np.zeros(len(q_n), np.int32)
    o1, l1 = oracle.sparse_mla_fp8(q, codes, scale, idx, q_seq, q_n, **kw)
    o2, l2 = oracle.sparse_mla_fp8(qh, codes, scale * 2, idx, q_seq, q_n, **kw)
    np.testing.assert_allclose(o2, 2 * o1, rtol=1e-13, atol=0)
    np.testing.assert_allclose(l2, l1, rtol=1e-13, atol=1e-13)
