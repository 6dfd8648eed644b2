"""Pins of the oracle's indexer distillation loss (forward): KL(p || softmax(I))
with p the heads' attention distributions summed over heads and L1-normalised
(DSA blog by marsggbo, section 5.1 for the dense stage, 5.2 for the sparse
stage over the selected set).

None re-types the oracle's formula: a zero query gives uniform p and a closed
form; one and several heads are checked against torch's softmax and kl_div in
fp64; index scores equal to ln p (up to a constant) give zero; the sparse
stage over every position is the dense stage; the loss is never negative.
"""
import numpy as np
import torch

from long_context_decode_indexer_b200.synth import encode_bf16, make_inputs


def _dec_bf16(bits):
    return torch.from_numpy(np.asarray(bits, np.uint16).view(np.int16)).view(torch.bfloat16).double()


def _case(h=4, n=300, seed=0):
    inp = make_inputs(1, L=n, h=h)
    rng = np.random.default_rng(seed)
    I = rng.standard_normal((1, n)) * 2.0
    return inp, I


def _torch_kl(inp, I, positions):
    """kl_div of the log-softmax of I against the head-mean softmax of S,
    over `positions`, with torch in fp64."""
    q = _dec_bf16(inp.q[0])                            # [h, 576]
    c = _dec_bf16(inp.kv[positions])                   # [m, 576]
    S = inp.scale * (q @ c.T)                          # [h, m]
    p = torch.softmax(S, dim=1).mean(dim=0)            # sum over heads, L1-normalised
    logr = torch.log_softmax(torch.from_numpy(I[0, positions]), dim=0)
    return float(torch.nn.functional.kl_div(logr, p, reduction="sum")), p.numpy()


def test_zero_query_gives_uniform_p_and_a_closed_form(oracle):
    inp, I = _case()
    inp.q[:] = 0
    kl, p = oracle.index_kl(inp.q, inp.kv, inp.q_seq, inp.q_n, I, scale=inp.scale,
                            seq_row0=inp.seq_row0, with_p=True)
    n = inp.q_n[0]
    assert np.allclose(p[0, :n], 1.0 / n, rtol=1e-13)
    lse = np.log(np.exp(I[0, :n] - I[0, :n].max()).sum()) + I[0, :n].max()
    assert abs(kl[0] - (-np.log(n) - np.mean(I[0, :n] - lse))) < 1e-12


def test_one_head_is_torch_kl_div(oracle):
    inp, I = _case(h=1)
    kl = oracle.index_kl(inp.q, inp.kv, inp.q_seq, inp.q_n, I, scale=inp.scale, seq_row0=inp.seq_row0)
    ref, _ = _torch_kl(inp, I, np.arange(inp.q_n[0]))
    assert abs(kl[0] - ref) < 1e-11 * max(1.0, abs(ref))


def test_several_heads_are_summed_then_normalised(oracle):
    inp, I = _case(h=16)
    kl, p = oracle.index_kl(inp.q, inp.kv, inp.q_seq, inp.q_n, I, scale=inp.scale,
                            seq_row0=inp.seq_row0, with_p=True)
    ref, p_ref = _torch_kl(inp, I, np.arange(inp.q_n[0]))
    assert np.allclose(p[0, :inp.q_n[0]], p_ref, rtol=1e-12, atol=1e-15)
    assert abs(kl[0] - ref) < 1e-11 * max(1.0, abs(ref))


def test_index_scores_equal_to_log_p_give_zero(oracle):
    inp, _ = _case(h=8)
    n = inp.q_n[0]
    _, p_ref = _torch_kl(inp, np.zeros((1, n)), np.arange(n))
    I = (np.log(p_ref) + 3.7)[None, :]                 # a constant shift changes nothing
    kl = oracle.index_kl(inp.q, inp.kv, inp.q_seq, inp.q_n, I, scale=inp.scale, seq_row0=inp.seq_row0)
    assert abs(kl[0]) < 1e-12


def test_sparse_stage_over_every_position_is_the_dense_stage(oracle):
    inp, I = _case(h=4, n=200)
    n = inp.q_n[0]
    dense, p_d = oracle.index_kl(inp.q, inp.kv, inp.q_seq, inp.q_n, I, scale=inp.scale,
                                 seq_row0=inp.seq_row0, with_p=True)
    idx = np.full((1, 256), -1, np.int32)
    idx[0, :n] = np.random.default_rng(2).permutation(n)
    idx[0] = idx[0, np.random.default_rng(3).permutation(256)]   # -1 interleaved
    sparse, p_s = oracle.index_kl(inp.q, inp.kv, inp.q_seq, inp.q_n, I, scale=inp.scale, idx=idx,
                                  seq_row0=inp.seq_row0, with_p=True)
    assert abs(dense[0] - sparse[0]) < 1e-12
    assert np.allclose(p_d, p_s, rtol=1e-12, atol=1e-16)


def test_sparse_stage_normalises_over_the_selected_set(oracle):
    inp, I = _case(h=4, n=300)
    sel = np.sort(np.random.default_rng(5).choice(300, 64, replace=False))
    idx = np.full((1, 64), -1, np.int32)
    idx[0] = sel
    kl, p = oracle.index_kl(inp.q, inp.kv, inp.q_seq, inp.q_n, I, scale=inp.scale, idx=idx,
                            seq_row0=inp.seq_row0, with_p=True)
    ref, p_ref = _torch_kl(inp, I, sel)
    assert abs(p[0].sum() - 1.0) < 1e-12 and np.all(np.delete(p[0], sel) == 0)
    assert np.allclose(p[0, sel], p_ref, rtol=1e-12)
    assert abs(kl[0] - ref) < 1e-11 * max(1.0, abs(ref))


def test_loss_is_never_negative(oracle):
    for seed in range(5):
        inp, I = _case(h=4, n=150, seed=seed)
        kl = oracle.index_kl(inp.q, inp.kv, inp.q_seq, inp.q_n, I * (seed + 1), scale=inp.scale,
                             seq_row0=inp.seq_row0)
        assert kl[0] >= -1e-14
