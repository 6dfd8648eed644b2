"""Pins of the fp64 oracle against what the pages and the mathematics fix.

None of these re-types the oracle's formula: each checks a value printed on a
page, a hand-worked example, a closed form, an invariant, a brute-force search,
or a special case that reduces to a library routine (torch).  Each is chosen so
that a plausible slip in the oracle (a dropped ReLU, a wrong head or query
index, a transposed operand, a wrong cache-row mapping, a tie broken the wrong
way, a mis-normalised softmax) fails at least one of them.
"""
import itertools
import math

import numpy as np
import pytest
import torch

from conftest import read_golden
from long_context_decode_indexer_b200.synth import encode_bf16, encode_e4m3, make_inputs, to_paged

# ---------------------------------------------------------------------------
# number formats
# ---------------------------------------------------------------------------


def test_e4m3_decoder_matches_torch_on_all_codes(oracle):
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()
    got = np.array([oracle.e4m3_to_f64(c) for c in codes])
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(got[ok], ref[ok])
    assert np.array_equal(np.signbit(got[ok]), np.signbit(ref[ok]))


def test_e4m3_decoder_spot_values_from_the_ocp_definition(oracle):
    assert oracle.e4m3_to_f64(0x7E) == 448.0          # largest finite
    assert oracle.e4m3_to_f64(0x01) == 2.0 ** -9      # smallest subnormal
    assert oracle.e4m3_to_f64(0x08) == 2.0 ** -6      # smallest normal
    assert oracle.e4m3_to_f64(0x38) == 1.0
    assert math.isnan(oracle.e4m3_to_f64(0x7F))
    v = oracle.e4m3_to_f64(0x80)
    assert v == 0.0 and math.copysign(1.0, v) < 0


def test_bf16_decoder_matches_torch(oracle):
    rng = np.random.default_rng(1)
    bits = rng.integers(0, 1 << 16, size=4000, dtype=np.uint16)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).double().numpy()
    got = np.array([oracle.bf16_to_f64(int(b)) for b in bits])
    ok = ~np.isnan(ref)
    assert np.array_equal(got[ok], ref[ok])
    assert np.all(np.isnan(got[~ok]))


# ---------------------------------------------------------------------------
# lightning-indexer score
# ---------------------------------------------------------------------------


def _hand_case():
    g = read_golden("indexer_hand.txt")
    q_idx = encode_e4m3(np.array([[g["q0h0"], g["q0h1"]], [g["q1h0"], g["q1h1"]]], np.float32))
    w = encode_bf16(np.array([g["w0"], g["w1"]], np.float32))
    kidx = encode_e4m3(np.array([g["k0"], g["k1"], g["k2"], g["k3"]], np.float32))
    return g, q_idx, w, kidx


def test_scores_hand_worked_example(oracle):
    g, q_idx, w, kidx = _hand_case()
    q_n = np.array(g["n"], np.int32)
    # both queries read the same sequence (rows 0..3)
    sc = oracle.indexer_scores(q_idx, w, kidx, q_seq=[0, 0], q_n=q_n, seq_row0=[0], ld=4)
    assert np.array_equal(sc[0], np.array(g["expected_q0"]))
    assert np.array_equal(sc[1], np.array(g["expected_q1"]))


def test_scores_hand_worked_example_with_key_scale(oracle):
    g, q_idx, w, kidx = _hand_case()
    ks = np.array(g["k_scale"], np.float32)
    sc = oracle.indexer_scores(q_idx[:1], w[:1], kidx, q_seq=[0], q_n=[4], seq_row0=[0],
                               k_scale=ks, ld=4)
    assert np.array_equal(sc[0], np.array(g["expected_q0_scaled"]))


def test_scores_hand_example_reads_the_right_sequence(oracle):
    # The same keys placed second in a two-sequence cache: query 0 reads
    # sequence 1 (rows 5..8), so the scores must not change.
    g, q_idx, w, kidx = _hand_case()
    junk = encode_e4m3(np.full((5, 4), 3.0, np.float32))
    cache = np.concatenate([junk, kidx])
    sc = oracle.indexer_scores(q_idx[:1], w[:1], cache, q_seq=[1], q_n=[4],
                               seq_row0=[0, 5], ld=4)
    assert np.array_equal(sc[0], np.array(g["expected_q0"]))


def test_scores_are_zero_when_every_dot_is_negative(oracle):
    rng = np.random.default_rng(2)
    q = np.abs(rng.standard_normal((1, 8, 64))).astype(np.float32) + 0.1
    k = -np.abs(rng.standard_normal((50, 64))).astype(np.float32) - 0.1
    w = rng.standard_normal((1, 8)).astype(np.float32)
    sc = oracle.indexer_scores(encode_e4m3(q), encode_bf16(w), encode_e4m3(k),
                               q_seq=[0], q_n=[50], seq_row0=[0])
    assert np.all(sc == 0.0)


def test_scores_reduce_to_one_matvec_when_every_dot_is_positive(oracle):
    # With all q.k > 0 the ReLU is the identity, so
    # I[s] = sum_j w_j (q_j . k_s) = (sum_j w_j q_j) . k_s : a single matvec.
    rng = np.random.default_rng(3)
    q = encode_e4m3(np.abs(rng.standard_normal((1, 6, 32))).astype(np.float32) + 0.05)
    k = encode_e4m3(np.abs(rng.standard_normal((40, 32))).astype(np.float32) + 0.05)
    w = encode_bf16(rng.standard_normal((1, 6)).astype(np.float32))
    sc = oracle.indexer_scores(q, w, k, q_seq=[0], q_n=[40], seq_row0=[0])
    qd = torch.from_numpy(q).view(torch.float8_e4m3fn).double()[0]
    kd = torch.from_numpy(k).view(torch.float8_e4m3fn).double()
    wd = torch.from_numpy(w.view(np.int16)).view(torch.bfloat16).double()[0]
    ref = torch.mv(kd, torch.mv(qd.T, wd)).numpy()
    np.testing.assert_allclose(sc[0], ref, rtol=1e-12, atol=1e-12)


def test_scores_scale_exactly_with_w_and_key_scale(oracle):
    inp = make_inputs(1, L=300)
    base = oracle.indexer_scores(inp.q_idx, inp.w, inp.kidx, inp.q_seq, inp.q_n,
                                 seq_row0=inp.seq_row0)
    # w * 2: bf16 doubling is exact, and so is every product and sum in fp64
    w2 = encode_bf16(torch.from_numpy(inp.w.view(np.int16)).view(torch.bfloat16).float().numpy() * 2)
    dbl = oracle.indexer_scores(inp.q_idx, w2, inp.kidx, inp.q_seq, inp.q_n, seq_row0=inp.seq_row0)
    assert np.array_equal(dbl, 2 * base)
    ks = np.full(inp.rows, 0.25, np.float32)
    quarter = oracle.indexer_scores(inp.q_idx, inp.w, inp.kidx, inp.q_seq, inp.q_n,
                                    seq_row0=inp.seq_row0, k_scale=ks)
    assert np.array_equal(quarter, base * 0.25)
    ones = oracle.indexer_scores(inp.q_idx, inp.w, inp.kidx, inp.q_seq, inp.q_n,
                                 seq_row0=inp.seq_row0, k_scale=np.ones(inp.rows, np.float32))
    assert np.array_equal(ones, base)


def test_scores_follow_the_rows_under_a_page_table(oracle):
    inp = make_inputs(2, nseq=3, L=700)
    pg = to_paged(inp)
    a = oracle.indexer_scores(inp.q_idx, inp.w, inp.kidx, inp.q_seq, inp.q_n, seq_row0=inp.seq_row0)
    b = oracle.indexer_scores(pg.q_idx, pg.w, pg.kidx, pg.q_seq, pg.q_n,
                              page_table=pg.page_table, page_size=pg.page_size)
    assert np.array_equal(a, b)


def test_scores_beyond_the_history_are_minus_inf(oracle):
    inp = make_inputs(1, L=200)
    sc = oracle.indexer_scores(inp.q_idx, inp.w, inp.kidx, inp.q_seq, inp.q_n,
                               seq_row0=inp.seq_row0, ld=256)
    assert np.all(np.isneginf(sc[:, 200:]))
    assert np.all(np.isfinite(sc[:, :200]))


# ---------------------------------------------------------------------------
# TopK
# ---------------------------------------------------------------------------


def test_topk_page_toy_example(oracle):
    g = read_golden("toy_topk.txt")
    idx, nsel = oracle.topk(np.array(g["scores"]), int(g["k"][0]))
    assert nsel == 2
    assert sorted((idx + 1).tolist()) == [int(v) for v in g["expected_positions_1based"]]


def _brute_force_topk(scores, k):
    """The unique k-subset whose every member beats every non-member under
    (higher score, then lower position)."""
    n = len(scores)
    if n <= k:
        return set(range(n))
    found = []
    for sub in itertools.combinations(range(n), k):
        inside = set(sub)
        ok = all((scores[a] > scores[b]) or (scores[a] == scores[b] and a < b)
                 for a in inside for b in range(n) if b not in inside)
        if ok:
            found.append(inside)
    assert len(found) == 1
    return found[0]


def test_topk_brute_force_with_ties(oracle):
    rng = np.random.default_rng(4)
    for trial in range(300):
        n = int(rng.integers(1, 9))
        k = int(rng.integers(1, 9))
        scores = rng.choice([-1.0, -0.0, 0.0, 0.5, 0.5, 1.0, 2.0], size=n)
        idx, nsel = oracle.topk(scores, k)
        assert nsel == min(n, k)
        assert np.all(idx[nsel:] == -1)
        assert set(idx[:nsel].tolist()) == _brute_force_topk(scores.tolist(), k), (scores, k)


def test_topk_keeps_everything_when_history_fits(oracle):
    for n in (0, 1, 5, 16):
        idx, nsel = oracle.topk(np.random.default_rng(n).standard_normal(n), 16)
        assert nsel == n
        assert idx[:n].tolist() == list(range(n)) and np.all(idx[n:] == -1)


def test_topk_boundary_n_equals_k_plus_one_drops_the_minimum(oracle):
    scores = np.array([3.0, 1.0, 2.0, 1.0, 5.0])        # n = 5, k = 4
    idx, _ = oracle.topk(scores, 4)
    assert sorted(idx.tolist()) == [0, 1, 2, 4]         # tie at 1.0: lower index kept


def test_topk_invariant_under_monotone_transforms(oracle):
    rng = np.random.default_rng(5)
    s = rng.standard_normal(5000)
    a, _ = oracle.topk(s, 300)
    b, _ = oracle.topk(np.exp(s) * 3.0 + 1.0, 300)
    c, _ = oracle.topk(np.arctan(s), 300)
    assert set(a.tolist()) == set(b.tolist()) == set(c.tolist())
    ref = set(np.argsort(-s, kind="stable")[:300].tolist())
    assert set(a.tolist()) == ref


def test_topk_signed_zeros_tie_by_position(oracle):
    s = np.array([-0.0, 0.0, -0.0, 0.0, -1.0])
    idx, _ = oracle.topk(s, 2)
    assert sorted(idx.tolist()) == [0, 1]


# ---------------------------------------------------------------------------
# sparse MQA-mode MLA attention
# ---------------------------------------------------------------------------


def _decoded(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).double()


def test_attention_single_row_is_that_row(oracle):
    inp = make_inputs(1, L=64)
    idx = np.full((1, 8), -1, np.int32)
    idx[0, 3] = 17
    out, lse = oracle.sparse_mla(inp.q, inp.kv, idx, inp.q_seq, inp.q_n, scale=inp.scale,
                                 seq_row0=inp.seq_row0)
    c = _decoded(inp.kv[17])
    assert np.array_equal(out[0], np.broadcast_to(c[:512].numpy(), out[0].shape))
    S = inp.scale * (_decoded(inp.q[0]) @ c).numpy()
    np.testing.assert_allclose(lse[0], S, rtol=1e-13, atol=1e-13)


def test_attention_equal_rows_give_that_row(oracle):
    inp = make_inputs(1, L=8)
    kv = np.repeat(inp.kv[:1], 8, axis=0)
    idx = np.arange(8, dtype=np.int32)[None]
    out, lse = oracle.sparse_mla(inp.q, kv, idx, inp.q_seq, inp.q_n, scale=inp.scale,
                                 seq_row0=inp.seq_row0)
    np.testing.assert_allclose(out[0], np.broadcast_to(_decoded(kv[0])[:512].numpy(), out[0].shape),
                               rtol=1e-14, atol=1e-14)


def test_attention_zero_scale_is_the_mean_and_log_count(oracle):
    inp = make_inputs(1, L=40)
    idx = np.array([[3, 7, 7, 20, -1, 39]], np.int32)    # 7 listed twice counts twice
    out, lse = oracle.sparse_mla(inp.q, inp.kv, idx, inp.q_seq, inp.q_n, scale=0.0,
                                 seq_row0=inp.seq_row0)
    vals = _decoded(inp.kv[[3, 7, 7, 20, 39]])[:, :512]
    np.testing.assert_allclose(out[0], np.broadcast_to(vals.mean(0).numpy(), out[0].shape),
                               rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(lse[0], math.log(5.0), rtol=1e-14)


def test_attention_matches_torch_sdpa(oracle):
    inp = make_inputs(1, L=500)
    rng = np.random.default_rng(6)
    sel = rng.choice(500, size=200, replace=False).astype(np.int32)
    idx = np.full((1, 256), -1, np.int32)
    idx[0, :200] = sel
    out, lse = oracle.sparse_mla(inp.q, inp.kv, idx, inp.q_seq, inp.q_n, scale=inp.scale,
                                 seq_row0=inp.seq_row0)
    qd = _decoded(inp.q[0])                       # [H, 576]
    kd = _decoded(inp.kv[sel])                    # [200, 576]
    ref = torch.nn.functional.scaled_dot_product_attention(
        qd[None, :, None, :], kd[None, None].expand(1, qd.shape[0], -1, -1),
        kd[None, None, :, :512].expand(1, qd.shape[0], -1, -1), scale=inp.scale)[0, :, 0]
    np.testing.assert_allclose(out[0], ref.numpy(), rtol=1e-10, atol=1e-12)
    ref_lse = torch.logsumexp(inp.scale * qd @ kd.T, dim=-1).numpy()
    np.testing.assert_allclose(lse[0], ref_lse, rtol=1e-12, atol=1e-12)


def test_attention_permutation_and_padding_invariant(oracle):
    inp = make_inputs(1, L=300)
    rng = np.random.default_rng(7)
    sel = rng.choice(300, size=100, replace=False).astype(np.int32)
    a = np.full((1, 128), -1, np.int32)
    a[0, :100] = sel
    b = np.full((1, 128), -1, np.int32)
    b[0, rng.choice(128, size=100, replace=False)] = rng.permutation(sel)
    oa, la = oracle.sparse_mla(inp.q, inp.kv, a, inp.q_seq, inp.q_n, scale=inp.scale, seq_row0=inp.seq_row0)
    ob, lb = oracle.sparse_mla(inp.q, inp.kv, b, inp.q_seq, inp.q_n, scale=inp.scale, seq_row0=inp.seq_row0)
    np.testing.assert_allclose(oa, ob, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(la, lb, rtol=1e-13, atol=1e-13)


def test_attention_ignores_entries_beyond_the_history_and_empty_sets(oracle):
    inp = make_inputs(1, L=50)
    idx = np.array([[60, -1, 55]], np.int32)          # nothing valid (n = 50)
    out, lse = oracle.sparse_mla(inp.q, inp.kv, idx, inp.q_seq, inp.q_n, scale=inp.scale,
                                 seq_row0=inp.seq_row0)
    assert np.all(out == 0.0) and np.all(np.isneginf(lse))


def test_sparse_equals_dense_when_history_fits_in_k(oracle):
    # n <= k: DSA keeps every position, so the result is dense attention.
    inp = make_inputs(2, nseq=3, L=1000, topk=1024)
    idx, out, lse = oracle.forward(inp.q_idx, inp.w, inp.kidx, inp.q, inp.kv, inp.q_seq,
                                   inp.q_n, k=1024, scale=inp.scale, seq_row0=inp.seq_row0)
    dout, dlse = oracle.dense_mla(inp.q, inp.kv, inp.q_seq, inp.q_n, scale=inp.scale,
                                  seq_row0=inp.seq_row0)
    np.testing.assert_allclose(out, dout, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(lse, dlse, rtol=1e-12, atol=1e-12)


def test_forward_composes_score_topk_attention(oracle):
    inp = make_inputs(1, L=1500, topk=256)
    idx, out, lse = oracle.forward(inp.q_idx, inp.w, inp.kidx, inp.q, inp.kv, inp.q_seq,
                                   inp.q_n, k=256, scale=inp.scale, seq_row0=inp.seq_row0)
    sc = oracle.indexer_scores(inp.q_idx, inp.w, inp.kidx, inp.q_seq, inp.q_n, seq_row0=inp.seq_row0)
    ref = set(np.argsort(-sc[0], kind="stable")[:256].tolist())
    assert set(idx[0].tolist()) == ref
    o2, l2 = oracle.sparse_mla(inp.q, inp.kv, idx, inp.q_seq, inp.q_n, scale=inp.scale,
                               seq_row0=inp.seq_row0)
    assert np.array_equal(out, o2) and np.array_equal(lse, l2)
