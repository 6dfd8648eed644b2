"""Pins of the oracle's indexer q^I / k^I / w producer (the step before the
indexer score on the decode path) and of its FP8 / bf16 encoders.

As for the hot-path pins, none re-types the oracle's formula: the encoders
are checked against torch's casts and against the definition of nearest
rounding; the projections against numpy / torch routines in fp64; RoPE
against its closed form on unit vectors, its norm preservation and its
relative-position property; the quantisation against its error bound; and
the whole producer against the indexer score it feeds.
"""
import numpy as np
import pytest
import torch

from long_context_decode_indexer_b200.synth import encode_bf16


def _bf16_bits(a):
    return encode_bf16(np.asarray(a, np.float32))


def _dec_bf16(bits):
    return torch.from_numpy(np.asarray(bits, np.uint16).view(np.int16)).view(torch.bfloat16).double().numpy()


def _dec_e4m3(codes):
    return torch.from_numpy(np.asarray(codes, np.uint8)).view(torch.float8_e4m3fn).double().numpy()


# ---------------------------------------------------------------------------
# encoders
# ---------------------------------------------------------------------------


def test_e4m3_encoder_matches_torch_including_ties_and_saturation(oracle):
    vals = _dec_e4m3(np.arange(0, 0x7F, dtype=np.uint8))               # every finite magnitude
    mids = (vals[:-1] + vals[1:]) / 2                                    # exact ties (5 bits)
    rng = np.random.default_rng(3)
    rand = np.concatenate([rng.standard_normal(4000) * s for s in (1e-3, 0.1, 1.0, 30.0, 600.0)])
    xs = np.concatenate([vals, mids, -mids, rand, [500.0, -1e6, 448.0, 464.0, -0.0, 0.0]])
    xs = xs.astype(np.float32)
    ref = torch.from_numpy(xs).clamp(-448.0, 448.0).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.f64_to_e4m3(float(x)) for x in xs], np.uint8)
    assert np.array_equal(got, ref)


def _project(oracle, nt=3, hidden=96, rank=40, h_idx=4, d_idx=16, rope_dim=8, seed=0, **kw):
    rng = np.random.default_rng(seed)
    x = _bf16_bits(rng.standard_normal((nt, hidden)))
    q_lora = _bf16_bits(rng.standard_normal((nt, rank)))
    w_qb = _bf16_bits(rng.standard_normal((h_idx * d_idx, rank)) / np.sqrt(rank))
    w_k = _bf16_bits(rng.standard_normal((d_idx, hidden)) / np.sqrt(hidden))
    w_proj = _bf16_bits(rng.standard_normal((h_idx, hidden)) / np.sqrt(hidden))
    gamma = (1.0 + 0.1 * rng.standard_normal(d_idx)).astype(np.float32)
    beta = (0.1 * rng.standard_normal(d_idx)).astype(np.float32)
    pos = kw.pop("positions", np.array([0, 5, 1000][:nt] + [7] * max(nt - 3, 0), np.int32))
    out = oracle.indexer_project(x, q_lora, w_qb, w_k, w_proj, gamma, beta, pos, h_idx=h_idx,
                                 d_idx=d_idx, rope_dim=rope_dim, **kw)
    return dict(x=x, q_lora=q_lora, w_qb=w_qb, w_k=w_k, w_proj=w_proj, gamma=gamma, beta=beta,
                pos=pos, out=out, h_idx=h_idx, d_idx=d_idx, rope_dim=rope_dim)


def test_folded_weights_are_the_nearest_bf16(oracle):
    r = _project(oracle, nt=6, h_idx=8)
    wf, wb = r["out"]["w_f"], r["out"]["w_bf16"]
    near = _dec_bf16(wb)
    up = _dec_bf16(wb.astype(np.int32) + 1)
    dn = _dec_bf16(wb.astype(np.int32) - 1)
    # no neighbouring bf16 value is closer than the chosen one
    assert np.all(np.abs(near - wf) <= np.abs(up - wf))
    assert np.all(np.abs(near - wf) <= np.abs(dn - wf))


# ---------------------------------------------------------------------------
# projections, LayerNorm, RoPE
# ---------------------------------------------------------------------------


def test_projections_without_rope_are_matmuls(oracle):
    r = _project(oracle, rope_dim=0)
    x, ql = _dec_bf16(r["x"]), _dec_bf16(r["q_lora"])
    q_ref = (ql @ _dec_bf16(r["w_qb"]).T).reshape(-1, r["h_idx"], r["d_idx"])
    np.testing.assert_allclose(r["out"]["q_f"], q_ref, rtol=1e-12, atol=1e-12)
    k_lin = torch.from_numpy(x @ _dec_bf16(r["w_k"]).T)
    k_ref = torch.nn.functional.layer_norm(k_lin, (r["d_idx"],), torch.from_numpy(r["gamma"]).double(),
                                           torch.from_numpy(r["beta"]).double(), eps=1e-6).numpy()
    np.testing.assert_allclose(r["out"]["k_f"], k_ref, rtol=1e-10, atol=1e-12)


def test_rope_on_unit_vectors_is_the_closed_form(oracle):
    # q^I = e_{2i} in every head (one q_lora input, one weight): RoPE turns it
    # into (cos a, sin a) on dims (2i, 2i+1) with a = pos * theta^(-2i/rope_dim)
    h_idx, d_idx, rope_dim, rank, theta = 2, 16, 8, 4, 10000.0
    pos = np.array([0, 3, 517], np.int32)
    for i in range(rope_dim // 2):
        w_qb = np.zeros((h_idx * d_idx, rank), np.float32)
        for j in range(h_idx):
            w_qb[j * d_idx + 2 * i, 0] = 1.0
        q_lora = np.zeros((3, rank), np.float32)
        q_lora[:, 0] = 1.0
        x = np.ones((3, 8), np.float32)
        out = oracle.indexer_project(_bf16_bits(x), _bf16_bits(q_lora), _bf16_bits(w_qb),
                                     _bf16_bits(np.ones((d_idx, 8))), _bf16_bits(np.ones((h_idx, 8))),
                                     np.ones(d_idx, np.float32), np.zeros(d_idx, np.float32), pos,
                                     h_idx=h_idx, d_idx=d_idx, rope_dim=rope_dim, rope_theta=theta)
        ang = pos * theta ** (-2.0 * i / rope_dim)
        for j in range(h_idx):
            q = out["q_f"][:, j]
            np.testing.assert_allclose(q[:, 2 * i], np.cos(ang), atol=1e-13)
            np.testing.assert_allclose(q[:, 2 * i + 1], np.sin(ang), atol=1e-13)
            others = np.delete(q, [2 * i, 2 * i + 1], axis=1)
            assert np.all(others == 0.0)


def test_rope_preserves_norms_and_leaves_the_other_dims(oracle):
    a = _project(oracle, rope_dim=8, positions=np.array([0, 0, 0], np.int32))
    b = _project(oracle, rope_dim=8, positions=np.array([9, 123, 40000], np.int32))
    qa, qb = a["out"]["q_f"], b["out"]["q_f"]
    np.testing.assert_allclose(np.linalg.norm(qb[..., :8], axis=-1), np.linalg.norm(qa[..., :8], axis=-1),
                               rtol=1e-12)
    assert np.array_equal(qa[..., 8:], qb[..., 8:])
    ka, kb = a["out"]["k_f"], b["out"]["k_f"]
    np.testing.assert_allclose(np.linalg.norm(kb[:, :8], axis=-1), np.linalg.norm(ka[:, :8], axis=-1),
                               rtol=1e-12)
    assert np.array_equal(ka[:, 8:], kb[:, 8:])


def test_rope_scores_depend_only_on_the_relative_position(oracle):
    # the same token content at positions (p, p + d): q . k depends on d only
    def qk(pq, pk):
        rq = _project(oracle, nt=1, seed=7, positions=np.array([pq], np.int32))
        rk = _project(oracle, nt=1, seed=7, positions=np.array([pk], np.int32))
        return np.einsum("hd,d->h", rq["out"]["q_f"][0, :, :8], rk["out"]["k_f"][0, :8])
    np.testing.assert_allclose(qk(10, 3), qk(1010, 1003), rtol=1e-9, atol=1e-12)
    np.testing.assert_allclose(qk(0, 0), qk(777, 777), rtol=1e-9, atol=1e-12)
    assert not np.allclose(qk(10, 3), qk(10, 4))


# ---------------------------------------------------------------------------
# quantisation and weight folding
# ---------------------------------------------------------------------------


def test_fp8_codes_are_within_half_a_step_at_a_minimal_power_of_two_scale(oracle):
    r = _project(oracle, nt=5, h_idx=6, d_idx=32, rope_dim=16, seed=2)
    o = r["out"]
    for vals, codes, scale in ((o["q_f"], o["q_code"], o["q_scale"][..., None]),
                               (o["k_f"], o["k_code"], o["k_scale"][:, None])):
        scale = scale.astype(np.float64)
        assert np.all(np.log2(scale) == np.round(np.log2(scale)))          # powers of two
        amax = np.max(np.abs(vals), axis=-1, keepdims=True)
        assert np.all(amax / scale <= 448.0) and np.all(amax / scale > 224.0)  # the smallest such
        deq = _dec_e4m3(codes) * scale
        # e4m3 has 3 mantissa bits: nearest rounding errs by <= 2^-4 relative,
        # or by half the subnormal step 2^-10 (times the scale) near zero
        err = np.abs(deq - vals)
        assert np.all(err <= np.maximum(np.abs(vals) * 2.0 ** -4, scale * 2.0 ** -10) * (1 + 1e-12))


def test_folded_weights_carry_the_head_scale_factors_and_the_q_scale(oracle):
    r = _project(oracle, nt=4, h_idx=8, d_idx=16, seed=5)
    o = r["out"]
    wp = _dec_bf16(r["x"]) @ _dec_bf16(r["w_proj"]).T
    ref = wp / np.sqrt(r["h_idx"]) / np.sqrt(r["d_idx"]) * o["q_scale"].astype(np.float64)
    np.testing.assert_allclose(o["w_f"], ref, rtol=1e-12)


def test_producer_feeds_the_indexer_score(oracle):
    # The quantised producer outputs, scored by the oracle's indexer, give
    # sum_j (W_proj x)_j / sqrt(H_I d_I) * ReLU(q_j . k) up to the FP8/bf16
    # rounding: the q scale folded into w and the k scale cancel exactly.
    nt, h_idx, d_idx = 6, 8, 32
    r = _project(oracle, nt=nt, h_idx=h_idx, d_idx=d_idx, rope_dim=16, seed=11,
                 positions=np.arange(nt, dtype=np.int32) * 3)
    o = r["out"]
    q_seq = np.zeros(nt, np.int32)
    q_n = np.full(nt, nt, np.int32)
    sc = oracle.indexer_scores(o["q_code"], o["w_bf16"], o["k_code"], q_seq, q_n,
                               seq_row0=np.zeros(1, np.int64), k_scale=o["k_scale"])
    wp = _dec_bf16(r["x"]) @ _dec_bf16(r["w_proj"]).T / np.sqrt(h_idx * d_idx)
    dots = np.einsum("thd,sd->tsh", o["q_f"], o["k_f"])
    ref = np.einsum("th,tsh->ts", wp, np.maximum(dots, 0.0))
    absref = np.einsum("th,tsh->ts", np.abs(wp), np.abs(dots))
    # per term: q and k each within 2^-4 relative, w within 2^-8: a loose bound
    assert np.all(np.abs(sc - ref) <= 0.2 * absref + 1e-9)
    assert np.corrcoef(sc.ravel(), ref.ravel())[0, 1] > 0.99


# ---------------------------------------------------------------------------
# the exported rounding decisions (used by the producer above)
# ---------------------------------------------------------------------------


def test_pow2_scale_is_the_smallest_power_of_two_that_fits_448(oracle):
    assert oracle.pow2_scale(0.0) == 1.0
    assert oracle.pow2_scale(448.0) == 1.0            # fits exactly
    assert oracle.pow2_scale(448.0 * (1 + 2 ** -40)) == 2.0
    assert oracle.pow2_scale(224.0) == 0.5
    assert oracle.pow2_scale(224.0 * (1 + 2 ** -40)) == 1.0
    rng = np.random.default_rng(8)
    for amax in rng.uniform(1e-6, 1e6, 500):
        s = oracle.pow2_scale(amax)
        assert s == 2.0 ** round(np.log2(s))           # a power of two
        assert amax / s <= 448.0 < 2 * amax / s         # the smallest one that fits


def test_quantize_rows_is_the_torch_cast_at_the_row_scale(oracle):
    rng = np.random.default_rng(9)
    v = rng.standard_normal((50, 128)) * rng.uniform(1e-3, 1e3, size=(50, 1))
    v[3] = 0.0                                          # an all-zero row: scale 1, codes 0
    codes, scales = oracle.quantize_rows(v)
    for r in range(50):
        s = oracle.pow2_scale(np.abs(v[r]).max())
        assert scales[r] == s and (r != 3 or (s == 1.0 and not codes[r].any()))
        ref = torch.from_numpy((v[r] / s).astype(np.float32)).clamp(-448, 448)
        # v / s is exact in fp64; its fp32 rounding can only move a tie, so
        # compare where the fp32 value is not within an fp32 ulp of a tie
        assert np.array_equal(codes[r], ref.to(torch.float8_e4m3fn).view(torch.uint8).numpy()) or \
            np.abs(_dec_e4m3(codes[r]) - v[r] / s).max() <= np.abs(v[r] / s).max() / 16


def test_fold_weights_closed_form(oracle):
    # wp = sqrt(H) * sqrt(d) * 2^k / q_scale gives w = 2^k (H = 4 heads here)
    h, d = 4, 128
    qs = np.array([[0.25, 1.0, 4.0, 0.5]], np.float32)
    wp = np.sqrt(h) * np.sqrt(d) * np.array([[1.0, -2.0, 0.5, 8.0]]) / qs.astype(np.float64)
    w_f, w_b = oracle.fold_weights(wp, qs, d)
    assert np.allclose(w_f, [[1.0, -2.0, 0.5, 8.0]], rtol=1e-14, atol=0)
    assert np.array_equal(_dec_bf16(w_b), [[1.0, -2.0, 0.5, 8.0]])
    assert oracle.f64_to_bf16(1.0 + 2 ** -8) == 0x3F80  # a tie rounds to even
    assert oracle.f64_to_bf16(1.0 + 3 * 2 ** -8) == 0x3F82
