"""GPU parity of the indexer producer (q^I, k^I, w and the cache append)
against the fp64 oracle.

Two kinds of check.  The values before rounding (after RoPE; w before
folding) come from fp32 tensor-core sums and must match the oracle's fp64
values to a tolerance the arithmetic gives.  The rounding decisions (the
power-of-two scales, the E4M3 codes, the bf16 weights) are compared in the
kernel's own precision: the oracle's quantiser applied to the kernel's fp32
values must give the kernel's bytes exactly.  Against the oracle's own bytes
(from fp64 values) a code may differ by one step only where the two values
straddle a rounding boundary.  Finally the produced cache feeds the fused
indexer, whose selection is checked against the oracle's scores.
"""
import numpy as np
import pytest
import torch

import oracle
from conftest import cuda_ok
from gpu_util import check_recall, ok_status
from long_context_decode_indexer_b200 import dsa
from long_context_decode_indexer_b200.batch import workspace
from long_context_decode_indexer_b200.synth import make_inputs, make_project_inputs, to_paged

pytestmark = [pytest.mark.gpu, pytest.mark.skipif(not cuda_ok(), reason="needs a CUDA GPU")]

SENTINEL = 0x5A
VALUE_REL = 2e-4   # fp32 sums of <= 7168 bf16 products (and LayerNorm) against fp64, per row rms


def _dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a))
    return (t.view(dtype) if dtype is not None else t).cuda()


def _run(pi, cache_rows, seq_row0=None, page_table=None, page_size=0):
    nt, H, d = pi.nt, pi.h_idx, pi.d_idx
    pp = dsa.make_project_params(nt=nt, hidden=pi.x.shape[1], q_lora_rank=pi.q_lora.shape[1],
                                 h_idx=H, d_idx=d, rope_dim=pi.rope_dim)
    # device copies stay referenced until the call's work is done (a dropped
    # temporary would return its memory to the allocator before the launch)
    q_seq = _dev(pi.q_seq)
    d_row0 = None if seq_row0 is None else _dev(seq_row0)
    d_pt = None if page_table is None else _dev(page_table)
    kv = dsa.make_kv(q_seq=q_seq, q_n=None, seq_row0=d_row0, page_table=d_pt,
                     page_size=page_size, cache_rows=cache_rows)
    ws = workspace(dsa.project_workspace_size(pp))
    out = dict(q_idx=torch.zeros((nt, H, d), dtype=torch.uint8, device="cuda"),
               q_scale=torch.zeros((nt, H), dtype=torch.float32, device="cuda"),
               w=torch.zeros((nt, H), dtype=torch.int16, device="cuda"),
               kidx=torch.full((cache_rows, d), SENTINEL, dtype=torch.uint8, device="cuda"),
               k_scale=torch.full((cache_rows,), -1.0, dtype=torch.float32, device="cuda"),
               q_f32=torch.zeros((nt, H, d), dtype=torch.float32, device="cuda"),
               k_f32=torch.zeros((nt, d), dtype=torch.float32, device="cuda"),
               w_f32=torch.zeros((nt, H), dtype=torch.float32, device="cuda"))
    dsa.indexer_project(pp, kv, _dev(pi.x, torch.int16), _dev(pi.q_lora, torch.int16),
                        _dev(pi.w_qb, torch.int16), _dev(pi.w_k, torch.int16),
                        _dev(pi.w_proj, torch.int16), _dev(pi.ln_gamma), _dev(pi.ln_beta),
                        _dev(pi.positions), out["q_idx"], out["q_scale"], out["w"], out["kidx"],
                        out["k_scale"], ws, q_f32=out["q_f32"], k_f32=out["k_f32"],
                        w_f32=out["w_f32"])
    ok_status(ws)
    return {k: v.cpu().numpy() for k, v in out.items()}


def _rows_of(pi, seq_row0=None, page_table=None, page_size=0):
    if page_table is None:
        return seq_row0[pi.q_seq].astype(np.int64) + pi.positions
    return (page_table[pi.q_seq, pi.positions // page_size].astype(np.int64) * page_size
            + pi.positions % page_size)


def _close(gpu, ref, what):
    g = gpu.reshape(-1, gpu.shape[-1]).astype(np.float64)
    r = ref.reshape(-1, ref.shape[-1])
    rms = np.sqrt((r ** 2).mean(axis=1, keepdims=True)) + 1e-30
    err = (np.abs(g - r) / rms).max()
    assert err <= VALUE_REL, "%s: max error %.3g of the row rms" % (what, err)


def _straddle_only(codes_g, codes_r, v32, v64):
    """Where the kernel's code differs from the oracle's, the kernel's fp32
    value and the oracle's fp64 value (both divided by the scale) lie on the
    two sides of the rounding boundary between the two codes."""
    diff = codes_g != codes_r
    if not diff.any():
        return 0
    dec = lambda c: torch.from_numpy(np.ascontiguousarray(c)).view(torch.float8_e4m3fn).double().numpy()
    a, b = dec(codes_g[diff]), dec(codes_r[diff])
    mid = (a + b) / 2
    straddle = (v32[diff] - mid) * (v64[diff] - mid) <= 0
    assert straddle.all(), "codes differ where the two values do not straddle a boundary"
    return int(diff.sum())


def _check(pi, g, rows):
    H, d = pi.h_idx, pi.d_idx
    ref = oracle.indexer_project(pi.x, pi.q_lora, pi.w_qb, pi.w_k, pi.w_proj, pi.ln_gamma,
                                 pi.ln_beta, pi.positions, h_idx=H, d_idx=d, rope_dim=pi.rope_dim)
    # values before rounding: fp32 tensor-core sums against fp64
    _close(g["q_f32"], ref["q_f"], "q^I")
    _close(g["k_f32"], ref["k_f"], "k^I")
    wp_ref = ref["w_f"] / ref["q_scale"].astype(np.float64) * np.sqrt(H) * np.sqrt(d)
    _close(g["w_f32"][None], wp_ref[None], "W_proj . x")
    # decisions in the kernel's precision: exact
    qc, qs = oracle.quantize_rows(g["q_f32"].reshape(-1, d).astype(np.float64))
    assert np.array_equal(qs.reshape(-1, H), g["q_scale"]), "q scales"
    assert np.array_equal(qc.reshape(g["q_idx"].shape), g["q_idx"]), "q codes"
    kc, ks = oracle.quantize_rows(g["k_f32"].astype(np.float64))
    assert np.array_equal(g["kidx"][rows], kc), "k codes in the cache rows"
    assert np.array_equal(g["k_scale"][rows], ks), "k scales in the cache"
    _, wb = oracle.fold_weights(g["w_f32"].astype(np.float64), g["q_scale"], d)
    assert np.array_equal(wb.view(np.int16), g["w"]), "folded weights"
    # every other cache row is untouched
    untouched = np.ones(len(g["kidx"]), bool)
    untouched[rows] = False
    assert np.all(g["kidx"][untouched] == SENTINEL) and np.all(g["k_scale"][untouched] == -1.0)
    # against the oracle's own bytes: the same except one step at a tie
    same_scale = g["q_scale"] == ref["q_scale"]
    assert same_scale.mean() >= 0.999
    qs = ref["q_scale"][..., None].astype(np.float64)
    n_q = _straddle_only(g["q_idx"][same_scale], ref["q_code"][same_scale],
                         (g["q_f32"] / qs)[same_scale], (ref["q_f"] / qs)[same_scale])
    same_k = g["k_scale"][rows] == ref["k_scale"]
    ks = ref["k_scale"][:, None].astype(np.float64)
    n_k = _straddle_only(g["kidx"][rows][same_k], ref["k_code"][same_k],
                         (g["k_f32"] / ks)[same_k], (ref["k_f"] / ks)[same_k])
    assert n_q <= 1e-3 * g["q_idx"].size and n_k <= 1e-3 * g["kidx"][rows].size


@pytest.mark.parametrize("case", ["decode_16_tokens", "prefill_600_paged", "small_heads"])
def test_producer_matches_the_oracle(case):
    if case == "decode_16_tokens":
        # the next token of 16 sequences at 128K context (cache of 16 short
        # segments standing in for the long histories: only the appended rows matter)
        pos = np.full(16, 131071, np.int32) - np.arange(16, dtype=np.int32) * 977
        pi = make_project_inputs(pos, q_seq=np.arange(16))
        seq_row0 = np.arange(16, dtype=np.int64) * 8 - pos.astype(np.int64) + 3   # token s -> row 8 s + 3
        rows = _rows_of(pi, seq_row0=seq_row0)
        g = _run(pi, 16 * 8, seq_row0=seq_row0)
    elif case == "prefill_600_paged":
        pi = make_project_inputs(np.arange(600, dtype=np.int32))
        pages = 10
        pt = np.random.default_rng(4).permutation(pages).astype(np.int32)[None, :]
        rows = _rows_of(pi, page_table=pt, page_size=64)
        g = _run(pi, pages * 64, page_table=pt, page_size=64)
    else:
        # 4 indexer heads of 64 dims (the tiny workload's indexer), narrow model
        pi = make_project_inputs(np.arange(37, dtype=np.int32) * 5, hidden=512, q_lora_rank=256,
                                 h_idx=4, d_idx=64, rope_dim=32)
        seq_row0 = np.zeros(1, np.int64)
        rows = _rows_of(pi, seq_row0=seq_row0)
        g = _run(pi, 200, seq_row0=seq_row0)
    assert np.all(rows >= 0)
    _check(pi, g, rows)


def test_produced_cache_feeds_the_fused_indexer():
    """A sequence's whole history and its next token through the producer
    (the history as one prefill, the token as decode), then the fused
    indexer + TopK over the produced cache: its selection against the
    oracle's scores of the same bytes, and against the all-oracle pipeline."""
    L = 5000
    hist = make_project_inputs(np.arange(L, dtype=np.int32), seed_offset=1)
    tok = make_project_inputs(np.array([L], np.int32), seed_offset=2)
    tok.w_qb, tok.w_k, tok.w_proj = hist.w_qb, hist.w_k, hist.w_proj      # one model
    tok.ln_gamma, tok.ln_beta = hist.ln_gamma, hist.ln_beta
    seq_row0 = np.zeros(1, np.int64)
    gh = _run(hist, L + 1, seq_row0=seq_row0)
    gt = _run(tok, L + 1, seq_row0=seq_row0)
    kidx = gh["kidx"].copy()
    kidx[L] = gt["kidx"][L]
    k_scale = gh["k_scale"].copy()
    k_scale[L] = gt["k_scale"][L]
    base = make_inputs(3, lengths=[L + 1], with_attention=False)
    import dataclasses
    inp = dataclasses.replace(base, q_idx=gt["q_idx"], w=gt["w"].view(np.uint16), kidx=kidx,
                              k_scale=k_scale, q_n=np.array([L + 1], np.int32))
    from gpu_util import gpu_indexer_topk
    from long_context_decode_indexer_b200.batch import upload
    idx, _ = gpu_indexer_topk(upload(inp))
    ref = oracle.indexer_scores(inp.q_idx, inp.w, inp.kidx, inp.q_seq, inp.q_n, seq_row0=seq_row0,
                                k_scale=k_scale)
    check_recall(idx, ref, inp.q_n, inp.topk)
    # the all-oracle pipeline: produce with the oracle, score, select
    oh = oracle.indexer_project(hist.x, hist.q_lora, hist.w_qb, hist.w_k, hist.w_proj, hist.ln_gamma,
                                hist.ln_beta, hist.positions, h_idx=64, d_idx=128)
    ot = oracle.indexer_project(tok.x, tok.q_lora, tok.w_qb, tok.w_k, tok.w_proj, tok.ln_gamma,
                                tok.ln_beta, tok.positions, h_idx=64, d_idx=128)
    o_k = np.concatenate([oh["k_code"], ot["k_code"]])
    o_ks = np.concatenate([oh["k_scale"], ot["k_scale"]])
    o_sc = oracle.indexer_scores(ot["q_code"], ot["w_bf16"], o_k, inp.q_seq, inp.q_n,
                                 seq_row0=seq_row0, k_scale=o_ks)
    o_idx, _ = oracle.topk(o_sc[0], inp.topk)
    overlap = len(set(idx[0].tolist()) & set(o_idx.tolist())) / inp.topk
    assert overlap >= 0.99, "selection overlap with the all-oracle pipeline %.4f" % overlap
