"""GPU parity of the sparse attention over an FP8 latent cache (e4m3 codes and
a power-of-two scale per row) against the fp64 oracle, and bit-for-bit
equality with the bf16 attention on a bf16 cache holding the decoded values
(every decoded value is exact in bf16, and after the gather both paths run
the same arithmetic)."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from conftest import cuda_ok
from gpu_util import check_attention, gpu_mla, ok_status, oracle_kw
from long_context_decode_indexer_b200 import dsa
from long_context_decode_indexer_b200.batch import upload, workspace
from long_context_decode_indexer_b200.synth import encode_bf16, make_fp8_latent, make_inputs

pytestmark = [pytest.mark.gpu, pytest.mark.skipif(not cuda_ok(), reason="needs a CUDA GPU")]


def gpu_mla_fp8(db, codes, scale, idx):
    i = db.inp
    p = db.params(topk=idx.shape[1])
    kv = db.kvdesc()
    ws = workspace(dsa.workspace_size(p, kv, dsa.OP_SPARSE_MLA_DECODE))
    c = torch.from_numpy(np.ascontiguousarray(codes)).cuda()
    s = torch.from_numpy(np.ascontiguousarray(scale)).cuda()
    idx_d = torch.from_numpy(np.ascontiguousarray(idx, np.int32)).cuda()
    out = torch.full((i.nq, i.h, i.d_v), 12345, dtype=torch.int16, device="cuda")
    lse = torch.full((i.nq, i.h), float("nan"), dtype=torch.float32, device="cuda")
    dsa.sparse_mla_decode_fp8(p, kv, db.q, c, c.stride(0), s, idx_d, out, lse, ws)
    ok_status(ws)
    return out, lse


def decoded_bf16(codes, scale):
    f = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float32).numpy() * scale[:, None]
    return encode_bf16(f)


def out_magnitude(ref_out):
    """Scale of the max-abs bound.  The 1e-2 bound is set for unit-normal
    latents, whose outputs (near-uniform softmax) stay far below 1; the FP8
    rows (code * 2^-3..2^3) give sharper softmaxes and outputs of up to tens,
    whose bf16 rounding alone is 2^-9 of their size: the bound becomes the
    larger of 1e-2 and four bf16 half-ulps of the largest output."""
    return max(1.0, 4 * 2.0 ** -9 * float(np.abs(ref_out).max()) / 1e-2)


def draw_idx(inp, seed, dup=False):
    rng = np.random.default_rng(seed)
    k = inp.topk
    idx = np.full((inp.nq, k), -1, np.int32)
    for qi in range(inp.nq):
        n = int(inp.q_n[qi])
        m = min(n, k)
        idx[qi, :m] = rng.choice(n, size=m, replace=False)
        if dup and m > 10:
            idx[qi, m // 2] = idx[qi, 0]
            idx[qi] = idx[qi, rng.permutation(k)]
    return idx


@pytest.mark.parametrize("case", ["v32", "padded_dups", "paged"])
def test_fp8_latent_matches_oracle_and_the_bf16_path(case):
    if case == "v32":
        inp = make_inputs(2, lengths=[5000, 3001])
    elif case == "padded_dups":
        inp = make_inputs(2, lengths=[600, 40, 3000], h=64)
    else:
        inp = make_inputs(5, lengths=[2500, 900])
    rows = inp.kv.shape[0]
    codes, scale = make_fp8_latent(rows, seed_offset=3)
    idx = draw_idx(inp, 5, dup=(case == "padded_dups"))
    db = upload(inp)
    out8, lse8 = gpu_mla_fp8(db, codes, scale, idx)
    o8 = out8.view(torch.bfloat16).double().cpu().numpy()
    l8 = lse8.double().cpu().numpy()
    # the bf16 path on the decoded values: the same bits
    db16 = upload(dataclasses.replace(inp, kv=decoded_bf16(codes, scale)))
    out16, lse16 = gpu_mla(db16, idx)
    assert np.array_equal(o8, out16), "FP8 path differs from the bf16 path on the decoded cache"
    assert np.array_equal(l8, lse16)
    ro, rl = oracle.sparse_mla_fp8(inp.q, codes, scale, idx, inp.q_seq, inp.q_n, scale=inp.scale,
                                   d_v=inp.d_v, **oracle_kw(inp))
    check_attention(o8, l8, ro, rl, magnitude=out_magnitude(ro))


def test_fp8_latent_at_v32_batch_sampled():
    """16 x 32K decode (the batched workload's shapes): every output against
    the bf16 path on the decoded cache, bit for bit; sampled queries against
    the oracle."""
    inp = make_inputs(2, nseq=16)
    codes, scale = make_fp8_latent(inp.kv.shape[0], seed_offset=4)
    idx = draw_idx(inp, 6)
    db = upload(inp)
    out8, lse8 = gpu_mla_fp8(db, codes, scale, idx)
    o8 = out8.view(torch.bfloat16).double().cpu().numpy()
    l8 = lse8.double().cpu().numpy()
    db16 = upload(dataclasses.replace(inp, kv=decoded_bf16(codes, scale)))
    out16, lse16 = gpu_mla(db16, idx)
    assert np.array_equal(o8, out16) and np.array_equal(l8, lse16)
    sel = np.array([0, 7, 15])
    ro, rl = oracle.sparse_mla_fp8(inp.q[sel], codes, scale, idx[sel], inp.q_seq[sel], inp.q_n[sel],
                                   scale=inp.scale, d_v=inp.d_v, **oracle_kw(inp))
    check_attention(o8[sel], l8[sel], ro, rl, magnitude=out_magnitude(ro))
