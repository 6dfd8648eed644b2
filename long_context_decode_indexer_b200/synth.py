"""Seeded synthetic inputs for the DSA decode path.

This module draws random numbers and encodes them into the storage formats the
path consumes (FP8 e4m3 codes, bf16 bits, int32 tables).  It holds none of the
method's arithmetic: no score, no selection, no attention.  Both the GPU path
(via tests / bench) and the fp64 oracle read the bytes it produces, so the two
sides never have to agree on a quantisation step.

Every tensor comes from its own PCG64 stream seeded by
``SeedSequence([1000 + config_id + seed_offset, stream])`` with these streams:
  0 context lengths, 1 page permutation, 2 q^I, 3 w, 4 k^I, 5 heavy-tail rows,
  6 q (attention query), 7 latent KV, 8 per-row key scales; and for the
  indexer producer (make_project_inputs): 9 x, 10 q_lora, 11 W_qb, 12 W_k,
  13 W_proj, 14 LayerNorm gamma / beta; and for the masked-MHA short prefill
  (make_mha_inputs): 15 q, 16 k, 17 v; and for the FP8 latent cache
  (make_fp8_latent): 18 codes, 19 row exponents.
Encodings: e4m3 via torch's float8_e4m3fn cast after clamping to +-448 (round
to nearest even, saturating); bf16 via torch's round-to-nearest-even cast.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np
import torch

# Shapes of the five workloads: tiny decode, batched decode at V3.2 shapes,
# long-context decode (128K), causal prefill (16K) and paged two-token decode.
CONFIGS = {
    1: dict(name="tiny_decode_4k", kind="decode", nseq=1, L=4096, h_idx=4, d_idx=64,
            w_std=0.5, topk=256, h=16, tail=False),
    2: dict(name="batched_decode_64x32k", kind="decode", nseq=64, L=32768, h_idx=64,
            d_idx=128, w_std=0.125, topk=2048, h=128, tail=True),
    3: dict(name="long_decode_16x128k", kind="decode", nseq=16, L=131072, h_idx=64,
            d_idx=128, w_std=0.125, topk=2048, h=128, tail=True),
    4: dict(name="causal_prefill_16k", kind="prefill", nseq=1, L=16384, h_idx=64,
            d_idx=128, w_std=0.125, topk=2048, h=128, tail=False),
    5: dict(name="paged_mtp_decode_128seq", kind="paged2", nseq=128, L=16384,
            h_idx=64, d_idx=128, w_std=0.125, topk=2048, h=128, tail=True),
}
D_QK = 576
D_V = 512
PAGE_SIZE = 64


@dataclasses.dataclass
class Inputs:
    """One batch of host-side inputs (numpy, storage formats)."""
    config_id: int
    name: str
    kind: str
    h_idx: int
    d_idx: int
    h: int
    d_qk: int
    d_v: int
    topk: int
    scale: float
    q_idx: np.ndarray            # [nq, h_idx, d_idx] uint8 e4m3 codes
    w: np.ndarray                # [nq, h_idx] uint16 bf16 bits
    kidx: np.ndarray             # [rows, d_idx] uint8 e4m3 codes
    k_scale: Optional[np.ndarray]  # [rows] float32 or None
    q: np.ndarray                # [nq, h, d_qk] uint16 bf16 bits
    kv: np.ndarray               # [rows, d_qk] uint16 bf16 bits
    q_seq: np.ndarray            # [nq] int32
    q_n: np.ndarray              # [nq] int32 visible positions per query
    seq_len: np.ndarray          # [nseq] int32 cache rows per sequence
    seq_row0: Optional[np.ndarray]   # [nseq] int64 (contiguous layout)
    page_table: Optional[np.ndarray]  # [nseq, max_pages] int32 (paged layout)
    page_size: int
    q_per_seq: int

    @property
    def nq(self) -> int:
        return int(self.q_n.shape[0])

    @property
    def nseq(self) -> int:
        return int(self.seq_len.shape[0])

    @property
    def rows(self) -> int:
        return int(self.kidx.shape[0])

    @property
    def max_n(self) -> int:
        return int(self.q_n.max()) if self.nq else 0


def _rng(config_id: int, seed_offset: int, stream: int) -> np.random.Generator:
    ss = np.random.SeedSequence([1000 + config_id + seed_offset, stream])
    return np.random.Generator(np.random.PCG64(ss))


def encode_e4m3(x: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).clamp_(-448.0, 448.0)
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def encode_bf16(x: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _normal_bf16(rng: np.random.Generator, shape, chunk: int = 1 << 24) -> np.ndarray:
    """N(0,1) drawn in float32 chunks and stored as bf16 bits."""
    total = int(np.prod(shape))
    out = np.empty(total, np.uint16)
    for start in range(0, total, chunk):
        n = min(chunk, total - start)
        out[start:start + n] = encode_bf16(rng.standard_normal(n, dtype=np.float32))
    return out.reshape(shape)


def context_lengths(config_id: int, *, seed_offset: int = 0, nseq: Optional[int] = None,
                    L: Optional[int] = None, ragged: bool = False,
                    lengths: Optional[np.ndarray] = None) -> np.ndarray:
    """Context length of every sequence of workload ``config_id`` (stream 0).

    decode : L for every sequence; ragged: U[1024, L] with sequence 0 at 2048
             and sequence 1 at 2049 (the short-history boundary).
    paged2 : round(exp(ln L + N(0,1))) clipped to [512, 131071] (the
             speculative token then sees at most 131072 positions).
    prefill: the one sequence of L tokens.
    """
    c = CONFIGS[config_id]
    kind = c["kind"]
    nseq = c["nseq"] if nseq is None else int(nseq)
    L = c["L"] if L is None else int(L)
    r_len = _rng(config_id, seed_offset, 0)
    if lengths is not None:
        return np.asarray(lengths, np.int64).copy()
    if kind == "paged2":
        z = r_len.standard_normal(nseq)
        return np.clip(np.round(np.exp(math.log(L) + 1.0 * z)), 512, 131071).astype(np.int64)
    if ragged:
        seq_ctx = r_len.integers(1024, L, size=nseq, endpoint=True).astype(np.int64)
        if nseq > 0:
            seq_ctx[0] = min(2048, L)
        if nseq > 1:
            seq_ctx[1] = min(2049, L)
        return seq_ctx
    return np.full(nseq, L, np.int64)


def make_inputs(config_id: int, *, seed_offset: int = 0, nseq: Optional[int] = None,
                L: Optional[int] = None, ragged: bool = False, paged: Optional[bool] = None,
                lengths: Optional[np.ndarray] = None, with_k_scale: bool = False,
                topk: Optional[int] = None, h: Optional[int] = None,
                h_idx: Optional[int] = None, d_idx: Optional[int] = None,
                with_attention: bool = True) -> Inputs:
    """Inputs of workload ``config_id`` (1..5), optionally resized for tests.

    decode  : one query per sequence; query n = L (rows 0..L-1 visible).
    prefill : one sequence of L tokens; query t sees n = t positions (s < t).
    paged2  : two queries per sequence (next token + one speculative token)
              with n = L and L + 1; cache rows L + 1; paged (64-token pages,
              physical pages a random permutation).
    ragged  : decode lengths ~ U[1024, L] per sequence, with sequence 0 at
              2048 and sequence 1 at 2049 (the short-history boundary).
    with_attention=False leaves q and the latent cache empty (indexer-only
    tests of long histories).
    """
    c = dict(CONFIGS[config_id])
    kind = c["kind"]
    nseq = c["nseq"] if nseq is None else int(nseq)
    L = c["L"] if L is None else int(L)
    h_idx = c["h_idx"] if h_idx is None else int(h_idx)
    d_idx = c["d_idx"] if d_idx is None else int(d_idx)
    h = c["h"] if h is None else int(h)
    k = c["topk"] if topk is None else int(topk)
    if paged is None:
        paged = kind == "paged2"

    seq_ctx = context_lengths(config_id, seed_offset=seed_offset, nseq=nseq, L=L,
                              ragged=ragged, lengths=lengths)
    nseq = len(seq_ctx)

    if kind == "prefill":
        assert nseq == 1
        q_seq = np.zeros(L, np.int32)
        q_n = np.arange(L, dtype=np.int32)
        seq_len = np.array([L], np.int64)
        q_per_seq = L
    elif kind == "paged2":
        q_seq = np.repeat(np.arange(nseq, dtype=np.int32), 2)
        q_n = np.stack([seq_ctx, seq_ctx + 1], axis=1).reshape(-1).astype(np.int32)
        seq_len = seq_ctx + 1
        q_per_seq = 2
    else:
        q_seq = np.arange(nseq, dtype=np.int32)
        q_n = seq_ctx.astype(np.int32)
        seq_len = seq_ctx.copy()
        q_per_seq = 1
    nq = len(q_n)

    # cache layout (stream 1 for the page permutation)
    if paged:
        pages = (seq_len + PAGE_SIZE - 1) // PAGE_SIZE
        total_pages = int(pages.sum())
        perm = _rng(config_id, seed_offset, 1).permutation(total_pages).astype(np.int32)
        max_pages = int(pages.max()) if nseq else 1
        page_table = np.full((nseq, max_pages), -1, np.int32)
        off = 0
        for i in range(nseq):
            page_table[i, :pages[i]] = perm[off:off + pages[i]]
            off += int(pages[i])
        rows = total_pages * PAGE_SIZE
        seq_row0 = None
        page_size = PAGE_SIZE
    else:
        seq_row0 = np.concatenate([[0], np.cumsum(seq_len)[:-1]]).astype(np.int64) if nseq else np.zeros(0, np.int64)
        rows = int(seq_len.sum())
        page_table = None
        page_size = 0

    # indexer query and head weights (streams 2, 3)
    q_idx = encode_e4m3(_rng(config_id, seed_offset, 2).standard_normal(
        (nq, h_idx, d_idx), dtype=np.float32))
    w = encode_bf16(_rng(config_id, seed_offset, 3).standard_normal(
        (nq, h_idx), dtype=np.float32) * np.float32(c["w_std"]))

    # index-K cache (stream 4), heavy tail (stream 5): per sequence, ceil(1% of
    # its rows) distinct positions scaled x3 before quantising.
    kf = _rng(config_id, seed_offset, 4).standard_normal((rows, d_idx), dtype=np.float32)
    if c["tail"]:
        r_tail = _rng(config_id, seed_offset, 5)
        for i in range(nseq):
            n_i = int(seq_len[i])
            cnt = int(math.ceil(0.01 * n_i))
            pos = r_tail.choice(n_i, size=cnt, replace=False)
            if paged:
                phys = page_table[i, pos // PAGE_SIZE].astype(np.int64) * PAGE_SIZE + pos % PAGE_SIZE
            else:
                phys = seq_row0[i] + pos
            kf[phys] *= np.float32(3.0)
    kidx = encode_e4m3(kf)
    del kf
    k_scale = None
    if with_k_scale:
        # powers of two in [1/4, 4] (e8m0-style block scales)
        k_scale = np.exp2(_rng(config_id, seed_offset, 8).integers(-2, 3, size=rows)).astype(np.float32)

    # attention query and latent cache (streams 6, 7)
    if with_attention:
        q = _normal_bf16(_rng(config_id, seed_offset, 6), (nq, h, D_QK))
        kv = _normal_bf16(_rng(config_id, seed_offset, 7), (rows, D_QK))
    else:
        q = np.zeros((nq, h, D_QK), np.uint16)
        kv = np.zeros((1, D_QK), np.uint16)

    return Inputs(config_id=config_id, name=c["name"], kind=kind, h_idx=h_idx,
                  d_idx=d_idx, h=h, d_qk=D_QK, d_v=D_V, topk=k,
                  scale=float(D_QK) ** -0.5, q_idx=q_idx, w=w, kidx=kidx,
                  k_scale=k_scale, q=q, kv=kv, q_seq=q_seq, q_n=q_n,
                  seq_len=seq_len.astype(np.int32), seq_row0=seq_row0,
                  page_table=page_table, page_size=page_size, q_per_seq=q_per_seq)


def to_paged(inp: Inputs, *, config_id: Optional[int] = None, seed_offset: int = 7,
             page_size: int = PAGE_SIZE) -> Inputs:
    """The same logical caches re-laid out in pages (random permutation)."""
    assert inp.page_table is None
    nseq = inp.nseq
    pages = (inp.seq_len.astype(np.int64) + page_size - 1) // page_size
    total = int(pages.sum())
    perm = _rng(config_id or inp.config_id, seed_offset, 1).permutation(total).astype(np.int32)
    max_pages = int(pages.max()) if nseq else 1
    pt = np.full((nseq, max_pages), -1, np.int32)
    off = 0
    kidx = np.zeros((total * page_size, inp.d_idx), np.uint8)
    kv = np.zeros((total * page_size, inp.d_qk), np.uint16)
    ks = None if inp.k_scale is None else np.ones(total * page_size, np.float32)
    for i in range(nseq):
        pt[i, :pages[i]] = perm[off:off + pages[i]]
        off += int(pages[i])
        n_i = int(inp.seq_len[i])
        pos = np.arange(n_i)
        phys = pt[i, pos // page_size].astype(np.int64) * page_size + pos % page_size
        src = inp.seq_row0[i] + pos
        kidx[phys] = inp.kidx[src]
        kv[phys] = inp.kv[src]
        if ks is not None:
            ks[phys] = inp.k_scale[src]
    return dataclasses.replace(inp, kidx=kidx, kv=kv, k_scale=ks, seq_row0=None,
                               page_table=pt, page_size=page_size)


@dataclasses.dataclass
class ProjectInputs:
    """Inputs of the indexer producer for nt tokens (host, storage formats)."""
    x: np.ndarray            # [nt, hidden] bf16 bits
    q_lora: np.ndarray       # [nt, q_lora_rank] bf16 bits
    w_qb: np.ndarray         # [h_idx * d_idx, q_lora_rank] bf16 bits
    w_k: np.ndarray          # [d_idx, hidden] bf16 bits
    w_proj: np.ndarray       # [h_idx, hidden] bf16 bits
    ln_gamma: np.ndarray     # [d_idx] float32
    ln_beta: np.ndarray      # [d_idx] float32
    positions: np.ndarray    # [nt] int32
    q_seq: np.ndarray        # [nt] int32 sequence of each token
    h_idx: int
    d_idx: int
    rope_dim: int

    @property
    def nt(self) -> int:
        return int(self.positions.shape[0])


def make_project_inputs(positions, q_seq=None, *, hidden: int = 7168, q_lora_rank: int = 1536,
                        h_idx: int = 64, d_idx: int = 128, rope_dim: int = 64,
                        seed_offset: int = 0) -> ProjectInputs:
    """Producer inputs at DeepSeek-V3.2 widths: x and q_lora ~ N(0,1); the
    weights ~ N(0, 1/fan_in) ([out, in]); LayerNorm gamma ~ 1 + N(0, 0.1^2),
    beta ~ N(0, 0.1^2); one token per entry of `positions` (its sequence in
    q_seq, default 0)."""
    positions = np.asarray(positions, np.int32)
    nt = len(positions)
    q_seq = np.zeros(nt, np.int32) if q_seq is None else np.asarray(q_seq, np.int32)
    cid = 3
    r = lambda stream: _rng(cid, seed_offset, stream)
    x = _normal_bf16(r(9), (nt, hidden))
    q_lora = _normal_bf16(r(10), (nt, q_lora_rank))
    w_qb = encode_bf16(r(11).standard_normal((h_idx * d_idx, q_lora_rank), dtype=np.float32)
                       * np.float32(q_lora_rank ** -0.5))
    w_k = encode_bf16(r(12).standard_normal((d_idx, hidden), dtype=np.float32) * np.float32(hidden ** -0.5))
    w_proj = encode_bf16(r(13).standard_normal((h_idx, hidden), dtype=np.float32) * np.float32(hidden ** -0.5))
    g = r(14)
    ln_gamma = (1.0 + 0.1 * g.standard_normal(d_idx)).astype(np.float32)
    ln_beta = (0.1 * g.standard_normal(d_idx)).astype(np.float32)
    return ProjectInputs(x=x, q_lora=q_lora, w_qb=w_qb, w_k=w_k, w_proj=w_proj, ln_gamma=ln_gamma,
                         ln_beta=ln_beta, positions=positions, q_seq=q_seq, h_idx=h_idx, d_idx=d_idx,
                         rope_dim=rope_dim)


@dataclasses.dataclass
class MhaInputs:
    """Per-head MHA q / k / v of one prefill sequence (bf16 bits)."""
    q: np.ndarray          # [L, h, d_qk]
    k: np.ndarray          # [L, h, d_qk]
    v: np.ndarray          # [L, h, d_v]
    q_seq: np.ndarray      # [L] int32 (all 0)
    q_n: np.ndarray        # [L] int32: token t sees s < t
    seq_row0: np.ndarray   # [1] int64
    scale: float


def make_mha_inputs(L: int, *, h: int = 128, d_qk: int = 192, d_v: int = 128,
                    seed_offset: int = 0) -> MhaInputs:
    """MHA-form prefill activations for one sequence of L tokens (the short
    prefill's masked MHA): q, k, v ~ N(0, 1) bf16, token t visible positions
    s < t (as the causal prefill workload), softmax scale d_qk^-1/2.  Drawn
    from the causal-prefill workload's seed."""
    cid = 4
    r = lambda stream: _rng(cid, seed_offset, stream)
    q = _normal_bf16(r(15), (L, h, d_qk))
    k = _normal_bf16(r(16), (L, h, d_qk))
    v = _normal_bf16(r(17), (L, h, d_v))
    return MhaInputs(q=q, k=k, v=v, q_seq=np.zeros(L, np.int32), q_n=np.arange(L, dtype=np.int32),
                     seq_row0=np.zeros(1, np.int64), scale=float(d_qk) ** -0.5)


def make_fp8_latent(rows: int, *, d_qk: int = D_QK, config_id: int = 3, seed_offset: int = 0):
    """An FP8 latent cache of `rows` rows: e4m3 codes of N(0,1) draws
    ([rows, d_qk] uint8) and one power-of-two scale per row, 2^U{-3..3}
    ([rows] fp32).  A row stands for code * scale."""
    r = lambda stream: _rng(config_id, seed_offset, stream)
    codes = np.empty((rows, d_qk), np.uint8)
    g = r(18)
    step = max(1, (1 << 24) // d_qk)
    for i in range(0, rows, step):
        j = min(rows, i + step)
        codes[i:j] = encode_e4m3(g.standard_normal((j - i, d_qk), dtype=np.float32))
    scale = np.ldexp(np.float32(1.0), r(19).integers(-3, 4, size=rows)).astype(np.float32)
    return codes, scale
