"""The seeded input generator follows the recipe the design notes state:
shapes per workload, one independent stream per tensor, the heavy tail on
the index keys, the short-history boundary of the ragged variant, the
lognormal lengths and the page tables of the paged workload."""
import numpy as np

from long_context_decode_indexer_b200.synth import (CONFIGS, PAGE_SIZE, context_lengths,
                                                    make_inputs, to_paged)


def _dec_e4m3(codes):
    import torch
    return torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy()


def test_shapes_follow_the_workload_table():
    for cid, c in CONFIGS.items():
        small = dict(nseq=2, L=600) if c["kind"] != "prefill" else dict(L=600)
        inp = make_inputs(cid, **small)
        assert inp.q_idx.shape[1:] == (c["h_idx"], c["d_idx"])
        assert inp.w.shape == (inp.nq, c["h_idx"])
        assert inp.kidx.shape[1] == c["d_idx"]
        assert inp.q.shape == (inp.nq, c["h"], 576)
        assert inp.kv.shape[1] == 576 and inp.kv.shape[0] == inp.kidx.shape[0]
        assert inp.topk == c["topk"] and abs(inp.scale - 576 ** -0.5) < 1e-15


def test_streams_are_independent_per_tensor():
    a = make_inputs(2, nseq=2, L=600)
    b = make_inputs(2, nseq=2, L=600, h=64)          # changes only the query tensor shape
    assert np.array_equal(a.kidx, b.kidx) and np.array_equal(a.q_idx, b.q_idx)
    assert np.array_equal(a.kv, b.kv)
    c = make_inputs(2, nseq=2, L=600, seed_offset=1)  # another replica
    assert not np.array_equal(a.kidx, c.kidx)
    # the key scales have a stream of their own: asking for them changes no
    # other tensor, and they are not a function of the heavy-tail draw
    d = make_inputs(2, nseq=2, L=600, with_k_scale=True)
    assert np.array_equal(a.kidx, d.kidx) and np.array_equal(a.q_idx, d.q_idx)
    assert np.array_equal(a.kv, d.kv) and np.array_equal(a.w, d.w)
    tail_rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([1002, 5])))
    same_as_tail = np.exp2(tail_rng.integers(-2, 3, size=d.rows)).astype(np.float32)
    assert not np.array_equal(d.k_scale, same_as_tail)
    assert set(np.unique(d.k_scale).tolist()) <= {0.25, 0.5, 1.0, 2.0, 4.0}


def test_heavy_tail_scales_one_percent_of_each_sequence():
    inp = make_inputs(2, nseq=3, L=4000)
    k = _dec_e4m3(inp.kidx).astype(np.float64)
    for s in range(3):
        rows = k[inp.seq_row0[s]:inp.seq_row0[s] + 4000]
        rms = np.sqrt((rows ** 2).mean(axis=1))
        big = (rms > 2.0).sum()                      # N(0,1) rows have rms ~1, x3 rows ~3
        assert big == int(np.ceil(0.01 * 4000))


def test_ragged_variant_pins_the_short_history_boundary():
    inp = make_inputs(3, nseq=5, L=9000, ragged=True)
    assert inp.q_n[0] == 2048 and inp.q_n[1] == 2049
    assert np.all((inp.q_n >= 1024) & (inp.q_n <= 9000))


def test_paged_workload_lengths_and_page_tables():
    inp = make_inputs(5, nseq=16)
    L = inp.seq_len.astype(np.int64) - 1             # context of the first query
    assert np.all((L >= 512) & (L <= 131071))
    assert inp.q_n.max() <= 131072                   # the speculative token too
    assert abs(np.median(np.log(L)) - np.log(16384)) < 0.6   # median 16384, sigma 1
    assert np.array_equal(inp.q_n[0::2], L) and np.array_equal(inp.q_n[1::2], L + 1)
    assert inp.page_size == PAGE_SIZE
    assert context_lengths(5).max() <= 131071        # the full 128-sequence draw
    clipped = context_lengths(5, L=1 << 22, nseq=8)  # a median far above the clip
    assert clipped.max() == 131071                   # n <= 131072 for the speculative token too
    assert np.array_equal(context_lengths(5, nseq=16), L)
    pages = (inp.seq_len.astype(np.int64) + PAGE_SIZE - 1) // PAGE_SIZE
    used = np.concatenate([inp.page_table[i, :pages[i]] for i in range(len(pages))])
    assert np.array_equal(np.sort(used), np.arange(pages.sum()))   # a permutation of all pages


def test_paged_copy_holds_the_same_rows():
    inp = make_inputs(3, nseq=2, L=700)
    pg = to_paged(inp, page_size=128)
    for s in range(2):
        for pos in (0, 127, 128, 699):
            src = inp.seq_row0[s] + pos
            dst = pg.page_table[s, pos // 128] * 128 + pos % 128
            assert np.array_equal(inp.kidx[src], pg.kidx[dst])
            assert np.array_equal(inp.kv[src], pg.kv[dst])
