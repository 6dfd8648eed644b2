"""The seeded input generator follows the recipe the design notes state:
shapes per workload, one independent stream per tensor, the heavy tail on
the index keys, the short-history boundary of the ragged variant, the
lognormal lengths and the page tables of the paged workload."""
import numpy as np

from long_context_decode_indexer_b200.synth import CONFIGS, PAGE_SIZE, make_inputs, to_paged


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
    assert np.all((L >= 512) & (L <= 131072))
    assert abs(np.median(np.log(L)) - np.log(16384)) < 0.6   # median 16384, sigma 1
    assert np.array_equal(inp.q_n[0::2], L) and np.array_equal(inp.q_n[1::2], L + 1)
    assert inp.page_size == PAGE_SIZE
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
