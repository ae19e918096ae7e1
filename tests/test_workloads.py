"""The seeded workload generator: determinism and the structure each recipe promises."""
import numpy as np

from sparse_mla_decoding_b200 import workloads as W


def test_deterministic_and_chunk_independent():
    w = W.TINY
    assert np.array_equal(W.queries(w), W.queries(w))
    lay = W.layout(w)
    rows = lay.num_blocks * 64
    a = list(W.cache_values(w, rows))
    b = list(W.cache_values(w, rows, chunk_rows=rows))
    assert np.array_equal(np.concatenate([x[1] for x in a]), np.concatenate([x[1] for x in b]))
    big = W.Workload("t", batch=1, s_q=1, h_q=16, topk=8, seed=5, seqlens=(3 * W.GEN_CHUNK_ROWS,))
    r = 3 * W.GEN_CHUNK_ROWS
    one = np.concatenate([x[1] for x in W.cache_values(big, r, chunk_rows=r)])
    three = np.concatenate([x[1] for x in W.cache_values(big, r, chunk_rows=W.GEN_CHUNK_ROWS)])
    assert np.array_equal(one, three)


def test_layout_is_a_block_permutation():
    w = W.Workload("v", batch=5, s_q=1, h_q=16, topk=8, seed=9, seqlens=(1, 64, 65, 200, 640))
    lay = W.layout(w)
    assert lay.num_used_blocks == 1 + 1 + 2 + 4 + 10
    used = np.concatenate([lay.block_table[i, :lay.blocks_per_req[i]] for i in range(5)])
    assert sorted(used.tolist()) == list(range(lay.num_used_blocks))
    for i in range(5):
        assert (lay.block_table[i, lay.blocks_per_req[i]:] == lay.spare_block).all()
    unused = W.unused_rows(lay)
    assert len(unused) == (64 - 1) + 0 + 63 + 56 + 0 + 64


def test_tiny_recipe():
    w = W.TINY
    lay = W.layout(w)
    idx = W.indices(w, lay.seqlens)
    assert idx.shape == (2, 1, 64)
    for b in range(2):
        row = idx[b, 0]
        assert (row == -1).sum() == 6
        v = row[row >= 0]
        assert len(set(v.tolist())) == len(v) and v.max() < lay.seqlens[b]


def test_recent_mix_and_causal_recipes():
    w = W.DECODE_H64_SQ2.with_(batch=2, seqlens=(32768, 32768))
    idx = W.indices(w, (32768, 32768))
    for b in range(2):
        for t in range(2):
            row = idx[b, t]
            assert (row == -1).sum() == 102
            v = row[row >= 0]
            assert len(set(v.tolist())) == len(v)
    full = W.DECODE_H64_SQ2.with_(batch=1, seqlens=(32768,), invalid_per_token=0)
    row = W.indices(full, (32768,))[0, 0]
    assert (row >= 32768 - 4096).sum() == 1024 and (row < 32768 - 4096).sum() == 1024
    c = W.PREFILL_SHAPED.with_(s_q=3)
    ci = W.indices(c, (65536,))
    for t in range(3):
        assert ci[0, t].max() < 61440 + t and len(set(ci[0, t].tolist())) == 2048


def test_varlen_lengths_in_range_and_poison_row():
    L = W.LONG_VARLEN.lengths()
    assert L.shape == (32,) and L.min() >= 4096 and L.max() <= 131072
    cache = np.zeros((4, 656), np.uint8)
    W.poison(cache, np.array([1, 3]))
    assert (cache[0] == 0).all() and (cache[1, :512] == 0x7F).all()
    assert np.isnan(cache[1, 512:528].view("<f4")).all()
    assert np.isnan(cache[3, 528:].view("<u2").astype(np.uint32).__lshift__(16).view(np.float32)).all()
