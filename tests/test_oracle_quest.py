"""Pins of the oracle's QUEST block metadata (CANN quest_prefill_metadata guide,
xdnf.cn/news/235188): per KV block and head, the per-channel max and min of K over the
block's tokens, one row per KV block in metadata blocks of block_size rows, the tail block
reduced over its valid tokens only, the unused rows of a request's last metadata block
zero. Here K is the dequantised q8 cache value code * scale.

Expected values come from a vectorised numpy reduction over the dequantised pool (a second
writing of the definition), a hand case, and invariances (moving physical blocks)."""
import numpy as np
import pytest

import oracle
from decode_attention_int8_b200 import inputs


def cache_of(w):
    return oracle.PagedCache(w.k, w.v, w.ks, w.vs, w.block_table, w.seq_lens,
                             w.cfg.n_q_heads, w.scale)


def numpy_metadata(w, meta_table, n_meta):
    bs, Hk, D = w.cfg.block_size, w.cfg.n_kv_heads, w.cfg.head_dim
    deq = w.k.astype(np.float32) * w.ks[..., None]  # fp32 products, as the definition
    mx = np.full((n_meta, bs, Hk, D), np.nan, np.float32)
    mn = np.full((n_meta, bs, Hk, D), np.nan, np.float32)
    for r, L in enumerate(w.seq_lens):
        nkv = -(-int(L) // bs)
        nmeta = -(-nkv // bs)
        for m in range(nmeta):
            mb = meta_table[r, m]
            mx[mb] = 0.0
            mn[mb] = 0.0
            for row in range(min(bs, nkv - m * bs)):
                j = m * bs + row
                n = min(bs, int(L) - j * bs)
                blk = deq[w.block_table[r, j], :n]  # [n][Hk][D]
                mx[mb, row] = blk.max(axis=0)
                mn[mb, row] = blk.min(axis=0)
    return mx, mn


@pytest.mark.parametrize("bs,lens,Hk", [
    (16, [1, 15, 16, 17, 256, 257, 300], 2),   # tails, one and several metadata blocks
    (32, [0, 1024, 1025, 33], 3),               # an empty request, a full metadata block
    (64, [4097, 64, 65], 1),                    # a second metadata block with one row
])
def test_matches_a_vectorised_reduction(bs, lens, Hk):
    w = inputs.make_custom(len(lens), Hk, Hk, 128, lens, bs, seed=bs,
                           k_dist="student_t3")
    meta, n_meta = inputs.quest_meta_table(lens, bs, seed=bs, extra_blocks=2)
    mx, mn = oracle.quest_metadata(cache_of(w), meta, n_meta)
    rx, rn = numpy_metadata(w, meta, n_meta)
    np.testing.assert_array_equal(mx, rx)
    np.testing.assert_array_equal(mn, rn)


def test_hand_case_tail_and_zero_rows():
    # one request of bs + 1 tokens: block 0 covers bs tokens, block 1 one token, so row 1
    # has max = min = that token's dequantised row; rows 2..bs-1 are zero
    bs, Hk, D = 16, 1, 64
    w = inputs.make_custom(1, 1, Hk, D, [bs + 1], bs, seed=3)
    meta, n_meta = inputs.quest_meta_table([bs + 1], bs, seed=3)
    mx, mn = oracle.quest_metadata(cache_of(w), meta, n_meta)
    mb = meta[0, 0]
    last = w.k[w.block_table[0, 1], 0, 0].astype(np.float32) * w.ks[w.block_table[0, 1], 0, 0]
    np.testing.assert_array_equal(mx[mb, 1, 0], last)
    np.testing.assert_array_equal(mn[mb, 1, 0], last)
    assert np.all(mx[mb, 2:] == 0.0) and np.all(mn[mb, 2:] == 0.0)
    blk0 = w.k[w.block_table[0, 0], :, 0].astype(np.float32) * w.ks[w.block_table[0, 0], :, 0,
                                                                    None]
    assert np.all(mx[mb, 0, 0] >= blk0) and np.all(mn[mb, 0, 0] <= blk0)
    assert np.all(np.any(mx[mb, 0, 0] == blk0, axis=0))


def test_invariant_to_physical_block_placement():
    bs = 16
    lens = [100, 37]
    w = inputs.make_custom(2, 4, 2, 128, lens, bs, seed=7, extra_blocks=5)
    meta, n_meta = inputs.quest_meta_table(lens, bs, seed=7)
    ref = oracle.quest_metadata(cache_of(w), meta, n_meta)
    perm = np.random.default_rng(1).permutation(w.num_blocks)
    inv = np.argsort(perm)
    w2 = inputs.Workload(w.cfg, w.q, w.k[inv], w.v[inv], w.ks[inv], w.vs[inv],
                         np.where(w.block_table >= 0, perm[np.maximum(w.block_table, 0)], -1)
                         .astype(np.int32), w.seq_lens, w.scale)
    got = oracle.quest_metadata(cache_of(w2), meta, n_meta)
    np.testing.assert_array_equal(got[0], ref[0])
    np.testing.assert_array_equal(got[1], ref[1])


def test_rejects_a_metadata_table_that_is_too_short():
    w = inputs.make_custom(1, 2, 2, 128, [300], 16, seed=1)
    with pytest.raises(oracle.OracleError):
        oracle.quest_metadata(cache_of(w), np.zeros((1, 1), np.int32), 4)  # needs 2 entries
