"""Decode over a q4_0 cache (q8kv_decode_attn_q4) against the fp64 oracle, with the same
tolerance as the q8 decode (max-abs <= 1e-4, rel-L2 <= 1e-5): groups 1 to 16 (powers of two,
and 3, 6, 12 with padding heads), block sizes 16 to 128 (48: not a power of two), lengths
around the 256-token chunks, Student-t data, empty sequences, the benchmark's 16 x
4096-token shape on sampled rows, agreement with the q8 kernel on a cache that holds the
same values, and bad block-table entries (flagged, their tokens skipped)."""
import numpy as np
import pytest
import torch

import decode_attention_int8_b200 as q8
import oracle
from decode_attention_int8_b200 import inputs
from gpu_util import assert_close, without_block

pytestmark = pytest.mark.gpu


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def run_q4(w):
    out = torch.full(w.q.shape, float("nan"), dtype=torch.float32, device="cuda")
    q8.q8kv_decode_attn_q4(out, dev(w.q), dev(w.k4), dev(w.v4), dev(w.kd.view(np.float16)),
                           dev(w.vd.view(np.float16)), dev(w.block_table), dev(w.seq_lens),
                           w.scale)
    torch.cuda.synchronize()
    return out.cpu().numpy()


def oracle_q4(w):
    return oracle.PagedCacheQ4(w.k4, w.v4, w.kd, w.vd, w.block_table, w.seq_lens,
                               w.cfg.n_q_heads, w.scale)


@pytest.mark.parametrize("G", [1, 2, 4, 8, 16])
@pytest.mark.parametrize("bs", [16, 48, 64, 128])
def test_groups_blocks_and_chunk_edges(G, bs):
    Hk = 2
    lens = [1, 255, 256, 257, 511, 1000, 0, 33]
    w = inputs.make_q4_custom(len(lens), G * Hk, Hk, 128, lens, bs, seed=G * 10 + bs)
    got = run_q4(w)
    assert np.all(got[6] == 0.0)
    assert_close(got, oracle.decode_q4_all(oracle_q4(w), w.q), f"G={G} bs={bs}")


def test_heavy_tails_and_bias():
    w = inputs.make_q4_custom(3, 32, 8, 128, [3000, 700, 5], 64, seed=9, k_dist="student_t3",
                              v_dist="student_t3", k_bias_std=4.0)
    assert_close(run_q4(w), oracle.decode_q4_all(oracle_q4(w), w.q), "t3 + bias")


def test_gqa_batch_shape_sampled_rows():
    w = inputs.make_q4(1)
    got = run_q4(w)
    rng = np.random.default_rng(0)
    pairs = np.stack([rng.integers(0, 16, 96), rng.integers(0, 32, 96)], axis=1)
    ref = oracle.decode_q4_pairs(oracle_q4(w), w.q, pairs)
    assert_close(got[pairs[:, 0], pairs[:, 1]], ref, "gqa_batch q4 sampled rows")


def test_agrees_with_the_q8_kernel_on_the_same_values():
    # codes in [-8, 7] and binary16 row scales: the q8 and q4_0 caches hold equal values
    rng = np.random.default_rng(5)
    w = inputs.make_custom(3, 32, 8, 128, [1, 900, 2000], 64, seed=5)
    codes = rng.integers(-8, 8, w.k.shape).astype(np.int8)
    vcodes = rng.integers(-8, 8, w.v.shape).astype(np.int8)
    ks = rng.uniform(0.01, 0.2, w.ks.shape).astype(np.float16).astype(np.float32)
    vs = rng.uniform(0.01, 0.2, w.vs.shape).astype(np.float16).astype(np.float32)
    pack = lambda c: ((c[..., 0::2].astype(np.int32) + 8) |
                      ((c[..., 1::2].astype(np.int32) + 8) << 4)).astype(np.uint8)
    rep = lambda s: np.repeat(s[..., None].astype(np.float16), 4, axis=-1)
    out8 = torch.empty(w.q.shape, dtype=torch.float32, device="cuda")
    q8.q8kv_decode_attn(out8, dev(w.q), dev(codes), dev(vcodes), dev(ks), dev(vs),
                        dev(w.block_table), dev(w.seq_lens), w.scale)
    out4 = torch.empty_like(out8)
    q8.q8kv_decode_attn_q4(out4, dev(w.q), dev(pack(codes)), dev(pack(vcodes)), dev(rep(ks)),
                           dev(rep(vs)), dev(w.block_table), dev(w.seq_lens), w.scale)
    torch.cuda.synchronize()
    assert_close(out4.cpu().numpy(), out8.cpu().numpy().astype(np.float64), "q4 vs q8 kernel")


@pytest.mark.parametrize("G", [3, 6, 12])
def test_groups_that_are_not_powers_of_two(G):
    # served by the next power-of-two instantiation, whose extra heads are padding
    Hk = 2
    lens = [300, 1, 600]
    w = inputs.make_q4_custom(len(lens), G * Hk, Hk, 128, lens, 64, seed=G)
    assert_close(run_q4(w), oracle.decode_q4_all(oracle_q4(w), w.q), f"G={G}")


def test_bad_block_table_entries_are_flagged_and_skipped():
    w = inputs.make_q4_custom(3, 8, 2, 128, [300, 520, 64], 16, seed=21)
    q8.q8kv_device_errors(clear=True)
    ref = run_q4(w)
    assert q8.q8kv_device_errors(clear=True) == 0
    # an entry past the pool: tokens 320-335 of sequence 1 are skipped, the flag is raised
    w.block_table[1, 20] = w.num_blocks + 5
    got = run_q4(w)
    assert q8.q8kv_device_errors(clear=True) & q8.DEVERR_BLOCK_TABLE
    np.testing.assert_array_equal(got[0], ref[0])
    np.testing.assert_array_equal(got[2], ref[2])
    # row 1 is attention over the tokens of its other blocks
    bt, lens = without_block(w.block_table, w.seq_lens, 1, 20, 16)
    kept = oracle.PagedCacheQ4(w.k4, w.v4, w.kd, w.vd, bt, lens, w.cfg.n_q_heads, w.scale)
    assert_close(got[1], oracle.decode_q4_all(kept, w.q)[1], "q4 block skipped")
    # a negative entry
    w.block_table[1, 20] = -3
    got = run_q4(w)
    assert q8.q8kv_device_errors(clear=True) & q8.DEVERR_BLOCK_TABLE
    assert_close(got[1], oracle.decode_q4_all(kept, w.q)[1], "q4 block skipped (negative)")


@pytest.mark.parametrize("G", [1, 4, 8, 16])
def test_many_ragged_sequences_with_empty_ones(G):
    # 40 ragged sequences (some empty) x 4 KV heads: about 1800 chunks of 256 tokens, more
    # than one wave of CTAs, with the chunks past each sequence's end left out of the merge,
    # and a bad block-table entry in the middle of the longest sequence
    rng = np.random.default_rng(40 + G)
    lens = rng.integers(0, 2700, 40)
    lens[[3, 17, 18, 30]] = 0
    lens[7] = 2700
    w = inputs.make_q4_custom(40, 4 * G, 4, 128, lens.tolist(), 32, seed=G)
    ref = oracle.decode_q4_all(oracle_q4(w), w.q)
    q8.q8kv_device_errors(clear=True)
    got = run_q4(w)
    assert q8.q8kv_device_errors(clear=True) == 0
    assert np.all(got[lens == 0] == 0.0)
    assert_close(got, ref, f"G={G} many chunks")
    w.block_table[7, 40] = -1  # tokens 1280-1311 of sequence 7 (its sixth chunk)
    got = run_q4(w)
    assert q8.q8kv_device_errors(clear=True) & q8.DEVERR_BLOCK_TABLE
    bt, kept_lens = without_block(w.block_table, w.seq_lens, 7, 40, 32)
    kept = oracle.PagedCacheQ4(w.k4, w.v4, w.kd, w.vd, bt, kept_lens, w.cfg.n_q_heads, w.scale)
    assert_close(got[7], oracle.decode_q4_all(kept, w.q)[7], f"G={G} bad entry mid-run")
    others = np.arange(40) != 7
    assert_close(got[others], ref[others], f"G={G} other rows")
