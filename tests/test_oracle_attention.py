"""Pins of the oracle's decode attention against what the pages and the mathematics fix.

- Closed forms: seq_len = 1 returns the dequantised V row; identical keys (or a zero
  query, or a zero softmax scale) return the mean of the dequantised V; one dominant key
  returns its V row; a two-token case against exp() by hand.
- Invariants from the Kestrel-LLM walk-through section 4 (debug task A): the token loop
  runs exactly seq_len times and M never decreases.
- Section 3 of the walk-through: the naive variant that stores all scores first is
  functionally equivalent to the single pass.
- A library routine: torch's scaled_dot_product_attention in fp64 on the dequantised
  tensors (dequantised q . dequantised k = sum_j dot_j qsc_j ks exactly in real numbers).
- Placement invariance (moving blocks and rewriting the block table) and the GQA mapping
  (replicating KV heads turns GQA into MHA with the same result).
"""
import math

import numpy as np
import pytest
import torch

import oracle
from decode_attention_int8_b200 import inputs

FL_1_127 = 2.0 ** -7 * (1 + 2.0 ** -7 + 2.0 ** -14 + 2.0 ** -21)  # fl32(1/127), by hand


def cache_of(w):
    return oracle.PagedCache(w.k, w.v, w.ks, w.vs, w.block_table, w.seq_lens,
                             w.cfg.n_q_heads, w.scale)


def hand_cache(k_rows, v_rows, ks, vs, n_q_heads, scale, bs=4):
    """A one-sequence cache from logical rows [L][Hk][D], identity block table."""
    k_rows = np.asarray(k_rows, np.int8)
    L, Hk, D = k_rows.shape
    P = max(1, -(-L // bs))
    k = np.zeros((P * bs, Hk, D), np.int8)
    v = np.zeros((P * bs, Hk, D), np.int8)
    kss = np.ones((P * bs, Hk), np.float32)
    vss = np.ones((P * bs, Hk), np.float32)
    k[:L], v[:L] = k_rows, np.asarray(v_rows, np.int8)
    kss[:L], vss[:L] = ks, vs
    bt = np.arange(P, dtype=np.int32)[None, :]
    return oracle.PagedCache(k.reshape(P, bs, Hk, D), v.reshape(P, bs, Hk, D),
                             kss.reshape(P, bs, Hk), vss.reshape(P, bs, Hk), bt,
                             np.array([L], np.int32), n_q_heads, scale)


def np_quantize(q):
    """The Q rule in numpy fp32 (input preparation for the library cross-check)."""
    blocks = np.asarray(q, np.float32).reshape(-1, 32)
    qm = np.abs(blocks).max(1)
    qm = np.where(qm < np.float32(1e-6), np.float32(1.0), qm).astype(np.float32)
    qsc = (qm * (np.float32(1.0) / np.float32(127.0))).astype(np.float32)
    iq = (np.float32(127.0) / qm).astype(np.float32)
    codes = np.clip(np.rint(blocks * iq[:, None]), -127, 127).astype(np.int8)
    return codes.reshape(np.shape(q)), qsc.reshape(*np.shape(q)[:-1], -1)


def sdpa_reference(w):
    """torch SDPA (fp64) on dequantised q, K, V gathered through the block table."""
    B, Hq, D = w.q.shape
    Hk, bs = w.cfg.n_kv_heads, w.cfg.block_size
    codes, qsc = np_quantize(w.q)
    qdeq = codes.astype(np.float64) * np.repeat(qsc.astype(np.float64), 32, axis=-1)
    out = np.zeros((B, Hq, D))
    for b in range(B):
        L = int(w.seq_lens[b])
        if L == 0:
            continue
        t = np.arange(L)
        slots = w.block_table[b, t // bs].astype(np.int64) * bs + t % bs
        kf = w.k.reshape(-1, Hk, D)[slots].astype(np.float64)
        vf = w.v.reshape(-1, Hk, D)[slots].astype(np.float64)
        kf *= w.ks.reshape(-1, Hk)[slots][..., None]
        vf *= w.vs.reshape(-1, Hk)[slots][..., None]
        G = Hq // Hk
        K = torch.from_numpy(kf).permute(1, 0, 2).repeat_interleave(G, 0)[None]
        V = torch.from_numpy(vf).permute(1, 0, 2).repeat_interleave(G, 0)[None]
        Q = torch.from_numpy(qdeq[b])[None, :, None, :]
        o = torch.nn.functional.scaled_dot_product_attention(Q, K, V, scale=float(w.scale))
        out[b] = o[0, :, 0, :].numpy()
    return out


def small_workload(seed=0, **kw):
    args = dict(B=3, n_q_heads=8, n_kv_heads=2, head_dim=64, seq_lens=[1, 37, 70],
                block_size=16, seed=seed)
    args.update(kw)
    return inputs.make_custom(**args)


# ------------------------------------------------------------------ closed forms


def test_seq_len_one_returns_dequantised_v_row():
    w = small_workload(seq_lens=[1, 1, 1])
    c = cache_of(w)
    out = oracle.decode_all(c, w.q)
    for b in range(w.cfg.B):
        slot = int(w.block_table[b, 0]) * w.cfg.block_size
        for h in range(w.cfg.n_q_heads):
            kvh = h // w.cfg.group
            expect = w.v.reshape(-1, 2, 64)[slot, kvh].astype(np.float64) * float(
                w.vs.reshape(-1, 2)[slot, kvh])
            np.testing.assert_array_equal(out[b, h], expect)


def test_identical_keys_return_mean_of_dequantised_v():
    rng = np.random.default_rng(1)
    L, Hk, D = 23, 1, 64
    krow = rng.integers(-127, 128, (Hk, D))
    k_rows = np.broadcast_to(krow, (L, Hk, D))
    v_rows = rng.integers(-127, 128, (L, Hk, D))
    vs = rng.uniform(0.01, 2.0, (L, Hk)).astype(np.float32)
    c = hand_cache(k_rows, v_rows, 0.37, vs, 4, 0.125)
    q = rng.standard_normal((1, 4, D)).astype(np.float32)
    expect = (v_rows.astype(np.float64) * vs[..., None].astype(np.float64)).mean(0)[0]
    out = oracle.decode_all(c, q)[0]
    for h in range(4):
        np.testing.assert_allclose(out[h], expect, rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("how", ["zero_q", "zero_scale"])
def test_flat_scores_return_mean(how):
    w = small_workload(seed=5)
    if how == "zero_q":
        w.q[:] = 0.0
    else:
        w.scale = 0.0
    c = cache_of(w)
    out = oracle.decode_all(c, w.q)
    Hk, D, bs = 2, 64, 16
    for b in range(w.cfg.B):
        L = int(w.seq_lens[b])
        t = np.arange(L)
        slots = w.block_table[b, t // bs].astype(np.int64) * bs + t % bs
        vdeq = w.v.reshape(-1, Hk, D)[slots] * w.vs.reshape(-1, Hk)[slots][..., None].astype(
            np.float64)
        for h in range(8):
            np.testing.assert_allclose(out[b, h], vdeq[:, h // 4].mean(0), rtol=1e-12,
                                       atol=1e-13)


@pytest.mark.parametrize("pos", [0, 9, 19])
def test_dominant_key_returns_its_v_row(pos):
    rng = np.random.default_rng(pos)
    L, D = 20, 128
    k_rows = np.zeros((L, 1, D), np.int8)
    k_rows[pos] = 127
    v_rows = rng.integers(-127, 128, (L, 1, D))
    vs = rng.uniform(0.1, 1.0, (L, 1)).astype(np.float32)
    q = np.ones((1, 1, D), np.float32)  # codes 127, qsc = fl(1/127)
    c = hand_cache(k_rows, v_rows, 1.0, vs, 1, 1.0 / math.sqrt(D))
    out = oracle.decode_all(c, q)[0, 0]
    # the winning score is 4 * 32 * 127 * 127 * fl(1/127) / sqrt(128) ~ 1436: every
    # other weight is exp(-1436) == 0 in fp64, so the result is the row itself
    np.testing.assert_array_equal(out, v_rows[pos, 0].astype(np.float64) * float(vs[pos, 0]))


def test_two_tokens_against_hand_exponentials():
    D = 128
    k_rows = np.stack([np.ones((1, D)), 2 * np.ones((1, D))]).astype(np.int8)
    v_rows = np.stack([np.full((1, D), 3), np.full((1, D), -5)]).astype(np.int8)
    ks = np.array([[0.5], [0.25]], np.float32)
    vs = np.array([[0.75], [0.125]], np.float32)
    scale = np.float32(0.0625)
    c = hand_cache(k_rows, v_rows, ks, vs, 1, scale)
    q = np.ones((1, 1, D), np.float32)
    out = oracle.decode_all(c, q)[0, 0]
    # codes of q are all 127 and each block scale is fl(1/127): dot_j = 32 * 127 * k
    s1 = 4 * (32 * 127 * 1) * FL_1_127 * 0.5 * 0.0625
    s2 = 4 * (32 * 127 * 2) * FL_1_127 * 0.25 * 0.0625
    e1, e2 = math.exp(s1), math.exp(s2)
    expect = (e1 * 3 * 0.75 + e2 * (-5) * 0.125) / (e1 + e2)
    np.testing.assert_allclose(out, expect, rtol=1e-14)
    np.testing.assert_allclose(oracle.scores(c, q, 0, 0), [s1, s2], rtol=1e-15)


def test_block_dots_closed_forms():
    D = 128
    L = 3
    k_rows = np.zeros((L, 1, D), np.int8)
    k_rows[0] = 1
    k_rows[1] = -2
    k_rows[2, 0, 70] = 5  # only channel 70 (block 2, lane 6) is non-zero
    c = hand_cache(k_rows, np.zeros((L, 1, D)), 1.0, 1.0, 1, 1.0)
    q = np.ones((1, 1, D), np.float32)
    q[0, 0, 70] = -1.0
    dots = oracle.block_dots(c, q, 0, 0)
    # block 2 holds one -127 code at channel 70; every other code is 127
    np.testing.assert_array_equal(dots[0], [4064, 4064, 4064 - 2 * 127, 4064])
    np.testing.assert_array_equal(dots[1], [-8128, -8128, -2 * (4064 - 2 * 127), -8128])
    np.testing.assert_array_equal(dots[2], [0, 0, -127 * 5, 0])


def test_block_dots_brute_force_tiny():
    w = small_workload(seed=11, B=2, seq_lens=[5, 3], head_dim=64, block_size=2)
    c = cache_of(w)
    codes, _ = oracle.quantize_q(w.q.reshape(-1))
    codes = codes.reshape(w.q.shape)
    for b in range(2):
        for h in range(8):
            dots = oracle.block_dots(c, w.q, b, h)
            for t in range(int(w.seq_lens[b])):
                blk = int(w.block_table[b][t // 2])
                row = w.k[blk][t % 2][h // 4]
                for j in range(2):
                    acc = 0
                    for i in range(32):
                        acc += int(codes[b, h, 32 * j + i]) * int(row[32 * j + i])
                    assert dots[t, j] == acc


# ------------------------------------------------------------------ invariants


def test_m_monotone_and_iteration_count():
    w = small_workload(seed=3, seq_lens=[1, 64, 203], block_size=32)
    c = cache_of(w)
    for b in range(w.cfg.B):
        for h in (0, 5):
            out, mt, n = oracle.decode_online(c, w.q, b, h, trace=True)
            L = int(w.seq_lens[b])
            assert n == L
            assert np.all(np.diff(mt) >= 0)
            s = oracle.scores(c, w.q, b, h)
            np.testing.assert_array_equal(mt, np.maximum.accumulate(s))


def test_single_pass_equals_three_pass():
    for seed in range(4):
        w = small_workload(seed=seed, seq_lens=[3, 50, 129], k_dist="student_t3")
        c = cache_of(w)
        for b in range(w.cfg.B):
            for h in range(w.cfg.n_q_heads):
                a = oracle.decode_online(c, w.q, b, h)
                t = oracle.decode_threepass(c, w.q, b, h)
                np.testing.assert_allclose(a, t, rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("seed,k_bias", [(0, 0.0), (1, 2.0), (2, 6.0)])
def test_matches_torch_sdpa_fp64(seed, k_bias):
    w = small_workload(seed=seed, k_bias_std=k_bias, seq_lens=[1, 77, 130], block_size=16,
                       n_q_heads=12, n_kv_heads=3, head_dim=128)
    c = cache_of(w)
    out = oracle.decode_all(c, w.q)
    ref = sdpa_reference(w)
    np.testing.assert_allclose(out, ref, rtol=1e-11, atol=1e-12)
    # the numpy quantisation used for the reference gives the oracle's codes
    codes, qsc = np_quantize(w.q)
    qi, qs = oracle.quantize_q(w.q.reshape(-1))
    np.testing.assert_array_equal(codes.reshape(-1), qi)
    np.testing.assert_array_equal(qsc.reshape(-1), qs)


def test_placement_invariance():
    w = small_workload(seed=9, seq_lens=[17, 40, 63], block_size=8, extra_blocks=5)
    c = cache_of(w)
    base = oracle.decode_all(c, w.q)
    rng = np.random.default_rng(0)
    perm = rng.permutation(w.num_blocks)  # new position of every physical block
    k2, v2 = np.empty_like(w.k), np.empty_like(w.v)
    ks2, vs2 = np.empty_like(w.ks), np.empty_like(w.vs)
    k2[perm], v2[perm], ks2[perm], vs2[perm] = w.k, w.v, w.ks, w.vs
    bt2 = np.where(w.block_table >= 0, perm[np.maximum(w.block_table, 0)], -1).astype(np.int32)
    c2 = oracle.PagedCache(k2, v2, ks2, vs2, bt2, w.seq_lens, w.cfg.n_q_heads, w.scale)
    np.testing.assert_array_equal(oracle.decode_all(c2, w.q), base)


def test_gqa_equals_mha_with_replicated_heads():
    w = small_workload(seed=4, seq_lens=[5, 33, 90])
    c = cache_of(w)
    base = oracle.decode_all(c, w.q)
    G = w.cfg.group
    rep = lambda a, ax: np.repeat(a, G, axis=ax)
    c2 = oracle.PagedCache(rep(w.k, 2), rep(w.v, 2), rep(w.ks, 2), rep(w.vs, 2), w.block_table,
                           w.seq_lens, w.cfg.n_q_heads, w.scale)
    np.testing.assert_array_equal(oracle.decode_all(c2, w.q), base)


def test_softmax_weights_sum_to_one():
    # constant dequantised V (codes 1, scale 1) gives exactly 1 up to rounding
    w = small_workload(seed=6, seq_lens=[9, 100, 257], block_size=32)
    w.v[:] = 1
    w.vs[:] = 1.0
    out = oracle.decode_all(cache_of(w), w.q)
    np.testing.assert_allclose(out, 1.0, rtol=1e-13)


def test_zero_length_sequence_gives_zero_row():
    w = small_workload(seed=2, seq_lens=[0, 5, 0])
    out = oracle.decode_all(cache_of(w), w.q)
    assert np.all(out[0] == 0) and np.all(out[2] == 0)
    assert np.any(out[1] != 0)


def test_pairs_match_all():
    w = small_workload(seed=8)
    c = cache_of(w)
    full = oracle.decode_all(c, w.q)
    pairs = [(2, 7), (0, 0), (1, 3)]
    got = oracle.decode_pairs(c, w.q, pairs)
    for i, (b, h) in enumerate(pairs):
        np.testing.assert_array_equal(got[i], full[b, h])


def test_rejects_out_of_range_inputs():
    w = small_workload(seed=1)
    bt = w.block_table.copy()
    bt[2, 0] = w.num_blocks  # one past the pool
    c = oracle.PagedCache(w.k, w.v, w.ks, w.vs, bt, w.seq_lens, 8, w.scale)
    with pytest.raises(oracle.OracleError):
        oracle.decode_all(c, w.q)
    lens = w.seq_lens.copy()
    lens[0] = w.max_blocks_per_seq * w.cfg.block_size + 1
    c = oracle.PagedCache(w.k, w.v, w.ks, w.vs, w.block_table, lens, 8, w.scale)
    with pytest.raises(oracle.OracleError):
        oracle.decode_all(c, w.q)


# ------------------------------------------------------------------ unquantised attention


def test_fp32_attention_matches_sdpa():
    w = inputs.make_custom(2, 4, 2, 64, [13, 40], 8, seed=12, keep_fp32=True)
    c = cache_of(w)
    Hk, D, bs = 2, 64, 8
    for b in range(2):
        L = int(w.seq_lens[b])
        t = np.arange(L)
        slots = w.block_table[b, t // bs].astype(np.int64) * bs + t % bs
        K = torch.from_numpy(w.k32.reshape(-1, Hk, D)[slots].astype(np.float64)).permute(1, 0, 2)
        V = torch.from_numpy(w.v32.reshape(-1, Hk, D)[slots].astype(np.float64)).permute(1, 0, 2)
        for h in range(4):
            Q = torch.from_numpy(w.q[b, h].astype(np.float64))[None, None, None]
            ref = torch.nn.functional.scaled_dot_product_attention(
                Q, K[h // 2][None, None], V[h // 2][None, None], scale=float(w.scale))
            got = oracle.attn_fp32(c, w.q, w.k32, w.v32, b, h)
            np.testing.assert_allclose(got, ref[0, 0, 0].numpy(), rtol=1e-12, atol=1e-13)
