"""Pins of the oracle's q4_0 KV-cache write (llama.cpp's q4_0 blocks, which the baguaai.com
FlashAttention page names as a quantised KV cache type; the slot placement of beaiera.top
"deepseek-attention-div64", "Top-K index global mapping"): blocks from the hand-derived
golden file written through the cache, random rows against the generator's vectorised
numpy quantiser (a separate writing of the rule), placement against sentinel-filled pools
(padding, slots past the pool, strided rows whose NaN tails are never read), the
non-finite-block rule, and a prompt written token by token that equals the generator's
q4_0 cache."""
import numpy as np
import pytest

import oracle
from decode_attention_int8_b200 import inputs
from test_oracle_q4 import golden

SENT8, SENT16 = 0xA5, 0xDEAD


def pools(P, bs, Hk, D):
    k4 = np.full((P, bs, Hk, D // 2), SENT8, np.uint8)
    kd = np.full((P, bs, Hk, D // 32), SENT16, np.uint16)
    return k4, k4.copy(), kd, kd.copy()


def np_q4(rows):
    return inputs.quantize_q4_0_rows(np.asarray(rows, np.float32))


def test_golden_blocks_through_the_write():
    cases = golden()
    D = 32 * len(cases)
    k_row = np.concatenate([c["x"] for c in cases])[None, None, :]  # one token, one head
    v_row = k_row[..., ::-1].copy()
    k4, v4, kd, vd = pools(2, 4, 1, D)
    flags = oracle.cache_write_q4(k4, v4, kd, vd, k_row, v_row, np.array([5], np.int64))
    assert flags == 0
    codes = np.empty(D, np.int32)
    codes[0::2] = k4[1, 1, 0] & 0xF
    codes[1::2] = k4[1, 1, 0] >> 4
    for j, c in enumerate(cases):
        np.testing.assert_array_equal(codes[32 * j:32 * (j + 1)], c["codes"], c["name"])
        assert kd[1, 1, 0, j] == c["d16"], c["name"]
    # every other slot untouched
    mask = np.ones((2, 4), bool)
    mask[1, 1] = False
    assert np.all(k4[mask] == SENT8) and np.all(kd[mask] == SENT16)


@pytest.mark.parametrize("D", [64, 128, 256])
def test_random_rows_match_the_generator_quantiser(D):
    rng = np.random.default_rng(D)
    P, bs, Hk, n = 6, 16, 4, 40
    x = rng.standard_normal((2, n, Hk, D)).astype(np.float32)
    x[:, ::3] = rng.standard_t(3, (2, len(range(0, n, 3)), Hk, D)).astype(np.float32)
    x *= (10.0 ** rng.integers(-4, 5, (2, n, Hk, 1))).astype(np.float32)
    slots = rng.permutation(P * bs)[:n].astype(np.int64)
    k4, v4, kd, vd = pools(P, bs, Hk, D)
    assert oracle.cache_write_q4(k4, v4, kd, vd, x[0], x[1], slots) == 0
    for which, (codes, d16) in enumerate(((k4, kd), (v4, vd))):
        ref_codes, ref_d = np_q4(x[which])
        got_codes = codes.reshape(P * bs, Hk, D // 2)[slots]
        got_d = d16.reshape(P * bs, Hk, D // 32)[slots]
        np.testing.assert_array_equal(got_codes, ref_codes)
        np.testing.assert_array_equal(got_d, ref_d)
        untouched = np.setdiff1d(np.arange(P * bs), slots)
        assert np.all(codes.reshape(P * bs, -1)[untouched] == SENT8)
        assert np.all(d16.reshape(P * bs, -1)[untouched] == SENT16)


def test_padding_slots_past_the_pool_and_strided_rows():
    rng = np.random.default_rng(7)
    P, bs, Hk, D = 3, 16, 2, 128
    n, stride = 6, 3 * 2 * 128  # a fused-QKV-like stride: the tail of every token is NaN
    kbuf = np.full((n, stride), np.nan, np.float32)
    vbuf = np.full((n, stride), np.nan, np.float32)
    rows_k = rng.standard_normal((n, Hk, D)).astype(np.float32)
    rows_v = rng.standard_normal((n, Hk, D)).astype(np.float32)
    kbuf[:, :Hk * D] = rows_k.reshape(n, -1)
    vbuf[:, :Hk * D] = rows_v.reshape(n, -1)
    slots = np.array([3, -1, 47, 48, 1000, 0], np.int64)  # 48 = P * bs is past the pool
    k4, v4, kd, vd = pools(P, bs, Hk, D)
    flags = oracle.cache_write_q4(k4, v4, kd, vd, kbuf, vbuf, slots, token_stride=stride)
    assert flags == oracle.FLAG_SLOT  # the NaN tails were never read
    written = [0, 2, 5]
    for which, (codes, d16, rows) in enumerate(((k4, kd, rows_k), (v4, vd, rows_v))):
        rc, rd = np_q4(rows[written])
        np.testing.assert_array_equal(codes.reshape(P * bs, Hk, -1)[slots[written]], rc)
        np.testing.assert_array_equal(d16.reshape(P * bs, Hk, -1)[slots[written]], rd)
        others = np.setdiff1d(np.arange(P * bs), slots[written])
        assert np.all(codes.reshape(P * bs, -1)[others] == SENT8)


def test_non_finite_blocks_and_zero_blocks():
    rng = np.random.default_rng(9)
    Hk, D = 1, 128
    x = rng.standard_normal((4, Hk, D)).astype(np.float32)
    x[0, 0, 40] = np.inf  # block 1 of token 0
    x[1, 0, 100] = np.nan  # block 3 of token 1
    x[2, 0, 0:32] = 0.0  # an all-zero block
    x[2, 0, 5] = -0.0
    k4, v4, kd, vd = pools(1, 16, Hk, D)
    flags = oracle.cache_write_q4(k4, v4, kd, vd, x, x.copy(), np.arange(4, dtype=np.int64))
    assert flags == oracle.FLAG_NONFINITE
    codes, d16 = k4[0, :4, 0], kd[0, :4, 0]
    bad = {(0, 1), (1, 3)}
    for t in range(4):
        for j in range(4):
            if (t, j) in bad:
                assert np.all(codes[t, 16 * j:16 * (j + 1)] == 0x88) and d16[t, j] == 0x7E00
            else:
                rc, rd = np_q4(np.nan_to_num(x[t, 0, 32 * j:32 * (j + 1)])[None])
                np.testing.assert_array_equal(codes[t, 16 * j:16 * (j + 1)], rc[0])
                if (t, j) == (2, 0):  # max|x| = 0: m = +0, d = +0 / -8 = -0, codes 8
                    assert d16[t, j] == 0x8000 and np.all(codes[t, :16] == 0x88)
                else:
                    assert d16[t, j] == rd[0, 0]
    np.testing.assert_array_equal(v4, k4)


def test_prompt_written_token_by_token_equals_the_generated_cache():
    lens = np.array([40, 1, 77], np.int32)
    w32 = inputs.make_custom(3, 8, 2, 128, lens, 16, seed=12, keep_fp32=True)  # fp32 draws
    w4 = inputs.make_q4_custom(3, 8, 2, 128, lens, 16, seed=12)  # the same draws as q4_0
    slots = inputs.prompt_slots(w4.block_table, lens, 16)
    P, bs, Hk, D = w32.k32.shape
    k_rows = w32.k32.reshape(P * bs, Hk, D)[slots]
    v_rows = w32.v32.reshape(P * bs, Hk, D)[slots]
    k4, v4, kd, vd = pools(P, bs, Hk, D)
    for i in range(len(slots)):  # one token per call
        assert oracle.cache_write_q4(k4, v4, kd, vd, k_rows[i:i + 1], v_rows[i:i + 1],
                                     slots[i:i + 1]) == 0
    for got, ref in ((k4, w4.k4), (v4, w4.v4), (kd, w4.kd), (vd, w4.vd)):
        np.testing.assert_array_equal(got.reshape(P * bs, -1)[slots],
                                      ref.reshape(P * bs, -1)[slots])
    # the decode over the written cache is the decode over the generated one
    c_w = oracle.PagedCacheQ4(k4, v4, kd, vd, w4.block_table, lens, 8, w4.scale)
    c_g = oracle.PagedCacheQ4(w4.k4, w4.v4, w4.kd, w4.vd, w4.block_table, lens, 8, w4.scale)
    np.testing.assert_array_equal(oracle.decode_q4_all(c_w, w4.q), oracle.decode_q4_all(c_g, w4.q))
