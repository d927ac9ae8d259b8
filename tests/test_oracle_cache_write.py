"""Pins of the oracle's KV-cache write: per-(token, KV head) q8 quantisation of new K and
V rows (Kestrel-LLM walk-through: one scale per (token, KV head), applied as
scale * 1/127, with the section 2 part 1 quantiser on whole rows) and their placement at
physical slots (beaiera.top "deepseek-attention-div64", "Top-K index global mapping":
slot = block * block_size + offset, negative entries skipped).

Expected values come from hand-derived rows (tests/golden/kvquant_cases.txt), from
properties of nearest-level quantisation, from the input generator's independent
vectorised quantiser, and, for placement, from the block-table arithmetic itself.
"""
import numpy as np
import pytest

import oracle
from conftest import load_golden_kvquant
from decode_attention_int8_b200 import inputs

SENTINEL_CODE = 99
SENTINEL_SCALE = -3.0


@pytest.mark.parametrize("case", load_golden_kvquant(), ids=lambda c: c["name"])
def test_golden_rows(case):
    codes, scale, flags = oracle.quantize_kv_row(case["x"])
    np.testing.assert_array_equal(codes, case["codes"])
    assert flags == case["flags"]
    bits = case["scale_bits"]
    if bits == "nan":
        assert np.isnan(scale)
    elif bits == "approx":
        ref = np.float32(np.max(np.abs(case["x"]))) / np.float32(127.0)
        assert abs(int(np.float32(scale).view(np.int32)) - int(ref.view(np.int32))) <= 2
    else:
        assert int(np.float32(scale).view(np.uint32)) == bits


def _rows(seed, n, D):
    rng = np.random.default_rng(seed)
    mag = rng.choice([1e-4, 1e-2, 1.0, 30.0, 1e4], size=(n, 1))
    x = rng.standard_normal((n, D)) * mag
    x[: n // 4] = rng.standard_t(3.0, (n // 4, D)) * mag[: n // 4]  # outlier-heavy rows
    return x.astype(np.float32)


@pytest.mark.parametrize("D", [64, 128, 256])
def test_row_properties(D):
    x = _rows(D, 512, D)
    for r in x:
        codes, scale, flags = oracle.quantize_kv_row(r)
        c = codes.astype(np.int64)
        assert flags == 0
        assert c.min() >= -127 and c.max() <= 127
        # the largest magnitude maps to +-127 with its sign
        i = int(np.argmax(np.abs(r)))
        assert c[i] == 127 * np.sign(r[i])
        # codes keep the sign of their input and sit within half a step of it
        assert np.all(np.sign(c) * np.sign(r) >= 0)
        err = np.abs(c * np.float64(scale) - r.astype(np.float64))
        assert np.all(err <= 0.5 * np.float64(scale) * (1 + 1e-5))
        # the stored multiplier is max|x| / 127 to within fp32 rounding
        assert abs(np.float64(scale) / (np.abs(r).max() / 127.0) - 1.0) < 2e-7


def test_power_of_two_equivariance():
    x = _rows(5, 64, 128)
    for r in x:
        c0, s0, _ = oracle.quantize_kv_row(r)
        for k in (-20, -3, 7, 30):
            if np.abs(r).max() * 2.0 ** k < 1e-6:
                continue  # the zero-row guard takes over (pinned by the golden rows)
            c1, s1, _ = oracle.quantize_kv_row(r * np.float32(2.0 ** k))
            np.testing.assert_array_equal(c1, c0)
            assert s1 == s0 * np.float32(2.0 ** k)


def test_agrees_with_the_generators_vectorised_quantiser():
    # inputs.quantize_rows is a separate numpy writing of the same rule (whole arrays at
    # once, numpy's own rint); the two must agree bit for bit
    x = _rows(11, 2048, 128)
    codes_v, scale_v = inputs.quantize_rows(x)
    for i, r in enumerate(x):
        codes, scale, _ = oracle.quantize_kv_row(r)
        np.testing.assert_array_equal(codes, codes_v[i])
        assert np.float32(scale).view(np.uint32) == scale_v[i].view(np.uint32)


def _pools(P, bs, Hk, D):
    k = np.full((P, bs, Hk, D), SENTINEL_CODE, np.int8)
    v = np.full((P, bs, Hk, D), SENTINEL_CODE, np.int8)
    ks = np.full((P, bs, Hk), SENTINEL_SCALE, np.float32)
    vs = np.full((P, bs, Hk), SENTINEL_SCALE, np.float32)
    return k, v, ks, vs


def test_rows_land_at_their_slots_and_nothing_else_changes():
    P, bs, Hk, D = 6, 16, 3, 64
    rng = np.random.default_rng(3)
    n = 40
    slots = rng.permutation(P * bs)[:n].astype(np.int64)
    slots[[3, 17, 30]] = -1  # padding entries
    stride = Hk * D + 8  # rows of a fused projection: 8 unrelated floats per token
    kbuf = rng.standard_normal((n, stride)).astype(np.float32)
    vbuf = rng.standard_normal((n, stride)).astype(np.float32)
    kbuf[:, Hk * D:] = np.nan  # never read
    vbuf[:, Hk * D:] = np.inf
    k, v, ks, vs = _pools(P, bs, Hk, D)
    flags = oracle.cache_write(k, v, ks, vs, kbuf, vbuf, slots, token_stride=stride)
    assert flags == 0
    kf, vf = k.reshape(P * bs, Hk, D), v.reshape(P * bs, Hk, D)
    ksf, vsf = ks.reshape(P * bs, Hk), vs.reshape(P * bs, Hk)
    written = np.zeros(P * bs, bool)
    for i, s in enumerate(slots):
        if s < 0:
            continue
        written[s] = True
        for h in range(Hk):
            ck, sk, _ = oracle.quantize_kv_row(kbuf[i, h * D:(h + 1) * D])
            cv, sv, _ = oracle.quantize_kv_row(vbuf[i, h * D:(h + 1) * D])
            np.testing.assert_array_equal(kf[s, h], ck)
            np.testing.assert_array_equal(vf[s, h], cv)
            assert ksf[s, h] == sk and vsf[s, h] == sv
    assert np.all(kf[~written] == SENTINEL_CODE) and np.all(vf[~written] == SENTINEL_CODE)
    assert np.all(ksf[~written] == SENTINEL_SCALE) and np.all(vsf[~written] == SENTINEL_SCALE)


def test_slot_past_the_pool_is_flagged_and_skipped():
    P, bs, Hk, D = 2, 16, 2, 64
    k, v, ks, vs = _pools(P, bs, Hk, D)
    x = np.ones((3, Hk, D), np.float32)
    flags = oracle.cache_write(k, v, ks, vs, x, x, np.array([P * bs, 5, P * bs + 100]))
    assert flags == oracle.FLAG_SLOT
    touched = (k.reshape(P * bs, Hk, D) != SENTINEL_CODE).any(axis=(1, 2))
    assert touched.tolist() == [i == 5 for i in range(P * bs)]


def test_non_finite_row_is_flagged():
    P, bs, Hk, D = 1, 16, 2, 64
    k, v, ks, vs = _pools(P, bs, Hk, D)
    kx = np.ones((1, Hk, D), np.float32)
    vx = np.ones((1, Hk, D), np.float32)
    vx[0, 1, 7] = np.nan
    flags = oracle.cache_write(k, v, ks, vs, kx, vx, np.array([4]))
    assert flags == oracle.FLAG_NONFINITE
    assert np.all(v[0, 4, 1] == 0) and np.isnan(vs[0, 4, 1])
    assert np.all(v[0, 4, 0] == 127) and vs[0, 4, 0] == np.float32(1.0) * (np.float32(1.0) /
                                                                        np.float32(127.0))
    assert np.all(k[0, 4] == 127)


def test_written_sequence_decodes_like_the_generated_cache():
    # Write the prompt of two sequences token by token through their block tables, then
    # check (1) the pools equal the generator's quantisation of the same rows placed by
    # the same tables, and (2) a one-token sequence decodes to its dequantised V row,
    # which is within half a step of the original fp32 row.
    B, Hq, Hk, D, bs = 2, 8, 2, 128, 16
    lens = np.array([37, 1], np.int32)
    w = inputs.make_custom(B, Hq, Hk, D, lens, bs, seed=9, keep_fp32=True)
    P = w.num_blocks
    k, v, ks, vs = _pools(P, bs, Hk, D)
    for b in range(B):
        t = np.arange(lens[b])
        slots = w.block_table[b, t // bs].astype(np.int64) * bs + t % bs
        kx = w.k32.reshape(P * bs, Hk, D)[slots]
        vx = w.v32.reshape(P * bs, Hk, D)[slots]
        assert oracle.cache_write(k, v, ks, vs, kx, vx, slots) == 0
    used = np.zeros(P * bs, bool)
    for b in range(B):
        t = np.arange(lens[b])
        used[w.block_table[b, t // bs].astype(np.int64) * bs + t % bs] = True
    np.testing.assert_array_equal(k.reshape(P * bs, Hk, D)[used], w.k.reshape(P * bs, Hk, D)[used])
    np.testing.assert_array_equal(v.reshape(P * bs, Hk, D)[used], w.v.reshape(P * bs, Hk, D)[used])
    np.testing.assert_array_equal(ks.reshape(P * bs, Hk)[used], w.ks.reshape(P * bs, Hk)[used])
    np.testing.assert_array_equal(vs.reshape(P * bs, Hk)[used], w.vs.reshape(P * bs, Hk)[used])
    cache = oracle.PagedCache(k, v, ks, vs, w.block_table, lens, Hq, w.scale)
    slot = int(w.block_table[1, 0]) * bs
    for h in range(Hq):
        kvh = h // (Hq // Hk)
        out = oracle.decode_online(cache, w.q, 1, h)
        vrow = v.reshape(P * bs, Hk, D)[slot, kvh].astype(np.float64)
        step = np.float64(vs.reshape(P * bs, Hk)[slot, kvh])
        np.testing.assert_array_equal(out, vrow * step)
        x32 = w.v32.reshape(P * bs, Hk, D)[slot, kvh].astype(np.float64)
        assert np.all(np.abs(out - x32) <= 0.5 * step * (1 + 1e-5))


def test_rejects_bad_arguments():
    k, v, ks, vs = _pools(1, 16, 2, 64)
    x = np.ones((2, 2, 64), np.float32)
    with pytest.raises(oracle.OracleError):
        oracle.cache_write(k, v, ks, vs, x, x, np.array([0, 1]), token_stride=64)
    with pytest.raises(oracle.OracleError):
        oracle.quantize_kv_row(np.zeros(0, np.float32))
