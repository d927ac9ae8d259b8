"""Pins of the oracle's q4_0 cache (llama.cpp's q4_0 blocks, which the baguaai.com
FlashAttention page names as a quantised KV cache type): the binary16 rounding against
numpy, the block quantiser against hand-derived blocks (tests/golden/q4_0_cases.txt) and
the generator's vectorised writing of it, and the q4_0 decode against (a) the pinned q8
decode on a cache holding the same values, (b) torch SDPA on the dequantised data, and
(c) the seq_len = 1 closed form."""
import os

import numpy as np
import pytest
import torch

import oracle
from decode_attention_int8_b200 import inputs
from test_oracle_attention import np_quantize

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def golden():
    cases, cur = [], None
    for raw in open(os.path.join(ROOT, "tests", "golden", "q4_0_cases.txt")):
        line = raw.strip()
        if not line or line.startswith("#"):
            continue
        key, *vals = line.split()
        if key == "case":
            cur = {"name": vals[0]}
            cases.append(cur)
        elif key == "x":
            cur["x"] = np.array([float(v) for v in vals], np.float32)
        elif key == "codes":
            cur["codes"] = np.array([int(v) for v in vals], np.int32)
        elif key == "d16":
            cur["d16"] = int(vals[0], 16)
    return cases


def unpack(packed):
    p = packed.astype(np.int32)
    out = np.empty(packed.shape[:-1] + (2 * packed.shape[-1],), np.int32)
    out[..., 0::2] = p & 0xF
    out[..., 1::2] = p >> 4
    return out


def test_binary16_rounding_matches_numpy():
    rng = np.random.default_rng(0)
    x = (rng.standard_normal(200000) * 10.0 ** rng.integers(-9, 6, 200000)).astype(np.float32)
    x = np.concatenate([x, np.array([65504, 65519, 65520, 1e-8, 6e-8, 2.98e-8, -0.0],
                                    np.float32)])
    with np.errstate(over="ignore"):
        ref = x.astype(np.float16).view(np.uint16)
    np.testing.assert_array_equal(oracle.f32_to_f16(x), ref)


@pytest.mark.parametrize("case", golden(), ids=lambda c: c["name"])
def test_golden_blocks(case):
    packed, d16 = oracle.quantize_q4_0(case["x"])
    np.testing.assert_array_equal(unpack(packed), case["codes"])
    assert int(d16[0]) == case["d16"]


def test_agrees_with_the_generators_vectorised_quantiser():
    rng = np.random.default_rng(3)
    x = (rng.standard_t(3.0, (4096, 128)) * rng.choice([1e-3, 1.0, 40.0], (4096, 1))).astype(
        np.float32)
    p0, d0 = oracle.quantize_q4_0(x)
    p1, d1 = inputs.quantize_q4_0_rows(x)
    np.testing.assert_array_equal(p0, p1)
    np.testing.assert_array_equal(d0, d1)


def test_block_properties():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((2048, 32)).astype(np.float32)
    packed, d16 = oracle.quantize_q4_0(x)
    codes = unpack(packed)
    d = d16.view(np.float16).astype(np.float64)[:, 0]
    deq = (codes - 8) * d[:, None]
    # the element of largest magnitude maps to code 0 (value -8 d = m up to binary16)
    i = np.argmax(np.abs(x), axis=1)
    assert np.all(codes[np.arange(2048), i] == 0)
    # every other value is within a step |d| (the rule rounds half down and clips at +7 d)
    err = np.abs(deq - x.astype(np.float64))
    assert np.all(err <= np.abs(d)[:, None] * 1.01 + 1e-6)


def q4_cache(w):
    return oracle.PagedCacheQ4(w.k4, w.v4, w.kd, w.vd, w.block_table, w.seq_lens,
                               w.cfg.n_q_heads, w.scale)


def test_decode_equals_the_q8_decode_on_the_same_values():
    # a q8 cache whose codes lie in [-8, 7] and whose row scales are binary16 numbers holds
    # exactly the values of the q4_0 cache with codes + 8 and those scales in every block
    rng = np.random.default_rng(5)
    w = inputs.make_custom(3, 8, 2, 128, [1, 40, 300], 16, seed=5)
    codes = rng.integers(-8, 8, w.k.shape).astype(np.int8)
    vcodes = rng.integers(-8, 8, w.v.shape).astype(np.int8)
    ks = (2.0 ** rng.integers(-8, 2, w.ks.shape) * rng.integers(1, 2048, w.ks.shape) /
          1024).astype(np.float16).astype(np.float32)
    vs = (2.0 ** rng.integers(-8, 2, w.vs.shape) * rng.integers(1, 2048, w.vs.shape) /
          1024).astype(np.float16).astype(np.float32)
    q8 = oracle.PagedCache(codes, vcodes, ks, vs, w.block_table, w.seq_lens, 8, w.scale)
    pack = lambda c: ((c[..., 0::2].astype(np.int32) + 8) |
                      ((c[..., 1::2].astype(np.int32) + 8) << 4)).astype(np.uint8)
    rep = lambda s: np.repeat(s[..., None].astype(np.float16).view(np.uint16), 4, axis=-1)
    q4 = oracle.PagedCacheQ4(pack(codes), pack(vcodes), rep(ks), rep(vs), w.block_table,
                             w.seq_lens, 8, w.scale)
    np.testing.assert_allclose(oracle.decode_q4_all(q4, w.q), oracle.decode_all(q8, w.q),
                               rtol=1e-12, atol=1e-14)


def test_decode_matches_sdpa_on_dequantised_data():
    w = inputs.make_q4_custom(2, 8, 2, 128, [33, 200], 16, seed=6, k_dist="student_t3")
    got = oracle.decode_q4_all(q4_cache(w), w.q)
    Hk, D, bs = 2, 128, 16
    codes, qsc = np_quantize(w.q)
    qdeq = codes.astype(np.float64) * np.repeat(qsc.astype(np.float64), 32, axis=-1)
    deq = lambda p, d: ((unpack(p) - 8).astype(np.float64) *
                        np.repeat(d.view(np.float16).astype(np.float64), 32, axis=-1))
    for b, L in enumerate(w.seq_lens):
        t = np.arange(L)
        slots = w.block_table[b, t // bs].astype(np.int64) * bs + t % bs
        kf = deq(w.k4.reshape(-1, Hk, D // 2)[slots], w.kd.reshape(-1, Hk, D // 32)[slots])
        vf = deq(w.v4.reshape(-1, Hk, D // 2)[slots], w.vd.reshape(-1, Hk, D // 32)[slots])
        K = torch.from_numpy(kf).permute(1, 0, 2).repeat_interleave(4, 0)[None]
        V = torch.from_numpy(vf).permute(1, 0, 2).repeat_interleave(4, 0)[None]
        Q = torch.from_numpy(qdeq[b])[None, :, None, :]
        ref = torch.nn.functional.scaled_dot_product_attention(Q, K, V, scale=float(w.scale))
        np.testing.assert_allclose(got[b], ref[0, :, 0, :].numpy(), rtol=1e-10, atol=1e-12)


def test_seq_len_one_returns_the_dequantised_v_row():
    w = inputs.make_q4_custom(2, 4, 1, 128, [1, 1], 16, seed=7)
    got = oracle.decode_q4_all(q4_cache(w), w.q)
    for b in range(2):
        slot = int(w.block_table[b, 0]) * 16
        v = ((unpack(w.v4.reshape(-1, 1, 64)[slot, 0]) - 8) *
             np.repeat(w.vd.reshape(-1, 1, 4)[slot, 0].view(np.float16).astype(np.float64), 32))
        for h in range(4):
            np.testing.assert_array_equal(got[b, h], v)
