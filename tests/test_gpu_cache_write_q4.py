"""Parity of the CUDA q4_0 KV-cache write (q8kv_cache_write_q4) with the oracle's, bit for
bit: packed 4-bit codes and binary16 block scales of every written row, untouched slots left
as they were, and the device error bits equal to the oracle's flags.

Covers head_dim 64/128/256, 1 to 8 KV heads, token counts from 1 to thousands (several
waves of the grid plus a ragged tail), padding slots, strided rows of a fused projection,
zero rows and zero blocks, magnitudes from 1e-7 to 30 (and scales that overflow binary16),
non-finite blocks, slots past the pool, magnitude ties, the hand-derived golden blocks, the
full q4_0 prompt fill of the 16 x 4096-token GQA workload against the generator's cache,
and a write followed by a q4_0 decode.
"""
import numpy as np
import pytest
import torch

import decode_attention_int8_b200 as q8
import oracle
from decode_attention_int8_b200 import inputs
from gpu_util import assert_close
from test_oracle_q4 import golden

pytestmark = pytest.mark.gpu

SENT8, SENT16 = 0xA5, 0xDEAD


def host_pools(P, bs, Hk, D):
    k4 = np.full((P, bs, Hk, D // 2), SENT8, np.uint8)
    kd = np.full((P, bs, Hk, D // 32), SENT16, np.uint16)
    return k4, k4.copy(), kd, kd.copy()


def gpu_write(pools, k_new, v_new, slots, Hk, D):
    """k_new, v_new: fp32 [n][stride] host arrays (row (i, h) at [i][h * D:(h + 1) * D])."""
    k4, v4 = (torch.from_numpy(a.copy()).cuda() for a in pools[:2])
    kd, vd = (torch.from_numpy(a.copy().view(np.int16)).cuda() for a in pools[2:])
    n = slots.shape[0]
    kb = torch.from_numpy(np.ascontiguousarray(k_new)).cuda()
    vb = torch.from_numpy(np.ascontiguousarray(v_new)).cuda()
    kn = kb[:, :Hk * D].view(n, Hk, D) if n else kb.view(0, Hk, D)
    vn = vb[:, :Hk * D].view(n, Hk, D) if n else vb.view(0, Hk, D)
    q8.q8kv_cache_write_q4(k4, v4, kd, vd, kn, vn, torch.from_numpy(slots).cuda())
    torch.cuda.synchronize()
    return (k4.cpu().numpy(), v4.cpu().numpy(), kd.cpu().numpy().view(np.uint16),
            vd.cpu().numpy().view(np.uint16))


def oracle_write(pools, k_new, v_new, slots):
    k4, v4, kd, vd = (a.copy() for a in pools)
    flags = oracle.cache_write_q4(k4, v4, kd, vd, k_new, v_new, slots,
                                  token_stride=k_new.shape[1])
    return (k4, v4, kd, vd), flags


def assert_pools_equal(got, ref, what=""):
    for g, r, name in zip(got, ref, ("k4", "v4", "kd", "vd")):
        bad = np.argwhere(g != r)
        assert bad.size == 0, f"{what} {name}: {len(bad)} mismatches, first at {bad[0].tolist()}"


def check(P, bs, Hk, D, rows: inputs.CacheRows):
    pools = host_pools(P, bs, Hk, D)
    q8.q8kv_device_errors(clear=True)
    got = gpu_write(pools, rows.k_new, rows.v_new, rows.slots, Hk, D)
    dev_flags = q8.q8kv_device_errors(clear=True)
    ref, flags = oracle_write(pools, rows.k_new, rows.v_new, rows.slots)
    assert_pools_equal(got, ref, f"P={P} bs={bs} Hk={Hk} D={D} n={rows.n_tokens}")
    assert dev_flags == flags
    return got


@pytest.mark.parametrize("D", [64, 128, 256])
@pytest.mark.parametrize("Hk", [1, 3, 8])
@pytest.mark.parametrize("n", [1, 37, 3000])
def test_scattered_rows_match_the_oracle(D, Hk, n):
    P, bs = 400, 16
    rows = inputs.make_cache_rows(n, Hk, D, P, bs, seed=D + Hk + n, pad_every=7)
    check(P, bs, Hk, D, rows)


def test_strided_rows_of_a_fused_projection():
    Hk, D, n = 4, 128, 500
    rows = inputs.make_cache_rows(n, Hk, D, 64, 32, seed=3, token_stride=3 * Hk * D)
    check(64, 32, Hk, D, rows)  # the NaN tails must never be read (no NONFINITE flag)


def test_non_finite_blocks_slots_past_the_pool_ties_and_overflow():
    rng = np.random.default_rng(5)
    Hk, D, n, P, bs = 2, 128, 12, 4, 16
    x = rng.standard_normal((2, n, Hk, D)).astype(np.float32)
    x[0, 0, 0, 40] = np.inf
    x[1, 1, 1, 100] = -np.inf
    x[0, 2, 0, 3] = np.nan
    x[:, 3, :, 32:64] = 0.0  # zero blocks
    x[:, 3, :, 35] = -0.0
    x[0, 4, 0, :32] = 1.0  # every element ties: the first wins
    x[0, 4, 0, 10] = -1.0
    x[1, 5, 1, 64:96] = np.float32(3e5)  # m = -6e5: d = 75000 is past binary16's range,
    x[1, 5, 1, 70] = np.float32(-6e5)  # so the stored scale is +inf (as the format does)
    x[0, 6, :, :] *= np.float32(1e-7)  # tiny values: subnormal binary16 scales
    k = x[0].reshape(n, -1)
    v = x[1].reshape(n, -1)
    slots = np.array([0, 1, 2, 3, 4, 5, 6, P * bs, -1, P * bs + 7, 20, 63], np.int64)
    pools = host_pools(P, bs, Hk, D)
    q8.q8kv_device_errors(clear=True)
    got = gpu_write(pools, k, v, slots, Hk, D)
    dev_flags = q8.q8kv_device_errors(clear=True)
    ref, flags = oracle_write(pools, k, v, slots)
    assert flags == oracle.FLAG_SLOT | oracle.FLAG_NONFINITE
    assert_pools_equal(got, ref, "edge rows")
    assert dev_flags == flags


def test_golden_blocks():
    cases = golden()
    D = 32 * len(cases)
    D = D if D in (64, 128, 256) else 256
    x = np.zeros((1, D), np.float32)
    for j, c in enumerate(cases[:D // 32]):
        x[0, 32 * j:32 * (j + 1)] = c["x"]
    pools = host_pools(1, 16, 1, D)
    got = gpu_write(pools, x, x[:, ::-1].copy(), np.array([9], np.int64), 1, D)
    codes = np.empty(D, np.int32)
    codes[0::2] = got[0][0, 9, 0] & 0xF
    codes[1::2] = got[0][0, 9, 0] >> 4
    for j, c in enumerate(cases[:D // 32]):
        np.testing.assert_array_equal(codes[32 * j:32 * (j + 1)], c["codes"], c["name"])
        assert got[2][0, 9, 0, j] == c["d16"], c["name"]


def test_prompt_fill_equals_the_generated_cache_and_decodes():
    """All 65536 tokens x 8 KV heads of the batched GQA workload, written from its fp32 draws
    at the slots of its block table: the pools equal the generator's q4_0 cache, and the q4_0
    decode over them equals the decode over the generated cache."""
    cfg = inputs.WORKLOADS[1]
    w32 = inputs.make(cfg, keep_fp32=True)
    w4 = inputs.make_q4(cfg)
    P, bs, Hk, D = w32.k32.shape
    slots = inputs.prompt_slots(w4.block_table, w4.seq_lens, bs)
    k_rows = w32.k32.reshape(P * bs, Hk * D)[slots]
    v_rows = w32.v32.reshape(P * bs, Hk * D)[slots]
    del w32
    pools = host_pools(P, bs, Hk, D)
    q8.q8kv_device_errors(clear=True)
    got = gpu_write(pools, k_rows, v_rows, slots, Hk, D)
    assert q8.q8kv_device_errors(clear=True) == 0
    for g, r, name in zip(got, (w4.k4, w4.v4, w4.kd, w4.vd), ("k4", "v4", "kd", "vd")):
        np.testing.assert_array_equal(g.reshape(P * bs, -1)[slots], r.reshape(P * bs, -1)[slots],
                                      name)
    # decode over the written pools on the device, against the oracle on sampled rows
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    out = torch.empty(w4.q.shape, dtype=torch.float32, device="cuda")
    q8.q8kv_decode_attn_q4(out, t(w4.q), t(got[0]), t(got[1]), t(got[2].view(np.int16)),
                           t(got[3].view(np.int16)), t(w4.block_table), t(w4.seq_lens), w4.scale)
    torch.cuda.synchronize()
    cache = oracle.PagedCacheQ4(w4.k4, w4.v4, w4.kd, w4.vd, w4.block_table, w4.seq_lens,
                                cfg.n_q_heads, w4.scale)
    rng = np.random.default_rng(1)
    pairs = [(int(b), int(h)) for b, h in zip(rng.integers(0, cfg.B, 48),
                                              rng.integers(0, cfg.n_q_heads, 48))]
    ref = oracle.decode_q4_pairs(cache, w4.q, pairs)
    got_rows = out.cpu().numpy()
    assert_close(np.stack([got_rows[b, h] for b, h in pairs]), ref, "decode after q4 write")


def test_rejected_arguments():
    k4 = torch.zeros((2, 16, 2, 64), dtype=torch.uint8, device="cuda")
    kd = torch.zeros((2, 16, 2, 4), dtype=torch.int16, device="cuda")
    rows = torch.zeros((3, 2, 128), dtype=torch.float32, device="cuda")
    slots = torch.zeros(3, dtype=torch.int64, device="cuda")
    with pytest.raises(ValueError):
        q8.q8kv_cache_write_q4(k4, k4.clone(), kd[..., :2], kd.clone(), rows, rows, slots)
    L = q8.lib()
    import ctypes
    P = lambda t: ctypes.c_void_p(t.data_ptr())
    # head_dim 96: not a supported width
    assert L.q8kv_cache_write_q4(P(k4), P(k4), P(kd), P(kd), P(rows), P(rows), P(slots), 3, 2,
                                 96, 16, 2, 0, None) == 2
    # misaligned scale pointer
    assert L.q8kv_cache_write_q4(P(k4), P(k4), ctypes.c_void_p(kd.data_ptr() + 2), P(kd),
                                 P(rows), P(rows), P(slots), 3, 2, 128, 16, 2, 0, None) == 1
    # zero tokens: nothing enqueued, null rows allowed
    assert L.q8kv_cache_write_q4(P(k4), P(k4), P(kd), P(kd), None, None, None, 0, 2, 128, 16, 2,
                                 0, None) == 0
