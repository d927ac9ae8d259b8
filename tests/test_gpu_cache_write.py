"""Parity of the CUDA KV-cache write (q8kv_cache_write) with the oracle's, bit for bit:
int8 codes and fp32 scales of every written row, untouched slots left as they were, and
the device error bits equal to the oracle's flags.

Covers head_dim 64/128/256, 1 to 8 KV heads, token counts from 1 to thousands (several
waves of the grid plus a ragged tail), padding slots, strided rows of a fused projection,
zero rows, rows below the 1e-6 guard, non-finite rows, slots past the pool, the hand-
derived golden rows, the full prompt fill of the 16 x 4096-token GQA workload, and a
write followed by a decode.
"""
import numpy as np
import pytest
import torch

import decode_attention_int8_b200 as q8
import oracle
from conftest import load_golden_kvquant
from decode_attention_int8_b200 import inputs
from gpu_util import assert_close, oracle_cache

pytestmark = pytest.mark.gpu

SENTINEL_CODE = 99
SENTINEL_SCALE = -3.0


def host_pools(P, bs, Hk, D):
    return (np.full((P, bs, Hk, D), SENTINEL_CODE, np.int8),
            np.full((P, bs, Hk, D), SENTINEL_CODE, np.int8),
            np.full((P, bs, Hk), SENTINEL_SCALE, np.float32),
            np.full((P, bs, Hk), SENTINEL_SCALE, np.float32))


def gpu_write(pools, rows: inputs.CacheRows, stream=None):
    """Copy pools and rows to the device, run the CUDA write, return the pools on the host."""
    k, v, ks, vs = (torch.from_numpy(a.copy()).cuda() for a in pools)
    n, Hk, D = rows.n_tokens, rows.n_kv_heads, rows.head_dim
    kb = torch.from_numpy(np.ascontiguousarray(rows.k_new)).cuda()
    vb = torch.from_numpy(np.ascontiguousarray(rows.v_new)).cuda()
    kn = kb[:, :Hk * D].view(n, Hk, D) if n else kb.view(0, Hk, D)
    vn = vb[:, :Hk * D].view(n, Hk, D) if n else vb.view(0, Hk, D)
    slots = torch.from_numpy(rows.slots).cuda()
    q8.q8kv_cache_write(k, v, ks, vs, kn, vn, slots, stream=stream)
    torch.cuda.synchronize()
    return tuple(t.cpu().numpy() for t in (k, v, ks, vs))


def oracle_write(pools, rows: inputs.CacheRows):
    k, v, ks, vs = (a.copy() for a in pools)
    flags = oracle.cache_write(k, v, ks, vs, rows.k_new, rows.v_new, rows.slots,
                               token_stride=rows.k_new.shape[1])
    return (k, v, ks, vs), flags


def assert_pools_equal(got, ref, what=""):
    names = ("k_blocks", "v_blocks", "kscale", "vscale")
    for g, r, name in zip(got, ref, names):
        if g.dtype == np.float32:
            g, r = g.view(np.uint32), r.view(np.uint32)  # bit equality, NaN included
        bad = np.argwhere(g != r)
        assert bad.size == 0, f"{what} {name}: {len(bad)} mismatches, first at {bad[0].tolist()}"


def check(P, bs, Hk, D, n, seed, pad_every=0, token_stride=None):
    rows = inputs.make_cache_rows(n, Hk, D, P, bs, seed=seed, pad_every=pad_every,
                                  token_stride=token_stride)
    pools = host_pools(P, bs, Hk, D)
    q8.q8kv_device_errors(clear=True)
    got = gpu_write(pools, rows)
    dev_flags = q8.q8kv_device_errors(clear=True)
    ref, flags = oracle_write(pools, rows)
    assert_pools_equal(got, ref, f"P={P} bs={bs} Hk={Hk} D={D} n={n}")
    assert dev_flags == flags
    return rows, got


@pytest.mark.parametrize("D", [64, 128, 256])
@pytest.mark.parametrize("Hk", [1, 3, 8])
@pytest.mark.parametrize("n", [1, 37, 3000])
def test_scattered_rows_match_the_oracle(D, Hk, n):
    bs = 16
    P = max(4, -(-n // bs) + 3)
    check(P, bs, Hk, D, n, seed=1000 + D + 10 * Hk + n, pad_every=7)


def test_many_waves_and_a_ragged_tail():
    # 8 * 148 blocks of 8 warps take 9472 rows per pass: 50001 tokens x 5 heads is 26+ passes
    check(P=3200, bs=16, Hk=5, D=128, n=50001, seed=7, pad_every=13)


@pytest.mark.parametrize("D", [64, 128, 256])
def test_strided_rows_of_a_fused_projection(D):
    # q, k and v of 4 query and 2 KV heads side by side: k_new starts at head 4, and the
    # NaN-filled neighbours must never be read (a read would set the non-finite bit)
    Hq, Hk, n, bs = 4, 2, 300, 32
    P = -(-n // bs) + 2
    rows = inputs.make_cache_rows(n, Hk, D, P, bs, seed=D, pad_every=11,
                                  token_stride=(Hq + 2 * Hk) * D)
    # move the rows to the K and V positions of the fused layout
    qkv = np.full((n, (Hq + 2 * Hk) * D), np.nan, np.float32)
    qkv[:, Hq * D:(Hq + Hk) * D] = rows.k_new[:, :Hk * D]
    qkv[:, (Hq + Hk) * D:] = rows.v_new[:, :Hk * D]
    pools = host_pools(P, bs, Hk, D)
    k, v, ks, vs = (torch.from_numpy(a.copy()).cuda() for a in pools)
    t = torch.from_numpy(qkv).cuda()
    kn = t[:, Hq * D:(Hq + Hk) * D].unflatten(1, (Hk, D))
    vn = t[:, (Hq + Hk) * D:].unflatten(1, (Hk, D))
    assert kn.stride(0) == (Hq + 2 * Hk) * D and not kn.is_contiguous()
    q8.q8kv_device_errors(clear=True)
    q8.q8kv_cache_write(k, v, ks, vs, kn, vn, torch.from_numpy(rows.slots).cuda())
    torch.cuda.synchronize()
    assert q8.q8kv_device_errors(clear=True) == 0
    got = tuple(x.cpu().numpy() for x in (k, v, ks, vs))
    ref, flags = oracle_write(pools, rows)
    assert flags == 0
    assert_pools_equal(got, ref, f"fused D={D}")


def test_golden_rows_on_the_gpu():
    cases = load_golden_kvquant()
    n, Hk, D = len(cases), 1, 64
    rows = inputs.CacheRows(np.stack([c["x"] for c in cases]), np.stack([c["x"] for c in cases]),
                            np.arange(n, dtype=np.int64), Hk, D)
    pools = host_pools(1, 16, Hk, D)
    q8.q8kv_device_errors(clear=True)
    k, v, ks, vs = gpu_write(pools, rows)
    dev_flags = q8.q8kv_device_errors(clear=True)
    expect_flags = 0
    for i, c in enumerate(cases):
        np.testing.assert_array_equal(k[0, i, 0], c["codes"], err_msg=c["name"])
        np.testing.assert_array_equal(v[0, i, 0], c["codes"], err_msg=c["name"])
        bits = c["scale_bits"]
        if bits == "nan":
            assert np.isnan(ks[0, i, 0]) and np.isnan(vs[0, i, 0])
        elif bits != "approx":
            assert int(ks[0, i, 0:1].view(np.uint32)[0]) == bits, c["name"]
        expect_flags |= c["flags"]
    assert dev_flags == expect_flags


def test_non_finite_rows_and_slots_past_the_pool():
    P, bs, Hk, D, n = 8, 16, 4, 128, 100
    rows = inputs.make_cache_rows(n, Hk, D, P, bs, seed=5)
    rows.k_new[3, 2 * D + 17] = np.inf
    rows.v_new[10, 5] = np.nan
    rows.k_new[11, 3 * D + 127] = -np.inf
    rows.slots[[20, 40]] = [P * bs, P * bs + 12345]
    pools = host_pools(P, bs, Hk, D)
    q8.q8kv_device_errors(clear=True)
    got = gpu_write(pools, rows)
    dev_flags = q8.q8kv_device_errors(clear=True)
    ref, flags = oracle_write(pools, rows)
    assert flags == q8.DEVERR_SLOT | q8.DEVERR_NONFINITE
    assert dev_flags == flags
    assert_pools_equal(got, ref, "non-finite / out of range")


def test_no_tokens_changes_nothing():
    pools = host_pools(2, 16, 2, 128)
    rows = inputs.CacheRows(np.zeros((0, 256), np.float32), np.zeros((0, 256), np.float32),
                            np.zeros(0, np.int64), 2, 128)
    got = gpu_write(pools, rows)
    assert_pools_equal(got, pools, "empty")


def test_prompt_fill_of_the_gqa_batch_workload():
    # the full-size write that the benchmark times: 16 x 4096 tokens x 8 KV heads, D 128,
    # slots of the workload's permuted 1024-block table
    cfg = inputs.WORKLOADS[1]
    rows = inputs.make_prompt_fill(cfg)
    P = int(rows.slots.max()) // cfg.block_size + 1
    pools = host_pools(P, cfg.block_size, cfg.n_kv_heads, cfg.head_dim)
    q8.q8kv_device_errors(clear=True)
    got = gpu_write(pools, rows)
    assert q8.q8kv_device_errors(clear=True) == 0
    ref, flags = oracle_write(pools, rows)
    assert flags == 0
    assert_pools_equal(got, ref, "prompt fill")


def test_write_then_decode():
    # fill a cache with the CUDA write, decode it with the CUDA decode kernel, and compare
    # with the oracle's decode of the oracle-written cache (the pools must be identical)
    B, Hq, Hk, D, bs = 3, 16, 4, 128, 64
    lens = np.array([1000, 1, 2500], np.int32)
    w = inputs.make_custom(B, Hq, Hk, D, lens, bs, seed=77)
    slots = inputs.prompt_slots(w.block_table, lens, bs)
    n = slots.shape[0]
    rng = np.random.default_rng(78)
    k32 = rng.standard_normal((n, Hk * D)).astype(np.float32)
    v32 = (rng.standard_t(3.0, (n, Hk * D))).astype(np.float32)
    rows = inputs.CacheRows(k32, v32, slots, Hk, D)
    pools = host_pools(w.num_blocks, bs, Hk, D)
    got = gpu_write(pools, rows)
    ref, flags = oracle_write(pools, rows)
    assert flags == 0
    assert_pools_equal(got, ref, "write before decode")
    k, v, ks, vs = (torch.from_numpy(a).cuda() for a in got)
    out = torch.full((B, Hq, D), float("nan"), dtype=torch.float32, device="cuda")
    q = torch.from_numpy(w.q).cuda()
    q8.q8kv_decode_attn(out, q, k, v, ks, vs, torch.from_numpy(w.block_table).cuda(),
                        torch.from_numpy(lens).cuda(), w.scale)
    torch.cuda.synchronize()
    wr = inputs.Workload(w.cfg, w.q, *ref, w.block_table, lens, w.scale)
    expect = oracle.decode_all(oracle_cache(wr), w.q)
    assert_close(out.cpu().numpy(), expect, "decode of the written cache")
