"""Multi-query decode (q8kv_decode_attn_multi) against the fp64 oracle: n_queries new
tokens per sequence share the K/V tiles, each query attending causally up to its own
position. Tolerance as for the single-query decode: max-abs <= 1e-4, rel-L2 <= 1e-5.

Covers every tiling the query rows can take (n_queries x group = 2 to 128 rows per KV
head: the packed path, one and two 8-row tiles, several 16-row slices), ragged lengths
around the causal window (shorter than n_queries, equal, tile and block boundaries), one
query (bit-equal to q8kv_decode_attn), the full-size 16 x 4096-token GQA workload with
4 queries per sequence on sampled rows, and the shape limit.
"""
import numpy as np
import pytest
import torch

import decode_attention_int8_b200 as q8
import oracle
from decode_attention_int8_b200 import inputs
from gpu_util import assert_close, oracle_cache, to_device

pytestmark = pytest.mark.gpu


def run_multi(w, q):
    d = to_device(w)
    qd = torch.from_numpy(np.ascontiguousarray(q)).cuda()
    out = torch.full(qd.shape, float("nan"), dtype=torch.float32, device="cuda")
    q8.q8kv_decode_attn_multi(out, qd, d["k"], d["v"], d["ks"], d["vs"], d["bt"], d["lens"],
                              w.scale)
    torch.cuda.synchronize()
    return out.cpu().numpy()


@pytest.mark.parametrize("nq,Hq,Hk", [
    (2, 4, 2),    # 4 rows per KV head: packed path
    (3, 8, 8),    # 3 rows (one padding row): packed path
    (2, 32, 8),   # 8 rows: one 8-row tile
    (4, 32, 8),   # 16 rows: two 8-row tiles
    (3, 32, 8),   # 12 rows
    (8, 32, 8),   # 32 rows: two 16-row slices, 4 KV heads per tile
    (8, 16, 2),   # 64 rows: four 16-row slices
    (16, 8, 1),   # 128 rows: the largest tiling (one KV head per tile)
    (16, 32, 8),  # 64 rows over 8 KV heads: 2-head tiles with 4-head scale boxes
    (5, 20, 4),   # 25 rows, 2 slices
])
@pytest.mark.parametrize("bs", [16, 64])
def test_tilings_and_causal_edges(nq, Hq, Hk, bs):
    lens = [1, nq - 1 if nq > 1 else 1, nq, nq + 1, 31, 32, 33, bs + nq - 1, 3 * bs + 5, 700]
    w = inputs.make_custom(len(lens), Hq, Hk, 128, lens, bs, seed=nq * 100 + Hq + bs)
    q = inputs.multi_queries(len(lens), nq, Hq, 128, seed=nq + bs)
    got = run_multi(w, q)
    ref = oracle.decode_multi(oracle_cache(w), q, nq)
    for b, L in enumerate(lens):
        for i in range(nq):
            if L - (nq - 1 - i) <= 0:
                assert np.all(got[b, i] == 0.0), f"b={b} i={i}: no visible token, not zero"
    assert_close(got, ref, f"nq={nq} Hq={Hq} Hk={Hk} bs={bs}")


def test_one_query_equals_the_single_query_call():
    w = inputs.make_custom(3, 32, 8, 128, [1000, 17, 4096], 64, seed=5)
    got = run_multi(w, w.q[:, None])
    d = to_device(w)
    out = torch.empty(d["q"].shape, dtype=torch.float32, device="cuda")
    q8.q8kv_decode_attn(out, d["q"], d["k"], d["v"], d["ks"], d["vs"], d["bt"], d["lens"],
                        w.scale)
    torch.cuda.synchronize()
    assert np.array_equal(got[:, 0], out.cpu().numpy())


def test_long_split_sequence_with_many_queries():
    # one long sequence split over every SM: the causal window sits in the last CTA's share
    nq, Hq, Hk = 8, 16, 4  # 32 rows per KV head
    w = inputs.make_custom(1, Hq, Hk, 128, [60001], 128, seed=11, k_bias_std=2.0)
    q = inputs.multi_queries(1, nq, Hq, 128, seed=11)
    assert_close(run_multi(w, q), oracle.decode_multi(oracle_cache(w), q, nq), "long, nq=8")


def test_gqa_batch_workload_with_four_queries():
    # the benchmark's 16 x 4096-token workload with 3 draft tokens + 1 (nq = 4), as timed
    # by bench.py; 160 sampled (sequence, query, head) rows against the oracle
    cfg = inputs.WORKLOADS[1]
    nq = 4
    w = inputs.make(cfg)
    q = inputs.multi_queries(cfg.B, nq, cfg.n_q_heads, cfg.head_dim, seed=cfg.seed)
    got = run_multi(w, q)
    rng = np.random.default_rng(0)
    rows = np.stack([rng.integers(0, cfg.B, 160), rng.integers(0, nq, 160),
                     rng.integers(0, cfg.n_q_heads, 160)], axis=1)
    ref = oracle.decode_multi_rows(oracle_cache(w), q, nq, rows)
    assert_close(got[rows[:, 0], rows[:, 1], rows[:, 2]], ref, "gqa_batch nq=4 sampled rows")


@pytest.mark.parametrize("nq,Hq,Hk", [
    (17, 64, 8),  # 136 rows per KV head: above the 128-row tiling
    (16, 24, 6),  # 64 rows per KV head with 6 KV heads: a tile holds 2 of them, and the
                  # scale rows of 6 heads (24 bytes) are no 16-byte multiple
])
def test_unsupported_row_counts(nq, Hq, Hk):
    w = inputs.make_custom(1, Hq, Hk, 128, [40], 16, seed=1)
    q = inputs.multi_queries(1, nq, Hq, 128)
    with pytest.raises(q8.Q8KVError) as e:
        run_multi(w, q)
    assert e.value.status == 2


# ------------------------------------------------------------------ tensor-memory kernel
# (9-32 query rows per KV head with n_queries > 1 run on q8kv_mq_tc.cuh)

@pytest.mark.parametrize("nq,Hq,Hk,bs", [
    (16, 1, 1, 64),    # 16 rows, one KV head: scales by bulk copy
    (12, 2, 1, 128),   # 24 rows padded to 32, a 128-token block per tile
    (10, 4, 4, 256),   # 10 rows padded to 16, a tile covers half a block
    (9, 16, 4, 16),    # 36 rows: above 32, the warp-MMA kernel
])
def test_tensor_memory_shapes(nq, Hq, Hk, bs):
    lens = [1, nq - 1, nq, 15, 127, 128, 129, 1000, 5000]
    w = inputs.make_custom(len(lens), Hq, Hk, 128, lens, bs, seed=nq + Hq + bs)
    q = inputs.multi_queries(len(lens), nq, Hq, 128, seed=bs)
    assert_close(run_multi(w, q), oracle.decode_multi(oracle_cache(w), q, nq),
                 f"nq={nq} Hq={Hq} Hk={Hk} bs={bs}")


def test_many_segments_per_cta():
    # 400 short sequences x 8 KV heads: each CTA switches segments many times, so the query
    # slots alternate and the later segments' rows are quantised by the helper warp
    rng = np.random.default_rng(21)
    lens = rng.integers(1, 300, 400)
    nq, Hq, Hk = 4, 32, 8
    w = inputs.make_custom(len(lens), Hq, Hk, 128, lens, 16, seed=21)
    q = inputs.multi_queries(len(lens), nq, Hq, 128, seed=21)
    assert_close(run_multi(w, q), oracle.decode_multi(oracle_cache(w), q, nq), "400 x nq=4")


@pytest.mark.parametrize("nq,Hq,Hk", [(8, 32, 8), (4, 32, 8)])
def test_tiny_and_huge_v_scales(nq, Hq, Hk):
    # V scales over 60 decades: each row's weights and its reference move with them; the
    # tolerance is relative to each output row's own magnitude
    lens = [500, 64, 3000]
    w = inputs.make_custom(len(lens), Hq, Hk, 128, lens, 32, seed=9 + nq)
    rng = np.random.default_rng(nq)
    w.vs *= (10.0 ** rng.uniform(-30, 30, w.vs.shape)).astype(np.float32)
    w.ks *= (10.0 ** rng.uniform(-2, 1, w.ks.shape)).astype(np.float32)
    q = inputs.multi_queries(len(lens), nq, Hq, 128, seed=nq)
    got = run_multi(w, q)
    ref = oracle.decode_multi(oracle_cache(w), q, nq)
    for b in range(len(lens)):
        for i in range(nq):
            for h in range(Hq):
                r = ref[b, i, h]
                assert np.linalg.norm(got[b, i, h] - r) <= 1e-5 * np.linalg.norm(r) + 1e-30, \
                    (b, i, h)
