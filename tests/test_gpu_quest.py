"""QUEST block metadata (q8kv_quest_metadata) against the oracle, bit for bit: the
per-channel max / min of the dequantised K of every KV block, the placement through the
metadata block table, the tail block, and the zero rows of a request's last metadata block
(rows no request owns are left untouched).

The grid follows the CANN guide's test matrix (xdnf.cn/news/235188, "functional
correctness"): basic (B 1-2, 4 or 8 KV heads, 1-128 blocks per request), edge (KV head
counts 1..33 including odd ones, block counts around 64 / 128 / 256), equal or random
request lengths, several metadata blocks per request, and a large batch."""
import numpy as np
import pytest
import torch

import decode_attention_int8_b200 as q8
import oracle
from decode_attention_int8_b200 import inputs
from gpu_util import oracle_cache

pytestmark = pytest.mark.gpu


def run(w, meta, n_meta):
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    bs, Hk, D = w.cfg.block_size, w.cfg.n_kv_heads, w.cfg.head_dim
    mx = torch.full((n_meta, bs, Hk, D), float("nan"), dtype=torch.float32, device="cuda")
    mn = torch.full_like(mx, float("nan"))
    q8.q8kv_device_errors(clear=True)
    q8.q8kv_quest_metadata(mx, mn, t(w.k), t(w.ks), t(w.block_table), t(w.seq_lens), t(meta))
    torch.cuda.synchronize()
    return mx.cpu().numpy(), mn.cpu().numpy(), q8.q8kv_device_errors(clear=True)


def check(B, Hk, mkbpr, same_len, seed, bs=128, k_dist="normal"):
    rng = np.random.default_rng(seed)
    full = mkbpr * bs
    lens = [full] * B if same_len else rng.integers(0, full + 1, B).tolist()
    w = inputs.make_custom(B, Hk, Hk, 128, lens, bs, seed=seed, k_dist=k_dist,
                           max_blocks_per_seq=mkbpr, extra_blocks=3)
    meta, n_meta = inputs.quest_meta_table(lens, bs, seed=seed, extra_blocks=2)
    mx, mn, err = run(w, meta, n_meta)
    rx, rn = oracle.quest_metadata(oracle_cache(w), meta, n_meta)
    assert err == 0
    for got, ref, name in ((mx, rx, "max"), (mn, rn, "min")):
        bad = np.argwhere(got.view(np.uint32) != ref.view(np.uint32))
        assert bad.size == 0, f"{name}: {len(bad)} mismatches, first {bad[0].tolist()}"


@pytest.mark.parametrize("B", [1, 2])
@pytest.mark.parametrize("Hk", [4, 8])
@pytest.mark.parametrize("mkbpr", [1, 64, 126, 128])
def test_basic(B, Hk, mkbpr):
    check(B, Hk, mkbpr, same_len=True, seed=B * 1000 + Hk * 10 + mkbpr)


@pytest.mark.parametrize("Hk", [1, 2, 7, 9, 16, 21, 33])
def test_edge_head_counts(Hk):
    check(2, Hk, 65, same_len=False, seed=Hk)


@pytest.mark.parametrize("mkbpr", [63, 64, 65, 127, 128, 129, 150, 255, 256, 257])
def test_edge_block_counts(mkbpr):
    check(2, 4, mkbpr, same_len=False, seed=mkbpr, k_dist="student_t3")


@pytest.mark.parametrize("bs", [16, 32, 64])
def test_other_block_sizes(bs):
    # a metadata block has block_size rows: with 16-token blocks it covers 256 tokens, so
    # requests of a few thousand tokens span many metadata blocks
    check(3, 8, 300, same_len=False, seed=bs, bs=bs)


def test_large_batch_random_lengths():
    check(24, 8, 40, same_len=False, seed=24)


def test_metadata_table_too_short_is_flagged():
    bs = 16
    w = inputs.make_custom(1, 2, 2, 128, [bs * bs + 1], bs, seed=1)  # needs 2 metadata blocks
    meta = np.array([[0]], np.int32)
    mx, mn, err = run(w, meta, 2)
    assert err == q8.DEVERR_META
    # the block that fits is still written
    rx, rn = oracle.quest_metadata(oracle_cache(w), np.array([[0, 1]], np.int32), 2)
    assert np.array_equal(mx[0], rx[0]) and np.array_equal(mn[0], rn[0])


@pytest.mark.parametrize("Hk", [8, 3])
def test_scales_at_the_edges_of_fp32(Hk):
    """Subnormal (down to the smallest), zero, tiny, huge and overflowing scales, with codes
    at -128, -127, 0 and 127: each product is one correctly rounded fp32 multiply with no
    flush to zero, and max and min equal the oracle's bit for bit (8 heads: the head count
    compiled in; 3 heads: read at run time). Zero scales carry non-negative codes only, so
    no product is -0: the oracle keeps the first of two equal zeros, and the sign of a zero
    extreme is not what this checks."""
    bs = 16
    lens = [300, 129, 17]
    w = inputs.make_custom(3, Hk, Hk, 128, lens, bs, seed=77, extra_blocks=3)
    rng = np.random.default_rng(77)
    special = np.array([1.4e-45, 1e-42, 1.1754942e-38, 2.0 ** -126, 0.0, 1e-30, 1.0, 3e36,
                        3.4e38], np.float32)
    ks, k = w.ks, w.k
    pick = rng.integers(0, len(special), ks.shape)
    on = rng.random(ks.shape) < 0.5
    ks[on] = special[pick[on]]
    edge = np.array([-128, -127, 0, 127], np.int8)
    kon = rng.random(k.shape) < 0.1
    k[kon] = edge[rng.integers(0, 4, k.shape)[kon]]
    zero = ks == 0
    k[zero] = np.abs(k[zero].astype(np.int16)).clip(0, 127).astype(np.int8)
    meta, n_meta = inputs.quest_meta_table(lens, bs, seed=77)
    mx, mn, err = run(w, meta, n_meta)
    rx, rn = oracle.quest_metadata(oracle_cache(w), meta, n_meta)
    assert err == 0
    assert np.isinf(rx).any() and (np.abs(rx[rx != 0]) < 1.1754944e-38).any()  # both edges hit
    for got, ref, name in ((mx, rx, "max"), (mn, rn, "min")):
        bad = np.argwhere(got.view(np.uint32) != ref.view(np.uint32))
        assert bad.size == 0, f"{name}: {len(bad)} mismatches, first {bad[0].tolist()}"
