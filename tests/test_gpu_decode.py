"""Decode-attention output of the CUDA library against the fp64 oracle.

Tolerance (fixed by the method's statement of work): max |gpu - oracle| <= 1e-4 and
||gpu - oracle||_2 / ||oracle||_2 <= 1e-5 over the output tensor.
"""
import math

import numpy as np
import pytest
import torch

import decode_attention_int8_b200 as q8
import oracle
from decode_attention_int8_b200 import inputs
from gpu_util import assert_close, oracle_cache, run_decode, to_device, without_block

pytestmark = pytest.mark.gpu


def check_full(w, what):
    got = run_decode(w).cpu().numpy()
    ref = oracle.decode_all(oracle_cache(w), w.q)
    return assert_close(got, ref, what)


# ------------------------------------------------------------------ edge grid

@pytest.mark.parametrize("bs", [16, 32, 64, 128])
@pytest.mark.parametrize("G", [1, 2, 4, 8, 16])
def test_edge_lengths(bs, G):
    Hk = 8 if G <= 4 else 4
    lens = [1, 2, bs - 1, bs, bs + 1, 2 * bs - 1, 15, 16, 17, 31, 33, 129]
    w = inputs.make_custom(len(lens), Hk * G, Hk, 128, lens, bs, seed=bs + G)
    check_full(w, f"bs={bs} G={G}")


@pytest.mark.parametrize("Hk", [1, 2, 4, 8, 12, 16, 32])
def test_kv_head_counts(Hk):
    lens = [7, 100, 257, 1]
    w = inputs.make_custom(len(lens), Hk * 4, Hk, 128, lens, 32, seed=Hk, k_dist="student_t3",
                           v_dist="student_t3")
    check_full(w, f"Hk={Hk}")


@pytest.mark.parametrize("G", [24, 32, 48, 64])
def test_large_groups(G):
    lens = [50, 300]
    w = inputs.make_custom(2, 2 * G, 2, 128, lens, 64, seed=G)
    check_full(w, f"G={G}")


@pytest.mark.parametrize("G,Hk", [(64, 8), (48, 4), (128, 4), (40, 12)])
def test_tiles_narrower_than_the_scale_box(G, Hk):
    # tiles of 1 or 2 KV heads out of 4+: the scales come in the aligned 4-head box around
    # the tile's heads, and the tile's column in it changes from one head chunk to the next
    lens = [77, 300, 1]
    w = inputs.make_custom(3, Hk * G, Hk, 128, lens, 32, seed=G + Hk)
    check_full(w, f"G={G} Hk={Hk}")


@pytest.mark.parametrize("B,Hq,Hk,ragged", [
    (16, 32, 8, False),  # the benchmark's head layout with shorter sequences
    (16, 32, 8, True),
    (30, 16, 4, False),  # about one sequence per SM
    (37, 8, 4, True),
    (9, 144, 16, False), # group 9 (two 8-row query tiles), 16 KV heads
])
def test_batches_near_the_sm_count(B, Hq, Hk, ragged):
    rng = np.random.default_rng(B + Hk)
    lens = (rng.integers(1, 3000, B) if ragged else np.full(B, 1500)).tolist()
    w = inputs.make_custom(B, Hq, Hk, 128, lens, 64, seed=B * Hk)
    check_full(w, f"B={B} Hq={Hq} Hk={Hk} ragged={ragged}")


def test_zero_query_blocks_and_identity_table():
    w = inputs.make_custom(3, 16, 4, 128, [40, 64, 9], 16, table="identity", seed=5)
    w.q[0, :, :32] = 0.0  # whole quant block zero
    w.q[1, 3, :] = 0.0  # whole head zero
    w.q[2, :, 64:96] = 5e-7  # block below the guard
    check_full(w, "zero blocks")


def test_zero_length_sequences_give_zero_rows():
    w = inputs.make_custom(4, 8, 2, 128, [0, 33, 0, 5], 16, seed=3)
    got = run_decode(w).cpu().numpy()
    assert np.all(got[0] == 0) and np.all(got[2] == 0)
    assert_close(got, oracle.decode_all(oracle_cache(w), w.q), "zero-length rows")


def test_all_sequences_empty():
    w = inputs.make_custom(3, 8, 2, 128, [0, 0, 0], 16, seed=4, max_blocks_per_seq=2)
    got = run_decode(w).cpu().numpy()
    assert np.all(got == 0)


def test_wide_score_range_and_outliers():
    w = inputs.make_custom(2, 32, 4, 128, [3000, 777], 128, k_bias_std=6.0, seed=8,
                           k_dist="student_t3", v_dist="student_t3")
    check_full(w, "bias 6 + t3")


def test_tiny_and_huge_v_scales():
    w = inputs.make_custom(2, 16, 2, 128, [500, 64], 32, seed=9)
    rng = np.random.default_rng(0)
    w.vs *= (10.0 ** rng.uniform(-30, 30, w.vs.shape)).astype(np.float32)
    w.ks *= (10.0 ** rng.uniform(-2, 1, w.ks.shape)).astype(np.float32)
    got = run_decode(w).cpu().numpy()
    ref = oracle.decode_all(oracle_cache(w), w.q)
    # tolerance relative to each row's magnitude (the rows span 60 decades)
    for b in range(2):
        for h in range(16):
            r = ref[b, h]
            nrm = np.linalg.norm(r)
            assert np.linalg.norm(got[b, h] - r) <= 1e-5 * nrm + 1e-30


def test_long_sequence_many_ctas():
    # one sequence spread over every SM: exercises the two-level combine
    w = inputs.make_custom(1, 32, 8, 128, [40000], 64, seed=10)
    check_full(w, "L=40000 B=1")


def test_many_short_sequences():
    rng = np.random.default_rng(11)
    lens = rng.integers(1, 40, 700)
    w = inputs.make_custom(len(lens), 16, 4, 128, lens, 16, seed=11)
    check_full(w, "700 short")


@pytest.mark.parametrize("B", [2049, 3000])
def test_batches_past_the_charged_split(B):
    # above 2048 sequences the work split charges no segment starts and the sequence
    # counts are not kept; both the decode kernel and the combine kernel (which recomputes
    # the split) take that path. Every 7th sequence is long enough to be split over CTAs,
    # some are empty.
    rng = np.random.default_rng(B)
    lens = rng.integers(0, 60, B)
    lens[::7] = rng.integers(800, 2500, len(lens[::7]))
    w = inputs.make_custom(B, 8, 2, 128, lens, 32, seed=B)
    got = run_decode(w).cpu().numpy()
    assert np.all(got[lens == 0] == 0)
    assert_close(got, oracle.decode_all(oracle_cache(w), w.q), f"B={B}")


def test_batch_limit_is_rejected_on_host():
    w = inputs.make_custom(16385, 8, 2, 128, np.ones(16385, np.int64), 16, seed=2)
    with pytest.raises(q8.Q8KVError) as e:
        run_decode(w)
    assert e.value.status == 2


# ------------------------------------------------------------------ API behaviour

def test_repeat_calls_identical_and_workspace_variant():
    w = inputs.make_custom(5, 32, 8, 128, [1000, 1, 4096, 300, 2500], 64, seed=12)
    d = to_device(w)
    a = run_decode(w, d).clone()
    b = run_decode(w, d).clone()
    assert torch.equal(a, b), "counters or workspace not reset between calls"
    nbytes = q8.q8kv_workspace_bytes(5, 32, 8, 128)
    assert nbytes > 0
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    q8.q8kv_workspace_init(ws)
    for _ in range(2):
        out = torch.empty_like(a)
        q8.q8kv_decode_attn_ws(out, d["q"], d["k"], d["v"], d["ks"], d["vs"], d["bt"], d["lens"],
                               w.scale, ws)
        torch.cuda.synchronize()
        assert torch.equal(out, a)
    small = torch.zeros(nbytes // 2, dtype=torch.uint8, device="cuda")
    with pytest.raises(q8.Q8KVError) as e:
        q8.q8kv_decode_attn_ws(torch.empty_like(a), d["q"], d["k"], d["v"], d["ks"], d["vs"],
                               d["bt"], d["lens"], w.scale, small)
    assert e.value.status == 4


def test_non_default_stream():
    w = inputs.make_custom(2, 16, 4, 128, [900, 33], 32, seed=13)
    d = to_device(w)
    s = torch.cuda.Stream()
    out = torch.empty(d["q"].shape, dtype=torch.float32, device="cuda")
    torch.cuda.synchronize()
    with torch.cuda.stream(s):
        q8.q8kv_decode_attn(out, d["q"], d["k"], d["v"], d["ks"], d["vs"], d["bt"], d["lens"],
                            w.scale)
    s.synchronize()
    assert_close(out.cpu().numpy(), oracle.decode_all(oracle_cache(w), w.q), "side stream")


def test_unsupported_shapes_rejected_on_host():
    w = inputs.make_custom(1, 8, 2, 64, [10], 16, seed=1)  # head_dim 64
    d = to_device(w)
    with pytest.raises(q8.Q8KVError) as e:
        run_decode(w, d)
    assert e.value.status == 2
    w = inputs.make_custom(1, 8, 2, 128, [10], 48, seed=1)  # block size not a power of two
    with pytest.raises(q8.Q8KVError) as e:
        run_decode(w)
    assert e.value.status == 2


def test_device_side_checks_flag_bad_tables_without_faulting():
    w = inputs.make_custom(3, 8, 2, 128, [40, 70, 16], 16, seed=14, extra_blocks=2)
    q8.q8kv_device_errors(clear=True)
    ref_ok = run_decode(w).cpu().numpy()
    assert q8.q8kv_device_errors(clear=True) == 0
    # an entry past the pool: that block's tokens are skipped, the flag is raised
    bad = inputs.make_custom(3, 8, 2, 128, [40, 70, 16], 16, seed=14, extra_blocks=2)
    entry = int(bad.block_table[1, 2])
    bad.block_table[1, 2] = bad.num_blocks + 5
    got = run_decode(bad).cpu().numpy()
    assert q8.q8kv_device_errors(clear=True) & q8.DEVERR_BLOCK_TABLE
    np.testing.assert_array_equal(got[0], ref_ok[0])
    np.testing.assert_array_equal(got[2], ref_ok[2])
    # row 1 is attention over the tokens of its other blocks
    bt, lens = without_block(bad.block_table, bad.seq_lens, 1, 2, 16)
    kept = oracle.PagedCache(bad.k, bad.v, bad.ks, bad.vs, bt, lens, 8, bad.scale)
    assert_close(got[1], oracle.decode_all(kept, bad.q)[1], "block skipped")
    # a negative entry, here in the sequence's last (partial) block
    bad.block_table[1, 2] = entry
    bad.block_table[1, 4] = -7
    got = run_decode(bad).cpu().numpy()
    assert q8.q8kv_device_errors(clear=True) & q8.DEVERR_BLOCK_TABLE
    bt, lens = without_block(bad.block_table, bad.seq_lens, 1, 4, 16)
    kept = oracle.PagedCache(bad.k, bad.v, bad.ks, bad.vs, bt, lens, 8, bad.scale)
    assert_close(got[1], oracle.decode_all(kept, bad.q)[1], "last block skipped")
    # seq_len above max_blocks_per_seq * block_size is clamped and flagged
    long = inputs.make_custom(3, 8, 2, 128, [40, 70, 16], 16, seed=14, extra_blocks=2)
    long.seq_lens[0] = long.max_blocks_per_seq * 16 + 100
    got = run_decode(long).cpu().numpy()
    assert q8.q8kv_device_errors(clear=True) & q8.DEVERR_SEQ_LEN
    clamped = inputs.make_custom(3, 8, 2, 128, [40, 70, 16], 16, seed=14, extra_blocks=2)
    clamped.seq_lens[0] = clamped.max_blocks_per_seq * 16
    clamped.block_table[0, :] = long.block_table[0, :]
    np.testing.assert_array_equal(got[0], run_decode(clamped).cpu().numpy()[0])
    # negative seq_len behaves as zero
    neg = inputs.make_custom(3, 8, 2, 128, [40, 70, 16], 16, seed=14, extra_blocks=2)
    neg.seq_lens[2] = -5
    got = run_decode(neg).cpu().numpy()
    assert q8.q8kv_device_errors(clear=True) & q8.DEVERR_SEQ_LEN
    assert np.all(got[2] == 0)


# ------------------------------------------------------------------ the five workloads

@pytest.mark.parametrize("idx", [0, 1, 2])
def test_workload_full_parity(idx):
    w = inputs.make(idx)
    max_abs, rel = check_full(w, inputs.WORKLOADS[idx].name)
    print(f"\n{inputs.WORKLOADS[idx].name}: max_abs={max_abs:.3e} rel_l2={rel:.3e}")


@pytest.mark.slow
@pytest.mark.parametrize("idx", [3, 4])
def test_workload_sampled_parity(idx):
    """Full-size runs; the oracle checks a sample of (sequence, head) rows."""
    w = inputs.make(idx)
    got = run_decode(w).cpu().numpy()
    assert np.all(np.isfinite(got))
    rng = np.random.default_rng(idx)
    B, Hq = w.cfg.B, w.cfg.n_q_heads
    pairs = [(int(b), int(h)) for b, h in zip(rng.integers(0, B, 96), rng.integers(0, Hq, 96))]
    # always include the longest and the shortest sequence
    for b in (int(np.argmax(w.seq_lens)), int(np.argmin(w.seq_lens))):
        pairs += [(b, 0), (b, Hq - 1)]
    ref = oracle.decode_pairs(oracle_cache(w), w.q, pairs)
    sel = np.stack([got[b, h] for b, h in pairs])
    max_abs, rel = assert_close(sel, ref, inputs.WORKLOADS[idx].name)
    print(f"\n{inputs.WORKLOADS[idx].name}: sampled {len(pairs)} rows max_abs={max_abs:.3e} "
          f"rel_l2={rel:.3e}")
