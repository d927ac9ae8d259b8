"""Host logic of bench.py that needs no GPU: both arms describe a workload with the same
config dict, the L2 policy follows the pool size, and the sampled-row parity report
compares against the oracle row by row."""
import json
import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402
import oracle  # noqa: E402
from decode_attention_int8_b200 import inputs  # noqa: E402


def test_pool_copies_exceed_four_times_l2():
    L2 = bench.L2_BYTES
    assert bench.n_pool_copies(4 * L2) == 1
    assert bench.n_pool_copies(5 * 10 ** 9) == 1
    n = bench.n_pool_copies(139 * 10 ** 6)
    assert n * 139 * 10 ** 6 > 4 * L2 and n <= 64
    assert bench.n_pool_copies(549_000) == 0  # too small to rotate: flushed instead


def test_reference_arm_prints_the_same_config_as_ours(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("WORLD_SIZE", "1")

    class Args:
        config = 0
        steps = 2
        warmup = 1
        gpus = 1

    assert bench.run_reference(Args()) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    w = inputs.make(0)
    assert line["config"] == json.loads(json.dumps(bench.workload_config(w, 1)))
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0


def test_default_workload_is_the_largest():
    cfgs = inputs.WORKLOADS
    units = [int(inputs._seq_lens(c).astype(np.int64).sum()) * c.n_kv_heads for c in cfgs]
    big = int(np.argmax(units))
    assert bench.DEFAULT_WORKLOAD == big == 4


def test_parity_rows_compares_against_the_oracle():
    w = inputs.make_custom(6, 16, 4, 128, [40, 1, 300, 0, 77, 129], 16, seed=3)
    cache = oracle.PagedCache(w.k, w.v, w.ks, w.vs, w.block_table, w.seq_lens, 16, w.scale)
    exact = oracle.decode_all(cache, w.q).astype(np.float32)
    r = bench.parity_rows(w, exact, 200, seed=0)  # every row
    assert r["rows"] == r["of_rows"] == 96 and r["within_tolerance"]
    r = bench.parity_rows(w, exact, 8, seed=1)  # sampled rows
    assert r["rows"] < 96 and r["within_tolerance"]
    bad = exact.copy()
    bad[:, :, 5] += 1e-3  # one channel of every row off by 1e-3
    r = bench.parity_rows(w, bad, 8, seed=1)
    assert not r["within_tolerance"] and r["max_abs"] == pytest.approx(1e-3, rel=1e-3)


def test_sampled_pairs_include_the_extremes():
    w = inputs.make_custom(5, 8, 2, 128, [10, 0, 500, 3, 40], 16, seed=2)
    pairs = bench.sample_pairs(w, 4, seed=0)
    assert all(w.seq_lens[b] > 0 for b, _ in pairs)
    assert (2, 0) in pairs and (2, 7) in pairs  # longest
    assert (3, 0) in pairs and (3, 7) in pairs  # shortest non-empty
