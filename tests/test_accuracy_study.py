"""Host side of the q8-vs-fp32 accuracy study (bench.py --accuracy-study): the fp32 rows
it regenerates are the ones the workload was quantised from, and its error figures are
consistent (with the oracle's own q8 output standing in for the CUDA output)."""
import numpy as np

import bench
import oracle
from decode_attention_int8_b200 import inputs


def test_regenerated_fp32_rows_are_the_quantised_ones():
    w = inputs.make_custom(2, 8, 2, 128, [5000, 300], 64, seed=3, keep_fp32=True,
                           k_bias_std=2.0, v_dist="student_t3")
    slots = np.array([0, 4095, 4096, 5100, 7, 5311])
    np.testing.assert_array_equal(inputs.fp32_rows(w, "k", slots),
                                  w.k32.reshape(-1, 2, 128)[slots])
    np.testing.assert_array_equal(inputs.fp32_rows(w, "v", slots),
                                  w.v32.reshape(-1, 2, 128)[slots])
    codes, scale = inputs.quantize_rows(inputs.fp32_rows(w, "k", slots))
    np.testing.assert_array_equal(codes, w.k.reshape(-1, 2, 128)[slots])
    np.testing.assert_array_equal(scale, w.ks.reshape(-1, 2)[slots])


def test_study_rows_with_the_oracle_standing_in():
    w = inputs.make_custom(3, 8, 2, 128, [500, 37, 0], 16, seed=4)
    cache = oracle.PagedCache(w.k, w.v, w.ks, w.vs, w.block_table, w.seq_lens, 8, w.scale)
    out = oracle.decode_all(cache, w.q).astype(np.float32)
    r = bench.accuracy_rows(w, out, 40, seed=0)
    assert r["rows"] > 0
    assert r["cuda_vs_oracle_q8_max_abs"] < 1e-6  # only the fp32 rounding of the stand-in
    a, b = r["cuda_q8_vs_fp32"], r["oracle_q8_vs_fp32"]
    for key in ("max_abs", "mean_abs", "rel_l2"):
        assert abs(a[key] - b[key]) <= 1e-6 * max(1.0, b[key])
    # int8 K and V with per-row scales and an int8 query: about 1 % relative error on
    # N(0, 1) data, far from both exactness and garbage
    assert 1e-3 < b["rel_l2"] < 5e-2
