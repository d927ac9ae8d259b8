"""Pins of the oracle's Q quantisation (Kestrel-LLM walk-through, section 2 part 1).

The expected codes and scales are hand-derived (tests/golden/qquant_cases.txt); the
random-data checks compare against closed-form properties of the rule, not against a
second copy of it.
"""
import numpy as np
import pytest

import oracle
from conftest import load_golden_qquant


@pytest.mark.parametrize("case", load_golden_qquant(), ids=lambda c: c["name"])
def test_golden_blocks(case):
    qi, qsc = oracle.quantize_q(case["q"])
    np.testing.assert_array_equal(qi, case["codes"])
    if case["qsc_bits"] is not None:
        assert int(qsc.view(np.uint32)[0]) == case["qsc_bits"]
    else:
        ref = np.float32(np.max(np.abs(case["q"]))) / np.float32(127.0)
        assert abs(int(qsc.view(np.int32)[0]) - int(ref.view(np.int32))) <= 2


def test_blocks_are_independent():
    cases = load_golden_qquant()
    q = np.concatenate([c["q"] for c in cases])
    qi, qsc = oracle.quantize_q(q)
    for i, c in enumerate(cases):
        np.testing.assert_array_equal(qi[32 * i:32 * i + 32], c["codes"])
    # reversing the block order reverses the result, block for block
    qr = np.concatenate([c["q"] for c in reversed(cases)])
    qi_r, qsc_r = oracle.quantize_q(qr)
    np.testing.assert_array_equal(qi_r.reshape(-1, 32), qi.reshape(-1, 32)[::-1])
    np.testing.assert_array_equal(qsc_r, qsc[::-1])


def test_random_block_properties():
    rng = np.random.default_rng(123)
    q = (rng.standard_normal(32 * 4096) * rng.choice([1e-3, 1.0, 50.0], 32 * 4096)).astype(
        np.float32)
    qi, qsc = oracle.quantize_q(q)
    blocks = q.reshape(-1, 32)
    codes = qi.reshape(-1, 32).astype(np.int64)
    # the largest magnitude of every non-degenerate block maps to +-127
    amax_idx = np.argmax(np.abs(blocks), axis=1)
    top = codes[np.arange(len(codes)), amax_idx]
    assert np.all(np.abs(top) == 127)
    # codes never leave [-127, 127] and keep the sign of their input
    assert codes.min() >= -127 and codes.max() <= 127
    assert np.all(np.sign(codes) * np.sign(blocks) >= 0)
    # dequantised values are within half a code step (plus fp32 slack) of the input
    deq = codes * qsc[:, None].astype(np.float64)
    err = np.abs(deq - blocks.astype(np.float64))
    assert np.all(err <= 0.5 * qsc[:, None] * (1 + 1e-5) + 1e-30)
    # the scale is max|q| / 127 to within an fp32 rounding
    rel = qsc / (np.abs(blocks).max(1) / 127.0) - 1.0
    assert np.all(np.abs(rel) < 2e-7)


def test_scale_equivariance_by_powers_of_two():
    # scaling a block by 2^k scales qsc by 2^k and leaves the codes unchanged
    rng = np.random.default_rng(7)
    q = rng.standard_normal(32 * 64).astype(np.float32)
    qi, qsc = oracle.quantize_q(q)
    for k in (-10, -3, 5, 40):
        qi2, qsc2 = oracle.quantize_q(q * np.float32(2.0 ** k))
        np.testing.assert_array_equal(qi2, qi)
        np.testing.assert_array_equal(qsc2, qsc * np.float32(2.0 ** k))


def test_rejects_bad_input():
    with pytest.raises(oracle.OracleError):
        oracle.quantize_q(np.zeros(31, np.float32))
    bad = np.zeros(32, np.float32)
    bad[3] = np.nan
    with pytest.raises(oracle.OracleError):
        oracle.quantize_q(bad)
