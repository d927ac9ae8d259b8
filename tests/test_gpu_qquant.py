"""GPU Q quantisation (the decode kernel's device routine, through q8kv_debug_quantize_q)
against the oracle and the hand-derived golden blocks: bit-exact codes and scales."""
import numpy as np
import pytest
import torch

import decode_attention_int8_b200 as q8
import oracle
from conftest import load_golden_qquant

pytestmark = pytest.mark.gpu


def gpu_quantize(q: np.ndarray):
    qd = torch.from_numpy(np.ascontiguousarray(q, np.float32)).cuda()
    qi = torch.empty(qd.shape, dtype=torch.int8, device="cuda")
    qsc = torch.empty(qd.shape[:-1] + (qd.shape[-1] // 32,), dtype=torch.float32, device="cuda")
    q8.q8kv_debug_quantize_q(qi, qsc, qd)
    torch.cuda.synchronize()
    return qi.cpu().numpy(), qsc.cpu().numpy()


def test_golden_blocks_bit_exact():
    cases = load_golden_qquant()
    q = np.concatenate([c["q"] for c in cases]).reshape(-1, 32)
    qi, qsc = gpu_quantize(q)
    for i, c in enumerate(cases):
        np.testing.assert_array_equal(qi[i], c["codes"], err_msg=c["name"])
        if c["qsc_bits"] is not None:
            assert int(qsc[i].view(np.uint32)[0]) == c["qsc_bits"], c["name"]


@pytest.mark.parametrize("D", [32, 128, 256])
def test_random_rows_match_oracle_bit_exact(D):
    rng = np.random.default_rng(D)
    n = 20000
    q = rng.standard_normal((n, D)).astype(np.float32)
    q *= rng.choice([1e-8, 1e-3, 1.0, 300.0], (n, 1)).astype(np.float32)
    q[::97] = 0.0  # all-zero rows
    q[5::101, :32] = np.float32(9e-7)  # blocks under the zero guard
    q[7::103, 3] = np.float32(1e-6)  # blocks exactly at the guard
    qi, qsc = gpu_quantize(q)
    ri, rs = oracle.quantize_q(q.reshape(-1))
    np.testing.assert_array_equal(qi.reshape(-1), ri)
    np.testing.assert_array_equal(qsc.reshape(-1).view(np.uint32), rs.view(np.uint32))


def test_ties_everywhere():
    # qm = 127 makes iq exactly 1: every half-integer input is a tie
    q = np.tile(np.arange(-126.5, 127.0, 1.0, dtype=np.float32), 4)[: 32 * 8].reshape(8, 32)
    q[:, 0] = 127.0
    qi, _ = gpu_quantize(q)
    ri, _ = oracle.quantize_q(q.reshape(-1))
    np.testing.assert_array_equal(qi.reshape(-1), ri)
