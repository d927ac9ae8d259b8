"""The decode kernel's int32 block dot products (its own TMA staging and int8 tensor-core
fragments, dumped through q8kv_debug_block_dots) equal the oracle's bit for bit."""
import numpy as np
import pytest
import torch

import decode_attention_int8_b200 as q8
import oracle
from decode_attention_int8_b200 import inputs
from gpu_util import assert_close, oracle_cache, to_device

pytestmark = pytest.mark.gpu

SHAPES = [
    # B, Hq, Hk, block, seq_lens
    (1, 8, 8, 16, [256]),
    (3, 32, 8, 64, [1, 65, 200]),
    (2, 32, 4, 128, [300, 129]),
    (4, 16, 1, 16, [17, 1, 48, 33]),
    (2, 64, 8, 128, [130, 5]),
    (2, 32, 2, 32, [95, 64]),
    (2, 64, 16, 64, [70, 3]),
    (2, 128, 8, 16, [40, 21]),  # group 16: two head rows per quad
    (1, 64, 2, 64, [77]),  # group 32: two head slices
]


@pytest.mark.parametrize("B,Hq,Hk,bs,lens", SHAPES)
def test_block_dots_bit_exact(B, Hq, Hk, bs, lens):
    w = inputs.make_custom(B, Hq, Hk, 128, lens, bs, seed=B * 100 + Hq + Hk + bs,
                           k_dist="student_t3")
    d = to_device(w)
    max_len = w.max_blocks_per_seq * bs
    dots = torch.full((B, Hq, max_len, 4), -(2 ** 31), dtype=torch.int32, device="cuda")
    out = torch.empty(d["q"].shape, dtype=torch.float32, device="cuda")
    q8.q8kv_debug_block_dots(dots, out, d["q"], d["k"], d["v"], d["ks"], d["vs"], d["bt"],
                             d["lens"], w.scale)
    torch.cuda.synchronize()
    got = dots.cpu().numpy()
    c = oracle_cache(w)
    for b in range(B):
        L = int(w.seq_lens[b])
        for h in range(Hq):
            ref = oracle.block_dots(c, w.q, b, h)
            np.testing.assert_array_equal(got[b, h, :L], ref, err_msg=f"b={b} h={h}")
            assert np.all(got[b, h, L:] == -(2 ** 31)), "wrote past seq_len"
    # the dumping instantiation computes the same attention output
    assert_close(out.cpu().numpy(), oracle.decode_all(c, w.q), "debug-instantiation output")
