"""The decode kernel's bounded pipeline waits, made to run out on purpose.

q8kv_debug_stall_pipeline injects one fault: the producer warp of one CTA never fills the
stage of its second tile (no arrive, no copy in flight). That CTA's consumer warps then wait
for a phase that never completes; after the given limit they set the time-out bit, skip the
rest of their work and keep their barriers, and the producer, waiting for stages the
consumers never release, gives up the same way. The call must complete, report
Q8KV_DEVERR_TIMEOUT, leave every row that CTA does not contribute to equal to the normal
call's, and leave the context usable for the next call. Nothing here faults or waits
without a bound."""
import numpy as np
import pytest
import torch

import decode_attention_int8_b200 as q8
import oracle
from decode_attention_int8_b200 import inputs
from gpu_util import assert_close, oracle_cache, run_decode, to_device

pytestmark = pytest.mark.gpu


def stalled(w, d, cta, limit_ns=100_000):
    out = torch.full(d["q"].shape, float("nan"), dtype=torch.float32, device="cuda")
    q8.q8kv_debug_stall_pipeline(out, d["q"], d["k"], d["v"], d["ks"], d["vs"], d["bt"],
                                 d["lens"], w.scale, stall_cta=cta, limit_ns=limit_ns)
    torch.cuda.synchronize()
    return out.cpu().numpy()


@pytest.mark.parametrize("Hq,first", [(32, True), (32, False), (64, True)])
def test_stalled_cta_times_out_and_the_rest_is_untouched(Hq, first):
    # 4 equal sequences of 8192 tokens: each CTA's share of the tiles lies inside one
    # sequence, so the first CTA touches only sequence 0 and the last only sequence 3
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    w = inputs.make_custom(4, Hq, 8, 128, [8192] * 4, 64, seed=31 + Hq)
    d = to_device(w)
    q8.q8kv_device_errors(clear=True)
    ref = run_decode(w, d).cpu().numpy()
    assert q8.q8kv_device_errors(clear=True) == 0
    cta = 0 if first else sms - 1
    got = stalled(w, d, cta)
    assert q8.q8kv_device_errors(clear=True) & q8.DEVERR_TIMEOUT
    keep = [1, 2, 3] if first else [0, 1, 2]
    np.testing.assert_array_equal(got[keep], ref[keep])
    cache = oracle_cache(w)
    pairs = [(b, h) for b in keep for h in (0, Hq // 2, Hq - 1)]
    assert_close(np.stack([got[b, h] for b, h in pairs]), oracle.decode_pairs(cache, w.q, pairs),
                 "rows outside the stalled CTA")
    # the context is still usable: the next normal call is clean and equal to the first
    again = run_decode(w, d).cpu().numpy()
    assert q8.q8kv_device_errors(clear=True) == 0
    np.testing.assert_array_equal(again, ref)


def test_stall_past_the_grid_injects_nothing():
    w = inputs.make_custom(2, 16, 4, 128, [3000, 700], 32, seed=33)
    d = to_device(w)
    q8.q8kv_device_errors(clear=True)
    ref = run_decode(w, d).cpu().numpy()
    got = stalled(w, d, 1 << 20)
    assert q8.q8kv_device_errors(clear=True) == 0
    np.testing.assert_array_equal(got, ref)


def test_limit_out_of_range_is_rejected_before_launch():
    w = inputs.make_custom(1, 8, 2, 128, [10], 16, seed=1)
    d = to_device(w)
    for cta, lim in [(-1, 100_000), (0, 10), (0, 2_000_000_000)]:
        with pytest.raises(q8.Q8KVError) as e:
            stalled(w, d, cta, lim)
        assert e.value.status == 1
