"""q8kv_decode_attn_static: the decode entry point whose scratch is a fixed device array
inside the library, so that a call allocates no device memory. It must give bit for bit
what q8kv_decode_attn gives (same plan, same kernel), call after call and across shapes,
and reject the shapes whose scratch would not fit before enqueueing anything.

The file name sorts last, so in a full run these calls come after every other test has
used the other entry points; the tests also pass when this file runs alone."""
import ctypes

import numpy as np
import pytest
import torch

import decode_attention_int8_b200 as q8
from decode_attention_int8_b200 import inputs

INVALID, UNSUPPORTED, WORKSPACE = 1, 2, 4


def _raw_static(**over):
    """The C entry point with fake (aligned, never dereferenced) pointers."""
    a = dict(out=0x10000, q=0x20000, k=0x30000, v=0x40000, ks=0x50000, vs=0x60000, bt=0x70000,
             lens=0x80000, B=2, Hq=8, Hk=2, D=128, bs=16, mbps=4, P=8, scale=0.088)
    a.update(over)
    P = lambda x: None if x is None else ctypes.c_void_p(x)
    return q8.lib().q8kv_decode_attn_static(P(a["out"]), P(a["q"]), P(a["k"]), P(a["v"]),
                                            P(a["ks"]), P(a["vs"]), P(a["bt"]), P(a["lens"]),
                                            a["B"], a["Hq"], a["Hk"], a["D"], a["bs"], a["mbps"],
                                            a["P"], a["scale"], None)


@pytest.mark.parametrize("over", [dict(out=None), dict(lens=None), dict(B=0), dict(Hq=9),
                                  dict(D=100), dict(scale=float("nan")), dict(k=0x30008)])
def test_bad_arguments_rejected_on_host(over):
    assert _raw_static(**over) == INVALID


def _device(w):
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    return dict(q=t(w.q), k=t(w.k), v=t(w.v), ks=t(w.ks), vs=t(w.vs), bt=t(w.block_table),
                lens=t(w.seq_lens))


def _args(d):
    return d["q"], d["k"], d["v"], d["ks"], d["vs"], d["bt"], d["lens"]


# Shapes with different tile head counts (so the partial-slot region is laid out
# differently from one call to the next) and ragged lengths that split across CTAs.
SHAPES = [
    dict(B=5, Hq=32, Hk=8, lens=[1000, 1, 4096, 300, 2500], bs=64, seed=41),
    dict(B=3, Hq=64, Hk=8, lens=[5000, 17, 1200], bs=128, seed=42),
    dict(B=2, Hq=8, Hk=8, lens=[3000, 64], bs=16, seed=43),
    dict(B=1, Hq=32, Hk=4, lens=[40000], bs=128, seed=44),
]


@pytest.mark.gpu
def test_two_calls_in_a_row_match_the_managed_entry_point():
    for sh in SHAPES:
        w = inputs.make_custom(sh["B"], sh["Hq"], sh["Hk"], 128, sh["lens"], sh["bs"],
                               seed=sh["seed"])
        d = _device(w)
        ref = torch.full(d["q"].shape, float("nan"), dtype=torch.float32, device="cuda")
        q8.q8kv_decode_attn(ref, *_args(d), w.scale)
        for call in range(2):
            out = torch.full_like(ref, float("nan"))
            q8.q8kv_decode_attn_static(out, *_args(d), w.scale)
            torch.cuda.synchronize()
            assert torch.equal(out, ref), f"{sh} call {call}: differs from q8kv_decode_attn"
    assert q8.q8kv_device_errors(clear=True) == 0


@pytest.mark.gpu
def test_calls_allocate_no_device_memory():
    w = inputs.make_custom(4, 32, 8, 128, [2048, 999, 1, 3000], 64, seed=45)
    d = _device(w)
    ref = torch.empty(d["q"].shape, dtype=torch.float32, device="cuda")
    q8.q8kv_decode_attn(ref, *_args(d), w.scale)  # loads the kernels' module
    outs = [torch.empty_like(ref) for _ in range(3)]
    torch.cuda.synchronize()
    free_before, _ = torch.cuda.mem_get_info()
    for out in outs:
        q8.q8kv_decode_attn_static(out, *_args(d), w.scale)
    torch.cuda.synchronize()
    free_after, _ = torch.cuda.mem_get_info()
    assert free_after == free_before
    for out in outs:
        assert torch.equal(out, ref)


@pytest.mark.gpu
@pytest.mark.parametrize("Hq,Hk", [(128, 8), (128, 1)])
def test_shapes_beyond_the_scratch_are_rejected(Hq, Hk):
    # 128 query heads per tile need about 20 MB of scratch on a 148-SM GPU (more than the
    # 12 MiB array); the managed and caller-workspace entry points still serve them.
    w = inputs.make_custom(1, Hq, Hk, 128, [100], 16, seed=46)
    need = q8.q8kv_workspace_bytes(1, Hq, Hk, 128)
    d = _device(w)
    out = torch.full(d["q"].shape, float("nan"), dtype=torch.float32, device="cuda")
    if need <= 12 * 1024 * 1024:
        pytest.skip(f"this device needs only {need} bytes for the shape")
    with pytest.raises(q8.Q8KVError) as e:
        q8.q8kv_decode_attn_static(out, *_args(d), w.scale)
    assert e.value.status == WORKSPACE
    torch.cuda.synchronize()
    assert torch.isnan(out).all(), "a rejected call must not write the output"
    ref = torch.empty_like(out)
    q8.q8kv_decode_attn(ref, *_args(d), w.scale)
    torch.cuda.synchronize()
    assert torch.isfinite(ref).all()


@pytest.mark.gpu
def test_unsupported_shape_rejected_like_the_managed_entry_point():
    w = inputs.make_custom(1, 8, 8, 128, [50], 16, seed=47)
    d = _device(w)
    out = torch.empty(d["q"].shape, dtype=torch.float32, device="cuda")
    P = lambda t: ctypes.c_void_p(t.data_ptr())
    args = (P(out), P(d["q"]), P(d["k"]), P(d["v"]), P(d["ks"]), P(d["vs"]), P(d["bt"]),
            P(d["lens"]), 1, 8, 8, 128, 24, 1, int(d["k"].shape[0]), ctypes.c_float(w.scale), None)
    assert q8.lib().q8kv_decode_attn_static(*args) == UNSUPPORTED  # block size not a power of 2
    assert q8.lib().q8kv_decode_attn(*args) == UNSUPPORTED
