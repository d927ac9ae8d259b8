"""The C-ABI library builds for sm_100a, loads without a GPU, exports every entry point
include/q8kv.h declares, and rejects bad arguments on the host before touching CUDA."""
import ctypes
import os
import re
import subprocess

import pytest

import decode_attention_int8_b200 as q8

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "q8kv.h")

OK, INVALID, UNSUPPORTED = 0, 1, 2


def declared_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(q8kv_\w+)\s*\(", text)))


def test_header_declares_the_binding_exports():
    assert declared_symbols() == sorted(q8.EXPORTS)


def test_library_exports_every_declared_symbol():
    L = q8.lib()
    out = subprocess.run(["nm", "-D", "--defined-only", q8.lib_path()], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (q8kv_\w+)", out))
    for name in declared_symbols():
        assert hasattr(L, name), name
        assert name in exported, name


def test_library_is_built_for_sm100a():
    from decode_attention_int8_b200 import build

    flags = " ".join(build.NVCC_FLAGS)
    assert "-gencode arch=compute_100a,code=sm_100a" in flags
    assert "compute_90" not in flags and "sm_90" not in flags


def test_status_strings_and_version():
    L = q8.lib()
    assert L.q8kv_status_string(0) == b"ok"
    assert L.q8kv_status_string(2) == b"unsupported shape"
    assert L.q8kv_status_string(99) == b"unknown status"
    assert L.q8kv_version() == 103


def _call(**over):
    """q8kv_decode_attn with fake (aligned, never dereferenced) pointers."""
    a = dict(out=0x10000, q=0x20000, k=0x30000, v=0x40000, ks=0x50000, vs=0x60000, bt=0x70000,
             lens=0x80000, B=2, Hq=8, Hk=2, D=128, bs=16, mbps=4, P=8, scale=0.088)
    a.update(over)
    P = lambda x: None if x is None else ctypes.c_void_p(x)
    return q8.lib().q8kv_decode_attn(P(a["out"]), P(a["q"]), P(a["k"]), P(a["v"]), P(a["ks"]),
                                     P(a["vs"]), P(a["bt"]), P(a["lens"]), a["B"], a["Hq"], a["Hk"],
                                     a["D"], a["bs"], a["mbps"], a["P"], a["scale"], None)


@pytest.mark.parametrize("field", ["out", "q", "k", "v", "ks", "vs", "bt", "lens"])
def test_null_pointer_rejected(field):
    assert _call(**{field: None}) == INVALID


@pytest.mark.parametrize("over", [dict(B=0), dict(B=-3), dict(Hq=0), dict(Hk=0), dict(Hq=9),
                                  dict(D=100), dict(bs=0), dict(mbps=0), dict(P=0),
                                  dict(scale=float("inf")), dict(scale=float("nan")),
                                  dict(q=0x20004), dict(k=0x30008), dict(out=0x10002)])
def test_bad_sizes_rejected(over):
    assert _call(**over) == INVALID


def test_workspace_bytes_of_invalid_shapes_is_zero():
    L = q8.lib()
    assert L.q8kv_workspace_bytes(0, 8, 2, 128) == 0
    assert L.q8kv_workspace_bytes(1, 9, 2, 128) == 0
    assert L.q8kv_workspace_bytes(1, 8, 2, 96) == 0  # head_dim other than 128
    assert L.q8kv_workspace_bytes(1, 1024, 4, 128) == 0  # group above 128


def test_debug_entry_points_reject_bad_arguments():
    L = q8.lib()
    P = ctypes.c_void_p
    assert L.q8kv_debug_quantize_q(None, P(0x1000), P(0x2000), 4, 128, None) == INVALID
    assert L.q8kv_debug_quantize_q(P(0x1000), P(0x1000), P(0x2000), 4, 100, None) == INVALID
    assert L.q8kv_debug_quantize_q(P(0x1000), P(0x1000), P(0x2000), 0, 128, None) == INVALID
    assert L.q8kv_debug_quantize_q(P(0x1000), P(0x1000), P(0x2004), 4, 128, None) == INVALID
    args = [P(0x10000 * i) for i in range(1, 9)] + [2, 8, 2, 128, 16, 4, 8, 0.1, None]
    assert L.q8kv_debug_block_dots(None, 64, *args) == INVALID
    assert L.q8kv_debug_block_dots(P(0x1000), 0, *args) == INVALID
    assert L.q8kv_debug_block_dots(P(0x1000), 63, *args) == INVALID  # < max_blocks * block_size
    assert L.q8kv_workspace_init(None, 16, None) == INVALID
    assert L.q8kv_device_errors(None, 0) == INVALID


def _write(**over):
    """q8kv_cache_write with fake (aligned, never dereferenced) pointers."""
    a = dict(k=0x10000, v=0x20000, ks=0x30000, vs=0x40000, kn=0x50000, vn=0x60000, sl=0x70000,
             n=4, Hk=2, D=128, bs=16, P=8, stride=0)
    a.update(over)
    P = lambda x: None if x is None else ctypes.c_void_p(x)
    return q8.lib().q8kv_cache_write(P(a["k"]), P(a["v"]), P(a["ks"]), P(a["vs"]), P(a["kn"]),
                                     P(a["vn"]), P(a["sl"]), a["n"], a["Hk"], a["D"], a["bs"],
                                     a["P"], a["stride"], None)


@pytest.mark.parametrize("field", ["k", "v", "ks", "vs", "kn", "vn", "sl"])
def test_cache_write_null_pointer_rejected(field):
    assert _write(**{field: None}) == INVALID


@pytest.mark.parametrize("over", [dict(n=-1), dict(Hk=0), dict(D=0), dict(D=100), dict(bs=0),
                                  dict(P=0), dict(stride=255), dict(stride=258), dict(kn=0x50004),
                                  dict(vn=0x60008), dict(k=0x10001), dict(ks=0x30002),
                                  dict(sl=0x70004)])
def test_cache_write_bad_arguments_rejected(over):
    assert _write(**over) == INVALID


@pytest.mark.parametrize("D", [32, 96, 160, 512])
def test_cache_write_unsupported_head_dim(D):
    assert _write(D=D) == UNSUPPORTED


def test_cache_write_of_no_tokens_enqueues_nothing():
    # returns before any CUDA call, so it succeeds even without a GPU; the row pointers of
    # an empty call may be null (an empty torch tensor has none)
    assert _write(n=0) == OK
    assert _write(n=0, kn=None, vn=None, sl=None) == OK
    assert _write(n=0, k=None) == INVALID


def test_quest_metadata_bad_arguments_rejected():
    L = q8.lib()
    P = ctypes.c_void_p
    ptrs = [P(0x10000 * i) for i in range(1, 8)]
    sizes = [2, 8, 128, 16, 4, 1, 8, 2]  # B, Hk, D, bs, mbps, mmbpr, num_blocks, num_meta
    for i in range(7):
        bad = list(ptrs)
        bad[i] = None
        assert L.q8kv_quest_metadata(*bad, *sizes, None) == INVALID
    for i in range(8):
        bad = list(sizes)
        bad[i] = 0
        assert L.q8kv_quest_metadata(*ptrs, *bad, None) == INVALID
    assert L.q8kv_quest_metadata(P(0x10004), *ptrs[1:], *sizes, None) == INVALID  # alignment
    odd = list(sizes)
    odd[2] = 64
    assert L.q8kv_quest_metadata(*ptrs, *odd, None) == UNSUPPORTED
    for i in (4, 5, 6, 7):  # a table or pool of 2^31 tokens or more (bs 16 x 2^27 entries)
        big = list(sizes)
        big[i] = 1 << 27
        assert L.q8kv_quest_metadata(*ptrs, *big, None) == UNSUPPORTED


def test_q4_decode_bad_arguments_rejected():
    L = q8.lib()
    P = ctypes.c_void_p
    ptrs = [P(0x10000 * i) for i in range(1, 9)]
    sizes = [2, 8, 2, 128, 16, 4, 8]  # B, Hq, Hk, D, bs, mbps, P
    for i in range(8):
        bad = list(ptrs)
        bad[i] = None
        assert L.q8kv_decode_attn_q4(*bad, *sizes, 0.1, None) == INVALID
    for i in range(7):
        bad = list(sizes)
        bad[i] = 0
        assert L.q8kv_decode_attn_q4(*ptrs, *bad, 0.1, None) == INVALID
    assert L.q8kv_decode_attn_q4(*ptrs, 2, 9, 2, 128, 16, 4, 8, 0.1, None) == INVALID
    assert L.q8kv_decode_attn_q4(*ptrs, *sizes, float("nan"), None) == INVALID
    odd = list(ptrs)
    odd[4] = P(0x50004)  # kd not 8-byte aligned
    assert L.q8kv_decode_attn_q4(*odd, *sizes, 0.1, None) == INVALID
    assert L.q8kv_decode_attn_q4(*ptrs, 2, 8, 2, 64, 16, 4, 8, 0.1, None) == UNSUPPORTED
    assert L.q8kv_decode_attn_q4(*ptrs, 2, 34, 2, 128, 16, 4, 8, 0.1, None) == UNSUPPORTED
