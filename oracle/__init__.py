"""CPU oracle for q8-KV single-query decode attention (test infrastructure only).

Only the test suite, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg
may import this package. The CUDA library never loads it and shares no code with it.

The arithmetic lives in ``q8kv_oracle.c`` (plain C, single-threaded, fp32 for the Q
quantisation that decides integers, fp64 for everything after the int32 dots). This
module compiles it on demand with gcc and wraps it with ctypes over numpy arrays.
See ``q8kv_oracle.h`` for the citations of each step.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "q8kv_oracle.c")
_HDR = os.path.join(_HERE, "q8kv_oracle.h")
_LIB = os.path.join(_HERE, "libq8kv_oracle.so")
CFLAGS = ["-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared", "-std=c11"]

_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/libq8kv_oracle.so`` (gcc, a second or two)."""
    newest_src = max(os.path.getmtime(_SRC), os.path.getmtime(_HDR))
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < newest_src:
        tmp = _LIB + ".tmp.%d" % os.getpid()
        subprocess.check_call(["gcc", *CFLAGS, _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class Cache(ctypes.Structure):
    """Mirror of ``q8kvo_cache``."""

    _fields_ = [
        ("k", ctypes.c_void_p),
        ("v", ctypes.c_void_p),
        ("ks", ctypes.c_void_p),
        ("vs", ctypes.c_void_p),
        ("block_table", ctypes.c_void_p),
        ("seq_lens", ctypes.c_void_p),
        ("B", ctypes.c_int),
        ("n_q_heads", ctypes.c_int),
        ("n_kv_heads", ctypes.c_int),
        ("head_dim", ctypes.c_int),
        ("block_size", ctypes.c_int),
        ("max_blocks_per_seq", ctypes.c_int),
        ("num_blocks", ctypes.c_int),
        ("scale", ctypes.c_float),
    ]


class CacheQ4(ctypes.Structure):
    """Mirror of ``q8kvo_cache_q4``."""

    _fields_ = [
        ("k4", ctypes.c_void_p),
        ("v4", ctypes.c_void_p),
        ("kd", ctypes.c_void_p),
        ("vd", ctypes.c_void_p),
        ("block_table", ctypes.c_void_p),
        ("seq_lens", ctypes.c_void_p),
        ("B", ctypes.c_int),
        ("n_q_heads", ctypes.c_int),
        ("n_kv_heads", ctypes.c_int),
        ("head_dim", ctypes.c_int),
        ("block_size", ctypes.c_int),
        ("max_blocks_per_seq", ctypes.c_int),
        ("num_blocks", ctypes.c_int),
        ("scale", ctypes.c_float),
    ]


def build_variant(mutant: int, out_path: str) -> str:
    """Compile the oracle with planted mistake ``mutant`` switched on (pin-strength test)."""
    subprocess.check_call(["gcc", *CFLAGS, f"-DQ8KVO_MUTANT={int(mutant)}", _SRC, "-o", out_path,
                           "-lm"])
    return out_path


def _load():
    global _lib
    with _lock:
        if _lib is None:
            # Q8KV_ORACLE_LIB selects a prebuilt variant (only the planted-mistake test sets it)
            lib = ctypes.CDLL(os.environ.get("Q8KV_ORACLE_LIB") or build())
            P = ctypes.c_void_p
            i, l = ctypes.c_int, ctypes.c_long
            cp = ctypes.POINTER(Cache)
            sigs = {
                "q8kvo_quantize_q": [P, l, P, P],
                "q8kvo_block_dots": [cp, P, i, i, P],
                "q8kvo_scores": [cp, P, i, i, P],
                "q8kvo_decode_online": [cp, P, i, i, P, P, P],
                "q8kvo_decode_threepass": [cp, P, i, i, P],
                "q8kvo_decode_all": [cp, P, P],
                "q8kvo_decode_pairs": [cp, P, P, l, P],
                "q8kvo_attn_fp32": [cp, P, P, P, i, i, P],
                "q8kvo_quantize_kv_row": [P, i, P, P, P],
                "q8kvo_decode_multi": [cp, P, i, P],
                "q8kvo_decode_multi_rows": [cp, P, i, P, l, P],
                "q8kvo_quest_metadata": [cp, P, i, i, P, P],
                "q8kvo_f32_to_f16": [P, l, P],
                "q8kvo_quantize_q4_0": [P, l, P, P],
                "q8kvo_decode_q4_all": [ctypes.POINTER(CacheQ4), P, P],
                "q8kvo_decode_q4_pairs": [ctypes.POINTER(CacheQ4), P, P, l, P],
                "q8kvo_cache_write": [P, P, P, P, P, P, P, l, i, i, i, i, l, P],
                "q8kvo_cache_write_q4": [P, P, P, P, P, P, P, l, i, i, i, i, l, P],
            }
            for name, args in sigs.items():
                fn = getattr(lib, name)
                fn.argtypes = args
                fn.restype = ctypes.c_int
            _lib = lib
    return _lib


class OracleError(RuntimeError):
    pass


FLAG_SLOT = 0x8
FLAG_NONFINITE = 0x10


def _ptr(a: np.ndarray | None):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _check(rc: int, what: str):
    if rc != 0:
        raise OracleError(f"{what} failed with oracle code {rc}")


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


class PagedCache:
    """Host-side paged q8 KV cache handed to the oracle (keeps the arrays alive)."""

    def __init__(self, k, v, ks, vs, block_table, seq_lens, n_q_heads, scale):
        self.k = _c(k, np.int8)
        self.v = _c(v, np.int8)
        self.ks = _c(ks, np.float32)
        self.vs = _c(vs, np.float32)
        self.block_table = _c(block_table, np.int32)
        self.seq_lens = _c(seq_lens, np.int32)
        P, bs, Hk, D = self.k.shape
        self.struct = Cache(
            _ptr(self.k), _ptr(self.v), _ptr(self.ks), _ptr(self.vs),
            _ptr(self.block_table), _ptr(self.seq_lens),
            int(self.seq_lens.shape[0]), int(n_q_heads), int(Hk), int(D), int(bs),
            int(self.block_table.shape[1]), int(P), float(np.float32(scale)),
        )

    @property
    def head_dim(self):
        return self.struct.head_dim

    @property
    def n_q_heads(self):
        return self.struct.n_q_heads

    @property
    def B(self):
        return self.struct.B

    def ref(self):
        return ctypes.byref(self.struct)


def quantize_q(q: np.ndarray):
    """int8 codes and per-32-block fp32 scales of a flat fp32 vector (len % 32 == 0)."""
    q = _c(q, np.float32).reshape(-1)
    qi = np.empty(q.shape, np.int8)
    qsc = np.empty(q.shape[0] // 32, np.float32)
    _check(_load().q8kvo_quantize_q(_ptr(q), q.shape[0], _ptr(qi), _ptr(qsc)), "quantize_q")
    return qi, qsc


def block_dots(cache: PagedCache, q: np.ndarray, b: int, h: int) -> np.ndarray:
    q = _c(q, np.float32)
    L = int(cache.seq_lens[b])
    out = np.zeros((L, cache.head_dim // 32), np.int32)
    _check(_load().q8kvo_block_dots(cache.ref(), _ptr(q), b, h, _ptr(out)), "block_dots")
    return out


def scores(cache: PagedCache, q: np.ndarray, b: int, h: int) -> np.ndarray:
    q = _c(q, np.float32)
    out = np.zeros(int(cache.seq_lens[b]), np.float64)
    _check(_load().q8kvo_scores(cache.ref(), _ptr(q), b, h, _ptr(out)), "scores")
    return out


def decode_online(cache: PagedCache, q: np.ndarray, b: int, h: int, trace: bool = False):
    """fp64 output row of (b, h); with ``trace`` also the M trace and iteration count."""
    q = _c(q, np.float32)
    out = np.zeros(cache.head_dim, np.float64)
    L = int(cache.seq_lens[b])
    mt = np.zeros(L, np.float64) if trace else None
    n_iter = ctypes.c_long(-1)
    _check(
        _load().q8kvo_decode_online(cache.ref(), _ptr(q), b, h, _ptr(out), _ptr(mt),
                                    ctypes.byref(n_iter)),
        "decode_online",
    )
    return (out, mt, n_iter.value) if trace else out


def decode_threepass(cache: PagedCache, q: np.ndarray, b: int, h: int) -> np.ndarray:
    q = _c(q, np.float32)
    out = np.zeros(cache.head_dim, np.float64)
    _check(_load().q8kvo_decode_threepass(cache.ref(), _ptr(q), b, h, _ptr(out)), "threepass")
    return out


def decode_all(cache: PagedCache, q: np.ndarray) -> np.ndarray:
    """fp64 output [B][n_q_heads][head_dim] of every (b, h)."""
    q = _c(q, np.float32)
    out = np.zeros((cache.B, cache.n_q_heads, cache.head_dim), np.float64)
    _check(_load().q8kvo_decode_all(cache.ref(), _ptr(q), _ptr(out)), "decode_all")
    return out


def decode_pairs(cache: PagedCache, q: np.ndarray, pairs) -> np.ndarray:
    """fp64 outputs [n][head_dim] of the chosen (b, h) pairs."""
    q = _c(q, np.float32)
    pairs = _c(pairs, np.int32).reshape(-1, 2)
    out = np.zeros((pairs.shape[0], cache.head_dim), np.float64)
    _check(_load().q8kvo_decode_pairs(cache.ref(), _ptr(q), _ptr(pairs), pairs.shape[0],
                                      _ptr(out)), "decode_pairs")
    return out


def decode_multi(cache: PagedCache, q: np.ndarray, n_queries: int) -> np.ndarray:
    """fp64 output [B][n_queries][n_q_heads][head_dim] of a causal multi-query decode:
    q is [B][n_queries][n_q_heads][head_dim], query i sees seq_lens[b] - (n_queries - 1 - i)
    tokens."""
    q = _c(q, np.float32)
    out = np.zeros((cache.B, n_queries, cache.n_q_heads, cache.head_dim), np.float64)
    _check(_load().q8kvo_decode_multi(cache.ref(), _ptr(q), int(n_queries), _ptr(out)),
           "decode_multi")
    return out


def decode_multi_rows(cache: PagedCache, q: np.ndarray, n_queries: int, rows) -> np.ndarray:
    """fp64 outputs [n][head_dim] of chosen (b, query index, head) rows."""
    q = _c(q, np.float32)
    rows = _c(rows, np.int32).reshape(-1, 3)
    out = np.zeros((rows.shape[0], cache.head_dim), np.float64)
    _check(_load().q8kvo_decode_multi_rows(cache.ref(), _ptr(q), int(n_queries), _ptr(rows),
                                           rows.shape[0], _ptr(out)), "decode_multi_rows")
    return out


def quest_metadata(cache: PagedCache, meta_table: np.ndarray, num_meta_blocks: int,
                   fill: float = np.nan):
    """(maxb, minb) fp32 [num_meta_blocks][block_size][n_kv_heads][head_dim] of the q8
    cache's K (rows no request owns keep ``fill``)."""
    meta_table = _c(meta_table, np.int32)
    bs, Hk, D = cache.struct.block_size, cache.struct.n_kv_heads, cache.head_dim
    maxb = np.full((num_meta_blocks, bs, Hk, D), fill, np.float32)
    minb = np.full((num_meta_blocks, bs, Hk, D), fill, np.float32)
    _check(_load().q8kvo_quest_metadata(cache.ref(), _ptr(meta_table), int(meta_table.shape[1]),
                                        int(num_meta_blocks), _ptr(maxb), _ptr(minb)),
           "quest_metadata")
    return maxb, minb


def attn_fp32(cache: PagedCache, q: np.ndarray, k32: np.ndarray, v32: np.ndarray, b: int,
              h: int) -> np.ndarray:
    """fp64 attention of the unquantised fp32 q/K/V (pools shaped like the int8 ones)."""
    q = _c(q, np.float32)
    k32 = _c(k32, np.float32)
    v32 = _c(v32, np.float32)
    out = np.zeros(cache.head_dim, np.float64)
    _check(_load().q8kvo_attn_fp32(cache.ref(), _ptr(q), _ptr(k32), _ptr(v32), b, h, _ptr(out)),
           "attn_fp32")
    return out


def quantize_kv_row(x: np.ndarray):
    """Cache quantisation of one K or V row: (int8 codes, fp32 scale, flags)."""
    x = _c(x, np.float32).reshape(-1)
    codes = np.empty(x.shape, np.int8)
    scale = np.zeros(1, np.float32)
    flags = ctypes.c_uint(0)
    _check(_load().q8kvo_quantize_kv_row(_ptr(x), x.shape[0], _ptr(codes), _ptr(scale),
                                         ctypes.byref(flags)), "quantize_kv_row")
    return codes, np.float32(scale[0]), int(flags.value)


def cache_write(k, v, ks, vs, k_new, v_new, slot_mapping, token_stride=None) -> int:
    """KV-cache write into the host pools k, v [P][bs][Hk][D] (int8) and ks, vs
    [P][bs][Hk] (fp32), modified in place, from k_new, v_new: fp32 arrays whose first axis
    is the token and whose rows (token i, head h) start at i * token_stride + h * D in the
    flattened array (token_stride defaults to Hk * D). Returns the flags."""
    for a, dt in ((k, np.int8), (v, np.int8), (ks, np.float32), (vs, np.float32)):
        if a.dtype != dt or not a.flags.c_contiguous:
            raise ValueError("pools must be C-contiguous int8 / fp32 arrays")
    P, bs, Hk, D = k.shape
    if v.shape != k.shape or ks.shape != (P, bs, Hk) or vs.shape != (P, bs, Hk):
        raise ValueError("pool shapes disagree")
    slots = _c(slot_mapping, np.int64).reshape(-1)
    n = slots.shape[0]
    stride = Hk * D if token_stride is None else int(token_stride)
    k_new = _c(k_new, np.float32).reshape(-1)
    v_new = _c(v_new, np.float32).reshape(-1)
    if n and (k_new.shape[0] < (n - 1) * stride + Hk * D or v_new.shape != k_new.shape):
        raise ValueError("k_new / v_new too small for the token count and stride")
    flags = ctypes.c_uint(0)
    _check(_load().q8kvo_cache_write(_ptr(k), _ptr(v), _ptr(ks), _ptr(vs), _ptr(k_new),
                                     _ptr(v_new), _ptr(slots), n, Hk, D, bs, P, stride,
                                     ctypes.byref(flags)), "cache_write")
    return int(flags.value)


def cache_write_q4(k4, v4, kd, vd, k_new, v_new, slot_mapping, token_stride=None) -> int:
    """q4_0 KV-cache write into the host pools k4, v4 [P][bs][Hk][D/2] (uint8) and kd, vd
    [P][bs][Hk][D/32] (uint16 binary16 bits), modified in place; k_new, v_new and the slots
    as cache_write. Returns the flags."""
    for a in (k4, v4, kd, vd):
        if not a.flags.c_contiguous:
            raise ValueError("pools must be C-contiguous")
    if k4.dtype != np.uint8 or v4.dtype != np.uint8 or kd.dtype != np.uint16 or \
            vd.dtype != np.uint16:
        raise ValueError("q4_0 pools are uint8 codes and uint16 scales")
    P, bs, Hk, D2 = k4.shape
    D = 2 * D2
    if v4.shape != k4.shape or kd.shape != (P, bs, Hk, D // 32) or vd.shape != kd.shape:
        raise ValueError("pool shapes disagree")
    slots = _c(slot_mapping, np.int64).reshape(-1)
    n = slots.shape[0]
    stride = Hk * D if token_stride is None else int(token_stride)
    k_new = _c(k_new, np.float32).reshape(-1)
    v_new = _c(v_new, np.float32).reshape(-1)
    if n and (k_new.shape[0] < (n - 1) * stride + Hk * D or v_new.shape != k_new.shape):
        raise ValueError("k_new / v_new too small for the token count and stride")
    flags = ctypes.c_uint(0)
    _check(_load().q8kvo_cache_write_q4(_ptr(k4), _ptr(v4), _ptr(kd), _ptr(vd), _ptr(k_new),
                                        _ptr(v_new), _ptr(slots), n, Hk, D, bs, P, stride,
                                        ctypes.byref(flags)), "cache_write_q4")
    return int(flags.value)


def f32_to_f16(x: np.ndarray) -> np.ndarray:
    """binary16 bits (uint16) of fp32 values, round to nearest even."""
    x = _c(x, np.float32)
    out = np.empty(x.shape, np.uint16)
    _check(_load().q8kvo_f32_to_f16(_ptr(x), x.size, _ptr(out)), "f32_to_f16")
    return out


def quantize_q4_0(x: np.ndarray):
    """q4_0 codes packed two per byte [..., n/2] and binary16 scales [..., n/32] of fp32
    rows [..., n] (n a multiple of 32)."""
    x = _c(x, np.float32)
    n = x.shape[-1]
    packed = np.empty(x.shape[:-1] + (n // 2,), np.uint8)
    d16 = np.empty(x.shape[:-1] + (n // 32,), np.uint16)
    _check(_load().q8kvo_quantize_q4_0(_ptr(x), x.size, _ptr(packed), _ptr(d16)), "quantize_q4_0")
    return packed, d16


class PagedCacheQ4:
    """Host-side paged q4_0 KV cache handed to the oracle (keeps the arrays alive)."""

    def __init__(self, k4, v4, kd, vd, block_table, seq_lens, n_q_heads, scale):
        self.k4, self.v4 = _c(k4, np.uint8), _c(v4, np.uint8)
        self.kd, self.vd = _c(kd, np.uint16), _c(vd, np.uint16)
        self.block_table = _c(block_table, np.int32)
        self.seq_lens = _c(seq_lens, np.int32)
        P, bs, Hk, half = self.k4.shape
        self.struct = CacheQ4(_ptr(self.k4), _ptr(self.v4), _ptr(self.kd), _ptr(self.vd),
                              _ptr(self.block_table), _ptr(self.seq_lens),
                              int(self.seq_lens.shape[0]), int(n_q_heads), int(Hk), 2 * int(half),
                              int(bs), int(self.block_table.shape[1]), int(P),
                              float(np.float32(scale)))

    def ref(self):
        return ctypes.byref(self.struct)


def decode_q4_all(cache: PagedCacheQ4, q: np.ndarray) -> np.ndarray:
    q = _c(q, np.float32)
    s = cache.struct
    out = np.zeros((s.B, s.n_q_heads, s.head_dim), np.float64)
    _check(_load().q8kvo_decode_q4_all(cache.ref(), _ptr(q), _ptr(out)), "decode_q4_all")
    return out


def decode_q4_pairs(cache: PagedCacheQ4, q: np.ndarray, pairs) -> np.ndarray:
    q = _c(q, np.float32)
    pairs = _c(pairs, np.int32).reshape(-1, 2)
    out = np.zeros((pairs.shape[0], cache.struct.head_dim), np.float64)
    _check(_load().q8kvo_decode_q4_pairs(cache.ref(), _ptr(q), _ptr(pairs), pairs.shape[0],
                                         _ptr(out)), "decode_q4_pairs")
    return out
