"""ctypes binding of libq8kv.so (the C ABI in include/q8kv.h).

Argument marshalling only: shapes and dtypes are read off torch tensors, device pointers
and the current CUDA stream are passed through, and a non-OK status raises Q8KVError.
Every step of the computation runs in the CUDA library; there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

from . import build as _build

_lock = threading.Lock()
_lib = None

Q8KV_OK = 0
DEVERR_SEQ_LEN = 0x1
DEVERR_BLOCK_TABLE = 0x2
DEVERR_TIMEOUT = 0x4
DEVERR_SLOT = 0x8
DEVERR_NONFINITE = 0x10
DEVERR_META = 0x20

EXPORTS = (
    "q8kv_decode_attn",
    "q8kv_decode_attn_multi",
    "q8kv_decode_attn_q4",
    "q8kv_workspace_bytes",
    "q8kv_workspace_init",
    "q8kv_decode_attn_ws",
    "q8kv_decode_attn_static",
    "q8kv_cache_write",
    "q8kv_cache_write_q4",
    "q8kv_quest_metadata",
    "q8kv_debug_quantize_q",
    "q8kv_debug_block_dots",
    "q8kv_debug_stall_pipeline",
    "q8kv_device_errors",
    "q8kv_status_string",
    "q8kv_last_cuda_error",
    "q8kv_version",
)


class Q8KVError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        msg = lib().q8kv_status_string(status).decode()
        if status == 3:
            msg += f" (cudaError {lib().q8kv_last_cuda_error()})"
        super().__init__(f"{what}: {msg} (status {status})")


def lib_path() -> str:
    return _build.LIB


def lib():
    """Load libq8kv.so, building it first when it is missing or older than its sources."""
    global _lib
    with _lock:
        if _lib is None:
            path = _build.LIB
            if not os.path.exists(path) or _build.stale():
                _build.build()
            L = ctypes.CDLL(path)
            P, I, F, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
            sig = {
                "q8kv_decode_attn": ([P] * 8 + [I] * 7 + [F, P], I),
                "q8kv_decode_attn_multi": ([P] * 8 + [I] * 8 + [F, P], I),
                "q8kv_decode_attn_q4": ([P] * 8 + [I] * 7 + [F, P], I),
                "q8kv_workspace_bytes": ([I, I, I, I], Z),
                "q8kv_workspace_init": ([P, Z, P], I),
                "q8kv_decode_attn_ws": ([P] * 8 + [I] * 7 + [F, P, Z, P], I),
                "q8kv_decode_attn_static": ([P] * 8 + [I] * 7 + [F, P], I),
                "q8kv_cache_write": ([P] * 7 + [I] * 5 + [ctypes.c_longlong, P], I),
                "q8kv_cache_write_q4": ([P] * 7 + [I] * 5 + [ctypes.c_longlong, P], I),
                "q8kv_quest_metadata": ([P] * 7 + [I] * 8 + [P], I),
                "q8kv_debug_quantize_q": ([P, P, P, I, I, P], I),
                "q8kv_debug_block_dots": ([P, I] + [P] * 8 + [I] * 7 + [F, P], I),
                "q8kv_debug_stall_pipeline": ([P] * 8 + [I] * 7 + [F, I, ctypes.c_ulonglong, P],
                                              I),
                "q8kv_device_errors": ([ctypes.POINTER(ctypes.c_uint), I], I),
                "q8kv_status_string": ([I], ctypes.c_char_p),
                "q8kv_last_cuda_error": ([], I),
                "q8kv_version": ([], I),
            }
            for name, (args, res) in sig.items():
                fn = getattr(L, name)
                fn.argtypes = args
                fn.restype = res
            _lib = L
    return _lib


def _ptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _need(t: torch.Tensor, name: str, dtype: torch.dtype, ndim: int):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype or t.dim() != ndim or not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name}: expected a contiguous CUDA {dtype} tensor with {ndim} dims, "
                         f"got {t.dtype} {tuple(t.shape)} on {t.device}")


def _geometry(out, q, k_blocks, v_blocks, kscale, vscale, block_table, seq_lens,
              contiguous=True):
    if contiguous:  # (a multi-query caller passes views of its checked 4-D tensors)
        _need(out, "out", torch.float32, 3)
        _need(q, "q", torch.float32, 3)
    _need(k_blocks, "k_blocks", torch.int8, 4)
    _need(v_blocks, "v_blocks", torch.int8, 4)
    _need(kscale, "kscale", torch.float32, 3)
    _need(vscale, "vscale", torch.float32, 3)
    _need(block_table, "block_table", torch.int32, 2)
    _need(seq_lens, "seq_lens", torch.int32, 1)
    B, Hq, D = q.shape
    P, bs, Hk, Dk = k_blocks.shape
    if tuple(out.shape) != (B, Hq, D) or Dk != D or tuple(v_blocks.shape) != (P, bs, Hk, D):
        raise ValueError("q/out/k_blocks/v_blocks shapes disagree")
    if tuple(kscale.shape) != (P, bs, Hk) or tuple(vscale.shape) != (P, bs, Hk):
        raise ValueError("kscale/vscale must be [num_blocks][block_size][n_kv_heads]")
    if block_table.shape[0] != B or tuple(seq_lens.shape) != (B,):
        raise ValueError("block_table/seq_lens batch dimension disagrees with q")
    return B, Hq, Hk, D, bs, int(block_table.shape[1]), P


def _check(status: int, what: str):
    if status != Q8KV_OK:
        raise Q8KVError(status, what)


def q8kv_decode_attn(out, q, k_blocks, v_blocks, kscale, vscale, block_table, seq_lens, scale,
                     stream=None):
    """Decode attention into ``out`` with the library-managed workspace."""
    geo = _geometry(out, q, k_blocks, v_blocks, kscale, vscale, block_table, seq_lens)
    _check(lib().q8kv_decode_attn(_ptr(out), _ptr(q), _ptr(k_blocks), _ptr(v_blocks),
                                  _ptr(kscale), _ptr(vscale), _ptr(block_table), _ptr(seq_lens),
                                  *geo, float(scale), _stream(stream)), "q8kv_decode_attn")
    return out


def q8kv_decode_attn_multi(out, q, k_blocks, v_blocks, kscale, vscale, block_table, seq_lens,
                           scale, stream=None):
    """Causal decode of n_queries new tokens per sequence: q, out [B][n_queries][Hq][D];
    query i of sequence b sees seq_lens[b] - (n_queries - 1 - i) tokens."""
    _need(out, "out", torch.float32, 4)
    _need(q, "q", torch.float32, 4)
    if tuple(out.shape) != tuple(q.shape):
        raise ValueError("out and q must have the same shape [B][n_queries][Hq][D]")
    B, nq, Hq, D = q.shape
    geo = _geometry(out[:, 0], q[:, 0], k_blocks, v_blocks, kscale, vscale, block_table,
                    seq_lens, contiguous=False)
    _check(lib().q8kv_decode_attn_multi(_ptr(out), _ptr(q), _ptr(k_blocks), _ptr(v_blocks),
                                        _ptr(kscale), _ptr(vscale), _ptr(block_table),
                                        _ptr(seq_lens), geo[0], nq, *geo[1:], float(scale),
                                        _stream(stream)), "q8kv_decode_attn_multi")
    return out


def q8kv_decode_attn_q4(out, q, k4_blocks, v4_blocks, kd, vd, block_table, seq_lens, scale,
                        stream=None):
    """Decode attention over a q4_0 cache: k4/v4 uint8 [P][bs][Hk][D/2] (two codes per byte,
    channel 2i in the low nibble), kd/vd binary16 [P][bs][Hk][D/32] (torch.float16, or
    16-bit integers holding the bits); q, out fp32 [B][Hq][D]."""
    _need(out, "out", torch.float32, 3)
    _need(q, "q", torch.float32, 3)
    _need(k4_blocks, "k4_blocks", torch.uint8, 4)
    _need(v4_blocks, "v4_blocks", torch.uint8, 4)
    for t, name in ((kd, "kd"), (vd, "vd")):
        if t.dtype not in (torch.float16, torch.int16, torch.uint16) or t.dim() != 4 or \
                not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name}: expected a contiguous CUDA 16-bit tensor with 4 dims")
    _need(block_table, "block_table", torch.int32, 2)
    _need(seq_lens, "seq_lens", torch.int32, 1)
    B, Hq, D = q.shape
    P, bs, Hk, half = k4_blocks.shape
    if tuple(out.shape) != (B, Hq, D) or 2 * half != D or tuple(v4_blocks.shape) != (P, bs, Hk, half):
        raise ValueError("q/out/k4/v4 shapes disagree")
    if tuple(kd.shape) != (P, bs, Hk, D // 32) or tuple(vd.shape) != (P, bs, Hk, D // 32):
        raise ValueError("kd/vd must be [num_blocks][block_size][n_kv_heads][head_dim/32]")
    _check(lib().q8kv_decode_attn_q4(_ptr(out), _ptr(q), _ptr(k4_blocks), _ptr(v4_blocks),
                                     _ptr(kd), _ptr(vd), _ptr(block_table), _ptr(seq_lens), B,
                                     Hq, Hk, D, bs, int(block_table.shape[1]), P, float(scale),
                                     _stream(stream)), "q8kv_decode_attn_q4")
    return out


def q8kv_workspace_bytes(B: int, n_q_heads: int, n_kv_heads: int, head_dim: int) -> int:
    return int(lib().q8kv_workspace_bytes(B, n_q_heads, n_kv_heads, head_dim))


def q8kv_workspace_init(workspace: torch.Tensor, stream=None):
    _check(lib().q8kv_workspace_init(_ptr(workspace), workspace.numel() * workspace.element_size(),
                                     _stream(stream)), "q8kv_workspace_init")


def q8kv_decode_attn_ws(out, q, k_blocks, v_blocks, kscale, vscale, block_table, seq_lens, scale,
                        workspace, stream=None):
    """Decode attention with a caller-owned (zero-initialised) workspace tensor."""
    geo = _geometry(out, q, k_blocks, v_blocks, kscale, vscale, block_table, seq_lens)
    if not workspace.is_cuda or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA tensor")
    _check(lib().q8kv_decode_attn_ws(_ptr(out), _ptr(q), _ptr(k_blocks), _ptr(v_blocks),
                                     _ptr(kscale), _ptr(vscale), _ptr(block_table),
                                     _ptr(seq_lens), *geo, float(scale), _ptr(workspace),
                                     workspace.numel() * workspace.element_size(),
                                     _stream(stream)), "q8kv_decode_attn_ws")
    return out


def q8kv_decode_attn_static(out, q, k_blocks, v_blocks, kscale, vscale, block_table, seq_lens,
                            scale, stream=None):
    """Decode attention with the library's fixed per-device scratch array (no allocation).

    Calls that may overlap on the GPU race on that array; order them on one stream."""
    geo = _geometry(out, q, k_blocks, v_blocks, kscale, vscale, block_table, seq_lens)
    _check(lib().q8kv_decode_attn_static(_ptr(out), _ptr(q), _ptr(k_blocks), _ptr(v_blocks),
                                         _ptr(kscale), _ptr(vscale), _ptr(block_table),
                                         _ptr(seq_lens), *geo, float(scale), _stream(stream)),
           "q8kv_decode_attn_static")
    return out


def q8kv_cache_write(k_blocks, v_blocks, kscale, vscale, k_new, v_new, slot_mapping,
                     stream=None):
    """Quantise the new rows k_new, v_new [n_tokens][n_kv_heads][head_dim] (fp32; the
    token dimension may be strided, e.g. a slice of a fused QKV projection) and store them
    at the physical slots slot_mapping [n_tokens] (int64; negative = padding) of the pools."""
    _need(k_blocks, "k_blocks", torch.int8, 4)
    _need(v_blocks, "v_blocks", torch.int8, 4)
    _need(kscale, "kscale", torch.float32, 3)
    _need(vscale, "vscale", torch.float32, 3)
    _need(slot_mapping, "slot_mapping", torch.int64, 1)
    P, bs, Hk, D = k_blocks.shape
    if tuple(v_blocks.shape) != (P, bs, Hk, D) or tuple(kscale.shape) != (P, bs, Hk) or \
            tuple(vscale.shape) != (P, bs, Hk):
        raise ValueError("pool shapes disagree")
    n = int(slot_mapping.shape[0])
    for t, name in ((k_new, "k_new"), (v_new, "v_new")):
        if not isinstance(t, torch.Tensor) or t.dtype != torch.float32 or not t.is_cuda:
            raise ValueError(f"{name}: expected a CUDA float32 tensor")
        if tuple(t.shape) != (n, Hk, D) or t.stride(2) != 1 or t.stride(1) != D:
            raise ValueError(f"{name}: expected shape {(n, Hk, D)} with contiguous rows, got "
                             f"{tuple(t.shape)} strides {t.stride()}")
    if n > 1 and k_new.stride(0) != v_new.stride(0):
        raise ValueError("k_new and v_new must have the same token stride")
    stride = int(k_new.stride(0)) if n > 1 else Hk * D
    _check(lib().q8kv_cache_write(_ptr(k_blocks), _ptr(v_blocks), _ptr(kscale), _ptr(vscale),
                                  _ptr(k_new), _ptr(v_new), _ptr(slot_mapping), n, Hk, D, bs, P,
                                  stride, _stream(stream)), "q8kv_cache_write")


def q8kv_cache_write_q4(k4_blocks, v4_blocks, kd, vd, k_new, v_new, slot_mapping, stream=None):
    """q4_0 cache write: quantise the new rows k_new, v_new [n_tokens][n_kv_heads][head_dim]
    (fp32; the token dimension may be strided) per 32-channel block and store codes (uint8
    [P][bs][Hk][D/2]) and binary16 scales (kd, vd [P][bs][Hk][D/32], torch.float16 or 16-bit
    integers holding the bits) at the slots slot_mapping [n_tokens] (int64; negative =
    padding)."""
    _need(k4_blocks, "k4_blocks", torch.uint8, 4)
    _need(v4_blocks, "v4_blocks", torch.uint8, 4)
    _need(slot_mapping, "slot_mapping", torch.int64, 1)
    P, bs, Hk, half = k4_blocks.shape
    D = 2 * half
    if tuple(v4_blocks.shape) != (P, bs, Hk, half):
        raise ValueError("k4/v4 shapes disagree")
    for t, name in ((kd, "kd"), (vd, "vd")):
        if t.dtype not in (torch.float16, torch.int16, torch.uint16) or not t.is_cuda or \
                not t.is_contiguous() or tuple(t.shape) != (P, bs, Hk, D // 32):
            raise ValueError(f"{name}: expected a contiguous CUDA 16-bit tensor "
                             f"{(P, bs, Hk, D // 32)}")
    n = int(slot_mapping.shape[0])
    for t, name in ((k_new, "k_new"), (v_new, "v_new")):
        if not isinstance(t, torch.Tensor) or t.dtype != torch.float32 or not t.is_cuda:
            raise ValueError(f"{name}: expected a CUDA float32 tensor")
        if tuple(t.shape) != (n, Hk, D) or t.stride(2) != 1 or t.stride(1) != D:
            raise ValueError(f"{name}: expected shape {(n, Hk, D)} with contiguous rows, got "
                             f"{tuple(t.shape)} strides {t.stride()}")
    if n > 1 and k_new.stride(0) != v_new.stride(0):
        raise ValueError("k_new and v_new must have the same token stride")
    stride = int(k_new.stride(0)) if n > 1 else Hk * D
    _check(lib().q8kv_cache_write_q4(_ptr(k4_blocks), _ptr(v4_blocks), _ptr(kd), _ptr(vd),
                                     _ptr(k_new), _ptr(v_new), _ptr(slot_mapping), n, Hk, D,
                                     bs, P, stride, _stream(stream)), "q8kv_cache_write_q4")


def q8kv_quest_metadata(maxblocks, minblocks, k_blocks, kscale, block_table, seq_lens,
                        meta_block_table, stream=None):
    """Per-block K metadata: maxblocks, minblocks fp32 [num_meta][block_size][Hk][D] get the
    per-channel max / min of the dequantised K of each KV block (row j % block_size of
    metadata block meta_block_table[r][j // block_size])."""
    _need(maxblocks, "maxblocks", torch.float32, 4)
    _need(minblocks, "minblocks", torch.float32, 4)
    _need(k_blocks, "k_blocks", torch.int8, 4)
    _need(kscale, "kscale", torch.float32, 3)
    _need(block_table, "block_table", torch.int32, 2)
    _need(seq_lens, "seq_lens", torch.int32, 1)
    _need(meta_block_table, "meta_block_table", torch.int32, 2)
    P, bs, Hk, D = k_blocks.shape
    nm = int(maxblocks.shape[0])
    if tuple(maxblocks.shape) != (nm, bs, Hk, D) or tuple(minblocks.shape) != (nm, bs, Hk, D):
        raise ValueError("maxblocks/minblocks must be [num_meta_blocks][block_size][Hk][D]")
    if tuple(kscale.shape) != (P, bs, Hk):
        raise ValueError("kscale must be [num_blocks][block_size][Hk]")
    B = int(seq_lens.shape[0])
    if block_table.shape[0] != B or meta_block_table.shape[0] != B:
        raise ValueError("block tables and seq_lens disagree on the batch size")
    _check(lib().q8kv_quest_metadata(_ptr(maxblocks), _ptr(minblocks), _ptr(k_blocks),
                                     _ptr(kscale), _ptr(block_table), _ptr(seq_lens),
                                     _ptr(meta_block_table), B, Hk, D, bs,
                                     int(block_table.shape[1]), int(meta_block_table.shape[1]),
                                     P, nm, _stream(stream)), "q8kv_quest_metadata")


def q8kv_debug_quantize_q(qi, qsc, q, stream=None):
    """int8 codes qi [..., D] and block scales qsc [..., D/32] of the fp32 rows of q [..., D]."""
    D = q.shape[-1]
    n_rows = q.numel() // D
    for t, dt in ((qi, torch.int8), (qsc, torch.float32), (q, torch.float32)):
        if t.dtype != dt or not t.is_cuda or not t.is_contiguous():
            raise ValueError("q8kv_debug_quantize_q: bad tensor")
    if qi.numel() != q.numel() or qsc.numel() != n_rows * (D // 32):
        raise ValueError("q8kv_debug_quantize_q: size mismatch")
    _check(lib().q8kv_debug_quantize_q(_ptr(qi), _ptr(qsc), _ptr(q), n_rows, D, _stream(stream)),
           "q8kv_debug_quantize_q")


def q8kv_debug_block_dots(dots, out, q, k_blocks, v_blocks, kscale, vscale, block_table,
                          seq_lens, scale, stream=None):
    """int32 block dots [B][Hq][max_len][D/32] from the decode kernel (and ``out``)."""
    geo = _geometry(out, q, k_blocks, v_blocks, kscale, vscale, block_table, seq_lens)
    _need(dots, "dots", torch.int32, 4)
    B, Hq, _, D, _, _, _ = geo
    if dots.shape[0] != B or dots.shape[1] != Hq or dots.shape[3] != D // 32:
        raise ValueError("dots must be [B][n_q_heads][max_seq_len][head_dim/32]")
    _check(lib().q8kv_debug_block_dots(_ptr(dots), int(dots.shape[2]), _ptr(out), _ptr(q),
                                       _ptr(k_blocks), _ptr(v_blocks), _ptr(kscale),
                                       _ptr(vscale), _ptr(block_table), _ptr(seq_lens), *geo,
                                       float(scale), _stream(stream)), "q8kv_debug_block_dots")


def q8kv_debug_stall_pipeline(out, q, k_blocks, v_blocks, kscale, vscale, block_table, seq_lens,
                              scale, stall_cta=0, limit_ns=100_000, stream=None):
    """q8kv_decode_attn with CTA ``stall_cta``'s pipeline stalled on purpose: its waits run
    out after ``limit_ns`` and set the time-out bit of the device error word."""
    geo = _geometry(out, q, k_blocks, v_blocks, kscale, vscale, block_table, seq_lens)
    _check(lib().q8kv_debug_stall_pipeline(_ptr(out), _ptr(q), _ptr(k_blocks), _ptr(v_blocks),
                                           _ptr(kscale), _ptr(vscale), _ptr(block_table),
                                           _ptr(seq_lens), *geo, float(scale), int(stall_cta),
                                           int(limit_ns), _stream(stream)),
           "q8kv_debug_stall_pipeline")


def q8kv_device_errors(clear: bool = True) -> int:
    flags = ctypes.c_uint(0)
    _check(lib().q8kv_device_errors(ctypes.byref(flags), 1 if clear else 0), "q8kv_device_errors")
    return int(flags.value)


def q8kv_version() -> int:
    return int(lib().q8kv_version())
