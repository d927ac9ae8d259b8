"""Seeded synthetic workloads for q8-KV decode attention.

This module only draws random inputs and lays them out; it holds none of the attention
arithmetic. Both the CUDA path and the CPU oracle consume what it returns.

Recipe (the five named workloads below, plus ``make_custom`` for test grids):
  - q: fp32, iid N(0, 1), shape [B][n_q_heads][head_dim].
  - K, V: fp32 drawn iid per element (N(0, 1), or Student-t with 3 degrees of freedom),
    K optionally plus a per-(KV head, channel) bias held constant over tokens, then
    quantised per (token, KV head) row with the cache-write rule (``quantize_rows``:
    scale = max|x| * fl(1/127), code = clamp(round-half-even(x * fl(127 / max|x|)),
    -127, 127), fp32). The pools are int8 [num_blocks][block_size][n_kv_heads][head_dim]
    with fp32 scales [num_blocks][block_size][n_kv_heads].
  - block_table: int32 [B][max_blocks_per_seq]; sequence b owns ceil(L_b / block_size)
    physical blocks, assigned in order ("identity") or from a random permutation of the
    pool ("permutation"); unused entries are -1.
  - softmax scale 1 / sqrt(head_dim) rounded to fp32.
Random numbers come from numpy PCG64 streams keyed by (seed, stream, chunk), so a
workload is identical whatever the thread count.
"""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field, replace

import numpy as np

# Stream identifiers of the PCG64 seed sequences.
(_S_Q, _S_K, _S_V, _S_TABLE, _S_BIAS, _S_LENS, _S_NEWK, _S_NEWV, _S_SLOTS, _S_MAG, _S_MQ,
 _S_META) = range(12)
_CHUNK_SLOTS = 4096  # pool slots generated per independent random stream


@dataclass(frozen=True)
class Config:
    name: str
    B: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    seq_len: int | tuple  # fixed length, or ("uniform", lo, hi) inclusive
    block_size: int
    table: str  # "identity" | "permutation"
    k_dist: str = "normal"  # "normal" | "student_t3"
    v_dist: str = "normal"
    k_bias_std: float = 0.0
    seed: int = 0
    description: str = ""

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    @property
    def max_seq_len(self) -> int:
        return self.seq_len if isinstance(self.seq_len, int) else int(self.seq_len[2])

    @property
    def max_blocks_per_seq(self) -> int:
        return -(-self.max_seq_len // self.block_size)


# The five workloads: shapes and distributions of long-context GQA decode over paged
# int8 caches (head_dim 128, contexts 256 to 128K).
WORKLOADS = [
    Config("tiny_mha", 1, 8, 8, 128, 256, 16, "identity", seed=0,
           description="B=1, 8/8 heads, L=256, block 16, identity table"),
    Config("gqa_batch", 16, 32, 8, 128, 4096, 64, "permutation", seed=1,
           description="B=16, 32/8 heads, L=4096, block 64, permuted 1024-block pool"),
    Config("long_context", 1, 32, 4, 128, 131072, 128, "permutation", k_bias_std=2.0, seed=2,
           description="B=1, 32/4 heads, L=131072, block 128, K + per-channel N(0, 2^2) bias"),
    Config("ragged_outliers", 64, 64, 8, 128, ("uniform", 1, 32768), 128, "permutation",
           k_dist="student_t3", v_dist="student_t3", seed=3,
           description="B=64, 64/8 heads, L~U[1,32768], block 128, Student-t(3) K/V"),
    Config("bandwidth", 256, 32, 8, 128, 8192, 64, "permutation", seed=4,
           description="B=256, 32/8 heads, L=8192, block 64, 32768-block pool"),
]


@dataclass
class Workload:
    cfg: Config
    q: np.ndarray  # fp32 [B][Hq][D]
    k: np.ndarray  # int8 [P][bs][Hk][D]
    v: np.ndarray
    ks: np.ndarray  # fp32 [P][bs][Hk]
    vs: np.ndarray
    block_table: np.ndarray  # int32 [B][max_blocks_per_seq]
    seq_lens: np.ndarray  # int32 [B]
    scale: float  # fp32 value
    k32: np.ndarray | None = field(default=None, repr=False)
    v32: np.ndarray | None = field(default=None, repr=False)

    @property
    def num_blocks(self) -> int:
        return int(self.k.shape[0])

    @property
    def max_blocks_per_seq(self) -> int:
        return int(self.block_table.shape[1])

    def algorithmic_bytes(self) -> int:
        """Bytes one call must move: every valid (token, KV head) K row, V row and both
        scales once, q read and out written (fp32), the used block-table entries and
        seq_lens."""
        c = self.cfg
        L = self.seq_lens.astype(np.int64)
        units = int(L.sum()) * c.n_kv_heads
        nblk = int(((L + c.block_size - 1) // c.block_size).sum())
        return (units * (2 * c.head_dim + 8) + c.B * c.n_q_heads * c.head_dim * 4 * 2
                + 4 * nblk + 4 * c.B)


def _rng(seed: int, stream: int, chunk: int = 0) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, stream, chunk])))


def _draw(rng: np.random.Generator, dist: str, shape) -> np.ndarray:
    if dist == "normal":
        return rng.standard_normal(shape, dtype=np.float32)
    if dist == "student_t3":
        return rng.standard_t(3.0, shape).astype(np.float32)
    raise ValueError(f"unknown distribution {dist!r}")


def quantize_rows(x: np.ndarray):
    """Per-row int8 quantisation that turns the drawn fp32 K/V into cache contents, with
    the same rule as the library's cache write: amax = max|x| (1 when below 1e-6),
    scale = amax * fl(1/127), code = clamp(rne(x * fl(127 / amax)), -127, 127), every
    operation rounded to fp32. Finite inputs only (the draws always are)."""
    x = np.asarray(x, np.float32)
    amax = np.max(np.abs(x), axis=-1)
    amax = np.where(amax < np.float32(1e-6), np.float32(1.0), amax).astype(np.float32)
    scale = (amax * (np.float32(1.0) / np.float32(127.0))).astype(np.float32)
    inv = (np.float32(127.0) / amax).astype(np.float32)
    codes = np.rint((x * inv[..., None]).astype(np.float32))
    codes = np.clip(codes, -127, 127).astype(np.int8)
    return codes, scale


def quantize_q4_0_rows(x: np.ndarray):
    """q4_0 blocks of 32 channels (llama.cpp's rule, this library's packing) of fp32 rows
    [..., D]: m = the value of largest magnitude with its sign, d = m / -8,
    code = min(15, trunc(x * (1 / d) + 8.5)) in fp32, d stored as binary16; codes packed
    two per byte (channel 2i low nibble, 2i + 1 high). Returns (packed uint8 [..., D/2],
    d uint16 binary16 bits [..., D/32])."""
    x = np.asarray(x, np.float32)
    blk = x.reshape(x.shape[:-1] + (x.shape[-1] // 32, 32))
    idx = np.argmax(np.abs(blk), axis=-1)
    m = np.take_along_axis(blk, idx[..., None], axis=-1)[..., 0]
    d = (m / np.float32(-8.0)).astype(np.float32)
    with np.errstate(divide="ignore"):
        inv = np.where(d != 0, np.float32(1.0) / d, np.float32(0.0)).astype(np.float32)
    t = (blk * inv[..., None]).astype(np.float32) + np.float32(8.5)
    q = np.minimum(15, np.trunc(t.astype(np.float32)).astype(np.int32))
    q = q.reshape(x.shape)
    packed = (q[..., 0::2] | (q[..., 1::2] << 4)).astype(np.uint8)
    with np.errstate(over="ignore"):  # |d| > 65504 rounds to infinity, as binary16 does
        return packed, d.astype(np.float16).view(np.uint16)


def _fill_pool(seed, stream, dist, P, bs, Hk, D, bias, keep_fp32, threads, q4=False):
    """Generate one pool and its scales chunk by chunk (deterministic per chunk): int8 codes
    and fp32 row scales, or (q4) packed 4-bit codes and binary16 block scales."""
    slots = P * bs
    if q4:
        codes = np.empty((slots, Hk, D // 2), np.uint8)
        scales = np.empty((slots, Hk, D // 32), np.uint16)
    else:
        codes = np.empty((slots, Hk, D), np.int8)
        scales = np.empty((slots, Hk), np.float32)
    raw = np.empty((slots, Hk, D), np.float32) if keep_fp32 else None
    n_chunks = -(-slots // _CHUNK_SLOTS)

    def work(i):
        lo, hi = i * _CHUNK_SLOTS, min(slots, (i + 1) * _CHUNK_SLOTS)
        x = _draw(_rng(seed, stream, i), dist, (hi - lo, Hk, D))
        if bias is not None:
            x += bias[None, :, :]
        c, s = quantize_q4_0_rows(x) if q4 else quantize_rows(x)
        codes[lo:hi] = c
        scales[lo:hi] = s
        if raw is not None:
            raw[lo:hi] = x

    if threads > 1 and n_chunks > 1:
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(work, range(n_chunks)))
    else:
        for i in range(n_chunks):
            work(i)
    shape = (P, bs, Hk, D)
    return (codes.reshape((P, bs) + codes.shape[1:]), scales.reshape((P, bs) + scales.shape[1:]),
            None if raw is None else raw.reshape(shape))


def _seq_lens(cfg: Config) -> np.ndarray:
    if isinstance(cfg.seq_len, int):
        return np.full(cfg.B, cfg.seq_len, np.int32)
    kind, lo, hi = cfg.seq_len
    if kind != "uniform":
        raise ValueError(kind)
    return _rng(cfg.seed, _S_LENS).integers(lo, hi + 1, size=cfg.B).astype(np.int32)


def build_block_table(seq_lens, block_size, max_blocks_per_seq, table, num_blocks, rng):
    """Assign ceil(L_b / block_size) distinct physical blocks to every sequence."""
    need = (np.asarray(seq_lens, np.int64) + block_size - 1) // block_size
    total = int(need.sum())
    if total > num_blocks:
        raise ValueError("pool too small")
    if table == "identity":
        order = np.arange(num_blocks, dtype=np.int64)
    elif table == "permutation":
        order = rng.permutation(num_blocks)
    else:
        raise ValueError(f"unknown table kind {table!r}")
    bt = np.full((len(seq_lens), max_blocks_per_seq), -1, np.int32)
    off = 0
    for b, n in enumerate(need):
        bt[b, :n] = order[off:off + n]
        off += n
    return bt


def make_custom(B, n_q_heads, n_kv_heads, head_dim, seq_lens, block_size, *, table="permutation",
                k_dist="normal", v_dist="normal", k_bias_std=0.0, seed=0, max_blocks_per_seq=None,
                extra_blocks=0, keep_fp32=False, threads=None, name="custom") -> Workload:
    """A workload with explicit per-sequence lengths (used by the test grids)."""
    seq_lens = np.asarray(seq_lens, np.int32).reshape(B)
    cfg = Config(name, B, n_q_heads, n_kv_heads, head_dim,
                 int(seq_lens.max(initial=0)), block_size, table, k_dist, v_dist, k_bias_std,
                 seed)
    return _make(cfg, seq_lens, max_blocks_per_seq, extra_blocks, keep_fp32, threads)


def make(cfg: Config | int, *, keep_fp32: bool = False, threads: int | None = None) -> Workload:
    """The named workload ``cfg`` (a Config or an index into WORKLOADS)."""
    if isinstance(cfg, int):
        cfg = WORKLOADS[cfg]
    return _make(cfg, _seq_lens(cfg), None, 0, keep_fp32, threads)


def _make(cfg: Config, seq_lens, max_blocks_per_seq, extra_blocks, keep_fp32, threads):
    threads = threads or min(32, os.cpu_count() or 1)
    bs, Hk, D = cfg.block_size, cfg.n_kv_heads, cfg.head_dim
    need = int(((seq_lens.astype(np.int64) + bs - 1) // bs).sum())
    P = max(1, need + int(extra_blocks))
    mbps = max_blocks_per_seq or max(1, -(-int(seq_lens.max(initial=0)) // bs))
    q = _rng(cfg.seed, _S_Q).standard_normal((cfg.B, cfg.n_q_heads, D), dtype=np.float32)
    bias = None
    if cfg.k_bias_std:
        bias = (_rng(cfg.seed, _S_BIAS).standard_normal((Hk, D), dtype=np.float32)
                * np.float32(cfg.k_bias_std))
    k, ks, k32 = _fill_pool(cfg.seed, _S_K, cfg.k_dist, P, bs, Hk, D, bias, keep_fp32, threads)
    v, vs, v32 = _fill_pool(cfg.seed, _S_V, cfg.v_dist, P, bs, Hk, D, None, keep_fp32, threads)
    bt = build_block_table(seq_lens, bs, mbps, cfg.table, P, _rng(cfg.seed, _S_TABLE))
    scale = float(np.float32(1.0) / np.float32(math.sqrt(D)))
    return Workload(cfg, q, k, v, ks, vs, bt, seq_lens.astype(np.int32), scale, k32, v32)


def with_config(cfg: Config, **kw) -> Config:
    return replace(cfg, **kw)


# ---------------------------------------------------------------- KV-cache write inputs


@dataclass
class CacheRows:
    """New K/V rows for the KV-cache write and where they go."""
    k_new: np.ndarray  # fp32 [n_tokens][token_stride] (row (i, h) at [i][h * D:(h + 1) * D])
    v_new: np.ndarray
    slots: np.ndarray  # int64 [n_tokens]; -1 = padding
    n_kv_heads: int
    head_dim: int

    @property
    def n_tokens(self) -> int:
        return int(self.slots.shape[0])

    def algorithmic_bytes(self) -> int:
        """Bytes one write must move: every non-padding (token, KV head) K and V row read
        (fp32) and written (int8 codes + fp32 scale), and the slot mapping read."""
        n = int(np.count_nonzero(self.slots >= 0))
        rows = n * self.n_kv_heads
        return rows * 2 * (4 * self.head_dim + self.head_dim + 4) + 8 * self.n_tokens


def _mixed_rows(seed, stream, n, Hk, D, threads):
    """Rows of N(0, 1) or Student-t(3) draws times a per-row magnitude in {1e-3, 1, 30},
    with about 1 row in 64 all zero and 1 in 64 below 1e-6 everywhere."""
    out = np.empty((n, Hk, D), np.float32)
    chunk = _CHUNK_SLOTS
    n_chunks = -(-n // chunk)

    def work(i):
        lo, hi = i * chunk, min(n, (i + 1) * chunk)
        rng = _rng(seed, stream, i)
        x = rng.standard_normal((hi - lo, Hk, D), dtype=np.float32)
        heavy = rng.random((hi - lo, Hk)) < 0.25
        if heavy.any():
            x[heavy] = rng.standard_t(3.0, (int(heavy.sum()), D)).astype(np.float32)
        kind = rng.integers(0, 64, size=(hi - lo, Hk))
        mag = np.choose(kind % 3, [np.float32(1e-3), np.float32(1.0), np.float32(30.0)])
        mag = np.where(kind == 0, np.float32(0.0), mag)
        mag = np.where(kind == 1, np.float32(1e-7), mag)
        out[lo:hi] = x * mag[..., None].astype(np.float32)

    if threads > 1 and n_chunks > 1:
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(work, range(n_chunks)))
    else:
        for i in range(n_chunks):
            work(i)
    return out


def _strided(rows: np.ndarray, token_stride: int | None, fill: float) -> np.ndarray:
    n, Hk, D = rows.shape
    stride = token_stride or Hk * D
    buf = np.full((n, stride), fill, np.float32)
    buf[:, :Hk * D] = rows.reshape(n, Hk * D)
    return buf


def make_cache_rows(n_tokens, n_kv_heads, head_dim, num_blocks, block_size, *, seed=0,
                    pad_every=0, token_stride=None, threads=None) -> CacheRows:
    """Rows for a scattered write: n_tokens distinct slots drawn from a random permutation
    of the pool, every pad_every-th token (if > 0) marked as padding (-1). With a
    token_stride above n_kv_heads * head_dim the unused tail of every token is NaN (it
    stands for the other heads of a fused projection and must never be read)."""
    threads = threads or min(32, os.cpu_count() or 1)
    n_slots = num_blocks * block_size
    if n_tokens > n_slots:
        raise ValueError("more tokens than slots")
    slots = _rng(seed, _S_SLOTS).permutation(n_slots)[:n_tokens].astype(np.int64)
    if pad_every > 0:
        slots[pad_every - 1::pad_every] = -1
    k = _mixed_rows(seed, _S_NEWK, n_tokens, n_kv_heads, head_dim, threads)
    v = _mixed_rows(seed, _S_NEWV, n_tokens, n_kv_heads, head_dim, threads)
    return CacheRows(_strided(k, token_stride, np.nan), _strided(v, token_stride, np.nan), slots,
                     n_kv_heads, head_dim)


def prompt_slots(block_table: np.ndarray, seq_lens, block_size: int) -> np.ndarray:
    """Slot of every token of every sequence, sequence after sequence (a prompt fill):
    block_table[b][t // block_size] * block_size + t % block_size."""
    parts = []
    for b, L in enumerate(np.asarray(seq_lens, np.int64)):
        t = np.arange(L, dtype=np.int64)
        parts.append(block_table[b, t // block_size].astype(np.int64) * block_size + t % block_size)
    return np.concatenate(parts) if parts else np.zeros(0, np.int64)


def make_prompt_fill(cfg: Config | int, *, threads: int | None = None) -> CacheRows:
    """Fresh fp32 K/V rows for every token of a named workload, with the slots its block
    table gives them: the write that fills that workload's whole cache."""
    if isinstance(cfg, int):
        cfg = WORKLOADS[cfg]
    threads = threads or min(32, os.cpu_count() or 1)
    lens = _seq_lens(cfg)
    bs = cfg.block_size
    need = int(((lens.astype(np.int64) + bs - 1) // bs).sum())
    mbps = max(1, -(-int(lens.max(initial=0)) // bs))
    bt = build_block_table(lens, bs, mbps, cfg.table, max(1, need), _rng(cfg.seed, _S_TABLE))
    slots = prompt_slots(bt, lens, bs)
    n = int(slots.shape[0])
    Hk, D = cfg.n_kv_heads, cfg.head_dim
    k = _mixed_rows(cfg.seed, _S_NEWK, n, Hk, D, threads)
    v = _mixed_rows(cfg.seed, _S_NEWV, n, Hk, D, threads)
    return CacheRows(k.reshape(n, Hk * D), v.reshape(n, Hk * D), slots, Hk, D)


# ---------------------------------------------------------------- several queries per sequence


def multi_queries(B: int, n_queries: int, n_q_heads: int, head_dim: int, *, seed: int = 0):
    """fp32 queries [B][n_queries][n_q_heads][head_dim], iid N(0, 1): the new tokens of a
    multi-token (speculative) decode step, one row per (sequence, new token, head)."""
    return _rng(seed, _S_MQ).standard_normal((B, n_queries, n_q_heads, head_dim),
                                             dtype=np.float32)


def fp32_rows(w: Workload, which: str, slots) -> np.ndarray:
    """The unquantised fp32 K ("k") or V ("v") rows [len(slots)][n_kv_heads][head_dim] that
    the workload's pool slots were quantised from, regenerated from the random streams of
    only the chunks that hold them (a sample of a large workload needs no full fp32 pool)."""
    c = w.cfg
    bs, Hk, D = c.block_size, c.n_kv_heads, c.head_dim
    n_slots = w.num_blocks * bs
    slots = np.asarray(slots, np.int64).reshape(-1)
    stream, dist = (_S_K, c.k_dist) if which == "k" else (_S_V, c.v_dist)
    bias = None
    if which == "k" and c.k_bias_std:
        bias = (_rng(c.seed, _S_BIAS).standard_normal((Hk, D), dtype=np.float32)
                * np.float32(c.k_bias_std))
    out = np.empty((slots.shape[0], Hk, D), np.float32)
    chunk_of = slots // _CHUNK_SLOTS
    for ch in np.unique(chunk_of):
        lo, hi = int(ch) * _CHUNK_SLOTS, min(n_slots, (int(ch) + 1) * _CHUNK_SLOTS)
        x = _draw(_rng(c.seed, stream, int(ch)), dist, (hi - lo, Hk, D))
        if bias is not None:
            x += bias[None, :, :]
        sel = chunk_of == ch
        out[sel] = x[slots[sel] - lo]
    return out


# ---------------------------------------------------------------- QUEST metadata tables


def quest_meta_table(seq_lens, block_size: int, *, seed: int = 0, extra_blocks: int = 0):
    """Metadata block table for per-block K metadata: request r needs
    ceil(ceil(L_r / block_size) / block_size) metadata blocks of block_size rows each; they
    are drawn from a random permutation of the pool (as the block table is). Returns
    (meta_table int32 [B][max_meta_per_seq] with -1 in unused entries, num_meta_blocks)."""
    L = np.asarray(seq_lens, np.int64)
    nkv = (L + block_size - 1) // block_size
    nmeta = (nkv + block_size - 1) // block_size
    mm = max(1, int(nmeta.max(initial=0)))
    total = max(1, int(nmeta.sum()) + int(extra_blocks))
    order = _rng(seed, _S_META).permutation(total)
    table = np.full((len(L), mm), -1, np.int32)
    off = 0
    for r, n in enumerate(nmeta):
        table[r, :n] = order[off:off + n]
        off += int(n)
    return table, total


# ---------------------------------------------------------------- q4_0 caches


@dataclass
class WorkloadQ4:
    """A workload whose cache is in the q4_0 format, drawn from the same random streams as
    the q8 workload of the same Config (so the two hold the same unquantised values)."""
    cfg: Config
    q: np.ndarray  # fp32 [B][Hq][D]
    k4: np.ndarray  # uint8 [P][bs][Hk][D/2]
    v4: np.ndarray
    kd: np.ndarray  # uint16 binary16 bits [P][bs][Hk][D/32]
    vd: np.ndarray
    block_table: np.ndarray
    seq_lens: np.ndarray
    scale: float
    k32: np.ndarray | None = field(default=None, repr=False)
    v32: np.ndarray | None = field(default=None, repr=False)

    @property
    def num_blocks(self) -> int:
        return int(self.k4.shape[0])

    @property
    def max_blocks_per_seq(self) -> int:
        return int(self.block_table.shape[1])

    def algorithmic_bytes(self) -> int:
        """Every valid (token, KV head) K and V row (D/2 code bytes + 2 * D/32 scale bytes
        each) once, q read and out written (fp32), the used block-table entries, seq_lens."""
        c = self.cfg
        L = self.seq_lens.astype(np.int64)
        units = int(L.sum()) * c.n_kv_heads
        nblk = int(((L + c.block_size - 1) // c.block_size).sum())
        row = c.head_dim // 2 + 2 * (c.head_dim // 32)
        return (units * 2 * row + c.B * c.n_q_heads * c.head_dim * 4 * 2 + 4 * nblk + 4 * c.B)


def make_q4(cfg: Config | int, *, seq_lens=None, keep_fp32: bool = False,
            threads: int | None = None) -> WorkloadQ4:
    """The named (or given) workload with a q4_0 cache."""
    if isinstance(cfg, int):
        cfg = WORKLOADS[cfg]
    threads = threads or min(32, os.cpu_count() or 1)
    seq_lens = _seq_lens(cfg) if seq_lens is None else np.asarray(seq_lens, np.int32)
    bs, Hk, D = cfg.block_size, cfg.n_kv_heads, cfg.head_dim
    need = int(((seq_lens.astype(np.int64) + bs - 1) // bs).sum())
    P = max(1, need)
    mbps = max(1, -(-int(seq_lens.max(initial=0)) // bs))
    q = _rng(cfg.seed, _S_Q).standard_normal((cfg.B, cfg.n_q_heads, D), dtype=np.float32)
    bias = None
    if cfg.k_bias_std:
        bias = (_rng(cfg.seed, _S_BIAS).standard_normal((Hk, D), dtype=np.float32)
                * np.float32(cfg.k_bias_std))
    k4, kd, k32 = _fill_pool(cfg.seed, _S_K, cfg.k_dist, P, bs, Hk, D, bias, keep_fp32,
                             threads, q4=True)
    v4, vd, v32 = _fill_pool(cfg.seed, _S_V, cfg.v_dist, P, bs, Hk, D, None, keep_fp32,
                             threads, q4=True)
    bt = build_block_table(seq_lens, bs, mbps, cfg.table, P, _rng(cfg.seed, _S_TABLE))
    scale = float(np.float32(1.0) / np.float32(math.sqrt(D)))
    return WorkloadQ4(cfg, q, k4, v4, kd, vd, bt, seq_lens.astype(np.int32), scale, k32, v32)


def make_q4_custom(B, n_q_heads, n_kv_heads, head_dim, seq_lens, block_size, *,
                   table="permutation", k_dist="normal", v_dist="normal", k_bias_std=0.0, seed=0,
                   keep_fp32=False, name="custom_q4") -> WorkloadQ4:
    seq_lens = np.asarray(seq_lens, np.int32).reshape(B)
    cfg = Config(name, B, n_q_heads, n_kv_heads, head_dim, int(seq_lens.max(initial=0)),
                 block_size, table, k_dist, v_dist, k_bias_std, seed)
    return make_q4(cfg, seq_lens=seq_lens, keep_fp32=keep_fp32)
