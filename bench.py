"""Benchmark of q8-KV single-query decode attention on B200.

One step = one q8kv_decode_attn call over one batch of the workload (the whole hot path:
Q quantisation, paged K/V streaming, int8 block dots, online softmax, V accumulation,
split combine), through the C ABI. Prints one JSON line (rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config I] [--impl reference]

Headline: the bandwidth-saturating workload (B = 256 sequences of 8192 tokens, 32 q heads
over 8 KV heads, 4.44 GB of K/V read per call), the largest of the five workloads and the
one that fits a single GPU with the most work; the metric is not quoted on any one
workload, so the largest is timed. The other four workloads, and the group-8 reading of
the 16 x 4096-token batch, follow as per-workload legs of the same line, each with its
own time, bandwidth, clocks and sampled-row parity against the oracle.

Metric: effective KV bandwidth = algorithmic bytes of one call / time per call, where the
algorithmic bytes are every valid (token, KV head) K row, V row and both scales once, plus
q read and out written in fp32, the used block-table entries and seq_lens.

Timing: inputs larger than L2 (the headline's 4.4 GB pool; smaller pools rotated over
copies whose total exceeds 4x the L2 size; the tiny workload flushes L2 before each call);
W untimed calls, then K calls bracketed by a barrier and a device synchronisation, timed
with CUDA events on the launching stream; the maximum over ranks is reported. Under
torchrun every rank runs its own copy of the workload on its own GPU (independent
sequences, no collective on the data path): weak scaling.
"""
from __future__ import annotations

import argparse
import ctypes
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "q8-KV decode attention: µs/call and effective KV GB/s (% of B200 HBM peak)"
UNIT = "GB/s"
DEFAULT_WORKLOAD = 4  # bandwidth: the largest single-GPU workload (4.44 GB per call)
L2_BYTES = 126 * 1024 * 1024
FALLBACK_PEAK_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0
LAUNCHES_PER_CALL = 2  # decode kernel + split combine kernel
PARITY_MAX_ABS, PARITY_REL_L2 = 1e-4, 1e-5  # output tolerance against the fp64 oracle


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--config", type=int, default=DEFAULT_WORKLOAD)
    ap.add_argument("--batch", type=int, default=0,
                    help="run the workload's recipe with this many sequences instead (a "
                         "smaller case of the same kernel, e.g. for an ncu capture)")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-legs", action="store_true",
                    help="skip the per-workload legs (the other workloads, group 8)")
    ap.add_argument("--no-accuracy", action="store_true",
                    help="skip the q8-vs-fp32 information report")
    ap.add_argument("--no-cache-write", action="store_true",
                    help="skip the KV-cache write information report")
    ap.add_argument("--no-multi-query", action="store_true",
                    help="skip the multi-query decode information report")
    ap.add_argument("--no-quest", action="store_true",
                    help="skip the QUEST block-metadata information report")
    ap.add_argument("--no-q4", action="store_true",
                    help="skip the q4_0-cache decode information report")
    ap.add_argument("--multi-query-only", type=int, default=0, metavar="NQ",
                    help="instead of the headline: only the multi-query report on the 16 x "
                         "4096-token GQA workload with NQ query tokens per sequence (one "
                         "JSON line; e.g. for an ncu capture of that call's kernels)")
    ap.add_argument("--accuracy-study", action="store_true",
                    help="instead of timing: the q8-vs-fp32 output error study over the "
                         "workloads and K/V distributions (one JSON line)")
    return ap.parse_args()


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def reduce_max(x: float, pg, device) -> float:
    """Maximum of a per-rank time over all ranks (the slowest rank bounds the job)."""
    if pg is None:
        return x
    import torch

    t = torch.tensor([x], dtype=torch.float64, device=device)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def whole_job_gbs(bytes_per_rank: int, world: int, ms_per_step: float) -> float:
    """Whole-job throughput: every rank processes its own copy of the workload."""
    return bytes_per_rank * world / (ms_per_step * 1e-3) / 1e9


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_PEAK_GBS, "fallback"


class ClockSampler:
    """SM clock and clock-event reasons of one GPU, polled through NVML every 2 ms in a
    background thread, so that even a timed region of a few milliseconds holds samples."""

    REASONS = (("hw_slowdown", 0x8), ("sw_thermal_slowdown", 0x20),
               ("hw_thermal_slowdown", 0x40), ("hw_power_brake_slowdown", 0x80),
               ("sw_power_cap", 0x4))

    def __init__(self, device):
        self.samples = []  # (host monotonic time, sm MHz, reason bits)
        self.h = None
        self.max_mhz = None
        self._stop = threading.Event()
        self.thread = None
        try:
            import pynvml
            import torch

            pynvml.nvmlInit()
            idx = torch.cuda._get_nvml_device_index(device)
            self.nvml = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(idx)
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM))
        except Exception:
            self.h = None

    def start(self):
        if self.h is None:
            return self
        nv = self.nvml

        def run():
            while not self._stop.is_set():
                try:
                    sm = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                    rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                    self.samples.append((time.monotonic(), float(sm), int(rs)))
                except Exception:
                    pass
                self._stop.wait(0.002)

        self.thread = threading.Thread(target=run, daemon=True)
        self.thread.start()
        return self

    def stop(self):
        self._stop.set()
        if self.thread is not None:
            self.thread.join(timeout=2)

    def summary(self, t0: float, t1: float):
        """Median SM clock and the union of reasons over the samples taken between host
        times t0 and t1 (the timed region); when none falls inside, the nearest sample
        on either side."""
        if self.h is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"],
                    "samples": 0}
        s = list(self.samples)
        inside = [x for x in s if t0 <= x[0] <= t1]
        if not inside and s:
            before = [x for x in s if x[0] < t0][-1:]
            after = [x for x in s if x[0] > t1][:1]
            inside = before + after
        bits = 0
        for x in inside:
            bits |= x[2]
        return {"sm_mhz": statistics.median([x[1] for x in inside]) if inside else None,
                "sm_max_mhz": self.max_mhz,
                "reasons": [n for n, b in self.REASONS if bits & b],
                "samples": len(inside)}


# ------------------------------------------------------------------ workloads on the device


def n_pool_copies(pool_bytes: int) -> int:
    """Device copies of the KV pool that the timed calls rotate over: enough for the copies
    to exceed 4x the L2 size, 1 when the pool alone is that large, 0 (flush L2 before every
    call instead) when even 64 copies would not be."""
    if pool_bytes >= 4 * L2_BYTES:
        return 1
    n = math.ceil(4 * L2_BYTES / pool_bytes) + 1
    return n if n <= 64 else 0


def pool_bytes_of(w) -> int:
    return int(w.k.nbytes + w.v.nbytes + w.ks.nbytes + w.vs.nbytes)


def l2_note(w) -> str:
    pb = pool_bytes_of(w)
    n = n_pool_copies(pb)
    if n == 1:
        return f"inputs larger than L2: {pb / 1e9:.2f} GB KV pool > {L2_BYTES / 1e6:.0f} MB L2"
    if n == 0:
        return (f"L2 flushed before every call (a {2 * L2_BYTES / 1e6:.0f} MB buffer written); "
                f"calls timed one at a time")
    return (f"inputs larger than L2: KV pool rotated over {n} copies "
            f"({n * pb / 1e6:.0f} MB > {L2_BYTES / 1e6:.0f} MB L2)")


def workload_config(w, world: int) -> dict:
    """The `config` of a JSON line; both arms print the same dict for the same workload."""
    c = w.cfg
    lens = w.seq_lens
    return {"workload": c.name, "B": c.B, "n_q_heads": c.n_q_heads, "n_kv_heads": c.n_kv_heads,
            "head_dim": c.head_dim, "kv_block_size": c.block_size,
            "seq_len": int(lens.max()) if lens.min() == lens.max() else
            f"ragged {int(lens.min())}..{int(lens.max())} (sum {int(lens.sum())})",
            "num_kv_blocks": w.num_blocks, "algorithmic_bytes": w.algorithmic_bytes(),
            "k_dist": c.k_dist, "v_dist": c.v_dist, "k_bias_std": c.k_bias_std, "seed": c.seed,
            "l2": l2_note(w), "parallelism": f"replicas{world}"}


def sample_pairs(w, n_rows: int, seed: int):
    """Random (sequence, head) rows of sequences with tokens, plus the first and last head of
    the longest and the shortest sequence."""
    import numpy as np

    rng = np.random.default_rng(seed)
    live = np.flatnonzero(w.seq_lens > 0)
    Hq = w.cfg.n_q_heads
    pairs = {(int(live[i]), int(h)) for i, h in zip(rng.integers(0, len(live), n_rows),
                                                    rng.integers(0, Hq, n_rows))}
    for b in (int(live[np.argmax(w.seq_lens[live])]), int(live[np.argmin(w.seq_lens[live])])):
        pairs |= {(b, 0), (b, Hq - 1)}
    return sorted(pairs)


def parity_rows(w, got, n_rows: int, seed: int) -> dict:
    """The CUDA output against the fp64 oracle on sampled rows (every row when the workload
    has at most n_rows): max |gpu - oracle| and relative L2, the outputs-equal column."""
    import numpy as np

    import oracle

    cache = oracle.PagedCache(w.k, w.v, w.ks, w.vs, w.block_table, w.seq_lens,
                              w.cfg.n_q_heads, w.scale)
    B, Hq = w.cfg.B, w.cfg.n_q_heads
    t = time.perf_counter()
    if B * Hq <= n_rows:
        ref = oracle.decode_all(cache, w.q).reshape(B * Hq, -1)
        sel = np.asarray(got, np.float64).reshape(B * Hq, -1)
        rows = B * Hq
    else:
        pairs = sample_pairs(w, n_rows, seed)
        ref = oracle.decode_pairs(cache, w.q, pairs)
        sel = np.stack([np.asarray(got[b, h], np.float64) for b, h in pairs])
        rows = len(pairs)
    d = sel - ref
    max_abs = float(np.abs(d).max())
    rel = float(np.linalg.norm(d) / max(np.linalg.norm(ref), 1e-300))
    return {"rows": rows, "of_rows": B * Hq, "max_abs": max_abs, "rel_l2": rel,
            "within_tolerance": bool(np.all(np.isfinite(sel)) and max_abs <= PARITY_MAX_ABS
                                     and rel <= PARITY_REL_L2),
            "tolerance": {"max_abs": PARITY_MAX_ABS, "rel_l2": PARITY_REL_L2},
            "oracle_s": round(time.perf_counter() - t, 2)}


class DeviceWorkload:
    """A workload on the device with its KV pool copies and prepared C-ABI argument sets
    (one per pool copy), so that a timed call costs one foreign call and no marshalling."""

    def __init__(self, w, dev, stream):
        import numpy as np
        import torch

        import decode_attention_int8_b200 as q8

        self.w, self.dev, self.stream = w, dev, stream
        t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)
        self.n_copies = n_pool_copies(pool_bytes_of(w))
        self.q = t(w.q)
        self.bt = t(w.block_table)
        self.lens = t(w.seq_lens)
        self.pools = [(t(w.k), t(w.v), t(w.ks), t(w.vs)) for _ in range(max(1, self.n_copies))]
        self.out = torch.empty(self.q.shape, dtype=torch.float32, device=dev)
        self.flush = (torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev)
                      if self.n_copies == 0 else None)
        c = w.cfg
        self.geo = (c.B, c.n_q_heads, c.n_kv_heads, c.head_dim, c.block_size,
                    w.max_blocks_per_seq, w.num_blocks)
        self.sp = ctypes.c_void_p(stream.cuda_stream)
        self.fn = q8.lib().q8kv_decode_attn
        self.q8 = q8
        self.argsets = [self.args(self.out, self.q, self.bt, self.lens, pool)
                        for pool in self.pools]

    def args(self, out, q, bt, lens, pool=None, stream=None):
        P = lambda x: ctypes.c_void_p(x.data_ptr())
        k, v, ks, vs = pool or self.pools[0]
        sp = self.sp if stream is None else ctypes.c_void_p(stream.cuda_stream)
        return (P(out), P(q), P(k), P(v), P(ks), P(vs), P(bt), P(lens), *self.geo,
                ctypes.c_float(self.w.scale), sp)

    def call(self, i: int):
        st = self.fn(*self.argsets[i % len(self.argsets)])
        if st != 0:
            raise self.q8.Q8KVError(st, "q8kv_decode_attn")

    def time_calls(self, n: int) -> float:
        """ms per call of n calls: back to back between two events on the launching stream
        (no event between calls, which would break the programmatic-dependent-launch overlap
        of consecutive calls), or, for a flushed workload, the median of calls timed one at
        a time after an L2 flush each."""
        import torch

        if self.flush is None:
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(self.stream)
            for i in range(n):
                self.call(i)
            e1.record(self.stream)
            e1.synchronize()
            return e0.elapsed_time(e1) / n
        times = []
        for i in range(n):
            self.flush.fill_(i & 0xff)
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(self.stream)
            self.call(i)
            e1.record(self.stream)
            e1.synchronize()
            times.append(e0.elapsed_time(e1))
        return statistics.median(times)

    def isolated_us(self, n: int) -> float:
        """Median of single calls between their own events (information)."""
        import torch

        iso = []
        for i in range(n):
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(self.stream)
            self.call(i)
            e1.record(self.stream)
            e1.synchronize()
            iso.append(e0.elapsed_time(e1))
        return statistics.median(iso) * 1e3

    def result(self):
        import torch

        self.call(0)
        torch.cuda.synchronize(self.dev)
        return self.out.cpu().numpy()


def e2e_pipelined(dw, steps: int, pg):
    """End to end through the C ABI with host buffers, as a serving loop runs it: every step
    copies that step's q, block table and seq_lens from pinned host memory to the device,
    runs the call, and copies `out` back to pinned host memory. The copies run on their own
    streams into double buffers, so step i + 1's inputs move while step i computes; the
    events between the streams keep every buffer's reads after its writes. Timed with two
    events on the compute stream around all steps."""
    import torch

    w, dev, comp = dw.w, dw.dev, dw.stream
    hq = torch.from_numpy(w.q).pin_memory()
    hbt = torch.from_numpy(w.block_table).pin_memory()
    hlens = torch.from_numpy(w.seq_lens).pin_memory()
    hout = [torch.empty(dw.out.shape, dtype=torch.float32).pin_memory() for _ in range(2)]
    dq = [torch.empty_like(dw.q) for _ in range(2)]
    dbt = [torch.empty_like(dw.bt) for _ in range(2)]
    dlens = [torch.empty_like(dw.lens) for _ in range(2)]
    dout = [torch.empty_like(dw.out) for _ in range(2)]
    args = [dw.args(dout[j], dq[j], dbt[j], dlens[j], stream=comp) for j in range(2)]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()
    ev_in, ev_comp, ev_out = [ev(), ev()], [ev(), ev()], [ev(), ev()]
    used = [False, False]

    def h2d(i):
        j = i % 2
        if used[j]:
            s_in.wait_event(ev_comp[j])  # the call that last read buffer j has finished
        with torch.cuda.stream(s_in):
            dq[j].copy_(hq, non_blocking=True)
            dbt[j].copy_(hbt, non_blocking=True)
            dlens[j].copy_(hlens, non_blocking=True)
        ev_in[j].record(s_in)

    def run(n):
        for j in range(2):
            used[j] = False
        h2d(0)
        for i in range(n):
            j = i % 2
            if i + 1 < n:
                h2d(i + 1)
            comp.wait_event(ev_in[j])
            if used[j]:
                comp.wait_event(ev_out[j])  # out[j] of step i - 2 has reached the host
            st = dw.fn(*args[j])
            if st != 0:
                raise dw.q8.Q8KVError(st, "q8kv_decode_attn")
            used[j] = True
            ev_comp[j].record(comp)
            s_out.wait_event(ev_comp[j])
            with torch.cuda.stream(s_out):
                hout[j].copy_(dout[j], non_blocking=True)
            ev_out[j].record(s_out)
        for j in range(2):
            comp.wait_event(ev_out[j])

    run(3)
    torch.cuda.synchronize(dev)
    if pg is not None:
        pg.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(comp)
    s_in.wait_event(e0)
    run(steps)
    e1.record(comp)
    torch.cuda.synchronize(dev)
    ms = reduce_max(e0.elapsed_time(e1) / steps, pg, dev)
    return ms, {"h2d_bytes_per_step": int(w.q.nbytes + w.block_table.nbytes + w.seq_lens.nbytes),
                "d2h_bytes_per_step": int(w.q.nbytes), "steps": steps,
                "pipeline": "inputs of step i+1 copied during step i (copy streams, double "
                            "buffers)"}


def bench_leg(w, dev, stream, min_calls=50, target_s=0.25, parity_n=64, seed=0):
    """One workload as an information leg of the line: µs per call (back to back, rotated
    pools or flushed L2), bandwidth, fractions of the measured and the nominal HBM peak,
    the clocks during its timed calls, and sampled-row parity against the oracle."""
    import torch

    dw = DeviceWorkload(w, dev, stream)
    for i in range(5):
        dw.call(i)
    torch.cuda.synchronize(dev)
    est = dw.time_calls(10)
    n = max(min_calls, int(target_s / max(est * 1e-3, 1e-6)))
    if dw.flush is not None:
        n = min(n, 400)
    sampler = ClockSampler(dev).start()
    time.sleep(0.02)
    h0 = time.monotonic()
    ms = dw.time_calls(n)
    h1 = time.monotonic()
    sampler.stop()
    algo = w.algorithmic_bytes()
    peak, peak_kind = measured_peak()
    gbs = algo / (ms * 1e-3) / 1e9
    got = dw.result()
    leg = {"config": workload_config(w, 1), "us_per_call": round(ms * 1e3, 3), "calls": n,
           "GB/s": round(gbs, 2), "frac_of_measured_hbm": round(gbs / peak, 4),
           "frac_of_8TBps_nominal": round(gbs / NOMINAL_HBM_GBS, 4), "peak_kind": peak_kind,
           "clocks": sampler.summary(h0, h1),
           "device_errors": dw.q8.q8kv_device_errors(clear=True),
           "parity_vs_oracle": parity_rows(w, got, parity_n, seed)}
    return leg, dw


def read_floor(nbytes: int, dev, stream, calls: int = 200) -> dict:
    """Context for a leg: a library kernel (torch's fp32 sum) reading the same number of
    bytes, timed like the leg (back-to-back calls, rotated over copies larger than 4x L2).
    What one call of that size costs a plain streaming read, launch and tail included."""
    import torch

    n = max(1, nbytes // 4)
    copies = max(1, n_pool_copies(4 * n))
    bufs = [torch.ones(n, dtype=torch.float32, device=dev) for _ in range(copies)]
    out = torch.empty((), dtype=torch.float32, device=dev)
    with torch.cuda.stream(stream):
        for i in range(10):
            torch.sum(bufs[i % copies], dim=0, out=out)
        torch.cuda.synchronize(dev)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(calls):
            torch.sum(bufs[i % copies], dim=0, out=out)
        e1.record(stream)
    torch.cuda.synchronize(dev)
    us = e0.elapsed_time(e1) / calls * 1e3
    peak, _ = measured_peak()
    del bufs
    return {"kernel": "torch.sum over fp32 (library)", "bytes": 4 * n,
            "us_per_call": round(us, 3), "frac_of_measured_hbm": round(4 * n / (us * 1e-6) / 1e9 / peak, 4)}


def cpu_sample_rate(w, seconds: float, seed: int = 0):
    """The oracle as it stands, single-threaded, on random (sequence, head) rows of the
    workload for about `seconds`; bytes counted pro rata to the rows done. Returns
    (GB/s, rows done, rows in the workload, elapsed s)."""
    import numpy as np

    import oracle

    cache = oracle.PagedCache(w.k, w.v, w.ks, w.vs, w.block_table, w.seq_lens,
                              w.cfg.n_q_heads, w.scale)
    B, Hq = w.cfg.B, w.cfg.n_q_heads
    pairs_all = [(b, h) for b in range(B) for h in range(Hq) if w.seq_lens[b] > 0]
    rng = np.random.default_rng(seed)
    done, t0 = 0, time.perf_counter()
    chunk = 1
    while True:
        sel = rng.choice(len(pairs_all), min(chunk, len(pairs_all)), replace=False)
        oracle.decode_pairs(cache, w.q, [pairs_all[j] for j in sel])
        done += len(sel)
        dt = time.perf_counter() - t0
        if dt >= seconds:
            break
        chunk = min(len(pairs_all), max(1, chunk * 2 if dt < seconds / 4 else chunk))
    gbs = w.algorithmic_bytes() * done / len(pairs_all) / dt / 1e9
    return gbs, done, len(pairs_all), dt


def cpu_baseline(w, seconds=12.0):
    gbs, done, total, dt = cpu_sample_rate(w, seconds)
    return {"value": round(gbs, 4), "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": f"{done} random (sequence, head) rows of {total} ({w.cfg.name}), "
                      f"{dt:.1f} s, single-threaded C oracle; bytes counted pro rata"}


def q8_vs_fp32(w, got, n_seqs=4, heads_per_seq=16, seed=0):
    """Information only: how far the q8 path's output is from attention over the unquantised
    fp32 q, K, V (plain fp64 numpy softmax(q K^T * scale) V on sampled (sequence, head)
    rows; each sampled sequence's fp32 rows are regenerated once from their random
    streams). This measures the int8 quantisation itself, not the kernel's arithmetic."""
    import numpy as np

    from decode_attention_int8_b200 import inputs

    c = w.cfg
    bs = c.block_size
    G = c.n_q_heads // c.n_kv_heads
    rng = np.random.default_rng(seed)
    live = np.flatnonzero(w.seq_lens > 0)
    diffs, refs = [], []
    for b in rng.choice(live, size=min(n_seqs, len(live)), replace=False):
        L = int(w.seq_lens[b])
        t = np.arange(L)
        slot = w.block_table[b, t // bs].astype(np.int64) * bs + t % bs
        k32 = inputs.fp32_rows(w, "k", slot)
        v32 = inputs.fp32_rows(w, "v", slot)
        for h in rng.choice(c.n_q_heads, size=min(heads_per_seq, c.n_q_heads), replace=False):
            kf = k32[:, h // G].astype(np.float64)
            vf = v32[:, h // G].astype(np.float64)
            sc = kf @ w.q[b, h].astype(np.float64) * w.scale
            pr = np.exp(sc - sc.max())
            ref = pr @ vf / pr.sum()
            refs.append(ref)
            diffs.append(np.asarray(got[b, h], np.float64) - ref)
    d, r = np.array(diffs), np.array(refs)
    return {"max_abs": float(np.abs(d).max()), "rel_l2": float(np.linalg.norm(d) / np.linalg.norm(r)),
            "rows": len(refs), "workload": c.name,
            "reference": "fp64 attention over the unquantised fp32 q, K, V"}


def _err_stats(got, ref):
    import numpy as np

    d = np.asarray(got, np.float64) - np.asarray(ref, np.float64)
    r = np.asarray(ref, np.float64)
    return {"max_abs": float(np.abs(d).max()), "mean_abs": float(np.abs(d).mean()),
            "rel_l2": float(np.linalg.norm(d) / np.linalg.norm(r)),
            "row_rel_l2_p99": float(np.percentile(np.linalg.norm(d, axis=1) /
                                                  np.maximum(np.linalg.norm(r, axis=1), 1e-300),
                                                  99))}


def accuracy_rows(w, out_gpu, n_rows, seed, max_seqs=8):
    """Error of the q8 path against attention over the unquantised fp32 q, K, V on sampled
    (sequence, head) rows: the CUDA output and the oracle's q8 decode, each against the
    oracle's fp64 attention of the fp32 data (the fp32 rows of the sampled sequences are
    regenerated from their random streams, so at most max_seqs sequences are sampled and
    the rows are spread over their heads)."""
    import numpy as np

    import oracle
    from decode_attention_int8_b200 import inputs

    c = w.cfg
    bs, Hk, D = c.block_size, c.n_kv_heads, c.head_dim
    rng = np.random.default_rng(seed)
    live = [b for b in range(c.B) if w.seq_lens[b] > 0]
    seqs = rng.choice(live, size=min(max_seqs, len(live), n_rows), replace=False)
    per = max(1, n_rows // len(seqs))
    pairs = sorted({(int(b), int(h)) for b in seqs
                    for h in rng.choice(c.n_q_heads, size=min(per, c.n_q_heads),
                                        replace=False)})
    cache = oracle.PagedCache(w.k, w.v, w.ks, w.vs, w.block_table, w.seq_lens, c.n_q_heads,
                              w.scale)
    q8_oracle = oracle.decode_pairs(cache, w.q, pairs)
    fp32, gpu = [], []
    for b in sorted({b for b, _ in pairs}):
        L = int(w.seq_lens[b])
        nblk = -(-L // bs)
        blocks = w.block_table[b, :nblk].astype(np.int64)
        slots = (blocks[:, None] * bs + np.arange(bs)[None, :]).reshape(-1)
        if w.k32 is not None:  # the workload kept its unquantised draws
            k32 = w.k32.reshape(-1, Hk, D)[slots].reshape(nblk, bs, Hk, D)
            v32 = w.v32.reshape(-1, Hk, D)[slots].reshape(nblk, bs, Hk, D)
        else:
            k32 = inputs.fp32_rows(w, "k", slots).reshape(nblk, bs, Hk, D)
            v32 = inputs.fp32_rows(w, "v", slots).reshape(nblk, bs, Hk, D)
        compact = oracle.PagedCache(w.k[blocks], w.v[blocks], w.ks[blocks], w.vs[blocks],
                                    np.arange(nblk, dtype=np.int32)[None, :],
                                    np.array([L], np.int32), c.n_q_heads, w.scale)
        for bb, h in pairs:
            if bb == b:
                fp32.append(oracle.attn_fp32(compact, w.q[b:b + 1], k32, v32, 0, h))
                gpu.append(out_gpu[b, h])
    fp32, gpu = np.array(fp32), np.array(gpu)
    return {"rows": len(pairs), "cuda_q8_vs_fp32": _err_stats(gpu, fp32),
            "oracle_q8_vs_fp32": _err_stats(q8_oracle, fp32),
            "cuda_vs_oracle_q8_max_abs": float(np.abs(gpu - q8_oracle).max())}


def run_accuracy_study(args):
    """The q8-vs-fp32 comparison the walk-through announces as its next article: how far the q8
    path's attention output is from attention over the unquantised fp32 data, per workload
    and per K/V distribution, for the CUDA kernel and for the oracle's q8 arithmetic."""
    import numpy as np
    import torch

    import decode_attention_int8_b200 as q8
    from decode_attention_int8_b200 import inputs

    _, rank, local = dist_env()
    if rank != 0:
        return 0
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)

    def gpu_out(w):
        t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)
        out = torch.empty(w.q.shape, dtype=torch.float32, device=dev)
        q8.q8kv_decode_attn(out, t(w.q), t(w.k), t(w.v), t(w.ks), t(w.vs), t(w.block_table),
                            t(w.seq_lens), w.scale)
        torch.cuda.synchronize(dev)
        return out.cpu().numpy()

    results = []
    # the first three workloads whole (their unquantised draws kept); the two multi-GB ones
    # with their recipe on 8 sequences (the fp32 copies of 4 GB pools would not fit the
    # host budget of this study)
    C = inputs.WORKLOADS
    lens3 = inputs._seq_lens(C[3])[:8]
    study = [(C[0], inputs.make(C[0], keep_fp32=True), 64),
             (C[1], inputs.make(C[1], keep_fp32=True), 256),
             (C[2], inputs.make(C[2], keep_fp32=True), 32),
             (C[3], inputs.make_custom(8, 64, 8, 128, lens3, 128, k_dist="student_t3",
                                       v_dist="student_t3", seed=3, keep_fp32=True,
                                       name="ragged_outliers (8 of its 64 sequences)"), 96),
             (C[4], inputs.make_custom(8, 32, 8, 128, [8192] * 8, 64, seed=4, keep_fp32=True,
                                       name="bandwidth (8 of its 256 sequences)"), 96)]
    for i, (cfg, w, n) in enumerate(study):
        r = accuracy_rows(w, gpu_out(w), n, seed=i)
        r.update({"workload": w.cfg.name, "k_dist": cfg.k_dist, "v_dist": cfg.v_dist,
                  "k_bias_std": cfg.k_bias_std})
        results.append(r)
        print(json.dumps({"partial": r}), flush=True)
    del study
    # distributions at one shape: 4 sequences of 4096 tokens, 32/8 heads, block 64
    for name, kw in [("normal", {}), ("student_t3 K and V", dict(k_dist="student_t3",
                                                                 v_dist="student_t3")),
                     ("K bias std 2", dict(k_bias_std=2.0)), ("K bias std 6", dict(k_bias_std=6.0)),
                     ("student_t3 K + bias 6", dict(k_dist="student_t3", k_bias_std=6.0))]:
        w = inputs.make_custom(4, 32, 8, 128, [4096] * 4, 64, seed=50, keep_fp32=True, **kw)
        r = accuracy_rows(w, gpu_out(w), 128, seed=50)
        r.update({"workload": f"4 x 4096 tokens, 32/8 heads: {name}"})
        results.append(r)
        print(json.dumps({"partial": r}), flush=True)
    print(json.dumps({"study": "q8 KV + q8 Q attention output vs fp64 attention over the "
                               "unquantised fp32 q, K, V", "results": results}), flush=True)
    return 0


def run_reference(args):
    """--impl reference: the oracle on the host cores, on this arm's workload and metric.
    Each step decodes a bounded random sample of (sequence, head) rows; the workload's
    algorithmic bytes are counted pro rata to the rows done."""
    world, rank, _ = dist_env()
    if rank != 0:
        return 0
    import numpy as np

    import oracle
    from decode_attention_int8_b200 import inputs

    w = make_workload(args)
    cache = oracle.PagedCache(w.k, w.v, w.ks, w.vs, w.block_table, w.seq_lens,
                              w.cfg.n_q_heads, w.scale)
    B, Hq = w.cfg.B, w.cfg.n_q_heads
    pairs_all = [(b, h) for b in range(B) for h in range(Hq) if w.seq_lens[b] > 0]
    # time one pair to size a step so that the whole run takes about two minutes
    t = time.perf_counter()
    oracle.decode_pairs(cache, w.q, pairs_all[:1])
    per_pair = max(time.perf_counter() - t, 1e-5)
    budget = min(2.0, 120.0 / max(1, args.steps + args.warmup))
    n_pairs = int(max(1, min(len(pairs_all), budget / per_pair)))
    rng = np.random.default_rng(0)

    def step():
        sel = rng.choice(len(pairs_all), n_pairs, replace=False)
        oracle.decode_pairs(cache, w.q, [pairs_all[j] for j in sel])
        return n_pairs

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    done = 0
    for _ in range(args.steps):
        done += step()
    dt = time.perf_counter() - t0
    gbs = w.algorithmic_bytes() * (done / len(pairs_all)) / dt / 1e9
    line = {"impl": "reference", "metric": METRIC, "value": round(gbs, 4), "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(dt / args.steps * 1e3, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(w, world),
            "cpu_baseline": {"value": round(gbs, 4), "unit": UNIT, "cores": 1, "kind": "oracle",
                             "sample": f"{n_pairs} random (sequence, head) rows per step of "
                                       f"{len(pairs_all)}; bytes counted pro rata"},
            "e2e": {"value": round(gbs, 4), "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def make_workload(args):
    """The workload of --config, or its recipe with --batch sequences."""
    from decode_attention_int8_b200 import inputs

    cfg = inputs.WORKLOADS[args.config]
    if getattr(args, "batch", 0):
        cfg = inputs.with_config(cfg, B=args.batch, name=f"{cfg.name}_b{args.batch}")
    return inputs.make(cfg)


# group-8 reading of the batched GQA workload's label: 64 q heads over its 8 KV heads
def group8_workload():
    from decode_attention_int8_b200 import inputs

    c = inputs.WORKLOADS[1]
    return inputs.make_custom(c.B, 64, c.n_kv_heads, c.head_dim, [c.seq_len] * c.B,
                              c.block_size, seed=c.seed, name="gqa_batch_group8")


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    if args.accuracy_study:
        return run_accuracy_study(args)
    if args.multi_query_only:
        return run_multi_query_only(args)
    world, rank, local = dist_env()
    import torch

    import decode_attention_int8_b200 as q8
    from decode_attention_int8_b200 import inputs

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
        pg = dist

    stream = torch.cuda.current_stream(dev)
    w = make_workload(args)
    algo = w.algorithmic_bytes()
    dw = DeviceWorkload(w, dev, stream)
    q8.q8kv_device_errors(clear=True)

    # warm-up (also sizes the library workspace outside the timed region)
    for i in range(max(args.warmup, 1)):
        dw.call(i)
    torch.cuda.synchronize(dev)

    def barrier():
        if pg is not None:
            pg.barrier()

    # timed region: K calls (back to back between two CUDA events on the launching stream,
    # or one at a time after an L2 flush for a pool too small to rotate)
    sampler = ClockSampler(dev).start()
    time.sleep(0.05)
    barrier()
    torch.cuda.synchronize(dev)
    host_t0 = time.monotonic()
    ms_per_step = dw.time_calls(args.steps)
    torch.cuda.synchronize(dev)
    host_t1 = time.monotonic()
    barrier()
    sampler.stop()
    clocks = sampler.summary(host_t0, host_t1)
    ms_per_step = reduce_max(ms_per_step, pg, dev)
    value = whole_job_gbs(algo, world, ms_per_step)
    isolated_us = dw.isolated_us(min(100, max(10, args.steps)))
    got = dw.result()
    dev_errors = q8.q8kv_device_errors(clear=True)

    e2e = None
    if not args.no_e2e:
        e2e_ms, e2e_info = e2e_pipelined(dw, max(10, args.steps), pg)
        e2e = {"value": round(whole_job_gbs(algo, world, e2e_ms), 2), "unit": UNIT,
               "us_per_step": round(e2e_ms * 1e3, 3), **e2e_info}

    peak, peak_kind = measured_peak()
    achieved = algo / (ms_per_step * 1e-3) / 1e9
    traffic = recorded_traffic(w.cfg.name, "decode")
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 6),
        "us_per_call": round(ms_per_step * 1e3, 3),
        "us_per_call_isolated": round(isolated_us, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "s8", "data": "synthetic",
        "config": workload_config(w, world),
        "roofline": {"bound": "hbm", "achieved": round(achieved, 2), "peak": peak,
                     "peak_kind": peak_kind, "unit": "GB/s", "frac": round(achieved / peak, 4),
                     "frac_of_8TBps_nominal": round(achieved / NOMINAL_HBM_GBS, 4),
                     "traffic": traffic,
                     "kernel": "q8kv::decode_kernel + q8kv::combine_kernel (one call)",
                     "kernel_us": round(ms_per_step * 1e3, 3)},
        "gpu_launches": LAUNCHES_PER_CALL * args.steps,
        "clocks": clocks,
        "device_errors": dev_errors,
    }
    if e2e is not None:
        line["e2e"] = e2e
    if rank == 0:
        line["parity_vs_oracle"] = parity_rows(w, got, 64, seed=args.config)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w)
    del dw
    torch.cuda.empty_cache()

    # information legs, after the timed region: every other workload (and the group-8
    # reading of the batched one), each timed and checked against the oracle on its own
    info = world == 1  # the scaling runs time the headline only
    if info and not args.no_legs:
        legs = {}
        others = [i for i in range(len(inputs.WORKLOADS)) if i != args.config]
        for i in others + ["group8"]:
            wi = group8_workload() if i == "group8" else inputs.make(i)
            leg, dwi = bench_leg(wi, dev, stream, seed=100 + (9 if i == "group8" else i))
            if wi.cfg.name in ("gqa_batch", "long_context"):
                # how close one call of this size can get: a plain read of the same bytes
                leg["read_floor"] = read_floor(wi.algorithmic_bytes(), dev, stream)
            if wi.cfg.name == "gqa_batch":
                if not args.no_multi_query:
                    # the same workload with n_queries new tokens per sequence (speculative
                    # decode), through q8kv_decode_attn_multi
                    line["multi_query"] = bench_multi_query(
                        wi, dwi.pools, dwi.bt, dwi.lens, dev, stream,
                        steps=max(10, min(args.steps, 2000)))
                if rank == 0 and world == 1 and not args.no_accuracy:
                    line["q8_vs_fp32"] = q8_vs_fp32(wi, dwi.result())
            legs[wi.cfg.name] = leg
            del dwi, wi
            torch.cuda.empty_cache()
        line["per_config"] = legs
    if info and not args.no_q4:
        line["q4_0_decode"] = bench_q4(dev, stream, steps=max(10, min(args.steps, 2000)))
        torch.cuda.empty_cache()
    if info and not args.no_cache_write:
        # the write path that fills the cache
        line["cache_write"] = bench_cache_write(dev, stream)
        torch.cuda.empty_cache()
    if info and not args.no_quest:
        line["quest_metadata"] = bench_quest(dev, stream)
    if pg is not None:
        pg.barrier()
        pg.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


CACHE_WRITE_SOURCES = ("q8kv_cache_write.cuh", "q8kv_cache_write_api.cuh", "q8kv_ptx.cuh")
QUEST_SOURCES = ("q8kv_quest.cuh", "q8kv_quest_api.cuh", "q8kv_ptx.cuh")
Q4_SOURCES = ("q8kv_q4.cuh", "q8kv_q4_api.cuh", "q8kv_ptx.cuh", "q8kv_qquant.cuh", "q8kv_decode.cuh")


def source_hash(kernel: str = "decode") -> str:
    """Hash of the sources a kernel is built from (traffic figures are valid only for the
    exact kernel): the cache write's, the QUEST metadata's or the q4_0 decode's own kernel
    and host files and the helpers they include, or, for the q8 decode call, every other
    source of the library (its kernels, helpers and plan)."""
    import hashlib

    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "decode_attention_int8_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        if kernel == "cache_write":
            mine = name in CACHE_WRITE_SOURCES
        elif kernel == "quest":
            mine = name in QUEST_SOURCES
        elif kernel == "q4":
            mine = name in Q4_SOURCES
        else:
            mine = not name.startswith(("q8kv_cache_write", "q8kv_quest", "q8kv_q4"))
        if not mine:
            continue
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(name: str, kernel: str = "decode"):
    """DRAM bytes per launch recorded under profiles/ for this workload and exact source."""
    tpath = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(tpath):
        return None
    h = source_hash(kernel)
    with open(tpath) as f:
        for ln in f:
            parts = ln.split()
            if len(parts) == 3 and not ln.startswith("#") and parts[0] == name and parts[1] == h:
                return int(parts[2])
    return None


def run_multi_query_only(args):
    """--multi-query-only NQ: the multi-query report alone (one GPU, one JSON line)."""
    import torch

    from decode_attention_int8_b200 import inputs

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    w = inputs.make(1)
    _, dw = bench_leg(w, dev, stream, min_calls=3, target_s=0.0, parity_n=8, seed=101)
    res = bench_multi_query(w, dw.pools, dw.bt, dw.lens, dev, stream,
                            steps=max(args.steps, 1), warmup=max(args.warmup, 1),
                            nqs=(args.multi_query_only,))
    print(json.dumps({"metric": METRIC, "unit": UNIT, "multi_query": res}), flush=True)
    return 0


def bench_multi_query(w, pools, bt, lens, dev, stream, steps, warmup=20, nqs=(2, 4, 8)):
    """Information: q8kv_decode_attn_multi on the benchmark workload with nq new query
    tokens per sequence (causal), timed like the single-query call (back-to-back calls
    between two events, the same rotated KV pools). Algorithmic bytes: the KV bytes of one
    single-query call plus nq times its q and out bytes."""
    import numpy as np
    import torch

    import decode_attention_int8_b200 as q8
    from decode_attention_int8_b200 import inputs

    c = w.cfg
    fn = q8.lib().q8kv_decode_attn_multi
    sp = ctypes.c_void_p(stream.cuda_stream)
    P_ = lambda x: ctypes.c_void_p(x.data_ptr())
    peak, _ = measured_peak()
    res = {}
    for nq in nqs:
        if nq * c.group > 128:
            continue
        q = torch.from_numpy(inputs.multi_queries(c.B, nq, c.n_q_heads, c.head_dim,
                                                  seed=c.seed)).to(dev)
        out = torch.empty_like(q)
        q8.q8kv_decode_attn_multi(out, q, *pools[0], bt, lens, w.scale, stream=stream)
        argsets = [(P_(out), P_(q), P_(k), P_(v), P_(ks), P_(vs), P_(bt), P_(lens), c.B, nq,
                    c.n_q_heads, c.n_kv_heads, c.head_dim, c.block_size, w.max_blocks_per_seq,
                    w.num_blocks, ctypes.c_float(w.scale), sp) for (k, v, ks, vs) in pools]
        for i in range(warmup):
            fn(*argsets[i % len(argsets)])
        torch.cuda.synchronize(dev)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(steps):
            st = fn(*argsets[i % len(argsets)])
            if st != 0:
                raise q8.Q8KVError(st, "q8kv_decode_attn_multi")
        e1.record(stream)
        torch.cuda.synchronize(dev)
        ms = e0.elapsed_time(e1) / steps
        algo = w.algorithmic_bytes() + (nq - 1) * 2 * int(w.q.nbytes)
        gbs = algo / (ms * 1e-3) / 1e9
        res[f"nq{nq}"] = {"us_per_call": round(ms * 1e3, 3), "GB/s": round(gbs, 2),
                          "frac_of_measured_hbm": round(gbs / peak, 4),
                          "query_rows_per_kv_head": nq * c.group,
                          "algorithmic_bytes": algo}
    res["workload"] = (f"{c.name} with nq new query tokens per sequence (causal), "
                       f"q/out [{c.B}][nq][{c.n_q_heads}][{c.head_dim}]")
    return res


def bench_quest(dev, stream, steps=20, warmup=3, B=20, L=32768, Hk=8, bs=128):
    """Information: QUEST block metadata (q8kv_quest_metadata) on the CANN guide's benchmark
    shape (N = 8 KV heads, D = 128, block 128, B = 20 requests of 32768 tokens), over the q8
    K pool. Algorithmic bytes: the K codes and scales of every token, the used block-table
    and metadata-table entries, and both metadata arrays' used rows written."""
    import numpy as np
    import torch

    import decode_attention_int8_b200 as q8
    from decode_attention_int8_b200 import inputs

    w = inputs.make_custom(B, Hk, Hk, 128, [L] * B, bs, seed=42)
    meta, n_meta = inputs.quest_meta_table(w.seq_lens, bs, seed=42)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)
    k, ks, bt, lens, mt = t(w.k), t(w.ks), t(w.block_table), t(w.seq_lens), t(meta)
    mx = torch.empty((n_meta, bs, Hk, 128), dtype=torch.float32, device=dev)
    mn = torch.empty_like(mx)
    q8.q8kv_quest_metadata(mx, mn, k, ks, bt, lens, mt, stream=stream)
    fn = q8.lib().q8kv_quest_metadata
    P_ = lambda x: ctypes.c_void_p(x.data_ptr())
    a = (P_(mx), P_(mn), P_(k), P_(ks), P_(bt), P_(lens), P_(mt), B, Hk, 128, bs,
         int(bt.shape[1]), int(mt.shape[1]), w.num_blocks, n_meta,
         ctypes.c_void_p(stream.cuda_stream))
    for _ in range(warmup):
        fn(*a)
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        st = fn(*a)
        if st != 0:
            raise q8.Q8KVError(st, "q8kv_quest_metadata")
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ms = e0.elapsed_time(e1) / steps
    nkv = -(-L // bs)
    nmeta = -(-nkv // bs)
    algo = (B * L * Hk * (128 + 4) + 4 * B * nkv + 4 * B * nmeta + 4 * B
            + 2 * B * nmeta * bs * Hk * 128 * 4)
    peak, peak_kind = measured_peak()
    gbs = algo / (ms * 1e-3) / 1e9
    return {"workload": f"{B} requests x {L} tokens, {Hk} KV heads, D 128, block {bs} "
                        f"(the CANN guide's benchmark shape), q8 K pool {w.k.nbytes / 1e6:.0f} MB",
            "us_per_call": round(ms * 1e3, 3), "calls": steps, "algorithmic_bytes": algo,
            "roofline": {"bound": "hbm", "achieved": round(gbs, 2), "peak": peak,
                         "peak_kind": peak_kind, "unit": "GB/s", "frac": round(gbs / peak, 4),
                         "traffic": recorded_traffic("quest_b20_l32768", "quest"),
                         "kernel": "q8kv::quest_metadata_kernel"},
            "device_errors": q8.q8kv_device_errors(clear=True)}


def bench_q4(dev, stream, steps=2000, warmup=20):
    """Information: q8kv_decode_attn_q4 on the benchmark's 16 x 4096-token GQA workload with
    a q4_0 cache drawn from the same random streams (pool rotated over copies larger than
    the L2, back-to-back calls between two events)."""
    import numpy as np
    import torch

    import decode_attention_int8_b200 as q8
    from decode_attention_int8_b200 import inputs

    w = inputs.make_q4(1)
    c = w.cfg
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)
    pool_bytes = w.k4.nbytes + w.v4.nbytes + w.kd.nbytes + w.vd.nbytes
    n_copies = max(2, math.ceil(4 * L2_BYTES / pool_bytes) + 1)
    pools = [(t(w.k4), t(w.v4), t(w.kd.view(np.float16)), t(w.vd.view(np.float16)))
             for _ in range(n_copies)]
    q, bt, lens = t(w.q), t(w.block_table), t(w.seq_lens)
    out = torch.empty(q.shape, dtype=torch.float32, device=dev)
    q8.q8kv_decode_attn_q4(out, q, *pools[0], bt, lens, w.scale, stream=stream)
    fn = q8.lib().q8kv_decode_attn_q4
    P_ = lambda x: ctypes.c_void_p(x.data_ptr())
    sp = ctypes.c_void_p(stream.cuda_stream)
    args = [(P_(out), P_(q), P_(k), P_(v), P_(kd), P_(vd), P_(bt), P_(lens), c.B, c.n_q_heads,
             c.n_kv_heads, c.head_dim, c.block_size, w.max_blocks_per_seq, w.num_blocks,
             ctypes.c_float(w.scale), sp) for (k, v, kd, vd) in pools]
    for i in range(warmup):
        fn(*args[i % n_copies])
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(steps):
        st = fn(*args[i % n_copies])
        if st != 0:
            raise q8.Q8KVError(st, "q8kv_decode_attn_q4")
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ms = e0.elapsed_time(e1) / steps
    algo = w.algorithmic_bytes()
    peak, peak_kind = measured_peak()
    gbs = algo / (ms * 1e-3) / 1e9
    return {"workload": f"{c.name} with a q4_0 cache ({algo / 1e6:.1f} MB per call)",
            "us_per_call": round(ms * 1e3, 3), "calls": steps, "algorithmic_bytes": algo,
            "roofline": {"bound": "hbm", "achieved": round(gbs, 2), "peak": peak,
                         "peak_kind": peak_kind, "unit": "GB/s", "frac": round(gbs / peak, 4),
                         "traffic": recorded_traffic("gqa_batch_q4", "q4"),
                         "kernel": "q8kv::q4_decode_kernel + q8kv::q4_combine_kernel"},
            "l2": f"pool rotated over {n_copies} copies"}


def bench_cache_write(dev, stream, steps=50, warmup=5, step_B=16):
    """Information: the KV-cache write (q8kv_cache_write), timed like the decode call.

    prompt_fill: fresh fp32 K/V rows for all 65536 tokens of the 16 x 4096-token GQA
    workload (8 KV heads, head_dim 128) written to the slots of its permuted block table;
    537 MB of fp32 rows in and 138 MB of codes and scales out per call, more than the L2.
    decode_step: one new token per sequence (16 x 8 rows), the append of a decode step,
    bound by launch latency rather than by bandwidth."""
    import numpy as np
    import torch

    import decode_attention_int8_b200 as q8
    from decode_attention_int8_b200 import inputs

    cfg = inputs.WORKLOADS[1]
    rows = inputs.make_prompt_fill(cfg)
    n, Hk, D, bs = rows.n_tokens, cfg.n_kv_heads, cfg.head_dim, cfg.block_size
    P = int(rows.slots.max()) // bs + 1
    k = torch.zeros((P, bs, Hk, D), dtype=torch.int8, device=dev)
    v = torch.zeros_like(k)
    ks = torch.zeros((P, bs, Hk), dtype=torch.float32, device=dev)
    vs = torch.zeros_like(ks)
    kn = torch.from_numpy(rows.k_new).to(dev).view(n, Hk, D)
    vn = torch.from_numpy(rows.v_new).to(dev).view(n, Hk, D)
    slots = torch.from_numpy(rows.slots).to(dev)
    step_idx = torch.arange(step_B, device=dev) * (n // step_B) + (n // step_B - 1)
    s_kn, s_vn, s_slots = kn[step_idx].contiguous(), vn[step_idx].contiguous(), slots[step_idx]

    # one binding call checks the arguments; the timed loops then call the C ABI with
    # prepared arguments (like the decode benchmark), so host overhead stays small
    q8.q8kv_cache_write(k, v, ks, vs, kn, vn, slots, stream=stream)
    fn = q8.lib().q8kv_cache_write
    sp = ctypes.c_void_p(stream.cuda_stream)
    P_ = lambda x: ctypes.c_void_p(x.data_ptr())

    def timed(kn_, vn_, slots_):
        a = (P_(k), P_(v), P_(ks), P_(vs), P_(kn_), P_(vn_), P_(slots_), int(slots_.shape[0]),
             Hk, D, bs, P, Hk * D, sp)
        for _ in range(warmup):
            fn(*a)
        torch.cuda.synchronize(dev)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            st = fn(*a)
            if st != 0:
                raise q8.Q8KVError(st, "q8kv_cache_write")
        e1.record(stream)
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1) / steps

    q8.q8kv_device_errors(clear=True)
    ms_fill = timed(kn, vn, slots)
    ms_step = timed(s_kn, s_vn, s_slots)
    errs = q8.q8kv_device_errors(clear=True)
    # the same prompt fill into q4_0 pools (q8kv_cache_write_q4)
    del k, v, ks, vs
    k4 = torch.zeros((P, bs, Hk, D // 2), dtype=torch.uint8, device=dev)
    v4 = torch.zeros_like(k4)
    kd = torch.zeros((P, bs, Hk, D // 32), dtype=torch.int16, device=dev)
    vd = torch.zeros_like(kd)
    q8.q8kv_cache_write_q4(k4, v4, kd, vd, kn, vn, slots, stream=stream)
    fn4 = q8.lib().q8kv_cache_write_q4
    a4 = (P_(k4), P_(v4), P_(kd), P_(vd), P_(kn), P_(vn), P_(slots), n, Hk, D, bs, P, Hk * D, sp)
    for _ in range(warmup):
        fn4(*a4)
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        st = fn4(*a4)
        if st != 0:
            raise q8.Q8KVError(st, "q8kv_cache_write_q4")
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ms_q4 = e0.elapsed_time(e1) / steps
    errs |= q8.q8kv_device_errors(clear=True)
    n_valid = int(np.count_nonzero(rows.slots >= 0))
    algo_q4 = n_valid * Hk * 2 * (4 * D + D // 2 + 2 * (D // 32)) + 8 * n
    algo = rows.algorithmic_bytes()
    peak, peak_kind = measured_peak()
    achieved = algo / (ms_fill * 1e-3) / 1e9
    step_bytes = step_B * Hk * 2 * (5 * D + 4) + 8 * step_B
    return {
        "prompt_fill": {
            "workload": f"gqa_batch prompt fill: {n} tokens x {Hk} KV heads x {D}, block {bs}, "
                        f"permuted {P}-block table",
            "us_per_call": round(ms_fill * 1e3, 3), "calls": steps,
            "algorithmic_bytes": algo,
            "roofline": {"bound": "hbm", "achieved": round(achieved, 2), "peak": peak,
                         "peak_kind": peak_kind, "unit": "GB/s", "frac": round(achieved / peak, 4),
                         "traffic": recorded_traffic("gqa_prompt_fill", "cache_write"),
                         "kernel": "q8kv::cache_write_kernel<128>"},
            "l2": "inputs (537 MB of fp32 rows) and outputs (138 MB) larger than L2"},
        "prompt_fill_q4": {
            "workload": "the same prompt fill into q4_0 pools (q8kv_cache_write_q4)",
            "us_per_call": round(ms_q4 * 1e3, 3), "calls": steps, "algorithmic_bytes": algo_q4,
            "roofline": {"bound": "hbm", "achieved": round(algo_q4 / (ms_q4 * 1e-3) / 1e9, 2),
                         "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
                         "frac": round(algo_q4 / (ms_q4 * 1e-3) / 1e9 / peak, 4),
                         "traffic": None, "kernel": "q8kv::cache_write_q4_kernel<128>"}},
        "decode_step": {"workload": f"one new token per sequence: {step_B} x {Hk} rows",
                        "us_per_call": round(ms_step * 1e3, 3), "calls": steps,
                        "algorithmic_bytes": step_bytes,
                        "note": "launch-latency bound (bytes fit in L2)"},
        "device_errors": errs,
    }


if __name__ == "__main__":
    sys.exit(main())
