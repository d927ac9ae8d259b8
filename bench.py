"""Benchmark of q8-KV single-query decode attention on B200.

One step = one q8kv_decode_attn call over one batch of the workload (the whole hot path:
Q quantisation, paged K/V streaming, int8 block dots, online softmax, V accumulation,
split combine), through the C ABI. Prints one JSON line (rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config I] [--impl reference]

Metric: effective KV bandwidth = algorithmic bytes of one call / time per call, where the
algorithmic bytes are every valid (token, KV head) K row, V row and both scales once, plus
q read and out written in fp32, the used block-table entries and seq_lens.

Timing: the KV pool is rotated over enough copies that their total exceeds 4x the L2 size,
so every call streams from HBM; W untimed calls, then K calls bracketed by a barrier and a
device synchronisation, timed with CUDA events on the launching stream; the maximum over
ranks is reported. Under torchrun every rank runs its own copy of the workload on its own
GPU (independent sequences, no collective on the data path): weak scaling.
"""
from __future__ import annotations

import argparse
import ctypes
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "q8-KV decode attention: µs/call and effective KV GB/s (% of B200 HBM peak)"
UNIT = "GB/s"
DEFAULT_WORKLOAD = 1  # the batched GQA decode workload the metric is quoted on
L2_BYTES = 126 * 1024 * 1024
FALLBACK_PEAK_GBS = 6650.0
LAUNCHES_PER_CALL = 2  # decode kernel + split combine kernel


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--config", type=int, default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
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
    """nvidia-smi clock / throttle samples of one GPU while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.window = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.monotonic(), line.strip()))

    def mark(self, t0: float, t1: float):
        """Keep only the samples taken between host times t0 and t1 (the timed region)."""
        self.window = (t0, t1)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.thread.join(timeout=2)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        lines = self.lines
        if self.window is not None:
            inside = [(t, ln) for t, ln in lines if self.window[0] <= t <= self.window[1]]
            lines = inside if inside else lines
        for _, ln in lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def workload_config(w, n_copies, extra):
    c = w.cfg
    lens = w.seq_lens
    d = {"workload": c.name, "B": c.B, "n_q_heads": c.n_q_heads, "n_kv_heads": c.n_kv_heads,
         "head_dim": c.head_dim, "kv_block_size": c.block_size,
         "seq_len": int(lens.max()) if lens.min() == lens.max() else
         f"ragged {int(lens.min())}..{int(lens.max())} (sum {int(lens.sum())})",
         "num_kv_blocks": w.num_blocks, "algorithmic_bytes": w.algorithmic_bytes(),
         "l2": f"inputs larger than L2: KV pool rotated over {n_copies} copies "
               f"({n_copies * (w.k.nbytes + w.v.nbytes + w.ks.nbytes + w.vs.nbytes) / 1e6:.0f} MB"
               f" > {L2_BYTES / 1e6:.0f} MB L2)"}
    d.update(extra)
    return d


def q8_vs_fp32(w, got, n_rows=64, seed=0):
    """Information only: how far the q8 path's output is from attention over the unquantised
    fp32 q, K, V (plain fp64 numpy softmax(q K^T * scale) V on a sample of (sequence, head)
    rows). This measures the int8 quantisation itself, not the kernel's arithmetic."""
    import numpy as np

    from decode_attention_int8_b200 import inputs

    c = w.cfg
    fp32_pool_bytes = 2 * 4 * w.k.size
    if fp32_pool_bytes > (2 << 30):
        return {"skipped": f"the unquantised fp32 pools would take {fp32_pool_bytes / 1e9:.1f} GB "
                           "of host memory"}
    w32 = inputs.make(c, keep_fp32=True)
    P, bs, Hk, D = w32.k.shape
    k32 = w32.k32.reshape(P * bs, Hk, D)
    v32 = w32.v32.reshape(P * bs, Hk, D)
    rng = np.random.default_rng(seed)
    G = c.n_q_heads // c.n_kv_heads
    diffs, refs = [], []
    for _ in range(n_rows):
        b = int(rng.integers(0, c.B))
        h = int(rng.integers(0, c.n_q_heads))
        L = int(w32.seq_lens[b])
        if L == 0:
            continue
        t = np.arange(L)
        slot = w32.block_table[b, t // bs].astype(np.int64) * bs + t % bs
        kf = k32[slot, h // G].astype(np.float64)
        vf = v32[slot, h // G].astype(np.float64)
        sc = kf @ w32.q[b, h].astype(np.float64) * w32.scale
        pr = np.exp(sc - sc.max())
        ref = pr @ vf / pr.sum()
        refs.append(ref)
        diffs.append(np.asarray(got[b, h], np.float64) - ref)
    d, r = np.array(diffs), np.array(refs)
    return {"max_abs": float(np.abs(d).max()), "rel_l2": float(np.linalg.norm(d) / np.linalg.norm(r)),
            "rows": len(refs), "reference": "fp64 attention over the unquantised fp32 q, K, V"}


def cpu_baseline(w, min_seconds=10.0):
    """The oracle as it stands, single-threaded, on whole passes over the workload."""
    import oracle

    cache = oracle.PagedCache(w.k, w.v, w.ks, w.vs, w.block_table, w.seq_lens,
                              w.cfg.n_q_heads, w.scale)
    reps, t0 = 0, time.perf_counter()
    while True:
        oracle.decode_all(cache, w.q)
        reps += 1
        dt = time.perf_counter() - t0
        if dt >= min_seconds:
            break
    gbs = w.algorithmic_bytes() * reps / dt / 1e9
    return {"value": round(gbs, 4), "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": f"whole workload ({w.cfg.B} sequences x {w.cfg.n_q_heads} heads), "
                      f"{reps} passes, {dt:.1f} s, single-threaded C oracle"}


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
    """--impl reference: the oracle on the host cores, on this arm's workload and metric."""
    world, rank, _ = dist_env()
    if rank != 0:
        return 0
    from decode_attention_int8_b200 import inputs
    import numpy as np
    import oracle

    w = inputs.make(args.config)
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

    def step(i):
        # a random sample of (sequence, head) rows; the workload's algorithmic bytes are
        # counted pro rata to the rows done
        sel = rng.choice(len(pairs_all), n_pairs, replace=False)
        oracle.decode_pairs(cache, w.q, [pairs_all[j] for j in sel])
        return n_pairs

    for i in range(args.warmup):
        step(i)
    t0 = time.perf_counter()
    done = 0
    for i in range(args.steps):
        done += step(i)
    dt = time.perf_counter() - t0
    frac = done / len(pairs_all)
    gbs = w.algorithmic_bytes() * frac / dt / 1e9
    line = {"impl": "reference", "metric": METRIC, "value": round(gbs, 4), "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(dt / args.steps * 1e3, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.cfg.name, "B": B, "n_q_heads": Hq,
                       "n_kv_heads": w.cfg.n_kv_heads, "head_dim": w.cfg.head_dim,
                       "kv_block_size": w.cfg.block_size},
            "cpu_baseline": {"value": round(gbs, 4), "unit": UNIT, "cores": 1, "kind": "oracle",
                             "sample": f"{n_pairs} random (sequence, head) rows per step of "
                                       f"{len(pairs_all)}; bytes counted pro rata"},
            "e2e": {"value": round(gbs, 4), "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    if args.accuracy_study:
        return run_accuracy_study(args)
    world, rank, local = dist_env()
    import numpy as np
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

    w = inputs.make(args.config)
    lib = q8.lib()
    algo = w.algorithmic_bytes()
    pool_bytes = w.k.nbytes + w.v.nbytes + w.ks.nbytes + w.vs.nbytes
    n_copies = max(2, math.ceil(4 * L2_BYTES / pool_bytes) + 1) if pool_bytes < 8 * L2_BYTES else 1
    n_copies = min(n_copies, 64)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)
    q = t(w.q)
    bt = t(w.block_table)
    lens = t(w.seq_lens)
    pools = [(t(w.k), t(w.v), t(w.ks), t(w.vs)) for _ in range(n_copies)]
    out = torch.empty(q.shape, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    sp = ctypes.c_void_p(stream.cuda_stream)
    c = w.cfg
    geo = (c.B, c.n_q_heads, c.n_kv_heads, c.head_dim, c.block_size, w.max_blocks_per_seq,
           w.num_blocks)
    P = lambda x: ctypes.c_void_p(x.data_ptr())
    argsets = [(P(out), P(q), P(k), P(v), P(ks), P(vs), P(bt), P(lens), *geo,
                ctypes.c_float(w.scale), sp) for (k, v, ks, vs) in pools]
    fn = lib.q8kv_decode_attn

    def call(i):
        st = fn(*argsets[i % n_copies])
        if st != 0:
            raise q8.Q8KVError(st, "q8kv_decode_attn")

    # warm-up (also sizes the library workspace outside the timed region)
    for i in range(max(args.warmup, 1)):
        call(i)
    torch.cuda.synchronize(dev)

    def barrier():
        if pg is not None:
            pg.barrier()

    # timed region: K back-to-back calls between two CUDA events on the launching stream
    # (events between the calls would sit between the kernels and break the programmatic
    # dependent launch overlap of consecutive calls)
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    barrier()
    torch.cuda.synchronize(dev)
    host_t0 = time.monotonic()
    t_begin = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_begin.record(stream)
    for i in range(args.steps):
        call(i)
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    host_t1 = time.monotonic()
    barrier()
    time.sleep(0.15)  # let the sampler deliver the last in-window line
    sampler.mark(host_t0, host_t1)
    clocks = sampler.stop()
    total_ms = t_begin.elapsed_time(t_end)
    total_ms = reduce_max(total_ms, pg, dev)
    ms_per_step = total_ms / args.steps
    kernel_ms = ms_per_step  # one step = the call's decode + combine kernels

    # information only, outside the timed region: one call at a time between its own events
    iso = []
    for i in range(min(200, max(20, args.steps))):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        call(i)
        e1.record(stream)
        e1.synchronize()
        iso.append(e0.elapsed_time(e1))
    isolated_us = statistics.median(iso) * 1e3
    value = whole_job_gbs(algo, world, ms_per_step)

    # end to end through the C ABI with host buffers: per step copy q / block table /
    # seq_lens from pinned host memory, decode, copy out back (the KV cache stays resident)
    e2e = None
    if not args.no_e2e:
        hq = torch.from_numpy(w.q).pin_memory()
        hbt = torch.from_numpy(w.block_table).pin_memory()
        hlens = torch.from_numpy(w.seq_lens).pin_memory()
        hout = torch.empty(out.shape, dtype=torch.float32).pin_memory()
        e2e_steps = max(10, min(args.steps, 2000))
        for i in range(3):
            q.copy_(hq, non_blocking=True)
            call(i)
            hout.copy_(out, non_blocking=True)
        torch.cuda.synchronize(dev)
        barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(e2e_steps):
            q.copy_(hq, non_blocking=True)
            bt.copy_(hbt, non_blocking=True)
            lens.copy_(hlens, non_blocking=True)
            call(i)
            hout.copy_(out, non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        e2e_ms = e0.elapsed_time(e1) / e2e_steps
        e2e_ms = reduce_max(e2e_ms, pg, dev)
        e2e = {"value": round(whole_job_gbs(algo, world, e2e_ms), 2), "unit": UNIT,
               "h2d_bytes_per_step": int(w.q.nbytes + w.block_table.nbytes + w.seq_lens.nbytes),
               "d2h_bytes_per_step": int(w.q.nbytes), "us_per_step": round(e2e_ms * 1e3, 3),
               "steps": e2e_steps}

    peak, peak_kind = measured_peak()
    achieved = algo / (kernel_ms * 1e-3) / 1e9
    traffic = recorded_traffic(c.name, "decode")
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 6),
        "us_per_call": round(ms_per_step * 1e3, 3),
        "us_per_call_isolated": round(isolated_us, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "s8", "data": "synthetic",
        "config": workload_config(w, n_copies, {"parallelism": f"replicas{world}"}),
        "roofline": {"bound": "hbm", "achieved": round(achieved, 2), "peak": peak,
                     "peak_kind": peak_kind, "unit": "GB/s", "frac": round(achieved / peak, 4),
                     "frac_of_8TBps_nominal": round(achieved / 8000.0, 4),
                     "traffic": traffic,
                     "kernel": "q8kv::decode_kernel + q8kv::combine_kernel (one call)",
                     "kernel_us": round(kernel_ms * 1e3, 3)},
        "gpu_launches": LAUNCHES_PER_CALL * args.steps,
        "clocks": clocks,
    }
    if e2e is not None:
        line["e2e"] = e2e
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w)
    if not args.no_multi_query:
        # information, after the timed region: the same workload with n_queries new tokens
        # per sequence (speculative decode), through q8kv_decode_attn_multi
        line["multi_query"] = bench_multi_query(w, pools, bt, lens, dev, stream,
                                                steps=max(10, min(args.steps, 2000)))
    if not args.no_q4:
        line["q4_0_decode"] = bench_q4(dev, stream, steps=max(10, min(args.steps, 2000)))
    if not args.no_cache_write or not args.no_quest:
        del pools, argsets
        torch.cuda.empty_cache()
    if not args.no_cache_write:
        # information, after the timed region: the write path that fills the cache
        line["cache_write"] = bench_cache_write(dev, stream)
    if not args.no_quest:
        line["quest_metadata"] = bench_quest(dev, stream)
    if rank == 0 and world == 1 and not args.no_accuracy:
        torch.cuda.synchronize(dev)
        line["q8_vs_fp32"] = q8_vs_fp32(w, out.cpu().numpy())
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
        "decode_step": {"workload": f"one new token per sequence: {step_B} x {Hk} rows",
                        "us_per_call": round(ms_step * 1e3, 3), "calls": steps,
                        "algorithmic_bytes": step_bytes,
                        "note": "launch-latency bound (bytes fit in L2)"},
        "device_errors": errs,
    }


if __name__ == "__main__":
    sys.exit(main())
