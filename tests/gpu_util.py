"""Shared helpers of the GPU tests: move a workload to the device, run the library through
its C ABI, and compare with the oracle."""
import numpy as np
import torch

import decode_attention_int8_b200 as q8
import oracle

MAX_ABS_TOL = 1e-4  # output tolerance against the fp64 oracle: max |gpu - oracle|
REL_L2_TOL = 1e-5  # and ||gpu - oracle||_2 / ||oracle||_2


def to_device(w, device="cuda"):
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(device)
    return dict(q=t(w.q), k=t(w.k), v=t(w.v), ks=t(w.ks), vs=t(w.vs), bt=t(w.block_table),
                lens=t(w.seq_lens))


def run_decode(w, d=None, out=None):
    d = d or to_device(w)
    if out is None:
        out = torch.full(d["q"].shape, float("nan"), dtype=torch.float32, device="cuda")
    q8.q8kv_decode_attn(out, d["q"], d["k"], d["v"], d["ks"], d["vs"], d["bt"], d["lens"], w.scale)
    torch.cuda.synchronize()
    return out


def oracle_cache(w):
    return oracle.PagedCache(w.k, w.v, w.ks, w.vs, w.block_table, w.seq_lens, w.cfg.n_q_heads,
                             w.scale)


def errors(got, ref):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    diff = got - ref
    max_abs = float(np.max(np.abs(diff))) if diff.size else 0.0
    nrm = float(np.linalg.norm(ref))
    rel = float(np.linalg.norm(diff) / nrm) if nrm > 0 else float(np.linalg.norm(diff))
    return max_abs, rel


def assert_close(got, ref, what=""):
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    max_abs, rel = errors(got, ref)
    assert max_abs <= MAX_ABS_TOL and rel <= REL_L2_TOL, (
        f"{what}: max_abs={max_abs:.3e} (tol {MAX_ABS_TOL}) rel_l2={rel:.3e} (tol {REL_L2_TOL})")
    return max_abs, rel


def without_block(block_table, seq_lens, b, j, bs):
    """The table and lengths of the same cache with logical block j of sequence b left out:
    the tokens a decode must attend to when that block's table entry is unusable (the
    decode has no positional term, so skipping a block's tokens is attention over the
    remaining ones)."""
    bt = np.array(block_table, copy=True)
    lens = np.array(seq_lens, copy=True)
    L = int(lens[b])
    nblk = -(-L // bs)
    assert 0 <= j < nblk
    dropped = min(bs, L - j * bs)
    row = list(bt[b, :nblk])
    del row[j]
    bt[b, :] = -1
    bt[b, :len(row)] = row
    lens[b] = L - dropped
    return bt, lens
