"""Pins of the oracle's multi-query decode: several new query tokens per sequence attend
to the q8 cache, each up to its own position (the multi-query "TILE" decode of the
llama.cpp change on baguaai.com's FlashAttention page, with the Kestrel-LLM single pass
per query row).

- One query per sequence is the single-query decode, bit for bit.
- Causality: query i equals the single-query decode of the sequence cut to its visible
  length seq_len - (n_queries - 1 - i) (a different code path: the cut is made through
  seq_lens).
- A library routine: torch's scaled_dot_product_attention in fp64 with an explicit causal
  mask on the dequantised tensors.
- Queries that see no token (seq_len < n_queries) return zero rows.
"""
import numpy as np
import pytest
import torch

import oracle
from decode_attention_int8_b200 import inputs
from test_oracle_attention import np_quantize


def cache_of(w, lens=None):
    return oracle.PagedCache(w.k, w.v, w.ks, w.vs, w.block_table,
                             w.seq_lens if lens is None else lens, w.cfg.n_q_heads, w.scale)


def workload(seed, lens, Hq=8, Hk=2, D=64, bs=16):
    return inputs.make_custom(len(lens), Hq, Hk, D, lens, bs, seed=seed)


def test_one_query_is_the_single_query_decode():
    w = workload(1, [1, 37, 70])
    c = cache_of(w)
    out = oracle.decode_multi(c, w.q[:, None], 1)
    np.testing.assert_array_equal(out[:, 0], oracle.decode_all(c, w.q))


@pytest.mark.parametrize("nq", [2, 3, 5])
def test_each_query_sees_the_cache_up_to_its_position(nq):
    lens = [1, 2, 17, 40, 64]
    w = workload(nq, lens)
    B, Hq, D = w.cfg.B, w.cfg.n_q_heads, w.cfg.head_dim
    q = inputs.multi_queries(B, nq, Hq, D, seed=nq)
    out = oracle.decode_multi(cache_of(w), q, nq)
    for i in range(nq):
        cut = np.maximum(np.asarray(lens) - (nq - 1 - i), 0).astype(np.int32)
        ref = oracle.decode_all(cache_of(w, cut), q[:, i])
        np.testing.assert_array_equal(out[:, i], ref)
    rows = [(b, i, h) for b in range(B) for i in range(nq) for h in (0, Hq - 1)]
    sel = oracle.decode_multi_rows(cache_of(w), q, nq, rows)
    for r, (b, i, h) in enumerate(rows):
        np.testing.assert_array_equal(sel[r], out[b, i, h])


def test_queries_without_visible_tokens_are_zero():
    nq = 4
    w = workload(3, [0, 1, 3, 4])
    q = inputs.multi_queries(4, nq, 8, 64, seed=3)
    out = oracle.decode_multi(cache_of(w), q, nq)
    for b, L in enumerate([0, 1, 3, 4]):
        for i in range(nq):
            visible = L - (nq - 1 - i)
            if visible <= 0:
                assert np.all(out[b, i] == 0.0)
            else:
                assert np.all(np.any(out[b, i] != 0.0, axis=-1))


@pytest.mark.parametrize("nq,G", [(2, 4), (4, 1), (3, 8)])
def test_matches_causal_sdpa_on_dequantised_data(nq, G):
    Hk, D, bs = 2, 64, 16
    Hq = G * Hk
    lens = [nq, 29, 50]
    w = workload(10 + nq, lens, Hq=Hq, Hk=Hk, D=D, bs=bs)
    B = len(lens)
    q = inputs.multi_queries(B, nq, Hq, D, seed=20 + nq)
    out = oracle.decode_multi(cache_of(w), q, nq)
    codes, qsc = np_quantize(q)
    qdeq = codes.astype(np.float64) * np.repeat(qsc.astype(np.float64), 32, axis=-1)
    for b, L in enumerate(lens):
        t = np.arange(L)
        slots = w.block_table[b, t // bs].astype(np.int64) * bs + t % bs
        kf = w.k.reshape(-1, Hk, D)[slots].astype(np.float64) * \
            w.ks.reshape(-1, Hk)[slots][..., None]
        vf = w.v.reshape(-1, Hk, D)[slots].astype(np.float64) * \
            w.vs.reshape(-1, Hk)[slots][..., None]
        K = torch.from_numpy(kf).permute(1, 0, 2).repeat_interleave(G, 0)[None]
        V = torch.from_numpy(vf).permute(1, 0, 2).repeat_interleave(G, 0)[None]
        Q = torch.from_numpy(qdeq[b]).permute(1, 0, 2)[None]  # [1][Hq][nq][D]
        allowed = torch.arange(L)[None, :] <= (L - nq + torch.arange(nq))[:, None]
        o = torch.nn.functional.scaled_dot_product_attention(Q, K, V, attn_mask=allowed,
                                                             scale=float(w.scale))
        ref = o[0].permute(1, 0, 2).numpy()  # [nq][Hq][D]
        np.testing.assert_allclose(out[b], ref, rtol=1e-10, atol=1e-12)


def test_rejects_bad_arguments():
    w = workload(4, [5])
    q = inputs.multi_queries(1, 2, 8, 64)
    with pytest.raises(oracle.OracleError):
        oracle.decode_multi(cache_of(w), q, 0)
    with pytest.raises(oracle.OracleError):
        oracle.decode_multi_rows(cache_of(w), q, 2, [(0, 2, 0)])
