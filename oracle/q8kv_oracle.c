/*
 * q8kv_oracle.c -- plain single-threaded CPU oracle for q8-KV single-query decode
 * attention. TEST INFRASTRUCTURE ONLY (see q8kv_oracle.h for what may call it).
 *
 * Build: gcc -O2 -ffp-contract=off -fno-fast-math -fPIC -shared (no -ffast-math, no
 * FMA contraction: the fp32 Q quantisation must round every operation separately).
 *
 * Readings of the pages taken here (the garbled spots in the Kestrel-LLM walk-through,
 * trdm.cn/news/511694, section 2 part 1):
 *   - the walk-through guards a block whose largest magnitude is tiny, but the comparison
 *     and assignment operators were lost in extraction; it is read as a less-than test
 *     against 1e-6 that replaces that largest magnitude with 1, so the block quantises to
 *     zeros;
 *   - the walk-through turns the scaled value into a code by clamping to [-128, 127] and
 *     truncating; this library instead rounds half to even and clamps to [-127, 127] (the
 *     rounding rule it fixes; the two differ by at most one step per element);
 *   - the K/V scale arrays hold the dequantisation multiplier itself (no extra 1/127)
 *     and are indexed by the physical slot: scale[slot * n_kv_heads + kv_head];
 *   - the running max starts at -infinity (the page's -1e9 gives the same result when
 *     every score exceeds -1e9);
 *   - on the new-maximum branch the token's own weight is exp(0) = 1;
 *   - seq_len == 0 yields an all-zero output row.
 */
#include "q8kv_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

/* Planted mistakes for the pin-strength test (tests/test_oracle_mutants.py): building
 * with -DQ8KVO_MUTANT=n switches on mistake n; the default build has none. */
#ifndef Q8KVO_MUTANT
#define Q8KVO_MUTANT 0
#endif
#define MUT(n) (Q8KVO_MUTANT == (n))

/* ---------------------------------------------------------------- Q quantisation */

/* Round to nearest, ties to even, written out so that it does not depend on the
 * floating-point environment. x is an fp32 value widened to double (exact). */
static double round_half_even(double x)
{
    double f = floor(x);
    double frac = x - f; /* exact: |x| < 2^24 here */
    if (frac > 0.5)
        return f + 1.0;
    if (frac < 0.5)
        return f;
    return (fmod(f, 2.0) == 0.0) ? f : f + 1.0;
}

/* One 32-element block, walk-through section 2 part 1:
 *   qm  = max |q_i|                      (fp32)
 *   if qm < 1e-6: qm = 1                  (all-zero block -> codes 0)
 *   qsc = qm * (1/127)                    (fp32)
 *   iq  = 127 / qm                        (fp32, correctly rounded)
 *   qi  = clamp(rne(q_i * iq), -127, 127) (product rounded to fp32 first) */
static void quantize_block(const float *qb, int8_t *qi, float *qsc)
{
    float qm = 0.0f;
    for (int i = 0; i < 32; ++i) {
        float a = fabsf(qb[i]);
        if (a > qm)
            qm = a;
    }
    if (MUT(8) ? (qm <= 1e-6f) : (qm < 1e-6f))
        qm = 1.0f;
    *qsc = qm * (1.0f / 127.0f);
    float iq = 127.0f / qm;
    for (int i = 0; i < 32; ++i) {
        float prod = qb[i] * iq;
        double r = MUT(3) ? trunc((double)prod) : round_half_even((double)prod);
        if (r > 127.0)
            r = 127.0;
        if (r < -127.0)
            r = -127.0;
        qi[i] = (int8_t)r;
    }
}

int q8kvo_quantize_q(const float *q, long n, int8_t *qi, float *qsc)
{
    if (!q || !qi || !qsc || n < 0 || (n % 32) != 0)
        return Q8KVO_EINVAL;
    for (long i = 0; i < n; ++i)
        if (!isfinite(q[i]))
            return Q8KVO_EINVAL;
    for (long b = 0; b < n / 32; ++b)
        quantize_block(q + 32 * b, qi + 32 * b, qsc + b);
    return Q8KVO_OK;
}

/* ---------------------------------------------------------------- KV-cache write */

/* One K or V row of n values for the cache. The walk-through keeps one scale per
 * (token, KV head) (trdm.cn/news/511694, the kernel signature's "per-token per-head"
 * kscale comment) and turns it into the dequantisation multiplier by one multiply with
 * 1/127 at use (section 2 part 2, kscale * KVQ_INV); the quantiser is the one section 2
 * part 1 gives for Q ("Q8_0 isomorphic"), applied to the whole row as one block:
 *   amax  = max |x_i|                       (fp32)
 *   if amax < 1e-6: amax = 1                (all-zero row -> codes 0, scale 1/127)
 *   scale = amax * (1/127)                  (fp32: the multiplier stored in the cache)
 *   inv   = 127 / amax                      (fp32, correctly rounded)
 *   code  = clamp(rne(x_i * inv), -127, 127) (product rounded to fp32 first)
 * A row holding an infinity or a NaN has no meaningful scale: its codes are 0, its scale
 * is a quiet NaN and *flags gets Q8KVO_FLAG_NONFINITE. */
static void quantize_kv_row(const float *x, int n, int8_t *codes, float *scale,
                            unsigned *flags)
{
    float amax = 0.0f;
    int finite = 1;
    for (int i = 0; i < n && !MUT(15); ++i) {
        if (!isfinite(x[i]))
            finite = 0;
        float a = fabsf(x[i]);
        if (a > amax)
            amax = a;
    }
    for (int i = 0; i < n && i < 32 && MUT(15); ++i) { /* planted: first 32 channels */
        if (!isfinite(x[i]))
            finite = 0;
        if (fabsf(x[i]) > amax)
            amax = fabsf(x[i]);
    }
    if (!finite) {
        for (int i = 0; i < n; ++i)
            codes[i] = 0;
        *scale = NAN;
        *flags |= Q8KVO_FLAG_NONFINITE;
        return;
    }
    if (amax < 1e-6f)
        amax = 1.0f;
    *scale = MUT(17) ? amax : amax * (1.0f / 127.0f);
    float inv = 127.0f / amax;
    for (int i = 0; i < n; ++i) {
        float prod = x[i] * inv;
        double r = MUT(16) ? trunc((double)prod) : round_half_even((double)prod);
        if (r > 127.0)
            r = 127.0;
        if (r < -127.0)
            r = -127.0;
        codes[i] = (int8_t)r;
    }
}

int q8kvo_quantize_kv_row(const float *x, int n, int8_t *codes, float *scale, unsigned *flags)
{
    if (!x || !codes || !scale || !flags || n <= 0)
        return Q8KVO_EINVAL;
    quantize_kv_row(x, n, codes, scale, flags);
    return Q8KVO_OK;
}

/* Write n_tokens new (token, KV head) rows of K and of V into the paged pools.
 * Token i goes to physical slot slot_mapping[i] = block * block_size + offset (the
 * block-table mapping of beaiera.top "deepseek-attention-div64", section "Top-K index
 * global mapping"); a negative slot marks a padding entry and is skipped, as the same
 * section prescribes for its -1 entries. A slot at or past num_blocks * block_size is
 * skipped too and sets Q8KVO_FLAG_SLOT. Row (i, h) of k_new starts at
 * k_new[i * token_stride + h * head_dim]; it lands at k[(slot * n_kv_heads + h) * head_dim]
 * and its scale at ks[slot * n_kv_heads + h] (same for V). Slots are taken in token order,
 * so when two tokens name one slot the later one wins. */
int q8kvo_cache_write(int8_t *k, int8_t *v, float *ks, float *vs, const float *k_new,
                      const float *v_new, const int64_t *slot_mapping, long n_tokens,
                      int n_kv_heads, int head_dim, int block_size, int num_blocks,
                      long token_stride, unsigned *flags)
{
    if (!k || !v || !ks || !vs || !k_new || !v_new || !slot_mapping || !flags)
        return Q8KVO_EINVAL;
    if (n_tokens < 0 || n_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 || num_blocks <= 0 ||
        token_stride < (long)n_kv_heads * head_dim)
        return Q8KVO_EINVAL;
    const int64_t n_slots = (int64_t)num_blocks * block_size;
    for (long i = 0; i < n_tokens; ++i) {
        int64_t slot = slot_mapping[i];
        if (slot < 0)
            continue;
        if (slot >= n_slots) {
            *flags |= Q8KVO_FLAG_SLOT;
            continue;
        }
        for (int h = 0; h < n_kv_heads; ++h) {
            int hd = MUT(18) ? (h + 1) % n_kv_heads : h;
            long src = i * token_stride + (long)h * head_dim;
            long row = (long)slot * n_kv_heads + hd;
            quantize_kv_row(k_new + src, head_dim, k + row * head_dim, ks + row, flags);
            quantize_kv_row(v_new + src, head_dim, v + row * head_dim, vs + row, flags);
        }
    }
    return Q8KVO_OK;
}

/* ---------------------------------------------------------------- cache access */

static int check_cache(const q8kvo_cache *c)
{
    if (!c || !c->block_table || !c->seq_lens)
        return Q8KVO_EINVAL;
    if (c->B <= 0 || c->n_q_heads <= 0 || c->n_kv_heads <= 0 || c->head_dim <= 0 ||
        (c->head_dim % 32) != 0 || c->block_size <= 0 || c->max_blocks_per_seq <= 0 ||
        c->num_blocks <= 0 || (c->n_q_heads % c->n_kv_heads) != 0 || !isfinite(c->scale))
        return Q8KVO_EINVAL;
    return Q8KVO_OK;
}

static int check_seq(const q8kvo_cache *c, int b, int h)
{
    if (b < 0 || b >= c->B || h < 0 || h >= c->n_q_heads)
        return Q8KVO_EINVAL;
    int L = c->seq_lens[b];
    if (L < 0 || (long)L > (long)c->max_blocks_per_seq * c->block_size)
        return Q8KVO_ERANGE;
    int nblk = (L + c->block_size - 1) / c->block_size;
    for (int i = 0; i < nblk; ++i) {
        int p = c->block_table[(long)b * c->max_blocks_per_seq + i];
        if (p < 0 || p >= c->num_blocks)
            return Q8KVO_ERANGE;
    }
    return Q8KVO_OK;
}

/* Physical slot of token t of sequence b (beaiera.top, "Top-K index global mapping";
 * Kestrel walk-through section 2 part 2: block t / kv_bs, offset t % kv_bs). */
static long slot_of(const q8kvo_cache *c, int b, int t)
{
    long blk = c->block_table[(long)b * c->max_blocks_per_seq + t / c->block_size];
    return blk * c->block_size + (MUT(5) ? (t + 1) % c->block_size : t % c->block_size);
}

/* GQA mapping of the llama2.c loop: kv_head = q_head / (n_q_heads / n_kv_heads). */
static int kv_head_of(const q8kvo_cache *c, int h)
{
    return MUT(2) ? h % c->n_kv_heads : h / (c->n_q_heads / c->n_kv_heads);
}

/* Quantised query of (b, h): codes and per-block scales. */
static int quantized_query(const q8kvo_cache *c, const float *q, int b, int h, int8_t *qi,
                           float *qsc)
{
    const float *qh = q + ((long)b * c->n_q_heads + h) * c->head_dim;
    return q8kvo_quantize_q(qh, c->head_dim, qi, qsc);
}

/* int32 dot of quant block j of the query with the same 32 channels of a K row. */
static int32_t block_dot(const int8_t *qi, const int8_t *krow, int j)
{
    int32_t acc = 0;
    for (int i = 0; i < 32; ++i)
        acc += (int32_t)qi[32 * j + i] * (int32_t)krow[32 * j + (MUT(14) ? (i + 1) % 32 : i)];
    return acc;
}

/* Score of token t: s = (sum_j dot_j * qsc_j) * ks * scale, in fp64 (section 2 part 2,
 * "block scales put back": the integer dot is the skeleton, the float scales are
 * applied while accumulating). */
static double score_of(const q8kvo_cache *c, const int8_t *qi, const float *qsc, int b, int kvh,
                       int t)
{
    long slot = slot_of(c, b, t);
    const int8_t *krow = c->k + (slot * c->n_kv_heads + kvh) * (long)c->head_dim;
    int nb = c->head_dim / 32;
    double s = 0.0;
    for (int j = 0; j < nb; ++j)
        s += (double)block_dot(qi, krow, j) * (double)qsc[MUT(7) ? 0 : j];
    double ks = MUT(1) ? 1.0 : (double)c->ks[slot * c->n_kv_heads + kvh];
    return s * ks * (double)c->scale * (MUT(13) ? (double)c->scale : 1.0);
}

int q8kvo_block_dots(const q8kvo_cache *c, const float *q, int b, int h, int32_t *dots)
{
    int rc = check_cache(c);
    if (rc)
        return rc;
    if (!c->k || !q || !dots)
        return Q8KVO_EINVAL;
    if ((rc = check_seq(c, b, h)))
        return rc;
    int D = c->head_dim, nb = D / 32, kvh = kv_head_of(c, h), L = c->seq_lens[b];
    int8_t *qi = (int8_t *)malloc((size_t)D);
    float *qsc = (float *)malloc(sizeof(float) * (size_t)nb);
    if (!qi || !qsc) {
        free(qi);
        free(qsc);
        return Q8KVO_ENOMEM;
    }
    rc = quantized_query(c, q, b, h, qi, qsc);
    for (int t = 0; rc == Q8KVO_OK && t < L; ++t) {
        long slot = slot_of(c, b, t);
        const int8_t *krow = c->k + (slot * c->n_kv_heads + kvh) * (long)D;
        for (int j = 0; j < nb; ++j)
            dots[(long)t * nb + j] = block_dot(qi, krow, j);
    }
    free(qi);
    free(qsc);
    return rc;
}

int q8kvo_scores(const q8kvo_cache *c, const float *q, int b, int h, double *s)
{
    int rc = check_cache(c);
    if (rc)
        return rc;
    if (!c->k || !c->ks || !q || !s)
        return Q8KVO_EINVAL;
    if ((rc = check_seq(c, b, h)))
        return rc;
    int D = c->head_dim, nb = D / 32, kvh = kv_head_of(c, h), L = c->seq_lens[b];
    int8_t *qi = (int8_t *)malloc((size_t)D);
    float *qsc = (float *)malloc(sizeof(float) * (size_t)nb);
    if (!qi || !qsc) {
        free(qi);
        free(qsc);
        return Q8KVO_ENOMEM;
    }
    rc = quantized_query(c, q, b, h, qi, qsc);
    for (int t = 0; rc == Q8KVO_OK && t < L; ++t)
        s[t] = score_of(c, qi, qsc, b, kvh, t);
    free(qi);
    free(qsc);
    return rc;
}

/* ---------------------------------------------------------------- single pass */

/* One (b, h), walk-through section 2 parts 1-3, token by token:
 *   if s > M:  f = exp(M - s); S *= f; acc *= f; M = s; w = 1
 *   else:      w = exp(s - M)
 *   S += w;  acc[d] += w * vs * V[d]
 * and finally out = acc / S. */
static int decode_row(const q8kvo_cache *c, const float *qh, int b, int h, int L, double *out,
                      double *m_trace, long *n_iter, int8_t *qi, float *qsc, double *acc)
{
    int D = c->head_dim, kvh = kv_head_of(c, h);
    int rc = q8kvo_quantize_q(qh, D, qi, qsc);
    if (rc)
        return rc;
    double M = -INFINITY, S = 0.0;
    for (int d = 0; d < D; ++d)
        acc[d] = 0.0;
    long iters = 0;
    for (int t = 0; t < L; ++t) {
        double s = score_of(c, qi, qsc, b, kvh, t);
        double w;
        if (s > M) {
            double f = exp(M - s);
            if (!MUT(10))
                S *= f;
            for (int d = 0; d < D && !MUT(4); ++d)
                acc[d] *= f;
            M = s;
            w = 1.0;
        } else {
            w = exp(s - M);
        }
        S += w;
        long slot = slot_of(c, b, t);
        const int8_t *vrow = c->v + (slot * c->n_kv_heads + kvh) * (long)D;
        double wv = w * (double)(MUT(6) ? c->ks : c->vs)[slot * c->n_kv_heads + kvh];
        for (int d = 0; d < D; ++d)
            acc[d] += wv * (double)vrow[d];
        if (m_trace)
            m_trace[t] = M;
        ++iters;
    }
    for (int d = 0; d < D; ++d)
        out[d] = (L > 0) ? acc[d] / S : 0.0;
    if (n_iter)
        *n_iter = iters;
    return Q8KVO_OK;
}

/* The single-query decode of (b, h): query row q[b][h], every cached token. */
static int decode_online_one(const q8kvo_cache *c, const float *q, int b, int h, double *out,
                             double *m_trace, long *n_iter, int8_t *qi, float *qsc, double *acc)
{
    const float *qh = q + ((long)b * c->n_q_heads + h) * c->head_dim;
    return decode_row(c, qh, b, h, c->seq_lens[b], out, m_trace, n_iter, qi, qsc, acc);
}

static int scratch_alloc(int D, int8_t **qi, float **qsc, double **acc)
{
    *qi = (int8_t *)malloc((size_t)D);
    *qsc = (float *)malloc(sizeof(float) * (size_t)(D / 32));
    *acc = (double *)malloc(sizeof(double) * (size_t)D);
    if (!*qi || !*qsc || !*acc) {
        free(*qi);
        free(*qsc);
        free(*acc);
        return Q8KVO_ENOMEM;
    }
    return Q8KVO_OK;
}

static int check_q8(const q8kvo_cache *c, const float *q, const void *out)
{
    int rc = check_cache(c);
    if (rc)
        return rc;
    if (!c->k || !c->v || !c->ks || !c->vs || !q || !out)
        return Q8KVO_EINVAL;
    return Q8KVO_OK;
}

int q8kvo_decode_online(const q8kvo_cache *c, const float *q, int b, int h, double *out,
                        double *m_trace, long *n_iter)
{
    int rc = check_q8(c, q, out);
    if (rc || (rc = check_seq(c, b, h)))
        return rc;
    int8_t *qi;
    float *qsc;
    double *acc;
    if ((rc = scratch_alloc(c->head_dim, &qi, &qsc, &acc)))
        return rc;
    rc = decode_online_one(c, q, b, h, out, m_trace, n_iter, qi, qsc, acc);
    free(qi);
    free(qsc);
    free(acc);
    return rc;
}

int q8kvo_decode_all(const q8kvo_cache *c, const float *q, double *out)
{
    int rc = check_q8(c, q, out);
    if (rc)
        return rc;
    for (int b = 0; b < c->B; ++b)
        if ((rc = check_seq(c, b, 0)))
            return rc;
    int8_t *qi;
    float *qsc;
    double *acc;
    if ((rc = scratch_alloc(c->head_dim, &qi, &qsc, &acc)))
        return rc;
    for (int b = 0; b < c->B && rc == Q8KVO_OK; ++b)
        for (int h = 0; h < c->n_q_heads && rc == Q8KVO_OK; ++h)
            rc = decode_online_one(c, q, b, h, out + ((long)b * c->n_q_heads + h) * c->head_dim,
                                   NULL, NULL, qi, qsc, acc);
    free(qi);
    free(qsc);
    free(acc);
    return rc;
}

int q8kvo_decode_pairs(const q8kvo_cache *c, const float *q, const int32_t *pairs, long n,
                       double *out)
{
    int rc = check_q8(c, q, out);
    if (rc)
        return rc;
    if (!pairs || n < 0)
        return Q8KVO_EINVAL;
    for (long i = 0; i < n; ++i)
        if ((rc = check_seq(c, pairs[2 * i], pairs[2 * i + 1])))
            return rc;
    int8_t *qi;
    float *qsc;
    double *acc;
    if ((rc = scratch_alloc(c->head_dim, &qi, &qsc, &acc)))
        return rc;
    for (long i = 0; i < n && rc == Q8KVO_OK; ++i)
        rc = decode_online_one(c, q, pairs[2 * i], pairs[2 * i + 1], out + i * c->head_dim, NULL,
                               NULL, qi, qsc, acc);
    free(qi);
    free(qsc);
    free(acc);
    return rc;
}

/* ---------------------------------------------------------------- several queries */

/* Tokens visible to query i of n_queries of sequence b: the new queries are the last
 * n_queries tokens of the sequence (already in the cache), and each attends to itself and
 * everything before it (causal), so query i sees seq_lens[b] - (n_queries - 1 - i)
 * tokens; fewer than none means none. */
static int visible_len(const q8kvo_cache *c, int b, int n_queries, int i)
{
    int L = c->seq_lens[b] - (n_queries - 1 - (MUT(19) ? 0 : i)) - (MUT(20) ? 1 : 0);
    return L > 0 ? L : 0;
}

int q8kvo_decode_multi(const q8kvo_cache *c, const float *q, int n_queries, double *out)
{
    int rc = check_q8(c, q, out);
    if (rc)
        return rc;
    if (n_queries <= 0)
        return Q8KVO_EINVAL;
    for (int b = 0; b < c->B; ++b)
        if ((rc = check_seq(c, b, 0)))
            return rc;
    int8_t *qi;
    float *qsc;
    double *acc;
    if ((rc = scratch_alloc(c->head_dim, &qi, &qsc, &acc)))
        return rc;
    const long D = c->head_dim;
    for (int b = 0; b < c->B && rc == Q8KVO_OK; ++b)
        for (int i = 0; i < n_queries && rc == Q8KVO_OK; ++i)
            for (int h = 0; h < c->n_q_heads && rc == Q8KVO_OK; ++h) {
                long row = ((long)b * n_queries + i) * c->n_q_heads + h;
                rc = decode_row(c, q + row * D, b, h, visible_len(c, b, n_queries, i),
                                out + row * D, NULL, NULL, qi, qsc, acc);
            }
    free(qi);
    free(qsc);
    free(acc);
    return rc;
}

int q8kvo_decode_multi_rows(const q8kvo_cache *c, const float *q, int n_queries,
                            const int32_t *rows, long n, double *out)
{
    int rc = check_q8(c, q, out);
    if (rc)
        return rc;
    if (n_queries <= 0 || !rows || n < 0)
        return Q8KVO_EINVAL;
    for (long r = 0; r < n; ++r) {
        int b = rows[3 * r], i = rows[3 * r + 1], h = rows[3 * r + 2];
        if (i < 0 || i >= n_queries)
            return Q8KVO_EINVAL;
        if ((rc = check_seq(c, b, h)))
            return rc;
    }
    int8_t *qi;
    float *qsc;
    double *acc;
    if ((rc = scratch_alloc(c->head_dim, &qi, &qsc, &acc)))
        return rc;
    const long D = c->head_dim;
    for (long r = 0; r < n && rc == Q8KVO_OK; ++r) {
        int b = rows[3 * r], i = rows[3 * r + 1], h = rows[3 * r + 2];
        long qrow = ((long)b * n_queries + i) * c->n_q_heads + h;
        rc = decode_row(c, q + qrow * D, b, h, visible_len(c, b, n_queries, i), out + r * D,
                        NULL, NULL, qi, qsc, acc);
    }
    free(qi);
    free(qsc);
    free(acc);
    return rc;
}

/* ---------------------------------------------------------------- QUEST metadata */

/* Per-block K metadata for QUEST-style block selection, following the CANN
 * quest_prefill_metadata guide (xdnf.cn/news/235188, "reference implementation" and
 * "source-level principles"): for request r with L = seq_lens[r] tokens, KV block j
 * (j < ceil(L / bs)) holds tokens [j * bs, min((j + 1) * bs, L)); its row of metadata block
 * m = j / bs (rows = bs per metadata block) is row j % bs of physical metadata block
 * meta_table[r][m], and for every KV head h and channel d
 *   maxb[.][j % bs][h][d] = max over the block's tokens of K[slot][h][d]
 *   minb[.][j % bs][h][d] = min over the same tokens
 * where K is the dequantised cache value code * kscale[slot][h] (fp32 product). Rows of the
 * request's last metadata block after its last KV block are zero in both. */
int q8kvo_quest_metadata(const q8kvo_cache *c, const int32_t *meta_table, int max_meta_per_seq,
                         int num_meta_blocks, float *maxb, float *minb)
{
    int rc = check_cache(c);
    if (rc)
        return rc;
    if (!c->k || !c->ks || !meta_table || !maxb || !minb || max_meta_per_seq <= 0 ||
        num_meta_blocks <= 0)
        return Q8KVO_EINVAL;
    const int bs = c->block_size, Hk = c->n_kv_heads, D = c->head_dim;
    const long row_floats = (long)Hk * D; /* one metadata row: every head's D channels */
    for (int r = 0; r < c->B; ++r) {
        if ((rc = check_seq(c, r, 0)))
            return rc;
        const int L = c->seq_lens[r];
        const int nkv = (L + bs - 1) / bs;
        const int nmeta = (nkv + bs - 1) / bs;
        if (nmeta > max_meta_per_seq)
            return Q8KVO_ERANGE;
        for (int m = 0; m < nmeta; ++m) {
            const int mb = meta_table[(long)r * max_meta_per_seq + m];
            if (mb < 0 || mb >= num_meta_blocks)
                return Q8KVO_ERANGE;
            for (int row = 0; row < bs; ++row) {
                const int j = m * bs + row;
                float *mx = maxb + ((long)mb * bs + row) * row_floats;
                float *mn = minb + ((long)mb * bs + row) * row_floats;
                if (j >= nkv) { /* after the request's last KV block */
                    for (long e = 0; e < row_floats; ++e)
                        mx[e] = mn[e] = MUT(22) ? 1.0f : 0.0f;
                    continue;
                }
                const int t0 = j * bs;
                const int t1 = MUT(21) ? t0 + bs : (t0 + bs < L ? t0 + bs : L);
                for (int h = 0; h < Hk; ++h)
                    for (int d = 0; d < D; ++d) {
                        float hi = -INFINITY, lo = INFINITY;
                        for (int t = t0; t < t1; ++t) {
                            const long slot = slot_of(c, r, t);
                            const float code = (float)c->k[(slot * Hk + h) * (long)D + d];
                            const float v = MUT(23) ? code : code * c->ks[slot * Hk + h];
                            if (v > hi)
                                hi = v;
                            if (v < lo)
                                lo = v;
                        }
                        mx[(long)h * D + d] = hi;
                        mn[(long)h * D + d] = lo;
                    }
            }
        }
    }
    return Q8KVO_OK;
}

/* ---------------------------------------------------------------- q4_0 KV cache */

/* IEEE binary16 from binary32, round to nearest even (written from the format definition:
 * 1 sign bit, 5 exponent bits with bias 15, 10 fraction bits; subnormals below 2^-14). */
static uint16_t f32_to_f16(float f)
{
    uint32_t x;
    memcpy(&x, &f, 4);
    uint32_t sign = (x >> 16) & 0x8000u;
    uint32_t ax = x & 0x7fffffffu;
    if (ax >= 0x7f800000u) /* inf or NaN */
        return (uint16_t)(sign | 0x7c00u | (ax > 0x7f800000u ? 0x200u : 0u));
    double a;
    float af;
    memcpy(&af, &ax, 4);
    a = (double)af;
    if (a >= 65520.0) /* rounds to infinity */
        return (uint16_t)(sign | 0x7c00u);
    int e;
    frexp(a, &e); /* a = m * 2^e, m in [0.5, 1) */
    int q = e - 1; /* a in [2^q, 2^(q+1)) */
    if (q < -14)
        q = -14; /* subnormal range: fixed spacing 2^-24 */
    double step = ldexp(1.0, q - 10);
    double n = a / step; /* exact: a power-of-two division */
    double r = floor(n);
    double frac = n - r;
    if (frac > 0.5 || (frac == 0.5 && fmod(r, 2.0) != 0.0))
        r += 1.0;
    double v = r * step; /* the rounded magnitude */
    if (v >= 65520.0)
        return (uint16_t)(sign | 0x7c00u);
    uint32_t bits;
    if (v < ldexp(1.0, -14)) {
        bits = (uint32_t)(v / ldexp(1.0, -24)); /* subnormal fraction */
    } else {
        int ee;
        double mm = frexp(v, &ee); /* v = mm * 2^ee, mm in [0.5, 1) */
        bits = ((uint32_t)(ee - 1 + 15) << 10) | ((uint32_t)((mm * 2.0 - 1.0) * 1024.0) & 0x3ffu);
    }
    return (uint16_t)(sign | bits);
}

static double f16_to_f64(uint16_t h)
{
    int sign = (h >> 15) & 1, e = (h >> 10) & 0x1f, f = h & 0x3ff;
    double v;
    if (e == 0)
        v = ldexp((double)f, -24);
    else if (e == 31)
        v = f ? NAN : INFINITY;
    else
        v = ldexp(1.0 + f / 1024.0, e - 15);
    return sign ? -v : v;
}

int q8kvo_f32_to_f16(const float *x, long n, uint16_t *out)
{
    if (!x || !out || n < 0)
        return Q8KVO_EINVAL;
    for (long i = 0; i < n; ++i)
        out[i] = f32_to_f16(x[i]);
    return Q8KVO_OK;
}

/* One 32-value block in the llama.cpp q4_0 format (baguaai.com FlashAttention page: the
 * q4_0 / q8_0 quantised KV caches of llama.cpp; the format is llama.cpp's):
 *   m    = the value of largest magnitude, sign kept (the first one on ties)
 *   d    = m / -8                          (fp32)
 *   id   = d != 0 ? 1 / d : 0              (fp32)
 *   q_i  = min(15, trunc(x_i * id + 8.5))  (fp32 products and sums; 0 <= q_i <= 15)
 *   stored: the 4-bit codes and d rounded to binary16; value = (q - 8) * d16.
 * Codes are packed two per byte: channel 2i in the low nibble of byte i, 2i + 1 in the high
 * nibble (this library's layout). */
static void quantize_q4_block(const float *x, uint8_t *packed, uint16_t *d16)
{
    float amax = 0.0f, m = 0.0f;
    for (int i = 0; i < 32; ++i)
        if (fabsf(x[i]) > amax) {
            amax = fabsf(x[i]);
            m = x[i];
        }
    const float d = m / -8.0f;
    const float id = d != 0.0f ? 1.0f / d : 0.0f;
    for (int i = 0; i < 32; i += 2) {
        int q[2];
        for (int k = 0; k < 2; ++k) {
            const float t = x[i + k] * id + 8.5f;
            int qi = (int)t; /* trunc; t >= 0 */
            q[k] = (qi > 15 && !MUT(27)) ? 15 : qi;
        }
        packed[i / 2] = (uint8_t)(MUT(24) ? (q[1] | (q[0] << 4)) : (q[0] | (q[1] << 4)));
    }
    *d16 = f32_to_f16(d);
}

int q8kvo_quantize_q4_0(const float *x, long n, uint8_t *packed, uint16_t *d16)
{
    if (!x || !packed || !d16 || n < 0 || (n % 32) != 0)
        return Q8KVO_EINVAL;
    for (long i = 0; i < n; ++i)
        if (!isfinite(x[i]))
            return Q8KVO_EINVAL;
    for (long b = 0; b < n / 32; ++b)
        quantize_q4_block(x + 32 * b, packed + 16 * b, d16 + b);
    return Q8KVO_OK;
}

/* KV-cache write in the q4_0 format: every (token, KV head) row of k_new and v_new (fp32,
 * row (i, h) at [i * token_stride + h * head_dim]) is quantised block by block with
 * quantize_q4_block and stored at physical slot slot_mapping[i]: codes at
 * k4[(slot * n_kv_heads + h) * head_dim / 2], block scales at
 * kd[(slot * n_kv_heads + h) * head_dim / 32] (the same for V). The slot rules are those of
 * q8kvo_cache_write (negative: skipped; at or past the pool: skipped, Q8KVO_FLAG_SLOT;
 * tokens in order, so a repeated slot keeps the later token). A 32-channel block holding an
 * infinity or a NaN has no q4_0 encoding: it is stored as codes 8 (value 0) with a NaN
 * scale (binary16 0x7e00), so that the value reads back as NaN, and sets
 * Q8KVO_FLAG_NONFINITE; the row's other blocks are quantised as usual. */
int q8kvo_cache_write_q4(uint8_t *k4, uint8_t *v4, uint16_t *kd, uint16_t *vd,
                         const float *k_new, const float *v_new, const int64_t *slot_mapping,
                         long n_tokens, int n_kv_heads, int head_dim, int block_size,
                         int num_blocks, long token_stride, unsigned *flags)
{
    if (!k4 || !v4 || !kd || !vd || !k_new || !v_new || !slot_mapping || !flags)
        return Q8KVO_EINVAL;
    if (n_tokens < 0 || n_kv_heads <= 0 || head_dim <= 0 || (head_dim % 32) != 0 ||
        block_size <= 0 || num_blocks <= 0 || token_stride < (long)n_kv_heads * head_dim)
        return Q8KVO_EINVAL;
    const int64_t n_slots = (int64_t)num_blocks * block_size;
    const int nb = head_dim / 32;
    for (long i = 0; i < n_tokens; ++i) {
        const int64_t slot = slot_mapping[i];
        if (slot < 0)
            continue;
        if (slot >= n_slots) {
            *flags |= Q8KVO_FLAG_SLOT;
            continue;
        }
        for (int h = 0; h < n_kv_heads; ++h) {
            const long row = (long)slot * n_kv_heads + (MUT(28) ? (h + 1) % n_kv_heads : h);
            for (int which = 0; which < 2; ++which) {
                const float *x = (which ? v_new : k_new) + i * token_stride + (long)h * head_dim;
                uint8_t *codes = (which ? v4 : k4) + row * (head_dim / 2);
                uint16_t *d16 = (which ? vd : kd) + row * nb;
                for (int j = 0; j < nb; ++j) {
                    int finite = 1;
                    for (int c = 0; c < 32; ++c)
                        finite &= isfinite(x[32 * j + c]) ? 1 : 0;
                    if (!finite) {
                        memset(codes + 16 * j, 0x88, 16);
                        d16[j] = 0x7e00u;
                        *flags |= Q8KVO_FLAG_NONFINITE;
                        continue;
                    }
                    quantize_q4_block(x + 32 * j, codes + 16 * j, d16 + j);
                }
            }
        }
    }
    return Q8KVO_OK;
}

static int q4_code(const uint8_t *row, int i)
{
    const uint8_t byte = row[i / 2];
    return (int)((i & 1) ? (byte >> 4) : (byte & 0x0f)) - (MUT(25) ? 0 : 8);
}

static int check_q4(const q8kvo_cache_q4 *c)
{
    if (!c || !c->k4 || !c->v4 || !c->kd || !c->vd || !c->block_table || !c->seq_lens)
        return Q8KVO_EINVAL;
    if (c->B <= 0 || c->n_q_heads <= 0 || c->n_kv_heads <= 0 || c->head_dim <= 0 ||
        (c->head_dim % 32) != 0 || c->block_size <= 0 || c->max_blocks_per_seq <= 0 ||
        c->num_blocks <= 0 || (c->n_q_heads % c->n_kv_heads) != 0 || !isfinite(c->scale))
        return Q8KVO_EINVAL;
    return Q8KVO_OK;
}

/* Decode of one (b, h) over a q4_0 cache, walk-through section 2 with the q4_0 blocks:
 *   dot_j = sum_{i in block j} qi_i * (code_i - 8)               (int32, exact)
 *   s_t   = (sum_j dot_j * qsc_j * dk_j) * scale                 (fp64)
 *   online softmax as for the q8 cache, acc[d] += w * dv_{j(d)} * (code_d - 8). */
static int decode_q4_row(const q8kvo_cache_q4 *c, const float *q, int b, int h, double *out,
                         int8_t *qi, float *qsc, double *acc)
{
    const int D = c->head_dim, nb = D / 32, Hk = c->n_kv_heads;
    const int kvh = h / (c->n_q_heads / Hk);
    int L = c->seq_lens[b];
    if (L < 0 || (long)L > (long)c->max_blocks_per_seq * c->block_size)
        return Q8KVO_ERANGE;
    int rc = q8kvo_quantize_q(q + ((long)b * c->n_q_heads + h) * D, D, qi, qsc);
    if (rc)
        return rc;
    double M = -INFINITY, S = 0.0;
    for (int d = 0; d < D; ++d)
        acc[d] = 0.0;
    for (int t = 0; t < L; ++t) {
        const int blk = c->block_table[(long)b * c->max_blocks_per_seq + t / c->block_size];
        if (blk < 0 || blk >= c->num_blocks)
            return Q8KVO_ERANGE;
        const long row = ((long)blk * c->block_size + t % c->block_size) * Hk + kvh;
        const uint8_t *krow = c->k4 + row * (D / 2);
        const uint8_t *vrow = c->v4 + row * (D / 2);
        const uint16_t *kd = c->kd + row * nb, *vd = c->vd + row * nb;
        double s = 0.0;
        for (int j = 0; j < nb; ++j) {
            int32_t dot = 0;
            for (int i = 32 * j; i < 32 * j + 32; ++i)
                dot += (int32_t)qi[i] * q4_code(krow, i);
            s += (double)dot * (double)qsc[j] * f16_to_f64(kd[MUT(26) ? 0 : j]);
        }
        s *= (double)c->scale;
        double w;
        if (s > M) {
            const double f = exp(M - s);
            S *= f;
            for (int d = 0; d < D; ++d)
                acc[d] *= f;
            M = s;
            w = 1.0;
        } else {
            w = exp(s - M);
        }
        S += w;
        for (int d = 0; d < D; ++d)
            acc[d] += w * f16_to_f64(vd[d / 32]) * (double)q4_code(vrow, d);
    }
    for (int d = 0; d < D; ++d)
        out[d] = L > 0 ? acc[d] / S : 0.0;
    return Q8KVO_OK;
}

int q8kvo_decode_q4_pairs(const q8kvo_cache_q4 *c, const float *q, const int32_t *pairs, long n,
                          double *out)
{
    int rc = check_q4(c);
    if (rc)
        return rc;
    if (!q || !pairs || !out || n < 0)
        return Q8KVO_EINVAL;
    int8_t *qi;
    float *qsc;
    double *acc;
    if ((rc = scratch_alloc(c->head_dim, &qi, &qsc, &acc)))
        return rc;
    for (long r = 0; r < n && rc == Q8KVO_OK; ++r) {
        const int b = pairs[2 * r], h = pairs[2 * r + 1];
        if (b < 0 || b >= c->B || h < 0 || h >= c->n_q_heads)
            rc = Q8KVO_EINVAL;
        else
            rc = decode_q4_row(c, q, b, h, out + r * c->head_dim, qi, qsc, acc);
    }
    free(qi);
    free(qsc);
    free(acc);
    return rc;
}

int q8kvo_decode_q4_all(const q8kvo_cache_q4 *c, const float *q, double *out)
{
    int rc = check_q4(c);
    if (rc)
        return rc;
    if (!q || !out)
        return Q8KVO_EINVAL;
    int8_t *qi;
    float *qsc;
    double *acc;
    if ((rc = scratch_alloc(c->head_dim, &qi, &qsc, &acc)))
        return rc;
    for (int b = 0; b < c->B && rc == Q8KVO_OK; ++b)
        for (int h = 0; h < c->n_q_heads && rc == Q8KVO_OK; ++h)
            rc = decode_q4_row(c, q, b, h, out + ((long)b * c->n_q_heads + h) * c->head_dim, qi,
                               qsc, acc);
    free(qi);
    free(qsc);
    free(acc);
    return rc;
}

/* ---------------------------------------------------------------- three pass */

/* The naive form the walk-through (section 3) contrasts with, laid out like the
 * llama2.c loop: all scores first, then the stable softmax (subtract the max,
 * exponentiate, sum, divide), then the weighted sum of dequantised V. */
int q8kvo_decode_threepass(const q8kvo_cache *c, const float *q, int b, int h, double *out)
{
    int rc = check_q8(c, q, out);
    if (rc || (rc = check_seq(c, b, h)))
        return rc;
    int D = c->head_dim, kvh = kv_head_of(c, h), L = c->seq_lens[b];
    for (int d = 0; d < D; ++d)
        out[d] = 0.0;
    if (L == 0)
        return Q8KVO_OK;
    double *s = (double *)malloc(sizeof(double) * (size_t)L);
    if (!s)
        return Q8KVO_ENOMEM;
    rc = q8kvo_scores(c, q, b, h, s);
    if (rc) {
        free(s);
        return rc;
    }
    double mx = s[0];
    for (int t = 1; t < L; ++t)
        if (s[t] > mx)
            mx = s[t];
    double sum = 0.0;
    for (int t = 0; t < L; ++t) {
        s[t] = exp(s[t] - mx);
        sum += s[t];
    }
    for (int t = 0; t < L; ++t) {
        long slot = slot_of(c, b, t);
        const int8_t *vrow = c->v + (slot * c->n_kv_heads + kvh) * (long)D;
        double a = s[t] / sum * (double)c->vs[slot * c->n_kv_heads + kvh];
        for (int d = 0; d < D; ++d)
            out[d] += a * (double)vrow[d];
    }
    free(s);
    return Q8KVO_OK;
}

/* ---------------------------------------------------------------- unquantised */

/* fp64 attention of the original fp32 q, K and V (no quantisation anywhere):
 * s_t = scale * q . k_t, stable softmax, weighted V. */
int q8kvo_attn_fp32(const q8kvo_cache *c, const float *q, const float *k32, const float *v32,
                    int b, int h, double *out)
{
    int rc = check_cache(c);
    if (rc)
        return rc;
    if (!q || !k32 || !v32 || !out)
        return Q8KVO_EINVAL;
    if ((rc = check_seq(c, b, h)))
        return rc;
    int D = c->head_dim, kvh = kv_head_of(c, h), L = c->seq_lens[b];
    const float *qh = q + ((long)b * c->n_q_heads + h) * D;
    for (int d = 0; d < D; ++d)
        out[d] = 0.0;
    if (L == 0)
        return Q8KVO_OK;
    double *s = (double *)malloc(sizeof(double) * (size_t)L);
    if (!s)
        return Q8KVO_ENOMEM;
    double mx = -INFINITY;
    for (int t = 0; t < L; ++t) {
        long slot = slot_of(c, b, t);
        const float *krow = k32 + (slot * c->n_kv_heads + kvh) * (long)D;
        double acc = 0.0;
        for (int d = 0; d < D; ++d)
            acc += (double)qh[d] * (double)krow[d];
        s[t] = acc * (double)c->scale;
        if (s[t] > mx)
            mx = s[t];
    }
    double sum = 0.0;
    for (int t = 0; t < L; ++t) {
        s[t] = exp(s[t] - mx);
        sum += s[t];
    }
    for (int t = 0; t < L; ++t) {
        long slot = slot_of(c, b, t);
        const float *vrow = v32 + (slot * c->n_kv_heads + kvh) * (long)D;
        double a = s[t] / sum;
        for (int d = 0; d < D; ++d)
            out[d] += a * (double)vrow[d];
    }
    free(s);
    return Q8KVO_OK;
}
