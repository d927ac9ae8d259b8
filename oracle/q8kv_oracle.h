/*
 * q8kv_oracle.h -- plain, slow, single-threaded CPU oracle for q8-KV single-query
 * decode attention.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path links, loads or calls this
 * code; only the test suite, the smoke check and the benchmark's CPU-baseline leg do.
 * It shares no source, header, table or helper with the CUDA library.
 *
 * What it computes follows the Kestrel-LLM walk-through "flash_attn_single_q_q8_neon"
 * (trdm.cn/news/511694):
 *   - section 2, part 1 ("Q quantised once"): Q -> int8 in 32-element blocks with a
 *     max-abs/127 scale per block, a zero-block guard, and a clamp;
 *   - section 2, part 2 ("online softmax running state"): per token, exact int8 block
 *     dot products into int32, each block scaled by its Q scale, then by the
 *     per-(token, KV head) K scale and the softmax scale; the running max M and sum S,
 *     with the accumulator rescaled whenever M rises; V accumulated as int8 V times
 *     (softmax weight x per-(token, head) V scale);
 *   - section 2, part 3 ("normalise the output"): one division by S at the end;
 *   - section 3 ("consequences of the change"): the naive variant that stores every
 *     score first is functionally equivalent (used here as a cross-check);
 *   - the opening and the kernel signature (KV compressed to q8 with one scale per
 *     (token, KV head), applied as scale * 1/127 at use): the KV-cache write that fills
 *     the pools, with the section 2 part 1 quantiser applied to whole rows.
 * The QUEST block metadata (per-channel max / min of K over each KV block) follows the
 * CANN quest_prefill_metadata guide (xdnf.cn/news/235188) on the q8 pool.
 * Several query tokens per sequence (the multi-query "TILE" decode of the llama.cpp
 * change on baguaai.com's FlashAttention page) are the same single pass per (sequence,
 * query, head), each query seeing the cache up to its own position (causal).
 * GQA head mapping kv_head = q_head / (n_q_heads / n_kv_heads) follows the llama2.c
 * attention loop (aicoding.csdn.net, "attention core logic").
 * The block-table -> slot mapping follows beaiera.top "deepseek-attention-div64",
 * section "Top-K index global mapping": slot = block_table[b][t / bs] * bs + t % bs.
 *
 * Precision: the Q quantisation runs in IEEE fp32 (it decides integers, so it is done
 * in the precision the GPU uses), everything after the int32 dots runs in fp64.
 * Rounding of the quantised Q: round-half-to-even, then clamp to [-127, 127].
 *
 * Pinning: every function here is pinned by the -m "not gpu" tests to hand-derived
 * golden cases, closed forms and library routines; see the test files named
 * test_oracle_*.py.
 */
#ifndef Q8KV_ORACLE_H
#define Q8KV_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Return codes of every oracle call. */
#define Q8KVO_OK 0
#define Q8KVO_EINVAL 1   /* null pointer, bad size, or non-finite input */
#define Q8KVO_ERANGE 2   /* seq_len or block-table entry outside the cache */
#define Q8KVO_ENOMEM 3

/* A paged q8 KV cache, exactly as the CUDA library receives it.
 *   k, v     int8  [num_blocks][block_size][n_kv_heads][head_dim]
 *   ks, vs   fp32  [num_blocks][block_size][n_kv_heads]   (dequant multipliers)
 *   block_table int32 [B][max_blocks_per_seq]
 *   seq_lens    int32 [B]
 * All pointers are host pointers owned by the caller. */
typedef struct {
    const int8_t *k;
    const int8_t *v;
    const float *ks;
    const float *vs;
    const int32_t *block_table;
    const int32_t *seq_lens;
    int B;
    int n_q_heads;
    int n_kv_heads;
    int head_dim;
    int block_size;
    int max_blocks_per_seq;
    int num_blocks;
    float scale;
} q8kvo_cache;

/* Quantise n fp32 values (n a multiple of 32) block by block.
 * qi[n] receives the int8 codes, qsc[n/32] the per-block fp32 scales. */
int q8kvo_quantize_q(const float *q, long n, int8_t *qi, float *qsc);

/* Flags of the KV-cache write (the same bits as the CUDA library's device error word). */
#define Q8KVO_FLAG_SLOT 0x8u       /* a slot at or past num_blocks * block_size (skipped) */
#define Q8KVO_FLAG_NONFINITE 0x10u /* a row held an infinity or a NaN (codes 0, scale NaN) */

/* Quantise one K or V row of n fp32 values for the cache: one fp32 dequantisation
 * multiplier for the row and n int8 codes (rule in q8kv_oracle.c). Non-finite rows set
 * Q8KVO_FLAG_NONFINITE in *flags. */
int q8kvo_quantize_kv_row(const float *x, int n, int8_t *codes, float *scale, unsigned *flags);

/* KV-cache write: quantise the n_tokens x n_kv_heads rows of k_new and v_new (fp32, row
 * (i, h) at [i * token_stride + h * head_dim]) and store codes and scales at physical slot
 * slot_mapping[i] of the pools k, v [num_blocks][block_size][n_kv_heads][head_dim] and
 * ks, vs [num_blocks][block_size][n_kv_heads]. Negative slots are skipped; slots past the
 * pool are skipped and set Q8KVO_FLAG_SLOT. */
int q8kvo_cache_write(int8_t *k, int8_t *v, float *ks, float *vs, const float *k_new,
                      const float *v_new, const int64_t *slot_mapping, long n_tokens,
                      int n_kv_heads, int head_dim, int block_size, int num_blocks,
                      long token_stride, unsigned *flags);

/* int32 dot product of each 32-element block of the quantised query of (b, h) with
 * the K row of every token of sequence b: dots[t][j], t < seq_lens[b], j < head_dim/32. */
int q8kvo_block_dots(const q8kvo_cache *c, const float *q, int b, int h, int32_t *dots);

/* Scores s[t] (fp64, natural-log units) of (b, h), exactly as the online pass uses them. */
int q8kvo_scores(const q8kvo_cache *c, const float *q, int b, int h, double *s);

/* Single-pass online-softmax decode of one (b, h): out[head_dim] in fp64.
 * m_trace (optional, length seq_lens[b]) receives M after each token;
 * n_iter (optional) receives the number of token iterations executed. */
int q8kvo_decode_online(const q8kvo_cache *c, const float *q, int b, int h,
                        double *out, double *m_trace, long *n_iter);

/* Decode with several new query tokens per sequence (speculative or multi-token decode):
 * q and out are [B][n_queries][n_q_heads][head_dim] (out in fp64); seq_lens[b] counts every
 * cached token including the n_queries new ones, and query i attends causally to tokens
 * t < seq_lens[b] - (n_queries - 1 - i); a query that sees no token gets a zero row.
 * n_queries = 1 is q8kvo_decode_all. */
int q8kvo_decode_multi(const q8kvo_cache *c, const float *q, int n_queries, double *out);

/* The same for n chosen rows: rows[3*r .. 3*r+2] = (b, query index i, head h);
 * out[n][head_dim] (fp64). */
int q8kvo_decode_multi_rows(const q8kvo_cache *c, const float *q, int n_queries,
                            const int32_t *rows, long n, double *out);

/* QUEST-style per-block K metadata (CANN quest_prefill_metadata guide, xdnf.cn/news/235188):
 * maxb, minb fp32 [num_meta_blocks][block_size][n_kv_heads][head_dim]; row j % bs of
 * metadata block meta_table[r][j / bs] holds the per-channel max / min of the dequantised
 * K over the tokens of request r's KV block j; unused rows of a request's last metadata
 * block are zero. meta_table int32 [B][max_meta_per_seq]. Other fields of c as above
 * (v, vs, n_q_heads and scale are not used). */
int q8kvo_quest_metadata(const q8kvo_cache *c, const int32_t *meta_table, int max_meta_per_seq,
                         int num_meta_blocks, float *maxb, float *minb);

/* A paged q4_0 KV cache (llama.cpp's q4_0 blocks, this library's packing):
 *   k4, v4   uint8  [num_blocks][block_size][n_kv_heads][head_dim / 2]  two 4-bit codes per
 *            byte: channel 2i in the low nibble of byte i, 2i + 1 in the high nibble
 *   kd, vd   binary16 bits [num_blocks][block_size][n_kv_heads][head_dim / 32]: the scale d
 *            of each 32-channel block; value = (code - 8) * d
 * Other fields as q8kvo_cache. */
typedef struct {
    const uint8_t *k4;
    const uint8_t *v4;
    const uint16_t *kd;
    const uint16_t *vd;
    const int32_t *block_table;
    const int32_t *seq_lens;
    int B;
    int n_q_heads;
    int n_kv_heads;
    int head_dim;
    int block_size;
    int max_blocks_per_seq;
    int num_blocks;
    float scale;
} q8kvo_cache_q4;

/* binary16 bits of n fp32 values, round to nearest even. */
int q8kvo_f32_to_f16(const float *x, long n, uint16_t *out);

/* q4_0 quantisation of n fp32 values (n a multiple of 32): packed [n / 2] codes and
 * d16 [n / 32] binary16 scales (rule in q8kv_oracle.c). */
int q8kvo_quantize_q4_0(const float *x, long n, uint8_t *packed, uint16_t *d16);

/* KV-cache write in the q4_0 format: the rows of k_new / v_new (as q8kvo_cache_write) are
 * quantised per 32-channel block (q8kvo_quantize_q4_0's rule) and stored at their slots of
 * k4, v4 [num_blocks][block_size][n_kv_heads][head_dim / 2] and kd, vd
 * [num_blocks][block_size][n_kv_heads][head_dim / 32]; slot rules and flags as
 * q8kvo_cache_write; a block holding inf or NaN is stored as codes 8 with a NaN scale
 * (Q8KVO_FLAG_NONFINITE). */
int q8kvo_cache_write_q4(uint8_t *k4, uint8_t *v4, uint16_t *kd, uint16_t *vd,
                         const float *k_new, const float *v_new, const int64_t *slot_mapping,
                         long n_tokens, int n_kv_heads, int head_dim, int block_size,
                         int num_blocks, long token_stride, unsigned *flags);

/* Single-query decode over a q4_0 cache (fp64 out [B][n_q_heads][head_dim], or the chosen
 * (b, h) pairs): the query quantisation and the online softmax of the q8 decode, with
 * the K and V values (code - 8) * d of their 32-channel blocks. */
int q8kvo_decode_q4_all(const q8kvo_cache_q4 *c, const float *q, double *out);
int q8kvo_decode_q4_pairs(const q8kvo_cache_q4 *c, const float *q, const int32_t *pairs, long n,
                          double *out);

/* Naive three-pass variant (all scores, then max, then exp/sum, then weighted V). */
int q8kvo_decode_threepass(const q8kvo_cache *c, const float *q, int b, int h, double *out);

/* Online decode of every (b, h): out[B][n_q_heads][head_dim] (fp64). */
int q8kvo_decode_all(const q8kvo_cache *c, const float *q, double *out);

/* Online decode of n chosen (b, h) pairs: pairs[2*i] = b, pairs[2*i+1] = h;
 * out[n][head_dim] (fp64). */
int q8kvo_decode_pairs(const q8kvo_cache *c, const float *q, const int32_t *pairs, long n,
                       double *out);

/* Unquantised attention of one (b, h) in fp64 from fp32 q and fp32 K/V pools laid out
 * like the int8 pools ([num_blocks][block_size][n_kv_heads][head_dim]); the q8 fields of
 * c (k, v, ks, vs) are ignored. Used to report the error of q8 against fp32 attention. */
int q8kvo_attn_fp32(const q8kvo_cache *c, const float *q, const float *k32, const float *v32,
                    int b, int h, double *out);

#ifdef __cplusplus
}
#endif
#endif
