/*
 * q8kv.h -- C ABI of the q8-KV single-query decode-attention library for NVIDIA B200
 * (sm_100a). Shared library: decode_attention_int8_b200/libq8kv.so.
 *
 * The operation (Kestrel-LLM walk-through "flash_attn_single_q_q8_neon",
 * trdm.cn/news/511694, section 2 parts 1-3): for every batch entry b and query head h,
 *   1. quantise q[b][h] once to int8 in 32-element blocks: qm = max|q| (if qm < 1e-6 then
 *      qm = 1), qsc_j = qm * fl(1/127), code = clamp(round-half-to-even(q * fl(127/qm)),
 *      -127, 127), all in IEEE fp32;
 *   2. for every token t < seq_lens[b], with kv = h / (n_q_heads / n_kv_heads) (the GQA
 *      mapping of the llama2.c loop, aicoding.csdn.net, "attention core logic") and
 *      slot = block_table[b][t / kv_block_size] * kv_block_size + t % kv_block_size
 *      (beaiera.top "deepseek-attention-div64", "Top-K index global mapping"):
 *        dot_j = sum over the 32 channels of block j of code * K[slot][kv]   (int32, exact)
 *        s_t   = (sum_j dot_j * qsc_j) * kscale[slot][kv] * scale
 *   3. out[b][h] = sum_t exp(s_t - M) * vscale[slot][kv] * V[slot][kv] / sum_t exp(s_t - M),
 *      computed in one pass with a running max M and running sum S (online softmax) and
 *      one division at the end.
 * The scan is split over the sequence across thread blocks (flash-decoding) and the
 * pieces are merged by a log-sum-exp combine kernel launched right after the decode
 * kernel on the same stream; the result equals the single pass up to fp32 rounding order.
 * Both kernels use programmatic dependent launch: each may be scheduled while the kernel
 * before it on the stream drains, and waits for that kernel to complete before it reads
 * or writes global memory.
 *
 * Layouts (all row-major, C order):
 *   q            fp32  [B][n_q_heads][head_dim]
 *   out          fp32  [B][n_q_heads][head_dim]
 *   k_blocks     int8  [num_kv_blocks][kv_block_size][n_kv_heads][head_dim]
 *   v_blocks     int8  same shape as k_blocks
 *   kscale       fp32  [num_kv_blocks][kv_block_size][n_kv_heads]  (dequant multipliers:
 *   vscale       fp32  same shape                                   value = code * scale)
 *   block_table  int32 [B][max_blocks_per_seq]  physical block of each logical block;
 *                      entries past ceil(seq_lens[b] / kv_block_size) are never read
 *   seq_lens     int32 [B]
 * The same block table indexes both pools and both scale arrays; scales are indexed by
 * the physical slot.
 *
 * Pointers: device pointers owned by the caller; the library never frees or retains
 * them. q, out, k_blocks, v_blocks, kscale, vscale must be 16-byte aligned (any torch or
 * cudaMalloc allocation is).
 *
 * Asynchrony: every call enqueues work on `stream` (NULL = legacy default stream) and
 * returns without synchronising. Q8KV_OK means the work was enqueued; faults surface at
 * the caller's next synchronisation.
 *
 * Errors: argument checks run on the host before any launch and return
 * Q8KV_ERR_INVALID_ARG or Q8KV_ERR_UNSUPPORTED without touching the GPU. Data that only
 * the device can see is checked in the kernel without trapping: a seq_len below 0 is
 * treated as 0, one above max_blocks_per_seq * kv_block_size is clamped, a block-table
 * entry outside [0, num_kv_blocks) makes the kernel skip that block's tokens; each of
 * these sets a bit in a device-side error word that q8kv_device_errors() reads.
 *
 * Supported shapes of the decode kernel: head_dim 128; kv_block_size a power of two in
 * [16, 256]; n_q_heads a multiple of n_kv_heads; query rows per KV head R (the group
 * n_q_heads / n_kv_heads, times n_queries for q8kv_decode_attn_multi) at most 128; a tile
 * holds up to 8 / ceil_pow2(R / 16) KV heads, and when it holds fewer than n_kv_heads (its
 * scales then come through a 2-D copy whose rows must be 16-byte multiples) n_kv_heads
 * must be a multiple of 4; B <= 16384; num_kv_blocks * kv_block_size < 2^31. Other shapes
 * return Q8KV_ERR_UNSUPPORTED.
 */
#ifndef Q8KV_H
#define Q8KV_H

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    Q8KV_OK = 0,
    Q8KV_ERR_INVALID_ARG = 1, /* null pointer, non-positive size, bad alignment, ... */
    Q8KV_ERR_UNSUPPORTED = 2, /* valid arguments outside the shapes the kernels handle */
    Q8KV_ERR_CUDA = 3,        /* a CUDA runtime call failed: see q8kv_last_cuda_error() */
    Q8KV_ERR_WORKSPACE = 4    /* workspace null or smaller than q8kv_workspace_bytes() */
} q8kv_status;

/* Device-side error bits reported by q8kv_device_errors(). */
#define Q8KV_DEVERR_SEQ_LEN 0x1u     /* a seq_len was negative or too long (clamped)     */
#define Q8KV_DEVERR_BLOCK_TABLE 0x2u /* a block-table entry was outside the pool (skipped) */
#define Q8KV_DEVERR_TIMEOUT 0x4u     /* a pipeline wait ran past its limit (kernel gave up) */
#define Q8KV_DEVERR_SLOT 0x8u        /* cache write: a slot past the pool (row skipped)     */
#define Q8KV_DEVERR_NONFINITE 0x10u  /* cache write: a row held inf or NaN (codes 0, NaN scale) */
#define Q8KV_DEVERR_META 0x20u       /* QUEST metadata: a metadata-table entry outside its pool
                                        (row skipped), or a table too short for a request */

/*
 * Decode attention with a library-managed workspace (one per device, grown on demand
 * under a lock, zero-initialised; the first call on a device, or a call that needs a
 * larger workspace, allocates and so must not happen during stream capture). Calls that
 * run concurrently on different streams of one device must use q8kv_decode_attn_ws with
 * separate workspaces.
 *
 *   out, q, k_blocks, v_blocks, kscale, vscale, block_table, seq_lens: see the layouts above
 *   B                  batch size (> 0)
 *   n_q_heads          query heads (> 0, a multiple of n_kv_heads)
 *   n_kv_heads         KV heads (> 0)
 *   head_dim           channels per head (128)
 *   kv_block_size      tokens per physical block
 *   max_blocks_per_seq row stride of block_table; seq_lens[b] <= max_blocks_per_seq *
 *                      kv_block_size
 *   num_kv_blocks      physical blocks in each pool (bounds every block-table entry)
 *   scale              softmax scale (finite; 1/sqrt(head_dim) in standard attention,
 *                      beaiera.top "deepseek-attention-div64", "derivation of the scale")
 */
q8kv_status q8kv_decode_attn(float *out, const float *q, const int8_t *k_blocks,
                             const int8_t *v_blocks, const float *kscale, const float *vscale,
                             const int32_t *block_table, const int32_t *seq_lens, int B,
                             int n_q_heads, int n_kv_heads, int head_dim, int kv_block_size,
                             int max_blocks_per_seq, int num_kv_blocks, float scale,
                             cudaStream_t stream);

/*
 * Decode attention with several new query tokens per sequence (speculative or multi-token
 * decode), library-managed workspace. The llama.cpp change on baguaai.com's FlashAttention
 * page moves quantised-KV decode from a per-query (VEC) kernel to a tiled (TILE) one; here
 * the n_queries tokens of a sequence share every K/V tile it streams, as extra rows of the
 * same tensor-core tiles, so the cache is read once for all of them.
 *
 *   q, out     fp32 [B][n_queries][n_q_heads][head_dim]
 *   seq_lens   tokens in the cache per sequence, the n_queries new ones included (they are
 *              its last n_queries tokens, written beforehand, e.g. by q8kv_cache_write)
 * Query i of sequence b attends causally to tokens t < seq_lens[b] - (n_queries - 1 - i),
 * with the single-query arithmetic of q8kv_decode_attn per (b, i, head); a query that sees
 * no token (seq_lens[b] < n_queries - i) gets a zero row. n_queries = 1 is
 * q8kv_decode_attn. Supported shapes: as above with R = n_queries * n_q_heads /
 * n_kv_heads rows per KV head. With n_queries > 1, 9 <= R <= 32 and n_kv_heads 1 or a
 * multiple of 4, the call runs on the fifth-generation tensor cores (tcgen05.mma with
 * int32 accumulators in tensor memory; rows padded to 16 or 32); other shapes on the warp
 * MMAs of q8kv_decode_attn. Both give the same results within the documented tolerance.
 * Other arguments, errors and asynchrony as q8kv_decode_attn.
 */
q8kv_status q8kv_decode_attn_multi(float *out, const float *q, const int8_t *k_blocks,
                                   const int8_t *v_blocks, const float *kscale,
                                   const float *vscale, const int32_t *block_table,
                                   const int32_t *seq_lens, int B, int n_queries, int n_q_heads,
                                   int n_kv_heads, int head_dim, int kv_block_size,
                                   int max_blocks_per_seq, int num_kv_blocks, float scale,
                                   cudaStream_t stream);

/*
 * Decode attention over a q4_0 KV cache (llama.cpp's q4_0 blocks, one of the quantised
 * KV-cache types of the llama.cpp change on baguaai.com's FlashAttention page),
 * library-managed workspace:
 *   k4_blocks, v4_blocks  uint8 [num_kv_blocks][kv_block_size][n_kv_heads][head_dim / 2]:
 *                         4-bit codes, channel 2i in the low nibble of byte i, 2i + 1 in
 *                         the high nibble
 *   kd, vd                binary16 bits [num_kv_blocks][kv_block_size][n_kv_heads]
 *                         [head_dim / 32]: the scale d of each 32-channel block
 * The value of channel c of a row is (code_c - 8) * d_(c / 32). With the query quantised
 * as in step 1 above, token t scores
 *   s_t = (sum_j dot_j * qsc_j * dk_tj) * scale,  dot_j = sum over block j of qi * (code - 8)
 * (exact int32), and out is the online-softmax average of the V values. Other arguments,
 * layouts and asynchrony as q8kv_decode_attn; kd and vd must be 8-byte aligned. Supported:
 * head_dim 128; group n_q_heads / n_kv_heads <= 16; B * n_kv_heads <= 65535. Two kernel
 * launches (per chunk of 256 tokens, then a merge of the chunks).
 */
q8kv_status q8kv_decode_attn_q4(float *out, const float *q, const uint8_t *k4_blocks,
                                const uint8_t *v4_blocks, const uint16_t *kd,
                                const uint16_t *vd, const int32_t *block_table,
                                const int32_t *seq_lens, int B, int n_q_heads, int n_kv_heads,
                                int head_dim, int kv_block_size, int max_blocks_per_seq,
                                int num_kv_blocks, float scale, cudaStream_t stream);

/* Bytes of workspace q8kv_decode_attn_ws needs for these sizes on the current device
 * (0 if the sizes are invalid or unsupported). */
size_t q8kv_workspace_bytes(int B, int n_q_heads, int n_kv_heads, int head_dim);

/* Zero a caller-owned workspace. Optional and without effect on results: no part of the
 * workspace needs an initial value (every call writes the partial results its combine
 * step reads before that step reads them); it only gives a fresh workspace defined
 * contents. */
q8kv_status q8kv_workspace_init(void *workspace, size_t workspace_bytes, cudaStream_t stream);

/* Same as q8kv_decode_attn with a caller-owned workspace (device memory of at least
 * q8kv_workspace_bytes() bytes, 256-byte aligned, any contents). The call allocates
 * nothing. Calls that overlap on the GPU must not share a workspace. */
q8kv_status q8kv_decode_attn_ws(float *out, const float *q, const int8_t *k_blocks,
                                const int8_t *v_blocks, const float *kscale,
                                const float *vscale, const int32_t *block_table,
                                const int32_t *seq_lens, int B, int n_q_heads, int n_kv_heads,
                                int head_dim, int kv_block_size, int max_blocks_per_seq,
                                int num_kv_blocks, float scale, void *workspace,
                                size_t workspace_bytes, cudaStream_t stream);

/* Size of the scratch array that q8kv_decode_attn_static uses (12 MiB per device). */
#define Q8KV_STATIC_SCRATCH_BYTES (12u * 1024u * 1024u)

/*
 * Same as q8kv_decode_attn, but the call allocates no device memory at all: the partial
 * results of the split sequences live in a fixed device array inside the library,
 * Q8KV_STATIC_SCRATCH_BYTES bytes per device. None of the source pages has a counterpart
 * to this entry point; they describe the computation, not where its scratch lives.
 *
 * Who needs it: a caller that must not allocate while it serves requests. Examples are a
 * server whose pool allocator hands out all device memory at start-up (a cudaMalloc then
 * fails, or takes memory the pool had counted on), and a timed decode step that cannot
 * afford the device-wide synchronisation of cudaFree or the latency of a first cudaMalloc.
 * q8kv_decode_attn allocates on its first call per device and again when a shape needs a
 * larger workspace; q8kv_decode_attn_ws makes the caller allocate one.
 *
 * Set-up: the first call on each device (with that device current) looks up the array's
 * address (cudaGetSymbolAddress) and the kernels' attributes; later calls reuse them.
 * Make that first call before any stream capture begins.
 *
 * Initial state: nothing in the array needs to start at zero. Every call's decode kernel
 * writes the partial results (2 slots per CTA) that the same call's combine kernel reads,
 * and the combine reads no other slot.
 *
 * Races: every call on one device uses the same array. Two calls that may run at the
 * same time on the GPU (different streams with no ordering between them, or threads
 * issuing to different streams) corrupt each other's results. Order them on one stream,
 * or use q8kv_decode_attn_ws with one workspace per stream. Calls of the other entry
 * points never touch this array.
 *
 * Errors: as q8kv_decode_attn, plus Q8KV_ERR_WORKSPACE (and nothing enqueued) when the
 * shape needs more than Q8KV_STATIC_SCRATCH_BYTES, i.e. when q8kv_workspace_bytes() for
 * it is larger. On a 148-SM B200 that happens when one tile covers more than 80 query
 * heads (a tile holds up to 8 KV heads and all their query heads): n_q_heads 128 with
 * n_kv_heads 8 or 1 is rejected, 64 with 8 fits.
 */
q8kv_status q8kv_decode_attn_static(float *out, const float *q, const int8_t *k_blocks,
                                    const int8_t *v_blocks, const float *kscale,
                                    const float *vscale, const int32_t *block_table,
                                    const int32_t *seq_lens, int B, int n_q_heads,
                                    int n_kv_heads, int head_dim, int kv_block_size,
                                    int max_blocks_per_seq, int num_kv_blocks, float scale,
                                    cudaStream_t stream);

/*
 * KV-cache write: quantise n_tokens new K rows and V rows per KV head and store them, with
 * their scales, at the given physical slots of the pools the decode entry points read.
 *
 * Quantisation of each (token, KV head) row of head_dim values, for K and V alike (the
 * walk-through's cache keeps one scale per (token, KV head), kernel signature comment, and
 * forms the dequantisation multiplier as scale * 1/127, section 2 part 2; the quantiser is
 * step 1's, taken over the whole row), in IEEE fp32:
 *   amax = max|x| (1 when below 1e-6), scale = amax * fl(1/127),
 *   code = clamp(round-half-to-even(x * fl(127 / amax)), -127, 127)
 * kscale / vscale receive `scale` (the multiplier value = code * scale of the layouts
 * above). A row holding an infinity or a NaN is stored as codes 0 with a NaN scale and
 * sets Q8KV_DEVERR_NONFINITE.
 *
 * Placement (beaiera.top "deepseek-attention-div64", "Top-K index global mapping"):
 * token i goes to slot s = slot_mapping[i] = block * kv_block_size + offset; row h lands at
 * k_blocks[s][h][:] with its scale at kscale[s][h] (the same for V). A negative slot marks
 * padding: the token is skipped. A slot >= num_kv_blocks * kv_block_size is skipped and
 * sets Q8KV_DEVERR_SLOT. Slots must be distinct within one call (two tokens naming one
 * slot race; which one lands is unspecified).
 *
 *   k_blocks, v_blocks, kscale, vscale: the pools (layouts above), written in place
 *   k_new, v_new  fp32; row (i, h) starts at element i * token_stride + h * head_dim
 *                 (16-byte aligned)
 *   slot_mapping  int64 [n_tokens]
 *   n_tokens      >= 0 (0: nothing is enqueued, and k_new, v_new, slot_mapping may be null)
 *   head_dim      64, 128 or 256 (other multiples of 32: Q8KV_ERR_UNSUPPORTED)
 *   token_stride  floats between consecutive tokens' rows (0 = n_kv_heads * head_dim;
 *                 otherwise >= that and a multiple of 4, e.g. the row stride of a fused
 *                 QKV projection)
 * One kernel launch, asynchronous on `stream`; it may be scheduled while the previous
 * kernel on the stream drains and waits for it before reading anything (programmatic
 * dependent launch), and a decode call enqueued after it sees the written rows.
 */
q8kv_status q8kv_cache_write(int8_t *k_blocks, int8_t *v_blocks, float *kscale, float *vscale,
                             const float *k_new, const float *v_new,
                             const int64_t *slot_mapping, int n_tokens, int n_kv_heads,
                             int head_dim, int kv_block_size, int num_kv_blocks,
                             long long token_stride, cudaStream_t stream);

/*
 * KV-cache write in the q4_0 format (llama.cpp's q4_0 blocks, one of the quantised KV-cache
 * types of the llama.cpp change on baguaai.com's FlashAttention page), into the pools
 * q8kv_decode_attn_q4 reads: every (token, KV head) row of K and of V is quantised per
 * 32-channel block, in IEEE fp32 with every operation rounded on its own:
 *   m = the value of largest magnitude, sign kept (the first one on ties; +0 for an
 *       all-zero block), d = m / -8, id = d != 0 ? 1 / d : 0,
 *   code = min(15, trunc(x * id + 8.5))  (0..15; value = (code - 8) * d)
 * d is stored as binary16 (round to nearest even; beyond 65504 it becomes infinity, as in
 * the format). Codes are packed two per byte, channel 2i in the low nibble of byte i. A block
 * holding an infinity or a NaN is stored as codes 8 with a NaN scale (0x7e00) and sets
 * Q8KV_DEVERR_NONFINITE (a decode over it returns NaN); the row's other blocks are
 * quantised as usual.
 *
 *   k4_blocks, v4_blocks  uint8 [num_kv_blocks][kv_block_size][n_kv_heads][head_dim / 2],
 *                         16-byte aligned, written in place
 *   kd, vd                binary16 bits [num_kv_blocks][kv_block_size][n_kv_heads]
 *                         [head_dim / 32], 8-byte aligned, written in place
 *   k_new, v_new, slot_mapping, n_tokens, token_stride: as q8kv_cache_write (the same slot
 *                         rules: negative = padding, skipped; past the pool = skipped with
 *                         Q8KV_DEVERR_SLOT; distinct slots within one call)
 *   head_dim              64, 128 or 256 (the q4_0 decode reads head_dim 128)
 * One kernel launch, asynchronous on `stream`, programmatic dependent launch as
 * q8kv_cache_write.
 */
q8kv_status q8kv_cache_write_q4(uint8_t *k4_blocks, uint8_t *v4_blocks, uint16_t *kd,
                                uint16_t *vd, const float *k_new, const float *v_new,
                                const int64_t *slot_mapping, int n_tokens, int n_kv_heads,
                                int head_dim, int kv_block_size, int num_kv_blocks,
                                long long token_stride, cudaStream_t stream);

/*
 * QUEST-style per-block K metadata (CANN quest_prefill_metadata guide, xdnf.cn/news/235188):
 * for every request r, KV block j < ceil(seq_lens[r] / kv_block_size) and KV head h, the
 * per-channel maximum and minimum of the dequantised K (code * kscale, one fp32 product)
 * over the block's tokens (the last block: only its tokens < seq_lens[r]). A metadata block
 * holds kv_block_size rows, one per KV block: KV block j of request r is row
 * j % kv_block_size of physical metadata block meta_block_table[r][j / kv_block_size].
 * The rows of a request's last metadata block after its last KV block are set to zero in
 * both arrays; metadata blocks no request uses are not touched. QUEST bounds q . k over a
 * block from these two vectors to choose the blocks a decode step reads.
 *
 *   maxblocks, minblocks  fp32 [num_meta_blocks][kv_block_size][n_kv_heads][head_dim],
 *                         16-byte aligned, written
 *   k_blocks, kscale      the K pool and its scales (layouts above); v is not read
 *   block_table, seq_lens as for decode
 *   meta_block_table      int32 [B][max_meta_blocks_per_seq]
 *   head_dim              128
 * Device-side checks: a seq_len outside [0, max_blocks_per_seq * kv_block_size] is clamped
 * (Q8KV_DEVERR_SEQ_LEN); a block-table entry outside the pool skips its row
 * (Q8KV_DEVERR_BLOCK_TABLE); a metadata-table entry outside [0, num_meta_blocks), or a
 * request needing more than max_meta_blocks_per_seq metadata blocks, sets
 * Q8KV_DEVERR_META (the rows it cannot place are skipped). Host-side: Q8KV_ERR_UNSUPPORTED
 * for head_dim != 128, or when max_blocks_per_seq, num_kv_blocks, num_meta_blocks or
 * max_meta_blocks_per_seq times kv_block_size reaches 2^31. One kernel launch, asynchronous
 * on `stream`, programmatic dependent launch as the other kernels.
 */
q8kv_status q8kv_quest_metadata(float *maxblocks, float *minblocks, const int8_t *k_blocks,
                                const float *kscale, const int32_t *block_table,
                                const int32_t *seq_lens, const int32_t *meta_block_table, int B,
                                int n_kv_heads, int head_dim, int kv_block_size,
                                int max_blocks_per_seq, int max_meta_blocks_per_seq,
                                int num_kv_blocks, int num_meta_blocks, cudaStream_t stream);

/* Debug: the Q quantisation alone (step 1) on n_rows rows of head_dim fp32 values
 * (head_dim a multiple of 32). qi int8 [n_rows][head_dim], qsc fp32
 * [n_rows][head_dim / 32]. Uses the device routine the decode kernel uses. */
q8kv_status q8kv_debug_quantize_q(int8_t *qi, float *qsc, const float *q, int n_rows,
                                  int head_dim, cudaStream_t stream);

/* Debug: the int32 block dot products of step 2, produced by the decode kernel itself
 * (same staging and tensor-core fragments) and written out as
 * dots int32 [B][n_q_heads][max_seq_len][head_dim / 32]; entries of tokens at or past
 * seq_lens[b] are left untouched. max_seq_len must be >= every seq_lens[b]. Also writes
 * `out` like q8kv_decode_attn. Uses the library-managed workspace. */
q8kv_status q8kv_debug_block_dots(int32_t *dots, int max_seq_len, float *out, const float *q,
                                  const int8_t *k_blocks, const int8_t *v_blocks,
                                  const float *kscale, const float *vscale,
                                  const int32_t *block_table, const int32_t *seq_lens, int B,
                                  int n_q_heads, int n_kv_heads, int head_dim,
                                  int kv_block_size, int max_blocks_per_seq, int num_kv_blocks,
                                  float scale, cudaStream_t stream);

/* Debug: q8kv_decode_attn with one pipeline fault injected, to exercise the bounded waits.
 * The producer warp of CTA stall_cta never arrives on, and never loads into, the stage of
 * that CTA's second tile (its first when it has only one), so nothing is in flight for that
 * stage and its phase never completes. That CTA's waits give up after limit_ns
 * (1e3 <= limit_ns <= 1e9; other CTAs keep the normal limit of one second): its consumer
 * warps stop computing and its producer stops issuing, Q8KV_DEVERR_TIMEOUT is set, and the
 * kernel returns normally, so the context stays usable. Rows whose split segments that CTA
 * contributes to are undefined; all other rows are what q8kv_decode_attn gives. A CTA
 * index past the grid injects nothing. Library-managed workspace, asynchronous. Returns
 * Q8KV_ERR_INVALID_ARG for stall_cta < 0 or limit_ns out of range. */
q8kv_status q8kv_debug_stall_pipeline(float *out, const float *q, const int8_t *k_blocks,
                                      const int8_t *v_blocks, const float *kscale,
                                      const float *vscale, const int32_t *block_table,
                                      const int32_t *seq_lens, int B, int n_q_heads,
                                      int n_kv_heads, int head_dim, int kv_block_size,
                                      int max_blocks_per_seq, int num_kv_blocks, float scale,
                                      int stall_cta, unsigned long long limit_ns,
                                      cudaStream_t stream);

/* Read (and, if clear != 0, reset) the device-side error word of the current device.
 * Synchronises the device. */
q8kv_status q8kv_device_errors(unsigned *flags, int clear);

/* Static description of a status code. */
const char *q8kv_status_string(q8kv_status status);

/* The cudaError_t of the last failing CUDA call made by this library on this thread
 * (0 if none). */
int q8kv_last_cuda_error(void);

/* Library ABI version (major * 100 + minor). */
int q8kv_version(void);

#ifdef __cplusplus
}
#endif
#endif
