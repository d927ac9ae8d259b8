// q8kv_quest.cuh -- QUEST-style per-block K metadata over the paged q8 cache.
//
// What it computes (CANN quest_prefill_metadata guide, xdnf.cn/news/235188, "reference
// implementation" and "source-level principles"): for request r with L = seq_lens[r]
// tokens, KV block j < ceil(L / bs) covers tokens [j * bs, min((j + 1) * bs, L)); its
// metadata row is row j % bs of metadata block meta_table[r][j / bs] (a metadata block
// has bs rows, so it summarises bs * bs tokens), and for every KV head h and channel d
//   maxb[row][h][d] = max over the block's tokens of K[slot][h][d]
//   minb[row][h][d] = min over the same tokens
// with K the dequantised cache value code * kscale[slot][h] (one fp32 product, so the
// result is exact and independent of the reduction order). Rows of a request's last
// metadata block after its last KV block are zero in both arrays. QUEST uses the two
// arrays to bound q . k over a block when choosing which blocks a decode step reads.
//
// How (B200): the page's AscendC kernel gives each vector core one (request, head) and
// walks its blocks with double-buffered copies; here every (request, metadata block, row,
// head) is one warp's work item, so thousands of independent warps keep HBM busy. A lane
// owns 4 channels: per token it loads one 32-bit word of codes (the warp reads the head's
// 128-byte row at once) and the row's scale.
//
// Two things set the pace, and the kernel is shaped by both:
// - Bytes in flight. Each warp streams its tokens in batches of 16 with two register
//   buffers: the loads of batch i + 1 are issued before batch i is reduced, a batch's 16
//   scales are one load spread over the lanes (not a copy in every lane), and an item's
//   three table entries are read in one round trip. On the benchmark shape the kernel
//   then runs as fast as a copy of it that only loads the same bytes.
// - Instruction issue. Per element the work is a byte-to-float conversion, a multiply, a
//   max and a min. The conversion instruction runs on the narrow XU pipe, which caps the
//   rate well below HBM's; so only bytes 0 and 2 of a word take it, and bytes 1 and 3 are
//   built in the integer pipe as the float 2^23 + (code + 128) (exponent byte 0x4B, the
//   code with its sign bit flipped as the low mantissa byte) minus 2^23 + 128, exact.
//   The subtraction and the multiply by the token's scale use the paired fp32 form
//   (sub/mul .rn.f32x2), each on channel c of two consecutive tokens, so one instruction
//   does two elements; both are correctly rounded, so every product equals the oracle's.
//   The head count is a template parameter where it is 1, 2, 4, 8, 16 or 32, so the loads
//   of a batch take their offsets as immediates.
// Items are ordered head-fastest, so neighbouring warps read neighbouring 128-byte rows
// of the same tokens and write neighbouring 512-byte rows of the same metadata row.
#pragma once

#include <cstdint>

#include "q8kv_decode.cuh" // the device error bits
#include "q8kv_ptx.cuh"

namespace q8kv {

constexpr unsigned kErrMeta = 0x20u; // metadata table entry outside its pool, or too short
constexpr int kQuestThreads = 256;
constexpr int kQuestWarps = kQuestThreads / 32;
constexpr int kQuestUnroll = 16;     // tokens per batch; two batches per warp in flight
constexpr int kQuestBlocksPerSM = 3; // 768 threads of up to 80 registers

struct QuestParams {
    float *maxb, *minb;           // [num_meta][bs][Hk][128]
    const int8_t *k;              // [num_blocks][bs][Hk][128]
    const float *ks;              // [num_blocks][bs][Hk]
    const int32_t *block_table;   // [B][mbps]
    const int32_t *seq_lens;      // [B]
    const int32_t *meta_table;    // [B][mmbpr]
    int B, Hk, bs, mbps, mmbpr, num_blocks, num_meta;
    unsigned *errors;
};

__device__ __forceinline__ void quest_store(float *base, long long row, int Hk, int h, int lane,
                                            float4 v)
{
    reinterpret_cast<float4 *>(base + ((size_t)row * Hk + h) * 128)[lane] = v;
}

// ---------------------------------------------------------------- paired fp32 arithmetic

__device__ __forceinline__ unsigned long long f32x2_pack(float a, float b)
{
    unsigned long long r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}

__device__ __forceinline__ void f32x2_unpack(unsigned long long r, float &a, float &b)
{
    asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(r));
}

__device__ __forceinline__ unsigned long long f32x2_mul_rn(unsigned long long a,
                                                          unsigned long long b)
{
    unsigned long long r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}

__device__ __forceinline__ unsigned long long f32x2_sub_rn(unsigned long long a,
                                                          unsigned long long b)
{
    unsigned long long r;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}

// ---------------------------------------------------------------- one item's tokens

template <int U> struct QuestBatch {
    uint32_t w[U]; // this lane's 4 codes of each token
    float s;       // the scale of token (lane % U): one load for the whole batch, taken by
                   // every lane with a shuffle when it is used (a per-lane copy of each
                   // token's scale would hold U registers for 4 bytes of data)
};

// The batch of tokens [t0, t0 + U) of an item whose first token's code word (this lane's)
// and scale are kw and ks; past the item's n tokens the last token is read again (only when
// CLAMP for the codes), which leaves max and min unchanged.
template <int U, int HK, bool CLAMP>
__device__ __forceinline__ void quest_load(QuestBatch<U> &b, const uint32_t *kw, const float *ks,
                                           int t0, int n, int Hk, int lane)
{
    const int hk = HK ? HK : Hk;
    const uint32_t *kb = kw + (long long)t0 * hk * 32;
#pragma unroll
    for (int u = 0; u < U; ++u) {
        const int du = CLAMP ? (t0 + u < n ? u : n - 1 - t0) : u;
        b.w[u] = __ldcs(kb + du * hk * 32);
    }
    const int ts = min(t0 + lane % U, n - 1);
    b.s = __ldcs(ks + (long long)ts * hk);
}

// Channel c (of this lane's 4) of tokens u and u + 1: code * scale for both, rounded once
// each, folded into the running max and min in token order.
template <int U>
__device__ __forceinline__ void quest_reduce(const QuestBatch<U> &b, float (&hi)[4],
                                             float (&lo)[4])
{
    const unsigned long long bias = f32x2_pack(8388736.f, 8388736.f); // 2^23 + 128
#pragma unroll
    for (int u = 0; u < U; u += 2) {
        const uint32_t w0 = b.w[u], w1 = b.w[u + 1];
        const uint32_t x0 = w0 ^ 0x80808080u, x1 = w1 ^ 0x80808080u; // code + 128 per byte
        const unsigned long long sp =
            f32x2_pack(__shfl_sync(0xffffffffu, b.s, u), __shfl_sync(0xffffffffu, b.s, u + 1));
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            unsigned long long v;
            if (c % 2 == 0) { // the conversion instruction
                v = f32x2_pack((float)(int8_t)((w0 >> (8 * c)) & 0xffu),
                               (float)(int8_t)((w1 >> (8 * c)) & 0xffu));
            } else { // 0x4B0000xx = 2^23 + xx, then minus 2^23 + 128
                const uint32_t sel = 0x7540u + c;
                v = f32x2_sub_rn(f32x2_pack(__uint_as_float(__byte_perm(x0, 0x4B000000u, sel)),
                                            __uint_as_float(__byte_perm(x1, 0x4B000000u, sel))),
                                 bias);
            }
            float a, d;
            f32x2_unpack(f32x2_mul_rn(v, sp), a, d);
            hi[c] = fmaxf(fmaxf(hi[c], a), d);
            lo[c] = fminf(fminf(lo[c], a), d);
        }
    }
}

// HK: the head count when it is a compile-time constant, else 0 (read from p.Hk).
template <int HK>
__global__ void __launch_bounds__(kQuestThreads, kQuestBlocksPerSM)
    quest_metadata_kernel(const __grid_constant__ QuestParams p)
{
    constexpr int U = kQuestUnroll;
    // the cache may have been written by the kernel before this one on the stream
    grid_dep_wait();
    grid_dep_launch();
    const int lane = threadIdx.x & 31;
    const int Hk = HK ? HK : p.Hk;
    const long long per_req = (long long)p.mmbpr * p.bs * Hk;
    const long long n_items = (long long)p.B * per_req;
    const bool narrow = n_items <= 0x7fffffffLL; // every item index fits in 32 bits
    const long long stride = (long long)gridDim.x * kQuestWarps;
    const int cap = p.mbps * p.bs;
    unsigned err = 0;
#pragma unroll 1
    for (long long it = (long long)blockIdx.x * kQuestWarps + (threadIdx.x >> 5); it < n_items;
         it += stride) {
        int r, j, h; // j = m * bs + row: KV block index within the request
        if (narrow) {
            r = (int)it / (int)per_req;
            const int rest = (int)it - r * (int)per_req;
            j = rest / Hk;
            h = rest - j * Hk;
        } else { // j < max_meta_per_seq * bs < 2^31 (checked on the host)
            r = (int)(it / per_req);
            const long long rest = it - (long long)r * per_req;
            j = (int)(rest / Hk);
            h = (int)(rest - (long long)j * Hk);
        }
        const int m = j / p.bs, row = j - m * p.bs;
        // the three table entries in one round trip
        int L = __ldg(p.seq_lens + r);
        const int mb = __ldg(p.meta_table + (long long)r * p.mmbpr + m);
        const int ph = j < p.mbps ? __ldg(p.block_table + (long long)r * p.mbps + j) : -1;
        if (L < 0 || L > cap) {
            err |= kErrSeqLen;
            L = L < 0 ? 0 : cap;
        }
        const int nkv = (L + p.bs - 1) / p.bs;
        const int nmeta = (nkv + p.bs - 1) / p.bs;
        if (nmeta > p.mmbpr && j == 0 && h == 0)
            err |= kErrMeta; // the table cannot hold all of this request's metadata blocks
        if (m >= nmeta)
            continue;
        if (mb < 0 || mb >= p.num_meta) {
            err |= kErrMeta;
            continue;
        }
        const long long orow = (long long)mb * p.bs + row;
        if (j >= nkv) { // after the request's last KV block
            const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
            quest_store(p.maxb, orow, Hk, h, lane, z);
            quest_store(p.minb, orow, Hk, h, lane, z);
            continue;
        }
        if (ph < 0 || ph >= p.num_blocks) {
            err |= kErrBlockTable;
            continue;
        }
        const int n = min(p.bs, L - j * p.bs);
        const long long e0 = (long long)ph * p.bs * Hk + h; // (first slot, head) row
        const uint32_t *kw = reinterpret_cast<const uint32_t *>(p.k + e0 * 128) + lane;
        const float *ks = p.ks + e0;
        float hi[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
        float lo[4] = {INFINITY, INFINITY, INFINITY, INFINITY};
        const int nfull = n / U, nb = (n + U - 1) / U;
        QuestBatch<U> A, B;
        auto load = [&](QuestBatch<U> &x, int i) {
            if (i < nfull)
                quest_load<U, HK, false>(x, kw, ks, i * U, n, Hk, lane);
            else
                quest_load<U, HK, true>(x, kw, ks, i * U, n, Hk, lane);
        };
        // batch i + 1 is in flight while batch i is reduced
        load(A, 0);
#pragma unroll 1
        for (int i = 0; i < nb; i += 2) {
            if (i + 1 < nb)
                load(B, i + 1);
            quest_reduce<U>(A, hi, lo);
            if (i + 1 >= nb)
                break;
            if (i + 2 < nb)
                load(A, i + 2);
            quest_reduce<U>(B, hi, lo);
        }
        quest_store(p.maxb, orow, Hk, h, lane, make_float4(hi[0], hi[1], hi[2], hi[3]));
        quest_store(p.minb, orow, Hk, h, lane, make_float4(lo[0], lo[1], lo[2], lo[3]));
    }
    if (err && lane == 0)
        atomicOr(p.errors, err);
}

} // namespace q8kv
