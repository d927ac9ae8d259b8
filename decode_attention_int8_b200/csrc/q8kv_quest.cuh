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
// 128-byte row at once) and the row's scale, 16 tokens per batch of independent loads.
// Per element the kernel issues about five instructions (byte to float, multiply by the
// scale, max, min, a share of the loads): on the 692 MB benchmark shape instruction issue,
// not HBM, sets the pace (measured alternatives, such as building the float from the byte
// with a permute and an add, or three-way max / min, issued more, not fewer).
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
constexpr int kQuestUnroll = 16;     // tokens whose loads are in flight together
constexpr int kQuestBlocksPerSM = 4; // 1024 threads of up to 64 registers: 16 tokens x 132 B
                                     // in flight per warp, about 68 KB per SM

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

__global__ void __launch_bounds__(kQuestThreads, kQuestBlocksPerSM)
    quest_metadata_kernel(const __grid_constant__ QuestParams p)
{
    // the cache may have been written by the kernel before this one on the stream
    grid_dep_wait();
    grid_dep_launch();
    const int lane = threadIdx.x & 31;
    const long long per_req = (long long)p.mmbpr * p.bs * p.Hk;
    const long long n_items = (long long)p.B * per_req;
    const long long stride = (long long)gridDim.x * kQuestWarps;
    const int cap = p.mbps * p.bs;
    unsigned err = 0;
#pragma unroll 1
    for (long long it = (long long)blockIdx.x * kQuestWarps + (threadIdx.x >> 5); it < n_items;
         it += stride) {
        const int r = (int)(it / per_req);
        const long long rest = it - (long long)r * per_req;
        const int h = (int)(rest % p.Hk);
        const int j = (int)(rest / p.Hk); // KV block index within the request: m * bs + row
        int L = __ldg(p.seq_lens + r);
        if (L < 0 || L > cap) {
            err |= kErrSeqLen;
            L = L < 0 ? 0 : cap;
        }
        const int nkv = (L + p.bs - 1) / p.bs;
        const int nmeta = (nkv + p.bs - 1) / p.bs;
        const int m = j / p.bs, row = j - m * p.bs;
        if (nmeta > p.mmbpr && j == 0 && h == 0)
            err |= kErrMeta; // the table cannot hold all of this request's metadata blocks
        if (m >= nmeta)
            continue;
        const int mb = __ldg(p.meta_table + (long long)r * p.mmbpr + m);
        if (mb < 0 || mb >= p.num_meta) {
            err |= kErrMeta;
            continue;
        }
        const long long orow = (long long)mb * p.bs + row;
        if (j >= nkv) { // after the request's last KV block
            const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
            quest_store(p.maxb, orow, p.Hk, h, lane, z);
            quest_store(p.minb, orow, p.Hk, h, lane, z);
            continue;
        }
        const int ph = __ldg(p.block_table + (long long)r * p.mbps + j);
        if (ph < 0 || ph >= p.num_blocks) {
            err |= kErrBlockTable;
            continue;
        }
        const int n = min(p.bs, L - j * p.bs);
        const long long e0 = (long long)ph * p.bs * p.Hk + h; // (first slot, head) row
        const unsigned int *kw = reinterpret_cast<const unsigned int *>(p.k + e0 * 128) + lane;
        const float *kscl = p.ks + e0;
        const int wstride = p.Hk * 32; // 32-bit words from one token's row to the next
        float hi[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
        float lo[4] = {INFINITY, INFINITY, INFINITY, INFINITY};
#pragma unroll 1
        for (int t0 = 0; t0 < n; t0 += kQuestUnroll) {
            uint32_t w[kQuestUnroll];
            float sc[kQuestUnroll];
#pragma unroll
            for (int u = 0; u < kQuestUnroll; ++u) {
                const int t = t0 + u < n ? t0 + u : n - 1; // repeats of a valid token are harmless
                w[u] = __ldcs(kw + t * wstride);
                sc[u] = __ldcs(kscl + t * p.Hk);
            }
            // products code * scale rounded once (fp32)
#pragma unroll
            for (int u = 0; u < kQuestUnroll; ++u)
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const float v =
                        __fmul_rn((float)(int8_t)((w[u] >> (8 * c)) & 0xffu), sc[u]);
                    hi[c] = fmaxf(hi[c], v);
                    lo[c] = fminf(lo[c], v);
                }
        }
        quest_store(p.maxb, orow, p.Hk, h, lane, make_float4(hi[0], hi[1], hi[2], hi[3]));
        quest_store(p.minb, orow, p.Hk, h, lane, make_float4(lo[0], lo[1], lo[2], lo[3]));
    }
    if (err && lane == 0)
        atomicOr(p.errors, err);
}

} // namespace q8kv
