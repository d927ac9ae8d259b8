// q8kv_q4.cuh -- single-query decode attention over a paged q4_0 KV cache.
//
// What it computes: the decode of q8kv_decode_attn (Kestrel-LLM walk-through
// "flash_attn_single_q_q8_neon", trdm.cn/news/511694, section 2: Q quantised once to int8
// in 32-element blocks, exact integer block dots, online softmax, one division at the end)
// over a cache in llama.cpp's q4_0 format, one of the quantised KV-cache types of the
// llama.cpp change on baguaai.com's FlashAttention page: every 32-channel block of a
// (token, KV head) row holds 4-bit codes and one binary16 scale d, value (code - 8) * d.
// So for query head h of KV head kv and token t
//   dot_j = sum over the block of qi * (code - 8)                (int32, exact)
//   s_t   = (sum_j dot_j * qsc_j * dk_tj) * scale
//   out   = sum_t exp(s_t - M) * (code_t - 8) * dv_t,block / sum_t exp(s_t - M).
// Codes are packed two per byte, channel 2i in the low nibble of byte i.
//
// How (B200): q4_0 halves the bytes per token again (72 B per row with its scales), and
// the per-block scales make every 32 channels of V a separate weight, which does not map
// onto the int8 tensor-core path of the q8 kernel; the work per byte is small enough for
// the CUDA cores. The sequence is cut into chunks of kQ4Chunk tokens (flash-decoding);
// one 256-thread CTA takes one (sequence, KV head, chunk) and all G query heads of the KV
// head:
//   * scores, lanes = tokens: each lane loads its token's 64-byte K row and 8 bytes of
//     scales, splits each 32-bit word of nibbles into the even and the odd channels with
//     two masks (no per-element unpacking), and forms each block dot with dp4a
//     (u8 codes x s8 query, the query stored in the same even / odd channel order in
//     shared memory) minus 8 times the block's query sum;
//   * softmax per chunk in shared memory (exp2, base-2 scores);
//   * the same lane also loads its token's V row and scales (with the K row: one round
//     trip after the block table) into shared memory;
//   * PV, lanes = channels: each warp walks its share of the chunk's tokens out of shared
//     memory, a lane reading the 2 bytes of its 4 channels, and the per-warp sums are
//     added in shared memory;
//   * the chunk's partial (acc, max, sum) goes to the workspace, and q4_combine_kernel
//     merges the chunks of every (sequence, head) with the usual log-sum-exp rescaling.
#pragma once

#include <cuda_fp16.h>

#include <cstdint>

#include "q8kv_decode.cuh" // device error bits, kD, kNB
#include "q8kv_ptx.cuh"
#include "q8kv_qquant.cuh"

namespace q8kv {

constexpr int kQ4Threads = 256;
constexpr int kQ4Warps = kQ4Threads / 32;
constexpr int kQ4Chunk = 256;   // tokens per CTA: one per lane of the 8 warps in the scores
constexpr int kQ4MaxG = 16;     // query heads per KV head
constexpr int kQ4Row = kD / 2;  // code bytes per (token, KV head) row
constexpr int kQ4SlotRow = kD + 4; // partial row: acc[128], M, S, pad

struct Q4Params {
    float *out;
    const float *q;
    const uint8_t *k4, *v4;
    const uint16_t *kd, *vd;
    const int32_t *block_table;
    const int32_t *seq_lens;
    float *partials; // [B * Hk][n_chunks][G][kQ4SlotRow]
    unsigned *errors;
    int B, Hq, Hk, G, bs, mbps, num_blocks, n_chunks;
    float scale_log2;
};

// Shared memory of one CTA (dynamic): query words, block sums and scales, the chunk's
// scores / weights, and the per-warp PV sums.
struct Q4Smem {
    uint32_t qw[kQ4MaxG][32]; // word 2m: channels 8m, 8m+2, 8m+4, 8m+6; word 2m+1: the odd
    int qsum[kQ4MaxG][kNB];   // sum of the block's query codes
    float qsc[kQ4MaxG][kNB];
    float ms[kQ4MaxG][2];     // chunk max and sum per head
};

// Dynamic shared memory: Q4Smem, the chunk's V codes [chunk][64 B] and V block scales
// [chunk][4] (fp32), the scores / weights [G][chunk], and the per-warp PV sums [8][G][128].
__host__ __device__ inline size_t q4_smem_bytes(int G)
{
    return sizeof(Q4Smem) + (size_t)kQ4Chunk * (kQ4Row + 4 * kNB) +
           sizeof(float) * (size_t)G * kQ4Chunk + sizeof(float) * (size_t)kQ4Warps * G * kD;
}

__device__ __forceinline__ int dp4a_us(uint32_t a_u8, uint32_t b_s8, int c)
{
    int d;
    asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a_u8), "r"(b_s8), "r"(c));
    return d;
}

__device__ __forceinline__ float half_bits_to_float(uint16_t h)
{
    return __half2float(__ushort_as_half(h));
}

// Physical slot of token t of sequence b, or -1 (and an error bit) for a bad table entry.
__device__ __forceinline__ long long q4_slot(const Q4Params &p, int b, int t, unsigned &err)
{
    const int ph = __ldg(p.block_table + (long long)b * p.mbps + t / p.bs);
    if (ph < 0 || ph >= p.num_blocks) {
        err |= kErrBlockTable;
        return -1;
    }
    return (long long)ph * p.bs + t % p.bs;
}

// GM: the largest group the instantiation serves (4, 8 or 16): the PV accumulators of the
// G heads live in registers, so smaller groups get a smaller, more resident kernel.
template <int GM>
__global__ void __launch_bounds__(kQ4Threads, GM <= 4 ? 4 : (GM <= 8 ? 3 : 2))
    q4_decode_kernel(const __grid_constant__ Q4Params p)
{
    extern __shared__ __align__(16) uint8_t q4_smem_raw[];
    Q4Smem &sm = *reinterpret_cast<Q4Smem *>(q4_smem_raw);
    uint4 *vbuf = reinterpret_cast<uint4 *>(q4_smem_raw + sizeof(Q4Smem));  // [chunk][4]
    float4 *vdbuf = reinterpret_cast<float4 *>(vbuf + kQ4Chunk * 4);       // [chunk]
    float *sc = reinterpret_cast<float *>(vdbuf + kQ4Chunk);                // [G][chunk]
    float *part = sc + p.G * kQ4Chunk;                                      // [warps][G][128]
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int bk = blockIdx.y, b = bk / p.Hk, kvh = bk - b * p.Hk;
    const int G = p.G;

    grid_dep_wait(); // q, the cache and the tables may come from the previous kernel
    grid_dep_launch();
    int L = __ldg(p.seq_lens + b);
    const int cap = p.mbps * p.bs;
    unsigned err = 0;
    if (L < 0 || L > cap) {
        if (blockIdx.x == 0 && tid == 0)
            atomicOr(p.errors, kErrSeqLen);
        L = L < 0 ? 0 : cap;
    }
    const int t0 = blockIdx.x * kQ4Chunk;
    if (t0 >= L)
        return; // the combine only reads the chunks that hold tokens
    const int nt = min(kQ4Chunk, L - t0);

    // ---- quantise the G query rows (4 blocks each; one quad of lanes per block)
    for (int blk = warp * 8 + (lane >> 2); blk - (lane >> 2) < 4 * G; blk += kQ4Warps * 8) {
        const int g = blk >> 2, j = blk & 3, part4 = lane & 3;
        const bool live = g < G;
        float v[8];
        const float *qr = p.q + ((long long)b * p.Hq + (long long)kvh * G + (live ? g : 0)) * kD +
                          32 * j + 8 * part4;
#pragma unroll
        for (int i = 0; i < 8; ++i)
            v[i] = live ? __ldg(qr + i) : 0.f;
        uint32_t lo, hi;
        float qs;
        quantize_block_quad(v, lo, hi, qs);
        int s8 = 0; // the block's code sum (the whole warp shuffles)
#pragma unroll
        for (int i = 0; i < 4; ++i)
            s8 += (int)(int8_t)(lo >> (8 * i)) + (int)(int8_t)(hi >> (8 * i));
        s8 += __shfl_xor_sync(0xffffffffu, s8, 1);
        s8 += __shfl_xor_sync(0xffffffffu, s8, 2);
        if (live) {
            // channels 8 * part4 + 0..7 of the block: even ones -> word 2m, odd -> 2m + 1
            const int m = 4 * j + part4;
            sm.qw[g][2 * m] = __byte_perm(lo, hi, 0x6420);
            sm.qw[g][2 * m + 1] = __byte_perm(lo, hi, 0x7531);
            if (part4 == 0) {
                sm.qsum[g][j] = s8;
                sm.qsc[g][j] = qs;
            }
        }
    }
    __syncthreads();

    // ---- scores: lane = token. The token's K and V rows are loaded together (one round
    // trip after the block table); V goes to shared memory for the PV pass.
    {
        const int tl = warp * 32 + lane; // token within the chunk
        const bool valid = tl < nt;
        long long slot = -1;
        if (valid)
            slot = q4_slot(p, b, t0 + tl, err);
        if (slot >= 0) {
            const long long row = slot * p.Hk + kvh;
            const uint4 *kr = reinterpret_cast<const uint4 *>(p.k4 + row * kQ4Row);
            const uint4 *vr = reinterpret_cast<const uint4 *>(p.v4 + row * kQ4Row);
            uint4 kw[4], vw[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                kw[i] = __ldcs(kr + i);
                vw[i] = __ldcs(vr + i);
            }
            const uint2 kdw = __ldcs(reinterpret_cast<const uint2 *>(p.kd + row * kNB));
            const uint2 vdw = __ldcs(reinterpret_cast<const uint2 *>(p.vd + row * kNB));
#pragma unroll
            for (int i = 0; i < 4; ++i)
                vbuf[tl * 4 + i] = vw[i];
            vdbuf[tl] = make_float4(half_bits_to_float((uint16_t)(vdw.x & 0xffffu)),
                                    half_bits_to_float((uint16_t)(vdw.x >> 16)),
                                    half_bits_to_float((uint16_t)(vdw.y & 0xffffu)),
                                    half_bits_to_float((uint16_t)(vdw.y >> 16)));
            float dk[kNB];
            dk[0] = half_bits_to_float((uint16_t)(kdw.x & 0xffffu));
            dk[1] = half_bits_to_float((uint16_t)(kdw.x >> 16));
            dk[2] = half_bits_to_float((uint16_t)(kdw.y & 0xffffu));
            dk[3] = half_bits_to_float((uint16_t)(kdw.y >> 16));
            // block j: 4 words (16 bytes, 32 channels); word k: channels 32j + 8k .. + 7
            for (int g = 0; g < G; ++g) {
                float s = 0.f;
#pragma unroll
                for (int j = 0; j < kNB; ++j) {
                    const uint32_t w[4] = {kw[j].x, kw[j].y, kw[j].z, kw[j].w};
                    int dot = 0;
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const uint32_t ev = w[k] & 0x0f0f0f0fu, od = (w[k] >> 4) & 0x0f0f0f0fu;
                        const int m = 4 * j + k;
                        dot = dp4a_us(ev, sm.qw[g][2 * m], dot);
                        dot = dp4a_us(od, sm.qw[g][2 * m + 1], dot);
                    }
                    dot -= 8 * sm.qsum[g][j];
                    s = fmaf((float)dot * sm.qsc[g][j], dk[j], s);
                }
                sc[g * kQ4Chunk + tl] = s * p.scale_log2;
            }
        } else {
            // no data: weight 0 against zero codes and a zero scale
#pragma unroll
            for (int i = 0; i < 4; ++i)
                vbuf[tl * 4 + i] = make_uint4(0u, 0u, 0u, 0u);
            vdbuf[tl] = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int g = 0; g < G; ++g)
                sc[g * kQ4Chunk + tl] = -INFINITY;
        }
    }
    __syncthreads();

    // ---- softmax over the chunk, per head (warp w takes heads w, w + 8)
    for (int g = warp; g < G; g += kQ4Warps) {
        float m = -INFINITY;
        for (int i = lane; i < kQ4Chunk; i += 32)
            m = fmaxf(m, sc[g * kQ4Chunk + i]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        const float ms = m == -INFINITY ? 0.f : m;
        float ssum = 0.f;
        for (int i = lane; i < kQ4Chunk; i += 32) {
            const float w = fast_exp2(sc[g * kQ4Chunk + i] - ms);
            sc[g * kQ4Chunk + i] = w;
            ssum += w;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            ssum += __shfl_xor_sync(0xffffffffu, ssum, o);
        if (lane == 0) {
            sm.ms[g][0] = m;
            sm.ms[g][1] = ssum;
        }
    }
    __syncthreads();

    // ---- PV: lane = 4 channels (4 * lane .. + 3, block lane / 8); warp w takes tokens w,
    // w + 8, ... of the chunk
    {
        float acc[GM][4];
#pragma unroll
        for (int g = 0; g < GM; ++g)
#pragma unroll
            for (int c = 0; c < 4; ++c)
                acc[g][c] = 0.f;
        const int jb = lane >> 3;
        const uint16_t *vb16 = reinterpret_cast<const uint16_t *>(vbuf);
        const float *vd32 = reinterpret_cast<const float *>(vdbuf);
        for (int tl = warp; tl < nt; tl += kQ4Warps) {
            const uint32_t nib = vb16[tl * kQ4Row / 2 + lane];
            const float dv = vd32[tl * 4 + jb];
            const float x0 = (float)((int)(nib & 0xfu) - 8), x1 = (float)((int)((nib >> 4) & 0xfu) - 8);
            const float x2 = (float)((int)((nib >> 8) & 0xfu) - 8), x3 = (float)((int)(nib >> 12) - 8);
#pragma unroll
            for (int g = 0; g < GM; ++g) {
                if (g < G) {
                    const float wv = sc[g * kQ4Chunk + tl] * dv;
                    acc[g][0] = fmaf(wv, x0, acc[g][0]);
                    acc[g][1] = fmaf(wv, x1, acc[g][1]);
                    acc[g][2] = fmaf(wv, x2, acc[g][2]);
                    acc[g][3] = fmaf(wv, x3, acc[g][3]);
                }
            }
        }
#pragma unroll
        for (int g = 0; g < GM; ++g)
            if (g < G)
                *reinterpret_cast<float4 *>(part + ((size_t)warp * G + g) * kD + 4 * lane) =
                    make_float4(acc[g][0], acc[g][1], acc[g][2], acc[g][3]);
    }
    __syncthreads();

    // ---- the chunk's partial: sum the warps' rows, then acc, M, S to the workspace
    float *dst = p.partials + (((size_t)bk * p.n_chunks + blockIdx.x) * G) * kQ4SlotRow;
    for (int e = tid; e < G * kD; e += kQ4Threads) {
        const int g = e / kD, d = e - g * kD;
        float s = 0.f;
#pragma unroll
        for (int w = 0; w < kQ4Warps; ++w)
            s += part[((size_t)w * G + g) * kD + d];
        dst[(size_t)g * kQ4SlotRow + d] = s;
    }
    for (int g = tid; g < G; g += kQ4Threads) {
        dst[(size_t)g * kQ4SlotRow + kD] = sm.ms[g][0];
        dst[(size_t)g * kQ4SlotRow + kD + 1] = sm.ms[g][1];
    }
    if (err)
        atomicOr(p.errors, err);
}

// Merge the chunks of every (sequence, query head): one warp per row, a lane per 4
// channels; maxima first, then the rescaled sums.
__global__ void __launch_bounds__(256) q4_combine_kernel(const __grid_constant__ Q4Params p)
{
    grid_dep_wait(); // the partials of the decode kernel before it
    grid_dep_launch();
    const int lane = threadIdx.x & 31;
    const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (row >= (long long)p.B * p.Hq)
        return;
    const int b = (int)(row / p.Hq), h = (int)(row - (long long)b * p.Hq);
    const int kvh = h / p.G, g = h - kvh * p.G;
    const int cap = p.mbps * p.bs;
    int L = __ldg(p.seq_lens + b);
    L = L < 0 ? 0 : (L > cap ? cap : L);
    const int n = (L + kQ4Chunk - 1) / kQ4Chunk;
    const float *base = p.partials + (((size_t)b * p.Hk + kvh) * p.n_chunks * p.G + g) * kQ4SlotRow;
    const size_t cstride = (size_t)p.G * kQ4SlotRow;
    float mx = -INFINITY;
    for (int c = 0; c < n; ++c)
        mx = fmaxf(mx, __ldcg(base + c * cstride + kD));
    float s = 0.f;
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int c = 0; c < n; ++c) {
        const float *r = base + c * cstride;
        const float mc = __ldcg(r + kD);
        const float f = mc == -INFINITY ? 0.f : exp2f(mc - mx);
        s += __ldcg(r + kD + 1) * f;
        const float4 x = __ldcg(reinterpret_cast<const float4 *>(r) + lane);
        a.x += x.x * f;
        a.y += x.y * f;
        a.z += x.z * f;
        a.w += x.w * f;
    }
    const float inv = s > 0.f ? 1.f / s : 0.f;
    reinterpret_cast<float4 *>(p.out + row * kD)[lane] =
        make_float4(a.x * inv, a.y * inv, a.z * inv, a.w * inv);
}

} // namespace q8kv
