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
// How (B200): the sequence is cut into chunks of kQ4Chunk = 256 tokens (flash-decoding);
// one 256-thread CTA takes one (sequence, KV head, chunk) and all G query heads of the KV
// head, and both contractions run on the int8 tensor cores (mma.sync m16n8k32):
//   * loads: each warp copies its 32-token slice (K and V rows, 64 bytes each, and their
//     scales) into shared memory with cp.async, one token per lane; a row's 16-byte
//     chunks sit at XOR-swizzled positions so that both ldmatrix patterns below are free
//     of bank conflicts;
//   * a nibble becomes a tensor-core operand with one or two logic instructions: for a
//     byte x = (odd << 4) | even, (x ^ 0x88) & 0xF0 is the signed byte 16 * (odd - 8) and
//     ((x << 4) ^ 0x80) & 0xF0 is 16 * (even - 8); the factor 16 is taken out in fp32;
//   * QK: the rows of the A operand are (block j, head h) pairs r = j * GT + h, and row r
//     holds q's block j only (zeros elsewhere), so one chained accumulator per row gives
//     exactly that block's dot; B = K^T by ldmatrix (8 tokens x 4 blocks per load). Each
//     dot is scaled by its own qsc * dk and the blocks of a head are summed in fp32;
//   * softmax: the chunk's maximum per head over the 8 warps (shared memory), base 2;
//   * PV: the weight w * dv_tj differs per 32-channel block, so a PV column is again a
//     (block, head) pair; each weight becomes an exact integer
//     P = round(w * dv * 2^(36 - e_j)), |P| < 2^22 (e_j the binary16 exponent field of the
//     chunk's largest |dv| in block j), whose three bytes are three B operands (two
//     unsigned, the top one signed). Warp w owns the 16 channels of parity (w & 1) in block
//     w / 2 and runs over all 8 slices: A = V^T by ldmatrix .trans (k = tokens in the
//     order tau of the QK accumulator layout, so P needs no shuffle), three MMAs per slice,
//     int32 sums over 4 slices at a time (|sum| < 2^22, so the fp32 view of
//     1.5 * 2^23 + sum is exact), recombined in fp32 and scaled by 2^(e_j - 32);
//   * the chunk's partial (acc, max, sum) goes to the workspace, and q4_combine_kernel
//     merges the chunks of every (sequence, head) with the usual log-sum-exp rescaling.
#pragma once

#include <cuda_fp16.h>

#include <cstdint>

#include "q8kv_decode.cuh" // device error bits, kD, kNB, kDotBias
#include "q8kv_ptx.cuh"
#include "q8kv_qquant.cuh"

namespace q8kv {

constexpr int kQ4Threads = 256;
constexpr int kQ4Warps = kQ4Threads / 32;
constexpr int kQ4Chunk = kQ4Warps * 32; // tokens per CTA: one 32-token slice per warp
constexpr int kQ4MaxG = 16;             // query heads per KV head
constexpr int kQ4Row = kD / 2;          // code bytes per (token, KV head) row
constexpr int kQ4SlotRow = kD + 4;      // partial row: acc[128], M, S, pad
constexpr int kQ4FoldEvery = 4;         // slices summed in int32 before an fp32 fold
constexpr float kQ4Bias = 12582912.0f;  // 1.5 * 2^23, the fp32 value of kDotBias

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
    int log2_bs; // log2(bs) when bs is a power of two, else -1
    float scale_log2;
};

// GT: the instantiated group (1, 2, 4, 8 or 16, at least G; heads G..GT-1 are padding).
template <int GT>
struct Q4Shape {
    static constexpr int R = 4 * GT;                   // (block, head) rows: r = j * GT + h
    static constexpr int MT = R <= 16 ? 1 : R / 16;    // QK m-tiles
    static constexpr int NS = R <= 8 ? 1 : R / 8;      // PV n-tiles (column sets)
    static constexpr int SPB = GT <= 8 ? 1 : GT / 8;   // PV n-tiles per 32-channel block
    static constexpr int NSLOT = GT <= 8 ? 1 : GT / 8; // heads whose scores a lane holds
};

template <int GT>
struct Q4Smem {
    uint8_t k[kQ4Chunk][kQ4Row]; // 16-byte chunks at position chunk ^ q4_swz(token)
    uint8_t v[kQ4Chunk][kQ4Row];
    float kdf[kQ4Chunk][kNB];    // the token's 4 block scales, converted once to fp32
    float vdf[kQ4Chunk][kNB];
    union {
        uint2 pb[kQ4Warps][Q4Shape<GT>::NS][3][32]; // P byte planes as PV B fragments
        struct {
            uint2 kd[kQ4Chunk]; // binary16 scales as copied; read only before the first
            uint2 vd[kQ4Chunk]; // barrier, long before the planes are written
        } raw;
    } u;
    uint32_t qw[GT][32]; // word 2m: channels 8m, 8m+2, 8m+4, 8m+6; word 2m+1: the odd ones
    float qsc[GT][kNB];
    float smax[kQ4Warps][GT];
    float ssum[kQ4Warps][GT];
    uint32_t dvmax[kQ4Warps][kNB]; // largest |dv| bit pattern of the warp's slice per block
    uint32_t valid[kQ4Warps];      // tokens of the slice with data
};

static_assert(sizeof(uint2) * kQ4Warps * 3 * 32 >= sizeof(uint2) * 2 * kQ4Chunk,
              "the raw scales must fit in the P planes of one n-tile");

template <int GT>
__host__ __device__ constexpr size_t q4_smem_bytes()
{
    return sizeof(Q4Smem<GT>);
}

// Chunk position of a row's 16-byte chunk: for 8 consecutive tokens (the QK ldmatrix) and
// for the tokens tau(0..7), tau(8..15) (the PV ldmatrix) the pairs (token & 1, swizzle)
// are all distinct, so each 8-row phase touches 8 different bank groups.
__device__ __forceinline__ uint32_t q4_swz(int tok)
{
    return (uint32_t)(((tok >> 1) & 1) | ((((tok >> 2) ^ (tok >> 3)) & 1) << 1));
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, uint32_t src_bytes)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
                 "r"(src_bytes)
                 : "memory");
}

__device__ __forceinline__ void cp_async8(uint32_t dst, const void *src, uint32_t src_bytes)
{
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8, %2;" ::"r"(dst), "l"(src),
                 "r"(src_bytes)
                 : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3,
                                        uint32_t addr)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

// 16 * (code - 8) as signed bytes, for the even (low-nibble) and odd channels of 4 bytes.
__device__ __forceinline__ uint32_t nib_even_s8x16(uint32_t x)
{
    return ((x << 4) ^ 0x80808080u) & 0xF0F0F0F0u;
}

__device__ __forceinline__ uint32_t nib_odd_s8x16(uint32_t x)
{
    return (x ^ 0x88888888u) & 0xF0F0F0F0u;
}

// Either of the two above: sh = 4 gives the even channels, sh = 0 the odd ones (the XOR
// with 0x88 and the mask leave the other nibble out either way).
__device__ __forceinline__ uint32_t nib_s8x16(uint32_t x, uint32_t sh)
{
    return ((x << sh) ^ 0x88888888u) & 0xF0F0F0F0u;
}

__device__ __forceinline__ float half_bits_to_float(uint16_t h)
{
    return __half2float(__ushort_as_half(h));
}

// Binary16 scale of block j (0..3) out of a token's 4 packed scales.
__device__ __forceinline__ float half_of(uint2 w, int j)
{
    const uint32_t x = (j & 2) ? w.y : w.x;
    return half_bits_to_float((uint16_t)(x >> ((j & 1) * 16)));
}

// Block-table entry of token t of sequence b (t below the table's capacity), read before
// the sequence's length is known so that both reads share one round trip.
__device__ __forceinline__ int q4_entry(const Q4Params &p, int b, int t)
{
    const int blk = p.log2_bs >= 0 ? t >> p.log2_bs : t / p.bs;
    return __ldg(p.block_table + (long long)b * p.mbps + blk);
}

// Physical slot of token t given its table entry, or -1 (and an error bit) for a bad entry.
__device__ __forceinline__ long long q4_slot(const Q4Params &p, int t, int ph, unsigned &err)
{
    if (ph < 0 || ph >= p.num_blocks) {
        err |= kErrBlockTable;
        return -1;
    }
    const int blk = p.log2_bs >= 0 ? t >> p.log2_bs : t / p.bs;
    return (long long)ph * p.bs + (t - blk * p.bs);
}

// Block of QK row r_base + g (r_base a multiple of 8, g < 8); compile-time for GT >= 8.
template <int GT>
__device__ __forceinline__ int q4_row_block(int r_base, int g)
{
    if constexpr (GT >= 8)
        return r_base / GT;
    else
        return (r_base + g) / GT;
}

// Does QK m-tile mt hold a row of block j?
template <int GT>
__host__ __device__ constexpr bool q4_tile_has_block(int mt, int j)
{
    return 16 * mt < (j + 1) * GT && j * GT < 16 * mt + 16;
}

template <int GT>
__global__ void __launch_bounds__(kQ4Threads, GT <= 4 ? 4 : (GT <= 8 ? 3 : 2))
    q4_decode_kernel(const __grid_constant__ Q4Params p)
{
    using S = Q4Shape<GT>;
    extern __shared__ __align__(128) uint8_t q4_smem_raw[];
    Q4Smem<GT> &sm = *reinterpret_cast<Q4Smem<GT> *>(q4_smem_raw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, c = lane & 3;
    const int bk = blockIdx.y, b = bk / p.Hk, kvh = bk - b * p.Hk;
    const int G = p.G;

    grid_dep_wait(); // q, the cache and the tables may come from the previous kernel
    grid_dep_launch();
    const int cap = p.mbps * p.bs;
    const int t0 = blockIdx.x * kQ4Chunk;
    const int tl = warp * 32 + lane; // this thread's token of the chunk
    // the length and this token's table entry in one round trip (the entry is used only if
    // the token turns out to be below the length)
    const int ph = t0 + tl < cap ? q4_entry(p, b, t0 + tl) : -1;
    int L = __ldg(p.seq_lens + b);
    unsigned err = 0;
    if (L < 0 || L > cap) {
        if (blockIdx.x == 0 && tid == 0)
            atomicOr(p.errors, kErrSeqLen);
        L = L < 0 ? 0 : cap;
    }
    if (t0 >= L)
        return; // the combine only reads the chunks that hold tokens
    const int nt = min(kQ4Chunk, L - t0);

    // ---- loads: lane = token of this warp's slice; tokens without data are zero-filled
    {
        long long slot = -1;
        if (tl < nt)
            slot = q4_slot(p, t0 + tl, ph, err);
        const bool ok = slot >= 0;
        const long long row = ok ? slot * p.Hk + kvh : 0;
        const uint32_t n16 = ok ? 16u : 0u, n8 = ok ? 8u : 0u;
        const uint8_t *kr = p.k4 + row * kQ4Row, *vr = p.v4 + row * kQ4Row;
        const uint32_t sw = q4_swz(tl);
        const uint32_t kdst = smem_addr(&sm.k[tl][0]), vdst = smem_addr(&sm.v[tl][0]);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            cp_async16(kdst + 16u * ((uint32_t)i ^ sw), kr + 16 * i, n16);
            cp_async16(vdst + 16u * ((uint32_t)i ^ sw), vr + 16 * i, n16);
        }
        cp_async8(smem_addr(&sm.u.raw.kd[tl]), p.kd + row * kNB, n8);
        cp_async8(smem_addr(&sm.u.raw.vd[tl]), p.vd + row * kNB, n8);
        asm volatile("cp.async.commit_group;" ::: "memory");
        const unsigned vm = __ballot_sync(kFullMask, ok);
        if (lane == 0)
            sm.valid[warp] = vm;
    }

    // ---- quantise the GT query rows (4 blocks each; one quad of lanes per block; rows
    // G..GT-1 are zero)
    for (int blk = warp * 8 + g; blk - g < 4 * GT; blk += kQ4Warps * 8) {
        const int h = blk >> 2, j = blk & 3;
        const bool live = blk < 4 * GT && h < G;
        float v[8];
        const float *qr = p.q + ((long long)b * p.Hq + (long long)kvh * G + (live ? h : 0)) * kD +
                          32 * j + 8 * c;
#pragma unroll
        for (int i = 0; i < 8; ++i)
            v[i] = live ? __ldg(qr + i) : 0.f;
        uint32_t lo, hi;
        float qs;
        quantize_block_quad(v, lo, hi, qs);
        if (blk < 4 * GT) {
            // channels 8c + 0..7 of the block: even ones -> word 2m, odd -> 2m + 1
            const int m = 4 * j + c;
            sm.qw[h][2 * m] = __byte_perm(lo, hi, 0x6420);
            sm.qw[h][2 * m + 1] = __byte_perm(lo, hi, 0x7531);
            if (c == 0)
                sm.qsc[h][j] = live ? qs : 0.f;
        }
    }

    // this lane's token: scales to fp32, and the slice's largest |dv| per block (the
    // lane's own copies are visible to it after the wait)
    asm volatile("cp.async.wait_all;" ::: "memory");
    {
        const uint2 kd = sm.u.raw.kd[tl], vd = sm.u.raw.vd[tl];
        *reinterpret_cast<float4 *>(&sm.kdf[tl][0]) =
            make_float4(half_of(kd, 0), half_of(kd, 1), half_of(kd, 2), half_of(kd, 3));
        *reinterpret_cast<float4 *>(&sm.vdf[tl][0]) =
            make_float4(half_of(vd, 0), half_of(vd, 1), half_of(vd, 2), half_of(vd, 3));
        const uint32_t a[4] = {vd.x & 0x7fffu, (vd.x >> 16) & 0x7fffu, vd.y & 0x7fffu,
                               (vd.y >> 16) & 0x7fffu};
#pragma unroll
        for (int j = 0; j < kNB; ++j) {
            const uint32_t m = __reduce_max_sync(kFullMask, a[j]);
            if (lane == 0)
                sm.dvmax[warp][j] = m;
        }
    }
    __syncthreads(); // query codes, every slice's K, V and scales

    // ---- QK on the tensor cores: this warp's 4 n-tiles of 8 tokens
    uint32_t qa[S::MT][kNB][4]; // A fragments: q's block j in the rows of block j, else 0
    float wq[S::MT][2];         // qsc * scale_log2 / 16 of rows g and g + 8 (0: padding)
    int jr[S::MT][2];           // the blocks of those rows
#pragma unroll
    for (int mt = 0; mt < S::MT; ++mt) {
#pragma unroll
        for (int hlf = 0; hlf < 2; ++hlf) {
            const int r = 16 * mt + 8 * hlf + g;
            const int j = q4_row_block<GT>(16 * mt + 8 * hlf, g);
            const int h = r % GT;
            jr[mt][hlf] = j & 3;
            wq[mt][hlf] = (r < S::R) ? sm.qsc[h][j & 3] * (p.scale_log2 * 0.0625f) : 0.f;
#pragma unroll
            for (int jj = 0; jj < kNB; ++jj) {
                const bool on = (j == jj) && r < S::R;
                qa[mt][jj][hlf] = on ? sm.qw[h][8 * jj + 2 * c] : 0u;
                qa[mt][jj][hlf + 2] = on ? sm.qw[h][8 * jj + 2 * c + 1] : 0u;
            }
        }
    }
    const unsigned vmask = sm.valid[warp];
    float sc[S::NSLOT][4][2]; // base-2 scores: head slot, n-tile, token 2c + e
#pragma unroll
    for (int ntile = 0; ntile < 4; ++ntile) {
        const int tk = warp * 32 + 8 * ntile + (lane & 7); // ldmatrix row; matrix = block
        const uint32_t addr =
            smem_addr(&sm.k[tk][0]) + 16u * ((uint32_t)(lane >> 3) ^ q4_swz(tk));
        uint32_t kr[4];
        ldsm_x4(kr[0], kr[1], kr[2], kr[3], addr);
        uint32_t kb0[4], kb1[4];
#pragma unroll
        for (int j = 0; j < kNB; ++j) {
            kb0[j] = nib_even_s8x16(kr[j]);
            kb1[j] = nib_odd_s8x16(kr[j]);
        }
        const int ta = warp * 32 + 8 * ntile + 2 * c;
#pragma unroll
        for (int s = 0; s < S::NSLOT; ++s) {
            sc[s][ntile][0] = 0.f;
            sc[s][ntile][1] = 0.f;
        }
#pragma unroll
        for (int mt = 0; mt < S::MT; ++mt) {
            int d[4] = {kDotBias, kDotBias, kDotBias, kDotBias};
#pragma unroll
            for (int j = 0; j < kNB; ++j)
                if (q4_tile_has_block<GT>(mt, j))
                    mma_s8_16832_acc(d, qa[mt][j][0], qa[mt][j][1], qa[mt][j][2], qa[mt][j][3],
                                     kb0[j], kb1[j], d);
#pragma unroll
            for (int hlf = 0; hlf < 2; ++hlf) {
                const int slot = (GT == 16) ? hlf : 0;
                const float x0 = __int_as_float(d[2 * hlf]) - kQ4Bias;
                const float x1 = __int_as_float(d[2 * hlf + 1]) - kQ4Bias;
                const int j = jr[mt][hlf];
                sc[slot][ntile][0] = fmaf(x0, wq[mt][hlf] * sm.kdf[ta][j], sc[slot][ntile][0]);
                sc[slot][ntile][1] =
                    fmaf(x1, wq[mt][hlf] * sm.kdf[ta + 1][j], sc[slot][ntile][1]);
            }
        }
    }
    // the blocks of one head sit in lanes whose g differs in the bits >= log2(GT)
#pragma unroll
    for (int s = 0; s < S::NSLOT; ++s)
#pragma unroll
        for (int ntile = 0; ntile < 4; ++ntile)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                float x = sc[s][ntile][e];
                if constexpr (GT <= 1)
                    x += __shfl_xor_sync(kFullMask, x, 4);
                if constexpr (GT <= 2)
                    x += __shfl_xor_sync(kFullMask, x, 8);
                if constexpr (GT <= 4)
                    x += __shfl_xor_sync(kFullMask, x, 16);
                const int t = 8 * ntile + 2 * c + e;
                sc[s][ntile][e] = ((vmask >> t) & 1u) ? x : -INFINITY;
            }

    // ---- softmax: the slice's maximum per head, then the chunk's
    const int hs = g % GT; // head of slot 0 (slot 1: hs + 8)
#pragma unroll
    for (int s = 0; s < S::NSLOT; ++s) {
        float m = -INFINITY;
#pragma unroll
        for (int ntile = 0; ntile < 4; ++ntile)
            m = fmaxf(m, fmaxf(sc[s][ntile][0], sc[s][ntile][1]));
        m = fmaxf(m, __shfl_xor_sync(kFullMask, m, 1));
        m = fmaxf(m, __shfl_xor_sync(kFullMask, m, 2));
        if (c == 0 && g < GT)
            sm.smax[warp][hs + 8 * s] = m;
    }
    __syncthreads();
    // binary16 exponent field of the chunk's largest |dv| in block j: lane (g, c) reads
    // warp g's value of block c; after the reduction over g, lane j holds block j's
    uint32_t emax_c = sm.dvmax[g][c];
    emax_c = max(emax_c, __shfl_xor_sync(kFullMask, emax_c, 4));
    emax_c = max(emax_c, __shfl_xor_sync(kFullMask, emax_c, 8));
    emax_c = max(emax_c, __shfl_xor_sync(kFullMask, emax_c, 16));
    emax_c >>= 10;
#pragma unroll
    for (int s = 0; s < S::NSLOT; ++s) {
        // the chunk's maximum: lane (g, c) reads warps c and c + 4, then the c lanes merge
        float m = fmaxf(sm.smax[c][hs + 8 * s], sm.smax[c + 4][hs + 8 * s]);
        m = fmaxf(m, __shfl_xor_sync(kFullMask, m, 1));
        m = fmaxf(m, __shfl_xor_sync(kFullMask, m, 2));
        const float mref = m == -INFINITY ? 0.f : m;
        float sum = 0.f;
#pragma unroll
        for (int ntile = 0; ntile < 4; ++ntile)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const float w = fast_exp2(sc[s][ntile][e] - mref);
                sc[s][ntile][e] = w;
                sum += w;
            }
        sum += __shfl_xor_sync(kFullMask, sum, 1);
        sum += __shfl_xor_sync(kFullMask, sum, 2);
        if (c == 0 && g < GT)
            sm.ssum[warp][hs + 8 * s] = sum;
    }

    // ---- P = round(w * dv * 2^(36 - e_j)) as byte planes, in PV B-fragment order: lane
    // (g, c) holds column g of n-tile ns, i.e. row 8 ns + g = (block, head), and the tokens
    // tau(4c + i) = 2c + (i & 1) + 8 (i >> 1) (+ 16 in the second register)
#pragma unroll
    for (int ns = 0; ns < S::NS; ++ns) {
        const int rr = 8 * ns + g;
        const int j = (rr / GT) & 3;
        const int slot = (GT == 16) ? (ns & 1) : 0;
        const bool live = rr < S::R;
        const float pscale = exp2i(36 - (int)__shfl_sync(kFullMask, emax_c, j));
        uint32_t planes[3][2];
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            int P[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int ntile = 2 * half + (i >> 1), e = i & 1;
                const int t = warp * 32 + 8 * ntile + 2 * c + e;
                const float dvs = sm.vdf[t][j] * pscale;
                const float x = fmaf(sc[slot][ntile][e], dvs, kQ4Bias);
                P[i] = live ? __float_as_int(x) - kDotBias : 0;
            }
            const uint32_t x01 = prmt((uint32_t)P[0], (uint32_t)P[1], 0x5140);
            const uint32_t x23 = prmt((uint32_t)P[2], (uint32_t)P[3], 0x5140);
            const uint32_t z01 = prmt((uint32_t)P[0], (uint32_t)P[1], 0x7362);
            const uint32_t z23 = prmt((uint32_t)P[2], (uint32_t)P[3], 0x7362);
            planes[0][half] = prmt(x01, x23, 0x5410);
            planes[1][half] = prmt(x01, x23, 0x7632);
            planes[2][half] = prmt(z01, z23, 0x5410);
        }
#pragma unroll
        for (int k = 0; k < 3; ++k)
            sm.u.pb[warp][ns][k][lane] = make_uint2(planes[k][0], planes[k][1]);
    }
    __syncthreads(); // every slice's P

    // ---- PV: warp w owns channels 32 jb + 2 m + par (m = 0..15), jb = w / 2, par = w & 1
    const int jb = warp >> 1, par = warp & 1;
    const uint32_t vsh = par ? 0u : 4u; // nibble of this warp's channels, moved to the top
    constexpr int SPB = S::SPB;
    const int ns0 = (jb * GT) / 8; // first n-tile holding block jb's columns
    const int kk = lane & 15;
    const int vtok = (lane >> 4) * 16 + 2 * (kk >> 2) + (kk & 1) + 8 * ((kk >> 1) & 1);
    const uint32_t vrow = smem_addr(&sm.v[vtok][0]) + 16u * ((uint32_t)jb ^ q4_swz(vtok));
    int acc[SPB][3][4];
    float o[SPB][4];
#pragma unroll
    for (int si = 0; si < SPB; ++si)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            o[si][e] = 0.f;
#pragma unroll
            for (int k = 0; k < 3; ++k)
                acc[si][k][e] = kDotBias;
        }
    // sum_t A P = D0 + 256 D1 + 65536 D2 = 256 x with A = 16 (code - 8) and
    // P = w dv 2^(36 - e), so sum_t w dv (code - 8) = x 2^(e - 32)
    const float oscale = exp2i((int)__shfl_sync(kFullMask, emax_c, jb) - 32);
#pragma unroll
    for (int sl = 0; sl < kQ4Warps; ++sl) {
        if (sl * 32 < nt) {
            uint32_t r[4];
            ldsm_x2_trans_b8(r[0], r[1], r[2], r[3], vrow + (uint32_t)(sl * 32 * kQ4Row));
            uint32_t a[4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
                a[i] = nib_s8x16(r[i], vsh);
#pragma unroll
            for (int si = 0; si < SPB; ++si) {
                const uint2 b0 = sm.u.pb[sl][ns0 + si][0][lane];
                const uint2 b1 = sm.u.pb[sl][ns0 + si][1][lane];
                const uint2 b2 = sm.u.pb[sl][ns0 + si][2][lane];
                mma_s8u8_16832_acc(acc[si][0], a[0], a[1], a[2], a[3], b0.x, b0.y, acc[si][0]);
                mma_s8u8_16832_acc(acc[si][1], a[0], a[1], a[2], a[3], b1.x, b1.y, acc[si][1]);
                mma_s8_16832_acc(acc[si][2], a[0], a[1], a[2], a[3], b2.x, b2.y, acc[si][2]);
            }
        }
        if ((sl % kQ4FoldEvery) == kQ4FoldEvery - 1) {
#pragma unroll
            for (int si = 0; si < SPB; ++si)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float f0 = __int_as_float(acc[si][0][e]) - kQ4Bias;
                    const float f1 = __int_as_float(acc[si][1][e]) - kQ4Bias;
                    const float f2 = __int_as_float(acc[si][2][e]) - kQ4Bias;
                    const float x = fmaf(f0, 1.0f / 256.0f, fmaf(f2, 256.0f, f1));
                    o[si][e] = fmaf(x, oscale, o[si][e]);
#pragma unroll
                    for (int k = 0; k < 3; ++k)
                        acc[si][k][e] = kDotBias;
                }
        }
    }

    // ---- the chunk's partial: acc of block jb's columns, then M and S per head
    float *dst = p.partials + (((size_t)bk * p.n_chunks + blockIdx.x) * G) * kQ4SlotRow;
#pragma unroll
    for (int si = 0; si < SPB; ++si)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int rr = 8 * (ns0 + si) + 2 * c + (e & 1);
            const int h = rr % GT;
            const int ch = 32 * jb + 2 * (g + 8 * (e >> 1)) + par;
            if (rr / GT == jb && h < G)
                dst[(size_t)h * kQ4SlotRow + ch] = o[si][e];
        }
    if (warp == 0 && lane < G) {
        float m = -INFINITY, s = 0.f;
#pragma unroll
        for (int w = 0; w < kQ4Warps; ++w) {
            m = fmaxf(m, sm.smax[w][lane]);
            s += sm.ssum[w][lane];
        }
        dst[(size_t)lane * kQ4SlotRow + kD] = m;
        dst[(size_t)lane * kQ4SlotRow + kD + 1] = s;
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
