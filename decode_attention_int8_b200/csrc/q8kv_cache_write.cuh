// q8kv_cache_write.cuh -- the KV-cache write: quantise new K and V rows to int8 with one
// fp32 scale per (token, KV head) and store them at their physical slots of the paged pools.
//
// What it computes: the cache the decode kernel reads holds, per (token, KV head), int8
// codes and one dequantisation multiplier (Kestrel-LLM walk-through
// "flash_attn_single_q_q8_neon", trdm.cn/news/511694: the kernel signature's per-token
// per-head kscale, turned into the multiplier as kscale * 1/127 in section 2 part 2). A row
// is quantised with the section 2 part 1 quantiser taken over the whole row:
//   amax = max|x| (1 when below 1e-6), scale = amax * fl(1/127), inv = fl(127 / amax),
//   code = clamp(round-half-even(fl(x * inv)), -127, 127)
// all in IEEE fp32 (explicitly rounded intrinsics: the codes are integers, so they must
// not depend on contraction or fast-math). A row holding an infinity or a NaN gets codes 0
// and a NaN scale, and sets a device error bit. Token i goes to physical slot
// slot_mapping[i] = block * block_size + offset (beaiera.top "deepseek-attention-div64",
// "Top-K index global mapping"); negative entries are padding and are skipped, as that
// section prescribes; a slot past the pool is skipped and sets a device error bit.
//
// How: the same page describes vLLM's fused cache-write kernel as one warp per (token,
// head) with 16-byte vector accesses. On B200 that layout spends more issue slots on the
// per-row scalar work (index arithmetic, the correctly rounded division, a 5-step
// reduction, all replicated over 32 lanes) than on the 128 elements, so here a row gets
// LPR = 8 lanes (16 for head_dim 256) and a warp takes 32 / LPR (token, KV head) pairs at
// once, with their K and V rows: each lane loads head_dim / LPR floats of each row as
// 16-byte streaming loads in which the row's LPR lanes cover 16 * LPR contiguous bytes
// (the rows are read once), the row maximum is a 3- or 4-step butterfly inside the lane
// group, and each lane stores 4 codes per 16-byte chunk, so every store instruction
// writes 4 * LPR contiguous bytes of each row. The pairs are taken in (token, head) order,
// so the scales of one slot (adjacent floats) come from neighbouring lanes. The grid is
// one wave of resident blocks striding over the pairs, with the (token, head) position
// advanced incrementally (no 64-bit division in the loop). The loads of a pair do not
// depend on its slot, so they are issued together with the slot load.
#pragma once

#include <cuda_fp16.h>

#include <cstdint>

#include "q8kv_ptx.cuh"

namespace q8kv {

constexpr unsigned kErrSlot = 0x8u;       // a slot past the pool (row skipped)
constexpr unsigned kErrNonFinite = 0x10u; // a row held an infinity or a NaN
constexpr int kWriteThreads = 256;
constexpr int kWriteWarps = kWriteThreads / 32;

// Lanes per row: 8 for head_dim 64 and 128, 16 for 256, so that a lane holds at most 16
// floats of each of its K and V rows.
__host__ __device__ constexpr int write_lanes_per_row(int D)
{
    return D == 256 ? 16 : 8;
}
// (token, KV head) pairs per warp and iteration.
__host__ __device__ constexpr int write_pairs_per_warp(int D)
{
    return 32 / write_lanes_per_row(D);
}
// Resident blocks per SM: 4 (1024 threads of up to 64 registers; a lane holds up to 32
// floats of K and V). Each warp has 4 KB of loads in flight, 128 KB per SM.
__host__ __device__ constexpr int write_blocks_per_sm(int)
{
    return 4;
}

struct CacheWriteParams {
    int8_t *k, *v;
    float *ks, *vs;
    const float *k_new, *v_new;
    const int64_t *slots;
    long long n_tokens;
    long long token_stride; // floats from one token's rows to the next token's
    long long n_slots;      // num_blocks * block_size
    int Hk;
    unsigned *errors;
};

// One lane's share of a row: C chunks of 4 floats; chunk c covers elements
// 4 * (sub + LPR * c) .. + 3, where sub is the lane's index inside the row's lane group.
template <int D>
struct RowFrag {
    static constexpr int LPR = write_lanes_per_row(D);
    static constexpr int C = D / (4 * LPR);
    float4 x[C];
};

template <int D>
__device__ __forceinline__ RowFrag<D> load_frag(const float *row, int sub)
{
    RowFrag<D> f;
#pragma unroll
    for (int c = 0; c < RowFrag<D>::C; ++c)
        f.x[c] = __ldcs(reinterpret_cast<const float4 *>(row) + sub + RowFrag<D>::LPR * c);
    return f;
}

// Maximum of |x| over the row (the lane group), and whether every element is finite.
template <int D>
__device__ __forceinline__ float row_amax(const RowFrag<D> &f, bool &finite)
{
    float m = 0.f;
    bool fin = true;
#pragma unroll
    for (int c = 0; c < RowFrag<D>::C; ++c) {
        const float a[4] = {fabsf(f.x[c].x), fabsf(f.x[c].y), fabsf(f.x[c].z), fabsf(f.x[c].w)};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            fin = fin && (a[i] <= 3.402823466e38f); // false for inf and NaN
            m = fmaxf(m, a[i]);
        }
    }
    unsigned bad = fin ? 0u : 1u;
#pragma unroll
    for (int o = RowFrag<D>::LPR / 2; o > 0; o >>= 1) {
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        bad |= __shfl_xor_sync(0xffffffffu, bad, o);
    }
    finite = bad == 0u;
    return m;
}

__device__ __forceinline__ uint32_t code_byte(float x, float inv)
{
    int c = __float2int_rn(__fmul_rn(x, inv));
    c = c > 127 ? 127 : (c < -127 ? -127 : c);
    return static_cast<uint32_t>(c) & 0xffu;
}

// Quantise one row (every lane of the warp takes part in the reductions) and, if `store`,
// write the lane's codes; returns the row's scale and sets `bad` for a non-finite row.
template <int D>
__device__ __forceinline__ float quantise_row(const RowFrag<D> &f, int8_t *dst, bool store,
                                              int sub, bool &bad)
{
    bool finite;
    float amax = row_amax<D>(f, finite);
    bad = !finite;
    float inv = 0.f, scale = __int_as_float(0x7fc00000); // quiet NaN for a non-finite row
    if (finite) {
        if (amax < 1e-6f)
            amax = 1.0f;
        scale = __fmul_rn(amax, 0x1.020408p-7f); // fl(1/127)
        inv = __fdiv_rn(127.0f, amax);
    }
    if (store) {
#pragma unroll
        for (int c = 0; c < RowFrag<D>::C; ++c) {
            uint32_t w = 0u;
            if (finite)
                w = code_byte(f.x[c].x, inv) | (code_byte(f.x[c].y, inv) << 8) |
                    (code_byte(f.x[c].z, inv) << 16) | (code_byte(f.x[c].w, inv) << 24);
            reinterpret_cast<uint32_t *>(dst)[sub + RowFrag<D>::LPR * c] = w;
        }
    }
    return scale;
}

template <int D>
__global__ void __launch_bounds__(kWriteThreads, write_blocks_per_sm(D))
    cache_write_kernel(const __grid_constant__ CacheWriteParams p)
{
    constexpr int LPR = write_lanes_per_row(D);
    constexpr int PPW = write_pairs_per_warp(D);
    // the new rows may come from the kernel before this one on the stream
    grid_dep_wait();
    grid_dep_launch();
    const int lane = threadIdx.x & 31, sub = lane % LPR;
    // this lane's (token, head) pair, advanced by `step` pairs per iteration
    const long long n_pairs = p.n_tokens * p.Hk;
    const long long step = (long long)gridDim.x * kWriteWarps * PPW;
    const long long wbase = ((long long)blockIdx.x * kWriteWarps + (threadIdx.x >> 5)) * PPW;
    const long long first = wbase + lane / LPR;
    long long tok = first / p.Hk;
    int h = (int)(first - tok * p.Hk);
    const long long dtok = step / p.Hk;
    const int dh = (int)(step - dtok * p.Hk);
    unsigned err = 0;
    // warp-uniform loop: the row reductions shuffle across the whole warp
#pragma unroll 1
    for (long long base = wbase; base < n_pairs; base += step) {
        long long slot = -1;
        RowFrag<D> fk, fv;
        if (tok < p.n_tokens) {
            const long long src = tok * p.token_stride + (long long)h * D;
            slot = __ldg(p.slots + tok);
            fk = load_frag<D>(p.k_new + src, sub);
            fv = load_frag<D>(p.v_new + src, sub);
        } else {
#pragma unroll
            for (int c = 0; c < RowFrag<D>::C; ++c)
                fk.x[c] = fv.x[c] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        if (slot >= p.n_slots) {
            err |= kErrSlot;
            slot = -1;
        }
        const bool store = slot >= 0; // negative: padding entry (or no pair)
        const long long row = store ? slot * p.Hk + h : 0;
        bool bad_k, bad_v;
        const float sk = quantise_row<D>(fk, p.k + row * D, store, sub, bad_k);
        const float sv = quantise_row<D>(fv, p.v + row * D, store, sub, bad_v);
        if (store) {
            if (sub == 0)
                p.ks[row] = sk;
            else if (sub == 1)
                p.vs[row] = sv;
            if (bad_k || bad_v)
                err |= kErrNonFinite;
        }
        tok += dtok;
        h += dh;
        if (h >= p.Hk) {
            h -= p.Hk;
            ++tok;
        }
    }
    if (err)
        atomicOr(p.errors, err);
}

// ------------------------------------------------------------------ q4_0 cache write
//
// The same write in llama.cpp's q4_0 format (one of the quantised KV-cache types of the
// llama.cpp change on baguaai.com's FlashAttention page), into the pools the q4_0 decode
// reads: per 32-channel block, m = the value of largest magnitude with its sign (the first
// one on ties; +0 for an all-zero block), d = m / -8, id = d != 0 ? 1 / d : 0,
// code = min(15, trunc(x * id + 8.5)), every operation rounded to fp32 on its own, d stored
// as binary16 (round to nearest even); codes packed two per byte, channel 2i in the low
// nibble of byte i. A block holding an infinity or a NaN is stored as codes 8 with a NaN
// scale and sets a device error bit.
//
// Lanes as in the q8 write: chunk c of a lane holds 4 consecutive channels of one block, and
// a block's 32 channels lie on 8 consecutive lanes, so the search for m is a 3-step
// butterfly over a 64-bit key (|x| bits, then the reversed channel index, so that the
// first channel wins a tie, then the sign); a lane stores the 2 code bytes of each of its
// chunks (16 contiguous bytes per block and store instruction).
struct CacheWriteQ4Params {
    uint8_t *k4, *v4;
    uint16_t *kd, *vd;
    const float *k_new, *v_new;
    const int64_t *slots;
    long long n_tokens;
    long long token_stride;
    long long n_slots;
    int Hk;
    unsigned *errors;
};

// Key of element i (channel `ch` of its block) for the largest-magnitude search.
__device__ __forceinline__ unsigned long long q4_key(float x, int ch)
{
    const uint32_t b = __float_as_uint(x);
    return ((unsigned long long)(b & 0x7fffffffu) << 32) | ((uint32_t)(31 - ch) << 1) | (b >> 31);
}

__device__ __forceinline__ uint32_t q4_code(float x, float id)
{
    const int c = __float2int_rz(__fadd_rn(__fmul_rn(x, id), 8.5f));
    return (uint32_t)(c > 15 ? 15 : c);
}

// One chunk of 4 channels (channel 4 * g8 .. 4 * g8 + 3 of its block, g8 = lane % 8 inside
// the block's lane group): returns the chunk's two code bytes as 16 bits and the block's
// binary16 scale; sets `bad` for a non-finite block.
__device__ __forceinline__ uint32_t q4_chunk(float4 x, int g8, uint16_t &d16, bool &bad)
{
    unsigned long long k = q4_key(x.x, 4 * g8);
    const unsigned long long k1 = q4_key(x.y, 4 * g8 + 1), k2 = q4_key(x.z, 4 * g8 + 2),
                             k3 = q4_key(x.w, 4 * g8 + 3);
    k = k1 > k ? k1 : k;
    k = k2 > k ? k2 : k;
    k = k3 > k ? k3 : k;
#pragma unroll
    for (int o = 1; o < 8; o <<= 1) {
        const unsigned long long t = __shfl_xor_sync(0xffffffffu, k, o);
        k = t > k ? t : k;
    }
    const uint32_t abits = (uint32_t)(k >> 32);
    bad = abits >= 0x7f800000u; // an infinity or a NaN in the block
    if (bad) {
        d16 = 0x7e00u;
        return 0x8888u;
    }
    // m with its sign; an all-zero block keeps m = +0 (d = +0 / -8 = -0)
    const float m = __uint_as_float(abits | (abits != 0u ? (uint32_t)(k & 1u) << 31 : 0u));
    // m / -8 and 1 / d, each correctly rounded: the quotient by a power of two is the product
    // by its reciprocal (the same exact value, so the same rounding), and the correctly
    // rounded reciprocal is the correctly rounded quotient 1 / d
    const float d = __fmul_rn(m, -0.125f);
    const float id = d != 0.0f ? __frcp_rn(d) : 0.0f;
    d16 = __half_as_ushort(__float2half_rn(d));
    return q4_code(x.x, id) | (q4_code(x.y, id) << 4) | (q4_code(x.z, id) << 8) |
           (q4_code(x.w, id) << 12);
}

template <int D>
__global__ void __launch_bounds__(kWriteThreads, write_blocks_per_sm(D))
    cache_write_q4_kernel(const __grid_constant__ CacheWriteQ4Params p)
{
    constexpr int LPR = write_lanes_per_row(D);
    constexpr int PPW = write_pairs_per_warp(D);
    constexpr int C = RowFrag<D>::C;
    // the new rows may come from the kernel before this one on the stream
    grid_dep_wait();
    grid_dep_launch();
    const int lane = threadIdx.x & 31, sub = lane % LPR, g8 = sub & 7;
    const long long n_pairs = p.n_tokens * p.Hk;
    const long long step = (long long)gridDim.x * kWriteWarps * PPW;
    const long long wbase = ((long long)blockIdx.x * kWriteWarps + (threadIdx.x >> 5)) * PPW;
    const long long first = wbase + lane / LPR;
    long long tok = first / p.Hk;
    int h = (int)(first - tok * p.Hk);
    const long long dtok = step / p.Hk;
    const int dh = (int)(step - dtok * p.Hk);
    unsigned err = 0;
#pragma unroll 1
    for (long long base = wbase; base < n_pairs; base += step) {
        long long slot = -1;
        RowFrag<D> fk, fv;
        if (tok < p.n_tokens) {
            const long long src = tok * p.token_stride + (long long)h * D;
            slot = __ldg(p.slots + tok);
            fk = load_frag<D>(p.k_new + src, sub);
            fv = load_frag<D>(p.v_new + src, sub);
        } else {
#pragma unroll
            for (int c = 0; c < C; ++c)
                fk.x[c] = fv.x[c] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        if (slot >= p.n_slots) {
            err |= kErrSlot;
            slot = -1;
        }
        const bool store = slot >= 0;
        const long long row = store ? slot * p.Hk + h : 0;
        uint8_t *kc = p.k4 + row * (D / 2), *vc = p.v4 + row * (D / 2);
        uint16_t *kdr = p.kd + row * (D / 32), *vdr = p.vd + row * (D / 32);
        bool bad = false;
#pragma unroll
        for (int c = 0; c < C; ++c) {
            // chunk c holds channels 4 * (sub + LPR * c) ..: block (sub + LPR * c) / 8
            const int blk = (sub + LPR * c) >> 3;
            uint16_t dk, dv;
            bool bk, bv;
            const uint32_t ck = q4_chunk(fk.x[c], g8, dk, bk);
            const uint32_t cv = q4_chunk(fv.x[c], g8, dv, bv);
            bad = bad || bk || bv;
            if (store) {
                reinterpret_cast<uint16_t *>(kc)[blk * 8 + g8] = (uint16_t)ck;
                reinterpret_cast<uint16_t *>(vc)[blk * 8 + g8] = (uint16_t)cv;
                // one lane per block writes its scales: K from g8 == c, V from g8 == 4 + c
                if (g8 == c)
                    kdr[blk] = dk;
                else if (g8 == 4 + c)
                    vdr[blk] = dv;
            }
        }
        if (store && bad)
            err |= kErrNonFinite;
        tok += dtok;
        h += dh;
        if (h >= p.Hk) {
            h -= p.Hk;
            ++tok;
        }
    }
    if (err)
        atomicOr(p.errors, err);
}

} // namespace q8kv
