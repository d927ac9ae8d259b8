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
// head) with 16-byte vector accesses; that shape suits B200 too. Here one warp owns one
// (token, KV head) pair and quantises its K and its V row together: each lane loads D/32
// consecutive floats of each row with 8- or 16-byte streaming loads (the rows are read
// once), the maximum is a 5-step butterfly over the warp, and each lane stores its D/32
// codes as one 2- or 4-byte word, so a warp writes each int8 row as one contiguous
// segment. Consecutive warps take consecutive KV heads of a token, so the scales of one
// slot (adjacent floats) are written by neighbouring warps. The grid is a whole number of
// resident blocks per SM and strides over the (token, head) pairs. The loads of a pair do
// not depend on its slot, so they are issued together with the slot load.
#pragma once

#include <cstdint>

#include "q8kv_ptx.cuh"

namespace q8kv {

constexpr unsigned kErrSlot = 0x8u;       // a slot past the pool (row skipped)
constexpr unsigned kErrNonFinite = 0x10u; // a row held an infinity or a NaN
constexpr int kWriteThreads = 256;
constexpr int kWriteWarps = kWriteThreads / 32;
// Resident blocks per SM: 8 (2048 threads, 32 registers each) where the row fits in that,
// 6 for head_dim 256 (its two 16-byte loads per row need more registers).
__host__ __device__ constexpr int write_blocks_per_sm(int D)
{
    return D == 256 ? 6 : 8;
}

struct CacheWriteParams {
    int8_t *k, *v;
    float *ks, *vs;
    const float *k_new, *v_new;
    const int64_t *slots;
    long long n_rows;       // n_tokens * Hk
    long long token_stride; // floats from one token's rows to the next token's
    long long n_slots;      // num_blocks * block_size
    int Hk;
    unsigned *errors;
};

// D/32 consecutive floats of one row per lane.
template <int D>
struct RowFrag {
    static constexpr int E = D / 32;
    float x[E];
};

template <int D>
__device__ __forceinline__ RowFrag<D> load_frag(const float *row, int lane)
{
    RowFrag<D> f;
    if constexpr (D == 64) {
        const float2 a = __ldcs(reinterpret_cast<const float2 *>(row) + lane);
        f.x[0] = a.x;
        f.x[1] = a.y;
    } else {
#pragma unroll
        for (int c = 0; c < D / 128; ++c) {
            const float4 a = __ldcs(reinterpret_cast<const float4 *>(row + 128 * c) + lane);
            f.x[4 * c + 0] = a.x;
            f.x[4 * c + 1] = a.y;
            f.x[4 * c + 2] = a.z;
            f.x[4 * c + 3] = a.w;
        }
    }
    return f;
}

// Row maximum of |x| over the warp, and whether every element of the row is finite.
template <int D>
__device__ __forceinline__ float row_amax(const RowFrag<D> &f, bool &finite)
{
    float m = 0.f;
    bool fin = true;
#pragma unroll
    for (int i = 0; i < RowFrag<D>::E; ++i) {
        const float a = fabsf(f.x[i]);
        fin = fin && (a <= 3.402823466e38f); // false for inf and NaN
        m = fmaxf(m, a);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    finite = __all_sync(0xffffffffu, fin);
    return m;
}

__device__ __forceinline__ uint32_t code_byte(float x, float inv)
{
    int c = __float2int_rn(__fmul_rn(x, inv));
    c = c > 127 ? 127 : (c < -127 ? -127 : c);
    return static_cast<uint32_t>(c) & 0xffu;
}

// Quantise the lane's fragment of one row and store its codes; returns the row's scale.
template <int D>
__device__ __forceinline__ float quantise_store(const RowFrag<D> &f, int8_t *dst, int lane,
                                                bool &bad)
{
    bool finite;
    float amax = row_amax<D>(f, finite);
    bad = !finite;
    float inv = 0.f, scale = __int_as_float(0x7fc00000); // quiet NaN for a non-finite row
    if (finite) {
        if (amax < 1e-6f)
            amax = 1.0f;
        scale = __fmul_rn(amax, __fdiv_rn(1.0f, 127.0f));
        inv = __fdiv_rn(127.0f, amax);
    }
    uint32_t w[RowFrag<D>::E];
#pragma unroll
    for (int i = 0; i < RowFrag<D>::E; ++i)
        w[i] = finite ? code_byte(f.x[i], inv) : 0u;
    if constexpr (D == 64) {
        reinterpret_cast<uint16_t *>(dst)[lane] = static_cast<uint16_t>(w[0] | (w[1] << 8));
    } else {
#pragma unroll
        for (int c = 0; c < D / 128; ++c)
            reinterpret_cast<uint32_t *>(dst + 128 * c)[lane] =
                w[4 * c] | (w[4 * c + 1] << 8) | (w[4 * c + 2] << 16) | (w[4 * c + 3] << 24);
    }
    return scale;
}

template <int D>
__global__ void __launch_bounds__(kWriteThreads, write_blocks_per_sm(D))
    cache_write_kernel(const __grid_constant__ CacheWriteParams p)
{
    // the new rows may come from the kernel before this one on the stream
    grid_dep_wait();
    grid_dep_launch();
    const int lane = threadIdx.x & 31;
    const long long nw = (long long)gridDim.x * kWriteWarps;
    unsigned err = 0;
#pragma unroll 1
    for (long long r = (long long)blockIdx.x * kWriteWarps + (threadIdx.x >> 5); r < p.n_rows;
         r += nw) {
        const long long tok = r / p.Hk;
        const int h = (int)(r - tok * p.Hk);
        const long long src = tok * p.token_stride + (long long)h * D;
        const long long slot = __ldg(p.slots + tok);
        const RowFrag<D> fk = load_frag<D>(p.k_new + src, lane);
        const RowFrag<D> fv = load_frag<D>(p.v_new + src, lane);
        if (slot < 0)
            continue; // padding entry
        if (slot >= p.n_slots) {
            err |= kErrSlot;
            continue;
        }
        const long long row = slot * p.Hk + h;
        bool bad_k, bad_v;
        const float sk = quantise_store<D>(fk, p.k + row * D, lane, bad_k);
        const float sv = quantise_store<D>(fv, p.v + row * D, lane, bad_v);
        if (lane == 0)
            p.ks[row] = sk;
        else if (lane == 1)
            p.vs[row] = sv;
        if (bad_k || bad_v)
            err |= kErrNonFinite;
    }
    if (err && lane == 0)
        atomicOr(p.errors, err);
}

} // namespace q8kv
