// q8kv_combine.cuh -- log-sum-exp combine of split-KV partial results (flash-decoding).
//
// When the decode kernel splits one segment (a sequence's tiles of one KV head chunk)
// across several CTAs, each CTA leaves a partial per query head: the unnormalised V
// accumulator acc (in units of 2^-A), its running maxima M (softmax scores) and A
// (score + log2 V scale) and its running sum S (in units of 2^-M), all base 2. The merged
// row is
//   mx = max_i M_i,  ax = max_i A_i,  S = sum_i S_i 2^(M_i - mx),
//   out = (sum_i acc_i 2^(A_i - ax)) * 2^(ax - mx) / S,
// i.e. the single-pass online softmax of the whole sequence (the running-max rescaling of
// the Kestrel-LLM walk-through "flash_attn_single_q_q8_neon", trdm.cn/news/511694,
// section 2 part 3, applied between pieces instead of between tokens).
//
// The decode kernel records, for every segment it split, a descriptor in the slot of the
// segment's first contributor: {b, hc, n contributors, first partial slot}; the other
// contributors' slots are 2 * (first CTA + k), k = 1..n-1. This kernel runs next on the
// stream (programmatic dependent launch: it is scheduled while the decode kernel drains
// and waits for its completion before reading anything). Its time is all latency (the
// partials are a few MB in L2), so it is laid out for few dependent steps:
//  * one load per thread of the descriptors and one block-wide scan compact them (the same
//    order in every CTA);
//  * the work is the list of units (segment, query head, 32-channel quarter), split evenly
//    over the CTAs in 32-bit arithmetic; a CTA takes up to 32 units at a time and gives
//    each unit 32 / units-in-batch rows of 8 threads that stride over the unit's inputs,
//    a thread issuing the loads of up to 8 inputs at once;
//  * a row merges its inputs with the maxima taken first, and the rows of a unit are then
//    merged pairwise with the associative log-sum-exp merge, by shuffles inside a warp and
//    one shared-memory step across warps.
#pragma once

#include <cstdint>

#include "q8kv_ptx.cuh"

namespace q8kv {

constexpr int kCombineThreads = 256;
constexpr int kCombineWarps = kCombineThreads / 32;
constexpr int kCombineMaxDesc = 2048;  // 2 * decode grid (the grid is at most 1024 CTAs)
constexpr int kCombineQuarter = 32;    // channels per unit
constexpr int kCombineSlotRow = 132;   // floats per partial row: acc[128], M, S, A, pad
constexpr int kCombineDescPerThread = kCombineMaxDesc / kCombineThreads;

struct CombineParams {
    float *out;
    const float *partials; // [n_desc slots] x heads_seg x kCombineSlotRow
    const int4 *desc;      // [n_desc] {b, hc, n (0: none), first slot}
    int n_desc;
    int Hq, heads_seg;
    int G, Gq, nq, HPC;    // query rows per KV head (nq tokens x Gq heads), tokens, KV heads
                           // per segment
};

constexpr int kCombineBatchIn = 8; // inputs a thread loads at once

// A piece of one output row: the maxima M and A, the sum S (units 2^-M) and 4 channels of
// the accumulator (units 2^-A).
struct LsePiece {
    float m, a, s;
    float4 acc;
};

__device__ __forceinline__ float lse_factor(float from, float to)
{
    return from == -INFINITY ? 0.f : exp2f(from - to);
}

// Merge of two pieces (associative and commutative up to rounding).
__device__ __forceinline__ LsePiece lse_merge(const LsePiece &x, const LsePiece &y)
{
    LsePiece r;
    r.m = fmaxf(x.m, y.m);
    r.a = fmaxf(x.a, y.a);
    const float fx = lse_factor(x.m, r.m), fy = lse_factor(y.m, r.m);
    const float gx = lse_factor(x.a, r.a), gy = lse_factor(y.a, r.a);
    r.s = x.s * fx + y.s * fy;
    r.acc = make_float4(x.acc.x * gx + y.acc.x * gy, x.acc.y * gx + y.acc.y * gy,
                        x.acc.z * gx + y.acc.z * gy, x.acc.w * gx + y.acc.w * gy);
    return r;
}

__device__ __forceinline__ LsePiece lse_shfl_xor(const LsePiece &x, int o)
{
    LsePiece r;
    r.m = __shfl_xor_sync(0xffffffffu, x.m, o);
    r.a = __shfl_xor_sync(0xffffffffu, x.a, o);
    r.s = __shfl_xor_sync(0xffffffffu, x.s, o);
    r.acc.x = __shfl_xor_sync(0xffffffffu, x.acc.x, o);
    r.acc.y = __shfl_xor_sync(0xffffffffu, x.acc.y, o);
    r.acc.z = __shfl_xor_sync(0xffffffffu, x.acc.z, o);
    r.acc.w = __shfl_xor_sync(0xffffffffu, x.acc.w, o);
    return r;
}

__global__ void __launch_bounds__(kCombineThreads)
    combine_kernel(const __grid_constant__ CombineParams p)
{
    __shared__ int4 sdesc[kCombineMaxDesc];
    __shared__ int wtot[kCombineWarps];
    __shared__ LsePiece xw[kCombineWarps][8]; // cross-warp step of a unit's merge

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // the decode kernel's partials and descriptors are complete and visible after this
    grid_dep_wait();
    grid_dep_launch();

    // ---- the descriptors that start a split segment, compacted in order: thread t holds
    // descriptors [t * per, (t + 1) * per)
    const int per = (p.n_desc + kCombineThreads - 1) / kCombineThreads; // <= 8
    int4 dv[kCombineDescPerThread];
    int cnt = 0;
#pragma unroll
    for (int k = 0; k < kCombineDescPerThread; ++k) {
        const int i = tid * per + k;
        dv[k] = (k < per && i < p.n_desc) ? __ldcg(&p.desc[i]) : make_int4(0, 0, 0, 0);
        cnt += dv[k].z > 0 ? 1 : 0;
    }
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o)
            incl += t;
    }
    if (lane == 31)
        wtot[warp] = incl;
    __syncthreads();
    int off = incl - cnt, nvalid = 0;
#pragma unroll
    for (int w = 0; w < kCombineWarps; ++w) {
        off += w < warp ? wtot[w] : 0;
        nvalid += wtot[w];
    }
#pragma unroll
    for (int k = 0; k < kCombineDescPerThread; ++k)
        if (dv[k].z > 0)
            sdesc[off++] = dv[k];
    __syncthreads();

    const int H = p.heads_seg;
    const int per_seg = H * (128 / kCombineQuarter);
    // T <= 2048 segments x 512 units < 2^21 and the grid is at most 1024 CTAs, so the
    // products below stay under 2^31
    const unsigned T = (unsigned)nvalid * (unsigned)per_seg;
    const int ubeg = (int)(T * blockIdx.x / gridDim.x);
    const int uend = (int)(T * (blockIdx.x + 1) / gridDim.x);

    const int fl = tid & 7, row = tid >> 3;
    for (int u0 = ubeg; u0 < uend; u0 += 32) {
        const int U = (uend - u0) < 32 ? (uend - u0) : 32;
        int upow = 1;
        while (upow < U)
            upow <<= 1;
        const int IG = 32 / upow; // rows per unit; row ig takes inputs ig, ig + IG, ...
        const int u = row / IG, ig = row - u * IG;
        const bool active = u < U;
        int b = 0, hc = 0, n = 0, first = 0, hl = 0, q = 0;
        if (active) {
            const int unit = u0 + u;
            const int d = unit / per_seg;
            const int rem = unit - d * per_seg;
            hl = rem >> 2;
            q = rem & 3;
            const int4 ds = sdesc[d];
            b = ds.x;
            hc = ds.y;
            n = ds.z;
            first = ds.w;
        }
        // this row's inputs: per chunk of kCombineBatchIn, all loads first, then the
        // maxima, then the rescaled sums (no chain of dependent exponentials)
        LsePiece x;
        x.m = -INFINITY;
        x.a = -INFINITY;
        x.s = 0.f;
        x.acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int i0 = ig; i0 < n; i0 += kCombineBatchIn * IG) {
            float4 hd[kCombineBatchIn], v[kCombineBatchIn];
#pragma unroll
            for (int k = 0; k < kCombineBatchIn; ++k) {
                const int i = i0 + k * IG;
                hd[k] = make_float4(-INFINITY, 0.f, -INFINITY, 0.f);
                v[k] = make_float4(0.f, 0.f, 0.f, 0.f);
                if (i < n) {
                    const int slot = i == 0 ? first : 2 * ((first >> 1) + i);
                    const float *rp = p.partials + ((size_t)slot * H + hl) * kCombineSlotRow;
                    hd[k] = __ldcg(reinterpret_cast<const float4 *>(rp + 128));
                    v[k] = __ldcg(reinterpret_cast<const float4 *>(rp + q * kCombineQuarter + 4 * fl));
                }
            }
            float mn = x.m, an = x.a;
#pragma unroll
            for (int k = 0; k < kCombineBatchIn; ++k) {
                mn = fmaxf(mn, hd[k].x);
                an = fmaxf(an, hd[k].z);
            }
            const float fo = lse_factor(x.m, mn), go = lse_factor(x.a, an);
            x.s *= fo;
            x.acc = make_float4(x.acc.x * go, x.acc.y * go, x.acc.z * go, x.acc.w * go);
#pragma unroll
            for (int k = 0; k < kCombineBatchIn; ++k) {
                const float fm = lse_factor(hd[k].x, mn), ga = lse_factor(hd[k].z, an);
                x.s += hd[k].y * fm;
                x.acc.x += v[k].x * ga;
                x.acc.y += v[k].y * ga;
                x.acc.z += v[k].z * ga;
                x.acc.w += v[k].w * ga;
            }
            x.m = mn;
            x.a = an;
        }
        // merge the unit's IG rows: rows r and r ^ 1 (lanes 8 apart) and r ^ 2 (16 apart)
        // share a warp; a unit of more than 4 rows spans IG / 4 whole warps
        if (IG >= 2)
            x = lse_merge(x, lse_shfl_xor(x, 8));
        if (IG >= 4)
            x = lse_merge(x, lse_shfl_xor(x, 16));
        if (IG >= 8) {
            if (lane < 8)
                xw[warp][lane] = x;
            __syncthreads();
            if (lane < 8 && (warp & (IG / 4 - 1)) == 0)
                for (int w = 1; w < IG / 4; ++w)
                    x = lse_merge(x, xw[warp + w][lane]);
            __syncthreads(); // xw is reused by the next batch
        }
        if (active && ig == 0) {
            const float f = x.s > 0.f ? exp2f(x.a - x.m) / x.s : 0.f;
            // segment row hl is query row hl % G of KV head hc * HPC + hl / G; that row is
            // query token hg / Gq, head kvh * Gq + hg % Gq of the [B][nq][Hq] output
            const int kvh = hc * p.HPC + hl / p.G, hg = hl % p.G;
            const int ti = hg / p.Gq;
            const long long orow =
                ((long long)b * p.nq + ti) * p.Hq + (long long)kvh * p.Gq + (hg - ti * p.Gq);
            float *dst = p.out + orow * 128 + q * kCombineQuarter + 4 * fl;
            *reinterpret_cast<float4 *>(dst) =
                make_float4(x.acc.x * f, x.acc.y * f, x.acc.z * f, x.acc.w * f);
        }
    }
}

} // namespace q8kv
