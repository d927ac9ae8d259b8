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
// Which segments the decode kernel split, and between which CTAs, follows from its work
// split alone: the same prefixes of the sequence lengths and the same CTA ranges, which this
// kernel recomputes (q8kv_decode.cuh) before it waits for the decode kernel. Reading the
// sequence lengths that early is safe: the only kernel before this one on the stream is the
// decode kernel of the same call, which never writes them, and this grid starts only after
// every decode CTA has passed its own dependency wait. Decode CTA j owns partial slots 2j
// (the segment its range starts in) and 2j + 1 (the segment it ends in); a split segment
// whose first contributor is j sits in slot 2j (when it starts exactly at j's first tile)
// or 2j + 1, and contributor k > 0 in slot 2 (j + k). This kernel runs next on the stream
// (programmatic dependent launch: it is scheduled while the decode kernel drains and waits
// for its completion before reading any partial). Its time is all latency (the partials
// are a few MB in L2), so it is laid out for few dependent steps:
//  * before the wait: the prefixes (one warp for up to 32 sequences), the CTA ranges, and
//    the split segments in CTA order (a block-wide scan compacts them);
//  * the work is the list of units (segment, query head, 32-channel quarter), split evenly
//    over the CTAs in 32-bit arithmetic; a CTA takes up to 32 units at a time and gives
//    each unit 32 / units-in-batch rows of 8 threads that stride over the unit's inputs,
//    a thread issuing the loads of up to 8 inputs at once;
//  * a row merges its inputs with the maxima taken first, and the rows of a unit are then
//    merged pairwise with the associative log-sum-exp merge, by shuffles inside a warp and
//    one shared-memory step across warps.
#pragma once

#include <cstdint>

#include "q8kv_decode.cuh"
#include "q8kv_ptx.cuh"

namespace q8kv {

constexpr int kCombineThreads = 256; // = kConsumerThreads: the decode's split helpers
                                     // synchronise 256 threads on named barrier 1
constexpr int kCombineWarps = kCombineThreads / 32;
constexpr int kCombineQuarter = 32;  // channels per unit
static_assert(kCombineThreads == kConsumerThreads, "the split helpers need 256 threads");
constexpr uint32_t kCombineStaticSmemMax = 4096; // bound on the kernel's static shared memory

// Dynamic shared memory of the combine kernel: split segments (one int4 per decode CTA),
// CTA ranges, then the prefixes.
struct CombineLayout {
    uint32_t off_desc, off_cstart, off_prefix, off_nseq, off_wsum, total;
};

__host__ __device__ inline CombineLayout combine_layout(int B, int grid)
{
    CombineLayout L;
    uint32_t o = 0;
    L.off_desc = o;
    o += 16u * (uint32_t)grid;
    L.off_cstart = o;
    o = align_up(o + 4u * (uint32_t)(grid + 1), 16);
    L.off_prefix = o;
    o = align_up(o + 4u * (uint32_t)(B + 1), 16);
    L.off_nseq = 0;
    if (B <= kPenaltyMaxB) {
        L.off_nseq = o;
        o = align_up(o + 4u * (uint32_t)(B + 1), 16);
    }
    L.off_wsum = o;
    o += 8u * kConsumerWarps;
    L.total = o;
    return L;
}

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
    combine_kernel(const __grid_constant__ DecodeParams p, int grid_dec)
{
    extern __shared__ __align__(16) uint8_t csm[];
    const CombineLayout cl = combine_layout(p.B, grid_dec);
    int4 *sdesc = reinterpret_cast<int4 *>(csm + cl.off_desc);
    int *cstart = reinterpret_cast<int *>(csm + cl.off_cstart);
    int *prefix = reinterpret_cast<int *>(csm + cl.off_prefix);
    int *nseq = cl.off_nseq ? reinterpret_cast<int *>(csm + cl.off_nseq) : nullptr;
    __shared__ int wtot[kCombineWarps];
    __shared__ LsePiece xw[kCombineWarps][8]; // cross-warp step of a unit's merge

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // ---- before the dependency wait: the decode kernel's work split (inputs only)
    build_prefix(p, prefix, nseq,
                 reinterpret_cast<volatile unsigned long long *>(csm + cl.off_wsum), tid, warp,
                 lane);
    consumer_bar();
    const Split sp = split_of(p, prefix, nseq, grid_dec);
    const int g = sp.gcta;
    for (int i = tid; i <= g; i += kCombineThreads)
        cstart[i] = cta_start(p, prefix, nseq, sp.pseg, sp.V, g, i);
    consumer_bar();
    // the split segment whose first contributor is decode CTA j (< g): the segment of its
    // last tile, when it starts inside j's range and ends past it (thread t takes
    // j = t, t + 256, ...; a block-wide scan compacts them in order)
    int nvalid = 0;
    for (int j0 = 0; j0 < g; j0 += kCombineThreads) {
        const int j = j0 + tid;
        int4 d = make_int4(0, 0, 0, 0);
        bool v = false;
        if (j < g) {
            const int t0 = cstart[j], t1 = cstart[j + 1];
            const SegCursor cu = cursor_at(p, prefix, t1 - 1);
            if (cu.seg0 >= t0 && cu.seg1 > t1) {
                const int last = cta_of_tile(cstart, g, cu.seg1 - 1);
                d = make_int4(cu.b, cu.hc, last - j + 1, 2 * j + (cu.seg0 == t0 ? 0 : 1));
                v = true;
            }
        }
        const unsigned m = __ballot_sync(0xffffffffu, v);
        if (lane == 0)
            wtot[warp] = __popc(m);
        consumer_bar();
        int off = nvalid, total = 0;
#pragma unroll
        for (int w = 0; w < kCombineWarps; ++w) {
            off += w < warp ? wtot[w] : 0;
            total += wtot[w];
        }
        if (v)
            sdesc[off + __popc(m & ((1u << lane) - 1u))] = d;
        nvalid += total;
        consumer_bar();
    }
    // the decode kernel's partials are complete and visible after this
    grid_dep_wait();
    grid_dep_launch();

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
                    const float *rp = p.partials + ((size_t)slot * H + hl) * kSlotRow;
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
