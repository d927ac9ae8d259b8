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
// and waits for its completion before reading anything). The work is the list of units
// (segment, query head, 32-channel quarter), split evenly over the CTAs; a CTA processes
// up to 32 units at a time, giving each unit 32 / units-in-batch rows of 8 threads that
// stride over the unit's inputs. A thread issues the loads of up to 8 inputs at once, so a
// unit usually costs one round trip to L2 whatever its input count; maxima are taken
// before any rescaling, so no exponential waits on another, and the rows of a unit are
// merged through shared memory the same way.
#pragma once

#include <cstdint>

#include "q8kv_ptx.cuh"

namespace q8kv {

constexpr int kCombineThreads = 256;
constexpr int kCombineMaxDesc = 2048;  // 2 * decode grid (the grid is at most 1024 CTAs)
constexpr int kCombineQuarter = 32;    // channels per unit
constexpr int kCombineSlotRow = 132;   // floats per partial row: acc[128], M, S, A, pad

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

__global__ void __launch_bounds__(kCombineThreads)
    combine_kernel(const __grid_constant__ CombineParams p)
{
    __shared__ int4 sdesc[kCombineMaxDesc];
    __shared__ int wcount[kCombineThreads / 32];
    __shared__ float4 part_acc[32][8];
    __shared__ float2 part_ma[32];
    __shared__ float part_s[32];

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // the decode kernel's partials and descriptors are complete and visible after this
    grid_dep_wait();
    grid_dep_launch();

    // compact copy of the descriptors that start a split segment (same order in every
    // CTA); all descriptor loads are issued before the first is used
    constexpr int kDescPerThread = kCombineMaxDesc / kCombineThreads;
    int4 dv[kDescPerThread];
#pragma unroll
    for (int k = 0; k < kDescPerThread; ++k) {
        const int i = k * kCombineThreads + tid;
        dv[k] = i < p.n_desc ? __ldcg(&p.desc[i]) : make_int4(0, 0, 0, 0);
    }
    int nvalid = 0;
#pragma unroll
    for (int k = 0; k < kDescPerThread; ++k) {
        if (k * kCombineThreads >= p.n_desc)
            break;
        const bool v = dv[k].z > 0;
        const unsigned m = __ballot_sync(0xffffffffu, v);
        if (lane == 0)
            wcount[warp] = __popc(m);
        __syncthreads();
        int off = nvalid;
        int total = 0;
        for (int w = 0; w < kCombineThreads / 32; ++w) {
            if (w < warp)
                off += wcount[w];
            total += wcount[w];
        }
        if (v)
            sdesc[off + __popc(m & ((1u << lane) - 1u))] = dv[k];
        nvalid += total;
        __syncthreads();
    }
    const int H = p.heads_seg;
    const int per_seg = H * (128 / kCombineQuarter);
    const long long T = (long long)nvalid * per_seg;
    const long long ubeg = T * blockIdx.x / gridDim.x, uend = T * (blockIdx.x + 1) / gridDim.x;

    const int fl = tid & 7, row = tid >> 3;
    for (long long u0 = ubeg; u0 < uend; u0 += 32) {
        const int U = (int)((uend - u0) < 32 ? (uend - u0) : 32);
        int upow = 1;
        while (upow < U)
            upow <<= 1;
        const int IG = 32 / upow; // rows per unit; row ig takes inputs ig, ig + IG, ...
        const int u = row / IG, ig = row % IG;
        const bool active = u < U;
        int b = 0, hc = 0, n = 0, first = 0, hl = 0, q = 0;
        if (active) {
            const long long unit = u0 + u;
            const int d = (int)(unit / per_seg);
            const int rem = (int)(unit - (long long)d * per_seg);
            hl = rem / (128 / kCombineQuarter);
            q = rem % (128 / kCombineQuarter);
            const int4 ds = sdesc[d];
            b = ds.x;
            hc = ds.y;
            n = ds.z;
            first = ds.w;
        }
        // this row's inputs: per chunk of kCombineBatchIn, all loads first, then the
        // maxima, then the rescaled sums (no chain of dependent exponentials)
        float m = -INFINITY, a = -INFINITY, s = 0.f;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int i0 = ig; i0 < n; i0 += kCombineBatchIn * IG) {
            float4 hd[kCombineBatchIn], x[kCombineBatchIn];
#pragma unroll
            for (int k = 0; k < kCombineBatchIn; ++k) {
                const int i = i0 + k * IG;
                hd[k] = make_float4(-INFINITY, 0.f, -INFINITY, 0.f);
                x[k] = make_float4(0.f, 0.f, 0.f, 0.f);
                if (i < n) {
                    const int slot = i == 0 ? first : 2 * ((first >> 1) + i);
                    const float *rp = p.partials + ((size_t)slot * H + hl) * kCombineSlotRow;
                    hd[k] = __ldcg(reinterpret_cast<const float4 *>(rp + 128));
                    x[k] = __ldcg(reinterpret_cast<const float4 *>(rp + q * kCombineQuarter + 4 * fl));
                }
            }
            float mn = m, an = a;
#pragma unroll
            for (int k = 0; k < kCombineBatchIn; ++k) {
                mn = fmaxf(mn, hd[k].x);
                an = fmaxf(an, hd[k].z);
            }
            const float fo = (m == -INFINITY) ? 0.f : exp2f(m - mn);
            const float go = (a == -INFINITY) ? 0.f : exp2f(a - an);
            s *= fo;
            acc = make_float4(acc.x * go, acc.y * go, acc.z * go, acc.w * go);
#pragma unroll
            for (int k = 0; k < kCombineBatchIn; ++k) {
                const float fm = (hd[k].x == -INFINITY) ? 0.f : exp2f(hd[k].x - mn);
                const float ga = (hd[k].z == -INFINITY) ? 0.f : exp2f(hd[k].z - an);
                s += hd[k].y * fm;
                acc.x += x[k].x * ga;
                acc.y += x[k].y * ga;
                acc.z += x[k].z * ga;
                acc.w += x[k].w * ga;
            }
            m = mn;
            a = an;
        }
        // merge the unit's rows: maxima first, then every row rescales its own piece, then
        // row 0 of the unit adds them up
        if (fl == 0)
            part_ma[row] = make_float2(m, a);
        __syncthreads();
        const int r0 = u * IG;
        float um = -INFINITY, ua = -INFINITY;
        if (active)
            for (int k = 0; k < IG; ++k) {
                const float2 o = part_ma[r0 + k];
                um = fmaxf(um, o.x);
                ua = fmaxf(ua, o.y);
            }
        const float fr = (m == -INFINITY) ? 0.f : exp2f(m - um);
        const float gr = (a == -INFINITY) ? 0.f : exp2f(a - ua);
        part_acc[row][fl] = make_float4(acc.x * gr, acc.y * gr, acc.z * gr, acc.w * gr);
        if (fl == 0)
            part_s[row] = s * fr;
        __syncthreads();
        if (active && ig == 0) {
            float4 t = part_acc[r0][fl];
            float st = part_s[r0];
            for (int k = 1; k < IG; ++k) {
                const float4 o = part_acc[r0 + k][fl];
                t.x += o.x;
                t.y += o.y;
                t.z += o.z;
                t.w += o.w;
                st += part_s[r0 + k];
            }
            const float f = st > 0.f ? exp2f(ua - um) / st : 0.f;
            // segment row hl is query row hl % G of KV head hc * HPC + hl / G; that row is
            // query token hg / Gq, head kvh * Gq + hg % Gq of the [B][nq][Hq] output
            const int kvh = hc * p.HPC + hl / p.G, hg = hl % p.G;
            const int ti = hg / p.Gq;
            const long long orow =
                ((long long)b * p.nq + ti) * p.Hq + (long long)kvh * p.Gq + (hg - ti * p.Gq);
            float *dst = p.out + orow * 128 + q * kCombineQuarter + 4 * fl;
            *reinterpret_cast<float4 *>(dst) = make_float4(t.x * f, t.y * f, t.z * f, t.w * f);
        }
        __syncthreads(); // part_* are reused by the next batch
    }
}

} // namespace q8kv
