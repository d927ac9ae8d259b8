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
// stride over the unit's inputs, so short and long input lists both keep loads in flight.
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
};

__device__ __forceinline__ float group_max(float v, int width)
{
    for (int o = (width < 32 ? width : 32) >> 1; o >= 1; o >>= 1)
        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

__device__ __forceinline__ float group_sum(float v, int width)
{
    for (int o = (width < 32 ? width : 32) >> 1; o >= 1; o >>= 1)
        v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__global__ void __launch_bounds__(kCombineThreads)
    combine_kernel(const __grid_constant__ CombineParams p)
{
    __shared__ int list[kCombineMaxDesc];
    __shared__ int wcount[kCombineThreads / 32];
    __shared__ float red[3][kCombineThreads / 32];
    __shared__ float4 part[32][8];

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // the decode kernel's partials and descriptors are complete and visible after this
    grid_dep_wait();
    grid_dep_launch();

    // compact list of the descriptors that start a split segment (same order in every CTA)
    int nvalid = 0;
    for (int base = 0; base < p.n_desc; base += kCombineThreads) {
        const int i = base + tid;
        const bool v = i < p.n_desc && __ldcg(&p.desc[i].z) > 0;
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
            list[off + __popc(m & ((1u << lane) - 1u))] = i;
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
        const int IG = 32 / upow;        // input-group rows per unit
        const int width = IG * 8;        // threads per unit (contiguous, aligned)
        const int u = row / IG, ig = row % IG;
        const bool active = u < U;
        int b = 0, hc = 0, n = 0, first = 0, hl = 0, q = 0;
        if (active) {
            const long long unit = u0 + u;
            const int d = (int)(unit / per_seg);
            const int rem = (int)(unit - (long long)d * per_seg);
            hl = rem / (128 / kCombineQuarter);
            q = rem % (128 / kCombineQuarter);
            const int4 ds = __ldcg(&p.desc[list[d]]);
            b = ds.x;
            hc = ds.y;
            n = ds.z;
            first = ds.w;
        }
        auto slot_of = [&](int i) { return i == 0 ? first : 2 * ((first >> 1) + i); };
        auto header = [&](int i) {
            return __ldcg(reinterpret_cast<const float4 *>(
                p.partials + ((size_t)slot_of(i) * H + hl) * kCombineSlotRow + 128));
        };
        // maxima of M and A over the unit's inputs
        float mx = -INFINITY, ax = -INFINITY;
        for (int i = ig * 8 + fl; i < n; i += width) {
            const float4 h = header(i);
            mx = fmaxf(mx, h.x);
            ax = fmaxf(ax, h.z);
        }
        mx = group_max(mx, width);
        ax = group_max(ax, width);
        if (width > 32) { // all threads agree on width, so the barriers are uniform
            if (lane == 0) {
                red[0][warp] = mx;
                red[1][warp] = ax;
            }
            __syncthreads();
            const int w0 = (u * width) >> 5, nw = width >> 5;
            mx = -INFINITY;
            ax = -INFINITY;
            for (int w = 0; w < nw && active; ++w) {
                mx = fmaxf(mx, red[0][w0 + w]);
                ax = fmaxf(ax, red[1][w0 + w]);
            }
            __syncthreads();
        }
        // S = sum_i S_i 2^(M_i - mx)
        float ssum = 0.f;
        for (int i = ig * 8 + fl; i < n; i += width) {
            const float4 h = header(i);
            if (h.x != -INFINITY)
                ssum += h.y * exp2f(h.x - mx);
        }
        ssum = group_sum(ssum, width);
        if (width > 32) {
            if (lane == 0)
                red[2][warp] = ssum;
            __syncthreads();
            const int w0 = (u * width) >> 5, nw = width >> 5;
            ssum = 0.f;
            for (int w = 0; w < nw && active; ++w)
                ssum += red[2][w0 + w];
        }
        // accumulators: row ig of the unit takes inputs ig, ig + IG, ...
        float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int i = ig; i < n; i += IG) {
            const size_t r = ((size_t)slot_of(i) * H + hl) * kCombineSlotRow;
            const float ai = __ldcg(p.partials + r + 130);
            const float f = (ai == -INFINITY) ? 0.f : exp2f(ai - ax);
            const float4 x = __ldcg(reinterpret_cast<const float4 *>(
                p.partials + r + q * kCombineQuarter + 4 * fl));
            a.x += f * x.x;
            a.y += f * x.y;
            a.z += f * x.z;
            a.w += f * x.w;
        }
        part[row][fl] = a;
        __syncthreads();
        if (active && ig == 0) {
            for (int k = 1; k < IG; ++k) {
                const float4 o = part[row + k][fl];
                a.x += o.x;
                a.y += o.y;
                a.z += o.z;
                a.w += o.w;
            }
            const float f = ssum > 0.f ? exp2f(ax - mx) / ssum : 0.f;
            float *dst = p.out + ((long long)b * p.Hq + (long long)hc * H + hl) * 128 +
                         q * kCombineQuarter + 4 * fl;
            *reinterpret_cast<float4 *>(dst) = make_float4(a.x * f, a.y * f, a.z * f, a.w * f);
        }
        __syncthreads(); // part[] is reused by the next batch
    }
}

} // namespace q8kv
