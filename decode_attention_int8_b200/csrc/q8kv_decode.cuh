// q8kv_decode.cuh -- the q8-KV single-query decode-attention kernel for sm_100a.
//
// What it computes (Kestrel-LLM walk-through "flash_attn_single_q_q8_neon",
// trdm.cn/news/511694, section 2 parts 1-3): per (sequence b, query head h) quantise q
// to int8 in 32-element blocks, take exact int32 block dot products with every int8 K
// row of the sequence, scale them by the Q block scale, the per-(token, KV head) K scale
// and the softmax scale, fold the scores into an online softmax (running max M, running
// sum S, accumulator rescaled when M rises), accumulate int8 V times weight times the
// per-(token, KV head) V scale, and divide by S once at the end.
//
// How (B200 design, none of it from the pages):
//  * One persistent CTA per SM. The work is the flat list of "tiles" (TT tokens x HPC KV
//    heads of one sequence), ordered sequence-major; CTA i takes a contiguous 1/grid
//    share of it, so load balance does not depend on how ragged the batch is. The list
//    is indexed through a per-sequence prefix sum every CTA builds in shared memory.
//  * Warp 8 is the producer: it resolves block-table entries 32 tiles at a time and
//    streams K and V tiles with TMA (3-D tensor maps, 128-byte swizzle, evict-first L2
//    policy) and the scales with bulk copies into an n-stage ring guarded by mbarriers.
//  * Warps 0-7 consume: each owns (KV head, 16-head slice of its query group, 16-token
//    subtile). QK is an int8 tensor-core MMA (m16n8k32, one MMA per 32-channel quant
//    block, so each MMA result is exactly one int32 block dot). PV is an f16 MMA
//    (m16n8k16) on exact f16 copies of the int8 V codes with the fp32 weights split into
//    hi + lo f16 halves (about 22 significant bits).
//  * The online softmax runs per 16-token subtile in base 2. The denominator S keeps the
//    softmax running max M; the V accumulator keeps its own running max A of
//    (score + log2 V scale), so the weight * V scale that enters the f16 halves is at
//    most 2^15 and the largest one is at least 2^14 (full f16 precision whatever the
//    spread of the V scales). Both are ordinary online maxima: rescale when they rise.
//  * Per-warp states are merged in shared memory. A segment that one CTA covers whole is
//    normalised and written out here; a CTA that covers only part of one leaves its
//    partial (M, S, A, acc) in the workspace, and the first contributor records the
//    segment in a descriptor for the log-sum-exp combine kernel (q8kv_combine.cuh) that
//    runs next on the stream. No CTA ever waits for another.
#pragma once

#include <cuda.h>

#include <cstdint>

#include "q8kv_ptx.cuh"
#include "q8kv_qquant.cuh"

namespace q8kv {

constexpr int kD = 128;             // head_dim handled by this kernel
constexpr int kNB = kD / 32;        // quant blocks per head
constexpr int kConsumerWarps = 8;   // warps 0-7 (two warpgroups)
constexpr int kProducerWarp = 8;    // warp 8 (its warpgroup, warps 8-11, gives registers away)
constexpr int kThreads = 12 * 32;
constexpr int kLaunchRegs = 168;    // per-thread registers at launch (65536 / 384, rounded)
constexpr int kProducerRegs = 56;   // after setmaxnreg.dec (producer warpgroup)
constexpr int kConsumerRegs = 224;  // after setmaxnreg.inc (consumer warpgroups)
static_assert(4 * 32 * kProducerRegs + 8 * 32 * kConsumerRegs <= kThreads * kLaunchRegs,
              "register split exceeds the launch allocation");
constexpr int kSub = 2;             // 16-token subtiles per consumer warp per stage
constexpr int kConsumerThreads = kConsumerWarps * 32;
constexpr int kMaxBoxes = 16;       // TMA boxes per stage
constexpr int kMaxStages = 8;
constexpr unsigned long long kWaitLimitNs = 1000000000ull; // 1 s per pipeline wait
constexpr int kSlotRow = kD + 4;    // per-head partial: kD accumulator floats, M, S, A, pad
constexpr float kVExpLimit = 100.f; // V-scale exponents are clamped to [-100, 100]
constexpr int kDotBias = 0x4B400000;    // bit pattern of 1.5 * 2^23
constexpr float kDotBiasF = 12582912.0f; // 1.5 * 2^23

// Device-side error bits (match Q8KV_DEVERR_* in q8kv.h).
constexpr unsigned kErrSeqLen = 0x1u;
constexpr unsigned kErrBlockTable = 0x2u;
constexpr unsigned kErrTimeout = 0x4u;

__host__ __device__ inline uint32_t align_up(uint32_t x, uint32_t a)
{
    return (x + a - 1) / a * a;
}

// Shared-memory carve-up, computed identically on host and device.
struct SmemLayout {
    uint32_t stage_bytes; // one ring slot: K | V | kscale | vscale
    uint32_t off_k, off_v, off_ks, off_vs; // within a slot
    uint32_t off_full, off_empty, off_mbar, off_mask, off_misc, off_slots, off_ptab, off_cstart,
        off_prefix, off_scratch;
    uint32_t total; // bytes from the 1024-aligned base
};

__host__ __device__ inline SmemLayout make_layout(int TT, int HPC, int n_stages, int B,
                                                  int scratch_floats, int grid)
{
    SmemLayout L;
    const uint32_t kv = (uint32_t)(TT * HPC * kD);
    const uint32_t sc = align_up((uint32_t)(TT * HPC * 4), 128);
    L.off_k = 0;
    L.off_v = kv;
    L.off_ks = 2 * kv;
    L.off_vs = 2 * kv + sc;
    L.stage_bytes = align_up(2 * kv + 2 * sc, 1024);
    uint32_t o = (uint32_t)n_stages * L.stage_bytes;
    L.off_full = o;
    o += 8 * kMaxStages;
    L.off_empty = o;
    o += 8 * kMaxStages;
    L.off_mbar = o;
    o += 8;
    L.off_mask = o;
    o += 4 * kMaxStages;
    L.off_misc = o;
    o += 64;
    L.off_slots = o;
    o += 4 * 32;
    L.off_ptab = o; // producer: physical slot of every box of the next 32 tiles
    o += 4 * 32 * kMaxBoxes;
    L.off_cstart = o;
    o = align_up(o + 4u * (uint32_t)(grid + 1), 16);
    L.off_prefix = o;
    o = align_up(o + 4u * (uint32_t)(B + 1), 16);
    L.off_scratch = o;
    o += 4u * (uint32_t)scratch_floats;
    L.total = o;
    return L;
}

struct DecodeParams {
    float *out;
    const float *q;
    const int32_t *block_table;
    const int32_t *seq_lens;
    const float *kscale;
    const float *vscale;
    float *partials;     // [2 * grid slots] x heads_seg x kSlotRow (kD acc, M, S, A, pad)
    int4 *split_desc;    // [2 * grid] {b, hc, contributors, first slot}; rewritten every call
    unsigned *errors;    // device error word
    int32_t *dbg_dots;   // [B][Hq][dbg_max_len][kNB] (debug instantiation only)
    int dbg_max_len;
    int B, Hq, Hk, G;
    int bs, mbps, num_blocks;
    int HPC, nhc, slices, pairs, subtiles, TT, box_tok, log2_box, n_boxes, n_stages;
    int scale_bulk;      // 1: scales by contiguous bulk copy (HPC == Hk); 0: 2-D tensor map
    int heads_seg;       // query heads per segment (HPC * G)
    int scratch_stride;  // floats per (subtile, pair) merge region
    float scale_log2;    // softmax scale * log2(e)
    SmemLayout lay;
};

__device__ __forceinline__ void consumer_bar()
{
    asm volatile("bar.sync 1, %0;" ::"n"(kConsumerThreads) : "memory");
}

__device__ __forceinline__ float ldcg_f(const float *p)
{
    return __ldcg(p);
}

__device__ __forceinline__ float4 ldcg_f4(const float *p)
{
    return __ldcg(reinterpret_cast<const float4 *>(p));
}

// CTA owning flat tile x: the largest i with cstart[i] <= x, where cstart[i] = i * N / g
// (the table every CTA builds once, so no 64-bit division runs after the prologue).
__device__ __forceinline__ int cta_of_tile(const int *cstart, int g, int x)
{
    int lo = 0, hi = g - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (cstart[mid] <= x)
            lo = mid;
        else
            hi = mid - 1;
    }
    return lo;
}

// Per-sequence tile prefix: prefix[b + 1] = sum over b' <= b of nhc * ceil(L_b' / TT).
__device__ void build_prefix(const DecodeParams &p, int *prefix, volatile int *wsum, int tid,
                             int warp, int lane)
{
    const int cap = p.mbps * p.bs;
    int carry = 0;
    for (int base = 0; base < p.B; base += kThreads) {
        const int b = base + tid;
        int v = 0;
        if (b < p.B) {
            int L = p.seq_lens[b];
            if (L < 0 || L > cap) {
                atomicOr(p.errors, kErrSeqLen);
                L = L < 0 ? 0 : cap;
            }
            v = ((L + p.TT - 1) / p.TT) * p.nhc;
        }
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int t = __shfl_up_sync(kFullMask, v, o);
            if (lane >= o)
                v += t;
        }
        if (lane == 31)
            wsum[warp] = v;
        __syncthreads();
        int off = carry, total = 0;
        for (int w = 0; w < kThreads / 32; ++w) {
            const int ws = wsum[w];
            if (w < warp)
                off += ws;
            total += ws;
        }
        if (b < p.B)
            prefix[b + 1] = off + v;
        carry += total;
        __syncthreads();
    }
    if (tid == 0)
        prefix[0] = 0;
}

__device__ __forceinline__ int clamp_len(int L, int cap)
{
    return L < 0 ? 0 : (L > cap ? cap : L);
}

// ------------------------------------------------------------------ producer warp

__device__ void produce(const DecodeParams &p, const CUtensorMap *tmK, const CUtensorMap *tmV,
                        const CUtensorMap *tmKs, const CUtensorMap *tmVs, uint8_t *smem,
                        const int *prefix, int t0, int t1, int lane)
{
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + p.lay.off_full);
    uint64_t *empty = reinterpret_cast<uint64_t *>(smem + p.lay.off_empty);
    int *mask = reinterpret_cast<int *>(smem + p.lay.off_mask);
    const uint64_t pol = l2_policy_evict_first();
    const int cap = p.mbps * p.bs;
    const uint32_t kv_box = (uint32_t)(p.box_tok * p.HPC * kD);
    const uint32_t sc_box = (uint32_t)(p.box_tok * p.HPC * 4);
    int stage = 0;
    uint32_t phase = 0, issued = 0, issued_par = 0;
    bool aborted = false;

    int *ptab = reinterpret_cast<int *>(smem + p.lay.off_ptab);
    for (int xb = t0; xb < t1 && !aborted; xb += 32) {
        // lane l resolves tile xb + l: its head chunk and the physical slot of every box
        const int x = xb + lane;
        int hc = 0;
        if (x < t1) {
            int lo = 0, hi = p.B - 1; // largest b with prefix[b] <= x
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (prefix[mid] <= x)
                    lo = mid;
                else
                    hi = mid - 1;
            }
            const int b = lo;
            const int pre = prefix[b];
            const int ntb = (prefix[b + 1] - pre) / p.nhc;
            const int local = x - pre;
            hc = local / ntb;
            const int lt = local - hc * ntb;
            const int tok0 = lt * p.TT;
            const int L = clamp_len(__ldg(p.seq_lens + b), cap);
            for (int bx = 0; bx < p.n_boxes; ++bx) {
                const int tk = tok0 + bx * p.box_tok;
                int sl = -1;
                if (tk < L) {
                    const int ph = __ldg(p.block_table + (long long)b * p.mbps + tk / p.bs);
                    if (ph >= 0 && ph < p.num_blocks)
                        sl = ph * p.bs + (tk % p.bs);
                    else
                        atomicOr(p.errors, kErrBlockTable);
                }
                ptab[lane * kMaxBoxes + bx] = sl;
            }
        }
        __syncwarp();
        const int n = (t1 - xb) < 32 ? (t1 - xb) : 32;
        for (int i = 0; i < n; ++i) {
            const int hci = __shfl_sync(kFullMask, hc, i);
            int ok = 1;
            if (lane == 0) {
                if (!mbar_wait(&empty[stage], phase ^ 1u, kWaitLimitNs)) {
                    ok = 0;
                    atomicOr(p.errors, kErrTimeout);
                } else {
                    const int *sl = ptab + i * kMaxBoxes;
                    uint32_t bytes = 0;
                    int loaded = 0;
                    for (int bx = 0; bx < p.n_boxes; ++bx)
                        if (sl[bx] >= 0) {
                            bytes += 2 * (kv_box + sc_box);
                            loaded |= 1 << bx;
                        }
                    // which boxes hold data; published by the release of the arrive below
                    mask[stage] = loaded;
                    mbar_arrive_expect_tx(&full[stage], bytes);
                    uint8_t *sb = smem + (size_t)stage * p.lay.stage_bytes;
                    for (int bx = 0; bx < p.n_boxes; ++bx) {
                        const int slot = sl[bx];
                        if (slot < 0)
                            continue;
                        tma_load_3d(sb + p.lay.off_k + bx * kv_box, tmK, &full[stage], 0, slot,
                                    hci * p.HPC, pol);
                        tma_load_3d(sb + p.lay.off_v + bx * kv_box, tmV, &full[stage], 0, slot,
                                    hci * p.HPC, pol);
                        if (p.scale_bulk) {
                            const long long e0 = (long long)slot * p.Hk;
                            bulk_load(sb + p.lay.off_ks + bx * sc_box, p.kscale + e0, sc_box,
                                      &full[stage], pol);
                            bulk_load(sb + p.lay.off_vs + bx * sc_box, p.vscale + e0, sc_box,
                                      &full[stage], pol);
                        } else {
                            tma_load_2d(sb + p.lay.off_ks + bx * sc_box, tmKs, &full[stage],
                                        hci * p.HPC, slot, pol);
                            tma_load_2d(sb + p.lay.off_vs + bx * sc_box, tmVs, &full[stage],
                                        hci * p.HPC, slot, pol);
                        }
                    }
                    issued |= 1u << stage;
                    issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
                }
            }
            ok = __shfl_sync(kFullMask, ok, 0);
            if (!ok) {
                aborted = true;
                break;
            }
            if (++stage == p.n_stages) {
                stage = 0;
                phase ^= 1u;
            }
        }
        __syncwarp(); // the table is rewritten for the next 32 tiles
    }
    // Every copy this warp issued must have landed before the CTA may exit.
    if (lane == 0) {
        for (int s = 0; s < p.n_stages; ++s)
            if ((issued >> s) & 1u)
                mbar_wait(&full[s], (issued_par >> s) & 1u, kWaitLimitNs);
    }
}

// ------------------------------------------------------------------ consumer warps

template <int NT>
struct WarpState {
    float acc[NT][8][4]; // PV accumulator fragments (columns = heads, rows = channels)
    float M[NT];         // softmax running max (base 2) of this lane's QK row head
    float S[NT];         // this lane's share of the running sum (units 2^-M)
    float A[NT];         // accumulator running max of score + log2(V scale) - 14
    uint32_t qa[kNB][4]; // int8 A fragments of the quantised query heads
    float qs[NT][kNB];   // Q block scales of rows g and g + 8
};

// Quantise this warp's query heads into int8 A fragments. Row g (and g + 8 when NT == 2)
// holds head slice * 16 + g (+ 8). In packed mode (group <= 4) rows g and g + 4 both hold
// head g & 3: the duplicate rows produce the same weights, which feed the low halves of the
// split PV operand (columns 4-7) while rows 0-3 feed the high halves (columns 0-3).
template <int NT>
struct QueryFrag {
    uint32_t qa[kNB][4];
    float qs[NT][kNB];
};

template <int NT, bool kPack>
__device__ __forceinline__ QueryFrag<NT> load_query(const DecodeParams &p, int b, int hc, int kl,
                                                 int slice, int g, int c)
{
    QueryFrag<NT> st;
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        if (r >= NT) {
#pragma unroll
            for (int j = 0; j < kNB; ++j) {
                st.qa[j][1] = 0u;
                st.qa[j][3] = 0u;
            }
            continue;
        }
        const int hg = kPack ? (g & 3) : slice * 16 + r * 8 + g;
        const bool valid = hg < p.G;
        const float *qrow =
            p.q + ((long long)b * p.Hq + (long long)(hc * p.HPC + kl) * p.G + hg) * kD;
        float v[kNB][8];
#pragma unroll
        for (int j = 0; j < kNB; ++j) {
            float4 x0 = make_float4(0.f, 0.f, 0.f, 0.f), x1 = x0;
            if (valid) {
                x0 = __ldg(reinterpret_cast<const float4 *>(qrow + 32 * j + 8 * c));
                x1 = __ldg(reinterpret_cast<const float4 *>(qrow + 32 * j + 8 * c + 4));
            }
            v[j][0] = x0.x;
            v[j][1] = x0.y;
            v[j][2] = x0.z;
            v[j][3] = x0.w;
            v[j][4] = x1.x;
            v[j][5] = x1.y;
            v[j][6] = x1.z;
            v[j][7] = x1.w;
        }
#pragma unroll
        for (int j = 0; j < kNB; ++j) {
            uint32_t lo, hi;
            quantize_block_quad(v[j], lo, hi, st.qs[r][j]);
            // MMA k positions 4c..4c+3 and 16+4c..16+4c+3 carry channels 8c..8c+7 of the
            // block; the K operand uses the same assignment, so each MMA is one block dot.
            st.qa[j][r == 0 ? 0 : 1] = lo;
            st.qa[j][r == 0 ? 2 : 3] = hi;
        }
    }
    return st;
}

template <int NT>
__device__ __forceinline__ void reset_state(WarpState<NT> &st)
{
#pragma unroll
    for (int pv = 0; pv < NT; ++pv) {
        st.M[pv] = -INFINITY;
        st.S[pv] = 0.f;
        st.A[pv] = -INFINITY;
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
            for (int k = 0; k < 4; ++k)
                st.acc[pv][i][k] = 0.f;
    }
}

// Per-thread shared-memory offsets that are the same for every stage. Subtile u of a
// warp covers stage tokens ts * 16 * kSub + 16 * u + [0, 16).
struct ThreadOffsets {
    uint32_t k[kSub][2][kNB]; // K fragment loads (subtile, QK n-tile, quant block)
    uint32_t v[kSub][4];      // V rows 2c, 2c+1, 2c+8, 2c+9 (channel chunk g)
    uint32_t s[kSub][2][2];   // scale of tokens nt*8 + 2c + e
    int tok[kSub][2][2];      // stage-local token index of (u, nt, e)
};

__device__ __forceinline__ ThreadOffsets make_offsets(const DecodeParams &p, int kl, int ts, int g,
                                                      int c)
{
    ThreadOffsets o;
    const int lb = p.log2_box, bt = p.box_tok, H = p.HPC;
    auto row_kv = [&](int tok) { return ((tok >> lb) * H + kl) * bt + (tok & (bt - 1)); };
    auto row_sc = [&](int tok) { return ((tok >> lb) * bt + (tok & (bt - 1))) * H + kl; };
#pragma unroll
    for (int u = 0; u < kSub; ++u) {
        const int t0 = (ts * kSub + u) * 16;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            const int r = row_kv(t0 + nt * 8 + g);
#pragma unroll
            for (int j = 0; j < kNB; ++j)
                o.k[u][nt][j] = p.lay.off_k + r * 128 + ((((2 * j) | (c >> 1)) ^ (r & 7)) << 4) +
                                ((c & 1) << 3);
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int tok = t0 + nt * 8 + 2 * c + e;
                o.tok[u][nt][e] = tok;
                o.s[u][nt][e] = 4 * row_sc(tok);
            }
        }
#pragma unroll
        for (int qv = 0; qv < 4; ++qv) {
            const int t = 2 * c + (qv & 1) + (qv >> 1) * 8;
            const int r = row_kv(t0 + t);
            o.v[u][qv] = p.lay.off_v + r * 128 + ((g ^ (r & 7)) << 4);
        }
    }
    return o;
}

__device__ __forceinline__ uint32_t word_of(const uint4 &v, int i)
{
    return i == 0 ? v.x : (i == 1 ? v.y : (i == 2 ? v.z : v.w));
}

// One stage: kSub 16-token subtiles of one KV head for this warp, folded into the online
// softmax as one block. kMasked: some tokens of the stage are past the sequence end or in a
// block that was not loaded.
template <int NT, bool kPack, bool kDump, bool kMasked>
__device__ __forceinline__ void process_stage(const DecodeParams &p, WarpState<NT> &st,
                                              const ThreadOffsets &o, const uint8_t *sb,
                                              int nvalid, int loaded, int b, int hc, int kl,
                                              int slice, int tok0, int g, int c)
{
    // ---- V rows first: their int8 -> f16 conversion overlaps the softmax chain below
    uint4 R[kSub][4];
#pragma unroll
    for (int u = 0; u < kSub; ++u)
#pragma unroll
        for (int qv = 0; qv < 4; ++qv)
            R[u][qv] = *reinterpret_cast<const uint4 *>(sb + o.v[u][qv]);
    // ---- scores: int8 MMA per quant block, exact int32 block dots. The accumulator
    // starts at the bit pattern of 1.5 * 2^23, so each result read as fp32 is
    // 1.5 * 2^23 + dot exactly (|dot| <= 32 * 127 * 127 < 2^22).
    float s[NT][kSub][2][2];
#pragma unroll
    for (int r = 0; r < NT; ++r)
#pragma unroll
        for (int u = 0; u < kSub; ++u)
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
                s[r][u][nt][0] = s[r][u][nt][1] = 0.f;
#pragma unroll
    for (int u = 0; u < kSub; ++u) {
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
            for (int j = 0; j < kNB; ++j) {
                const uint2 kk = *reinterpret_cast<const uint2 *>(sb + o.k[u][nt][j]);
                int d[4];
                mma_s8_16832_biased(d, st.qa[j][0], NT == 2 ? st.qa[j][1] : 0u, st.qa[j][2],
                                    NT == 2 ? st.qa[j][3] : 0u, kk.x, kk.y);
                if constexpr (kDump) {
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int r = q >> 1, e = q & 1;
                        const int hg = kPack ? g : slice * 16 + r * 8 + g;
                        const bool row_ok = kPack ? (r == 0 && g < 4) : (r < NT);
                        const int tl = o.tok[u][nt][e];
                        if (row_ok && hg < p.G && tl < nvalid &&
                            ((loaded >> (tl >> p.log2_box)) & 1)) {
                            const long long h = (long long)(hc * p.HPC + kl) * p.G + hg;
                            p.dbg_dots[(((long long)b * p.Hq + h) * p.dbg_max_len + tok0 + tl) *
                                           kNB +
                                       j] = d[q] - kDotBias;
                        }
                    }
                }
                s[0][u][nt][0] += (__int_as_float(d[0]) - kDotBiasF) * st.qs[0][j];
                s[0][u][nt][1] += (__int_as_float(d[1]) - kDotBiasF) * st.qs[0][j];
                if constexpr (NT == 2) {
                    s[NT - 1][u][nt][0] += (__int_as_float(d[2]) - kDotBiasF) * st.qs[NT - 1][j];
                    s[NT - 1][u][nt][1] += (__int_as_float(d[3]) - kDotBiasF) * st.qs[NT - 1][j];
                }
            }
        }
    }
    // ---- per-token K and V scales; masking of tokens past the sequence end
    float kss[kSub][2][2], vsv[kSub][2][2], vex[kSub][2][2];
    bool val[kSub][2][2];
#pragma unroll
    for (int u = 0; u < kSub; ++u)
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int tl = o.tok[u][nt][e];
                val[u][nt][e] = !kMasked || (tl < nvalid && ((loaded >> (tl >> p.log2_box)) & 1));
                kss[u][nt][e] =
                    *reinterpret_cast<const float *>(sb + p.lay.off_ks + o.s[u][nt][e]) *
                    p.scale_log2;
                const float vv =
                    *reinterpret_cast<const float *>(sb + p.lay.off_vs + o.s[u][nt][e]);
                vsv[u][nt][e] = val[u][nt][e] ? vv : 0.f;
                // floor(log2 |vs|) from the exponent field, clamped to [-100, 100]
                vex[u][nt][e] = fminf(fmaxf(exponent_as_float(vv), -kVExpLimit), kVExpLimit);
            }
    // ---- online softmax (base 2), blockwise over the stage's tokens. M: running max of the
    // scores (denominator). A: running max of score + log2(vs) - 14 (numerator), so that
    // every weight * vs * 2^(M - A) entering the f16 MMA is below 2^15.
    float alpha_a[NT];
    uint32_t bh[NT][kSub][2], bl[NT][kSub][2];
#pragma unroll
    for (int r = 0; r < NT; ++r) {
        float m = -INFINITY, a = -INFINITY;
#pragma unroll
        for (int u = 0; u < kSub; ++u)
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const float v = val[u][nt][e] ? s[r][u][nt][e] * kss[u][nt][e] : -INFINITY;
                    s[r][u][nt][e] = v;
                    m = fmaxf(m, v);
                    a = fmaxf(a, v + vex[u][nt][e]);
                }
        m = fmaxf(m, __shfl_xor_sync(kFullMask, m, 1));
        a = fmaxf(a, __shfl_xor_sync(kFullMask, a, 1));
        m = fmaxf(m, __shfl_xor_sync(kFullMask, m, 2));
        a = fmaxf(a, __shfl_xor_sync(kFullMask, a, 2));
        const float mn = fmaxf(st.M[r], m);
        const float an = fmaxf(st.A[r], a - 14.f);
        const float ms = (mn == -INFINITY) ? 0.f : mn;
        const float as = (an == -INFINITY) ? 0.f : an;
        const float alpha_s = exp2f(st.M[r] - ms);
        alpha_a[r] = exp2f(st.A[r] - as);
        st.M[r] = mn;
        st.A[r] = an;
        const float cvs = exp2f(ms - as); // 2^(M - A), within [2^-86, 2^114]
        float ws = 0.f;
#pragma unroll
        for (int u = 0; u < kSub; ++u) {
            float pw[2][2];
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const float w = exp2f(s[r][u][nt][e] - ms);
                    ws += w;
                    pw[nt][e] = w * (vsv[u][nt][e] * cvs);
                }
            // weights as split f16 B operands (column n = head g, k = token)
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                const __half2 h = __floats2half2_rn(pw[nt][0], pw[nt][1]);
                const float r0 = pw[nt][0] - __low2float(h), r1 = pw[nt][1] - __high2float(h);
                bh[r][u][nt] = *reinterpret_cast<const uint32_t *>(&h);
                bl[r][u][nt] = pack_f16x2(r0, r1);
            }
        }
        st.S[r] = st.S[r] * alpha_s + ws;
    }
    // ---- rescale factors of the accumulator columns (in packed mode rows 4-7 repeat rows
    // 0-3, so the source lane of column col carries head col & 3 either way)
    float f0[NT], f1[NT];
#pragma unroll
    for (int pv = 0; pv < NT; ++pv) {
        f0[pv] = __shfl_sync(kFullMask, alpha_a[pv], 8 * c);
        f1[pv] = __shfl_sync(kFullMask, alpha_a[pv], 8 * c + 4);
    }
    // ---- PV: rows = channels 16g + 2i (+1), k = tokens, columns = heads (packed mode:
    // columns 0-3 high halves of heads 0-3, columns 4-7 their low halves). The stage's
    // products are summed in a fresh tensor-core accumulator and folded into the running
    // one with one round-to-nearest FFMA (which also applies the rescale factor): the
    // tensor-core accumulation does not round to nearest, so chaining every stage of a
    // long scan through it would let its error grow with the scan length.
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        float d[NT][4];
#pragma unroll
        for (int u = 0; u < kSub; ++u) {
            const uint32_t w0 = word_of(R[u][0], i >> 1), w1 = word_of(R[u][1], i >> 1);
            const uint32_t w2 = word_of(R[u][2], i >> 1), w3 = word_of(R[u][3], i >> 1);
            const uint32_t sl = (i & 1) ? 0x0602u : 0x0400u;
            const uint32_t sh = (i & 1) ? 0x0703u : 0x0501u;
            const uint32_t a0 = s8pair_to_f16x2(prmt(w0, w1, sl));
            const uint32_t a1 = s8pair_to_f16x2(prmt(w0, w1, sh));
            const uint32_t a2 = s8pair_to_f16x2(prmt(w2, w3, sl));
            const uint32_t a3 = s8pair_to_f16x2(prmt(w2, w3, sh));
#pragma unroll
            for (int pv = 0; pv < NT; ++pv) {
                const uint32_t b0 = (kPack && g >= 4) ? bl[pv][u][0] : bh[pv][u][0];
                const uint32_t b1 = (kPack && g >= 4) ? bl[pv][u][1] : bh[pv][u][1];
                if (u == 0)
                    mma_f16_16816_zero_c(d[pv], a0, a1, a2, a3, b0, b1);
                else
                    mma_f16_16816(d[pv], a0, a1, a2, a3, b0, b1);
                if constexpr (!kPack)
                    mma_f16_16816(d[pv], a0, a1, a2, a3, bl[pv][u][0], bl[pv][u][1]);
            }
        }
#pragma unroll
        for (int pv = 0; pv < NT; ++pv) {
            st.acc[pv][i][0] = fmaf(st.acc[pv][i][0], f0[pv], d[pv][0]);
            st.acc[pv][i][1] = fmaf(st.acc[pv][i][1], f1[pv], d[pv][1]);
            st.acc[pv][i][2] = fmaf(st.acc[pv][i][2], f0[pv], d[pv][2]);
            st.acc[pv][i][3] = fmaf(st.acc[pv][i][3], f1[pv], d[pv][3]);
        }
    }
}

// Write the 16 channels 16g..16g+15 of column head (pv, col) scaled by f.
template <int NT>
__device__ __forceinline__ void store_row16(float *dst, const WarpState<NT> &st, int pv, int q,
                                            float f)
{
#pragma unroll
    for (int i = 0; i < 8; i += 2) {
        const float4 v = make_float4(st.acc[pv][i][q] * f, st.acc[pv][i][q + 2] * f,
                                     st.acc[pv][i + 1][q] * f, st.acc[pv][i + 1][q + 2] * f);
        *reinterpret_cast<float4 *>(dst + 2 * i) = v;
    }
}

// End of a segment (all of this CTA's tiles of sequence b, head chunk hc).
template <int NT, bool kPack>
__device__ __forceinline__ void finalize_segment(const DecodeParams &p, WarpState<NT> &st,
                                                 uint8_t *smem, int b,
                                 int hc, int kl, int slice, int pair, int ts, int g, int c,
                                 int ctid, const int *prefix, const int *cstart, int gcta,
                                 int t0, int t1)
{
    // complete this lane's row sums
#pragma unroll
    for (int r = 0; r < NT; ++r) {
        st.S[r] += __shfl_xor_sync(kFullMask, st.S[r], 1);
        st.S[r] += __shfl_xor_sync(kFullMask, st.S[r], 2);
    }

    // merge the token subtiles of each (KV head, slice) pair inside the CTA (the scratch
    // holds accumulator element e of lane l at e * 32 + l: conflict-free bank access)
    if (p.subtiles > 1) {
        float *scr = reinterpret_cast<float *>(smem + p.lay.off_scratch);
        const int lane = g * 4 + c;
        if (ts > 0) {
            float *reg = scr + (size_t)((ts - 1) * p.pairs + pair) * p.scratch_stride;
#pragma unroll
            for (int pv = 0; pv < NT; ++pv)
#pragma unroll
                for (int i = 0; i < 8; ++i)
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        reg[((pv * 8 + i) * 4 + k) * 32 + lane] = st.acc[pv][i][k];
            if (c == 0) {
#pragma unroll
                for (int r = 0; r < NT; ++r) {
                    reg[32 * 32 * NT + r * 8 + g] = st.M[r];
                    reg[32 * 32 * NT + 16 + r * 8 + g] = st.S[r];
                    reg[32 * 32 * NT + 32 + r * 8 + g] = st.A[r];
                }
            }
        }
        consumer_bar();
        if (ts == 0) {
            for (int k = 1; k < p.subtiles; ++k) {
                const float *reg = scr + (size_t)((k - 1) * p.pairs + pair) * p.scratch_stride;
#pragma unroll
                for (int pv = 0; pv < NT; ++pv) {
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        const int col = 2 * c + q;
                        const float am = __shfl_sync(kFullMask, st.A[pv], 4 * col);
                        const float ao = reg[32 * 32 * NT + 32 + pv * 8 + col];
                        const float an = fmaxf(am, ao);
                        const float fa = (am == -INFINITY) ? 0.f : exp2f(am - an);
                        const float fo = (ao == -INFINITY) ? 0.f : exp2f(ao - an);
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            st.acc[pv][i][q] = st.acc[pv][i][q] * fa +
                                               reg[((pv * 8 + i) * 4 + q) * 32 + lane] * fo;
                            st.acc[pv][i][q + 2] =
                                st.acc[pv][i][q + 2] * fa +
                                reg[((pv * 8 + i) * 4 + q + 2) * 32 + lane] * fo;
                        }
                    }
                }
#pragma unroll
                for (int r = 0; r < NT; ++r) {
                    const float mo = reg[32 * 32 * NT + r * 8 + g];
                    const float so = reg[32 * 32 * NT + 16 + r * 8 + g];
                    const float ao = reg[32 * 32 * NT + 32 + r * 8 + g];
                    const float mn = fmaxf(st.M[r], mo);
                    const float fa = (st.M[r] == -INFINITY) ? 0.f : exp2f(st.M[r] - mn);
                    const float fo = (mo == -INFINITY) ? 0.f : exp2f(mo - mn);
                    st.S[r] = st.S[r] * fa + so * fo;
                    st.M[r] = mn;
                    st.A[r] = fmaxf(st.A[r], ao);
                }
            }
        }
        consumer_bar();
    }

    // packed mode: column col + 4 holds the low half of column col's head
    if constexpr (kPack) {
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
            for (int k = 0; k < 4; ++k)
                st.acc[0][i][k] += __shfl_xor_sync(kFullMask, st.acc[0][i][k], 2);
    }
    const bool col_lane = !kPack || c < 2; // lanes whose columns are real heads
    const int pre = prefix[b];
    const int ntb = (prefix[b + 1] - pre) / p.nhc;
    const int seg0 = pre + hc * ntb, seg1 = seg0 + ntb;
    const bool complete = seg0 >= t0 && seg1 <= t1;
    if (complete) {
        if (ts == 0) {
#pragma unroll
            for (int pv = 0; pv < NT; ++pv)
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    const int col = 2 * c + q;
                    const float sc = __shfl_sync(kFullMask, st.S[pv], 4 * col);
                    const float mc = __shfl_sync(kFullMask, st.M[pv], 4 * col);
                    const float ac = __shfl_sync(kFullMask, st.A[pv], 4 * col);
                    const int hg = slice * 16 + pv * 8 + col;
                    if (col_lane && hg < p.G) {
                        const long long h = (long long)(hc * p.HPC + kl) * p.G + hg;
                        float *dst = p.out + ((long long)b * p.Hq + h) * kD + 16 * g;
                        store_row16(dst, st, pv, q, sc > 0.f ? exp2f(ac - mc) / sc : 0.f);
                    }
                }
        }
        return;
    }

    // partial: this CTA's share of the segment goes to its workspace slot (0: the segment
    // this CTA's range starts in, 1: the one it ends in); the first contributor describes
    // the segment for the combine kernel
    const int which = (seg0 <= t0) ? 0 : 1;
    const int H = p.heads_seg;
    if (ts == 0) {
        float *slotp = p.partials + (size_t)(2 * blockIdx.x + which) * H * kSlotRow;
#pragma unroll
        for (int pv = 0; pv < NT; ++pv)
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                const int hg = slice * 16 + pv * 8 + 2 * c + q;
                if (col_lane && hg < p.G)
                    store_row16(slotp + (size_t)(kl * p.G + hg) * kSlotRow + 16 * g, st, pv, q,
                                1.0f);
            }
        if (c == 0) {
#pragma unroll
            for (int r = 0; r < NT; ++r) {
                const int hg = slice * 16 + r * 8 + g;
                if ((!kPack || g < 4) && hg < p.G)
                    *reinterpret_cast<float4 *>(slotp + (size_t)(kl * p.G + hg) * kSlotRow + kD) =
                        make_float4(st.M[r], st.S[r], st.A[r], 0.f);
            }
        }
    }
    if (ctid == 0 && seg0 >= t0) {
        const int last = cta_of_tile(cstart, gcta, seg1 - 1);
        const int slot = 2 * (int)blockIdx.x + which;
        p.split_desc[slot] = make_int4(b, hc, last - (int)blockIdx.x + 1, slot);
    }
}

// The consumer's view of the flat tile list: which sequence / head chunk tile x is.
// Consumers derive it from the prefix sums themselves, so their control flow (and every
// named barrier they take) never depends on data arriving.
struct SegCursor {
    int b, hc, ntb, L, seg0, seg1;
};

__device__ __forceinline__ SegCursor cursor_at(const DecodeParams &p, const int *prefix, int x)
{
    SegCursor cu;
    int lo = 0, hi = p.B - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (prefix[mid] <= x)
            lo = mid;
        else
            hi = mid - 1;
    }
    cu.b = lo;
    const int pre = prefix[lo];
    cu.ntb = (prefix[lo + 1] - pre) / p.nhc;
    cu.hc = (x - pre) / cu.ntb;
    cu.seg0 = pre + cu.hc * cu.ntb;
    cu.seg1 = cu.seg0 + cu.ntb;
    cu.L = clamp_len(__ldg(p.seq_lens + lo), p.mbps * p.bs);
    return cu;
}

template <int NT, bool kPack, bool kDump>
__device__ void consume(const DecodeParams &p, uint8_t *smem, const int *prefix,
                        const int *cstart, int t0, int t1, int gcta, int warp, int lane)
{
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + p.lay.off_full);
    uint64_t *empty = reinterpret_cast<uint64_t *>(smem + p.lay.off_empty);
    const int pair = warp % p.pairs, ts = warp / p.pairs;
    const int kl = pair / p.slices, slice = pair % p.slices;
    const int g = lane >> 2, c = lane & 3;
    const ThreadOffsets o = make_offsets(p, kl, ts, g, c);
    WarpState<NT> st;
    reset_state(st);
#pragma unroll
    for (int j = 0; j < kNB; ++j)
#pragma unroll
        for (int k = 0; k < 4; ++k)
            st.qa[j][k] = 0u;
#pragma unroll
    for (int r = 0; r < NT; ++r)
#pragma unroll
        for (int j = 0; j < kNB; ++j)
            st.qs[r][j] = 0.f;

    bool dead = false; // set when a pipeline wait timed out: skip work, keep the barriers
    int stage = 0;
    uint32_t phase = 0;
    // Outer loop: one segment (this CTA's tiles of one sequence and head chunk) per pass.
    // The inner loop over the segment's tiles holds only wait / compute / release, so the
    // hot code stays small enough for the instruction cache.
    for (int x = t0; x < t1;) {
        const SegCursor cu = cursor_at(p, prefix, x);
        const int x_end = cu.seg1 < t1 ? cu.seg1 : t1;
        {
            const QueryFrag<NT> qf = load_query<NT, kPack>(p, cu.b, cu.hc, kl, slice, g, c);
#pragma unroll
            for (int j = 0; j < kNB; ++j) {
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    st.qa[j][k] = qf.qa[j][k];
#pragma unroll
                for (int r = 0; r < NT; ++r)
                    st.qs[r][j] = qf.qs[r][j];
            }
            reset_state(st);
        }
        for (; x < x_end; ++x) {
            const int tok0 = (x - cu.seg0) * p.TT;
            const int nvalid = min(p.TT, cu.L - tok0);
            if (!dead && !mbar_wait(&full[stage], phase, kWaitLimitNs)) {
                dead = true;
                atomicOr(p.errors, kErrTimeout);
            }
            if (!dead) {
                const int loaded = reinterpret_cast<volatile int *>(smem + p.lay.off_mask)[stage];
                const uint8_t *sb = smem + (size_t)stage * p.lay.stage_bytes;
                process_stage<NT, kPack, kDump, true>(p, st, o, sb, nvalid, loaded, cu.b, cu.hc,
                                                      kl, slice, tok0, g, c);
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(&empty[stage]);
            }
            if (++stage == p.n_stages) {
                stage = 0;
                phase ^= 1u;
            }
        }
        finalize_segment<NT, kPack>(p, st, smem, cu.b, cu.hc, kl, slice, pair, ts, g, c,
                                    warp * 32 + lane, prefix, cstart, gcta, t0, t1);
    }
}

template <int NT, bool kPack, bool kDump>
__global__ void __launch_bounds__(kThreads, 1)
    decode_kernel(const __grid_constant__ DecodeParams p, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmKs,
                  const __grid_constant__ CUtensorMap tmVs)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + p.lay.off_full);
    uint64_t *empty = reinterpret_cast<uint64_t *>(smem + p.lay.off_empty);
    int *prefix = reinterpret_cast<int *>(smem + p.lay.off_prefix);
    volatile int *misc = reinterpret_cast<volatile int *>(smem + p.lay.off_misc);

    if (tid == 0) {
        for (int s = 0; s < p.n_stages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kConsumerWarps);
        }
        mbar_init(reinterpret_cast<uint64_t *>(smem + p.lay.off_mbar), 1);
        fence_mbar_init();
    }
    if (warp == kProducerWarp && lane == 0) {
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
        if (!p.scale_bulk) {
            tma_prefetch_desc(&tmKs);
            tma_prefetch_desc(&tmVs);
        }
    }
    // Everything above touches only shared memory and kernel parameters; from here on the
    // previous kernel on the stream (another call's combine, which reads the workspace, or
    // a producer of the inputs) must be complete.
    grid_dep_wait();
    grid_dep_launch();
    if (tid == 0) { // no split segment recorded yet in this CTA's descriptor slots
        p.split_desc[2 * blockIdx.x] = make_int4(0, 0, 0, 0);
        p.split_desc[2 * blockIdx.x + 1] = make_int4(0, 0, 0, 0);
    }
    build_prefix(p, prefix, misc + 2, tid, warp, lane);
    __syncthreads();

    const int N = prefix[p.B];
    int *cstart = reinterpret_cast<int *>(smem + p.lay.off_cstart);
    // rows of empty sequences are zero
    for (int b = blockIdx.x; b < p.B; b += gridDim.x) {
        if (prefix[b + 1] != prefix[b])
            continue;
        float4 *row = reinterpret_cast<float4 *>(p.out + (long long)b * p.Hq * kD);
        for (int i = tid; i < p.Hq * kD / 4; i += kThreads)
            row[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    const int gcta = N < (int)gridDim.x ? N : (int)gridDim.x;
    {
        const int qn = N / (gcta > 0 ? gcta : 1), rn = N - qn * (gcta > 0 ? gcta : 1);
        for (int i = tid; i <= gcta; i += kThreads)
            cstart[i] = i * qn + (i * rn) / gcta; // == floor(i * N / gcta)
    }
    __syncthreads();
    if ((int)blockIdx.x >= gcta)
        return;
    const int t0 = cstart[blockIdx.x], t1 = cstart[blockIdx.x + 1];
    // Warp specialisation: the producer warpgroup hands most of its registers to the two
    // consumer warpgroups (the sums match the launch allocation, checked by static_assert).
    if (warp >= kConsumerWarps) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kProducerRegs));
        if (warp == kProducerWarp)
            produce(p, &tmK, &tmV, &tmKs, &tmVs, smem, prefix, t0, t1, lane);
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kConsumerRegs));
        consume<NT, kPack, kDump>(p, smem, prefix, cstart, t0, t1, gcta, warp, lane);
    }
}

} // namespace q8kv
