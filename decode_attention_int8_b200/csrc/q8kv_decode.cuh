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
//    block, so each MMA result is exactly one int32 block dot). PV is an int8 x u8
//    tensor-core MMA too: V^T straight from the swizzled tile through ldmatrix .trans, and
//    the weights as exact 23-bit integers split into byte planes (one n-tile each).
//  * The online softmax runs per stage in base 2. The denominator S keeps the softmax
//    running max M; the V accumulator keeps its own running max A of
//    (score + log2 V scale), so the integer weight w * vs * 2^(M - A + 8) is below 2^23
//    and the largest one of a stage is at least 2^22 (22 significant bits whatever the
//    spread of the V scales). Both are ordinary online maxima: rescale when they rise.
//  * Per-warp states are merged in shared memory. A segment that one CTA covers whole is
//    normalised and written out here; a CTA that covers only part of one leaves its
//    partial (M, S, A, acc) in the workspace for the log-sum-exp combine kernel
//    (q8kv_combine.cuh) that runs next on the stream and recomputes the same work split to
//    find the split segments. No CTA ever waits for another.
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
// Per-thread registers after setmaxnreg: the producer warpgroup gives registers to the two
// consumer warpgroups. One 8-row query tile (NT == 1) fits in 200 consumer registers with
// 96 left to the producer (no spills); the packed path's int32 PV accumulators and two
// query tiles take 224 (with 216 the packed path spilled 2.5x as much and ran 0.35 us
// slower on the 16 x 4096-token workload).
template <int NT, bool kPack>
struct RegSplit {
    static constexpr int producer = kPack ? 56 : (NT == 1 ? 96 : 56);
    static constexpr int consumer = kPack ? 224 : (NT == 1 ? 200 : 224);
    static_assert(4 * 32 * producer + 8 * 32 * consumer <= kThreads * kLaunchRegs,
                  "register split exceeds the launch allocation");
};
constexpr int kSub = 2;             // 16-token subtiles per consumer warp per stage
constexpr int kConsumerThreads = kConsumerWarps * 32;
constexpr int kMaxBoxes = 16;       // TMA boxes per stage
constexpr int kMaxStages = 8;
constexpr unsigned long long kWaitLimitNs = 1000000000ull; // 1 s per pipeline wait
constexpr int kSlotRow = kD + 4;    // per-head partial: kD accumulator floats, M, S, A, pad
// Work split: a segment that starts in the middle of a CTA's range costs that CTA about
// four to five tiles' time (the finished segment's accumulators are folded, reduced and
// written and the next query is set up, by code that runs once and is fetched cold while
// the K/V stream loads the memory system; per-CTA timestamps on the 16 x 4096-token
// workload put the CTAs that switch segments 2-3 us behind the others when charged three
// tiles). The split therefore charges every segment start kSegPenaltyTiles extra tiles,
// when the batch is small enough to keep the count of sequences with tokens in shared
// memory and every CTA's share is at least twice that (so that no share fits inside one
// segment's charge, which would leave a CTA without tiles in the middle of a segment).
constexpr int kSegPenaltyTiles = 5;
constexpr int kPenaltyMaxB = 2048;
constexpr int kDotBias = 0x4B400000;    // bit pattern of 1.5 * 2^23
constexpr float kDotBiasF = 12582912.0f; // 1.5 * 2^23

// Device-side error bits (match Q8KV_DEVERR_* in q8kv.h).
constexpr unsigned kErrSeqLen = 0x1u;
constexpr unsigned kErrBlockTable = 0x2u;
constexpr unsigned kErrTimeout = 0x4u;

constexpr int kPscanLen = 40; // >= 33 ints: prefix[0..32] of a batch of up to 32 sequences

__host__ __device__ inline uint32_t align_up(uint32_t x, uint32_t a)
{
    return (x + a - 1) / a * a;
}

// Shared-memory carve-up, computed identically on host and device.
struct SmemLayout {
    uint32_t stage_bytes; // one ring slot: K | V | kscale | vscale
    uint32_t off_k, off_v, off_ks, off_vs; // within a slot
    uint32_t sc_gap;      // bytes from a stage's K scales to its V scales (TT * sc_heads * 4)
    uint32_t off_full, off_empty, off_mask, off_misc, off_pscan, off_ptab, off_cstart,
        off_prefix, off_scratch;
    uint32_t off_nseq;  // prefix count of sequences with tokens (B <= kPenaltyMaxB), else 0
    uint32_t off_qbuf;  // quantised query of a CTA's second segment (0 bytes when it did not fit)
    uint32_t qbuf_rows; // query rows per (KV head, slice) pair kept there; 0 = no buffer
    uint32_t total;     // bytes from the 1024-aligned base
};

__host__ __device__ inline SmemLayout make_layout(int TT, int HPC, int sc_heads, int n_stages,
                                                  int B, int scratch_floats, int grid)
{
    SmemLayout L;
    const uint32_t kv = (uint32_t)(TT * HPC * kD);
    L.sc_gap = align_up((uint32_t)(TT * sc_heads * 4), 128);
    L.off_k = 0;
    L.off_v = kv;
    L.off_ks = 2 * kv;
    L.off_vs = 2 * kv + L.sc_gap;
    L.stage_bytes = align_up(2 * kv + 2 * L.sc_gap, 1024);
    uint32_t o = (uint32_t)n_stages * L.stage_bytes;
    L.off_full = o;
    o += 8 * kMaxStages;
    L.off_empty = o;
    o += 8 * kMaxStages;
    L.off_mask = o;
    o += 4 * kMaxStages;
    L.off_misc = o; // 8-byte aligned: the prefix scan's per-warp 64-bit sums
    o += 128;
    L.off_pscan = o; // producer's own copy of the tile and sequence prefixes (B <= 32)
    o += 4 * 2 * kPscanLen;
    L.off_ptab = o; // producer: physical slot of every box of the next 32 tiles
    o += 4 * 32 * kMaxBoxes;
    L.off_cstart = o;
    o = align_up(o + 4u * (uint32_t)(grid + 1), 16);
    L.off_prefix = o;
    o = align_up(o + 4u * (uint32_t)(B + 1), 16);
    L.off_scratch = o;
    o += 4u * (uint32_t)scratch_floats;
    L.off_nseq = 0;
    if (B <= kPenaltyMaxB) {
        L.off_nseq = align_up(o, 16);
        o = L.off_nseq + 4u * (uint32_t)(B + 1);
    }
    L.off_qbuf = align_up(o, 16);
    L.qbuf_rows = 0;
    L.total = o;
    return L;
}

// Bytes per query row in the second-segment buffer: 32 code words (lane-fragment order) and
// the 4 block scales.
constexpr uint32_t kQRowBytes = 32 * 4 + kNB * 4;

struct DecodeParams {
    float *out;
    const float *q;
    const int32_t *block_table;
    const int32_t *seq_lens;
    const float *kscale;
    const float *vscale;
    float *partials;     // [2 * grid slots] x heads_seg x kSlotRow (kD acc, M, S, A, pad)
    unsigned *errors;    // device error word
    int32_t *dbg_dots;   // [B][Hq][dbg_max_len][kNB] (debug instantiation only)
    int dbg_max_len;
    int B, Hq, Hk, G;    // G: query rows per KV head = nq * Gq (the tiling's group)
    int nq, Gq;          // query tokens per sequence; query heads per KV head
    int bs, mbps, num_blocks;
    int HPC, nhc, slices, pairs, subtiles, TT, box_tok, log2_box, n_boxes, n_stages;
    int scale_bulk;      // 1: scales by contiguous bulk copy (HPC == Hk); 0: 2-D tensor map
    int sc_heads;        // KV heads per scale box: HPC, or 4 when a tile holds fewer heads
                         // (a box row must be 16 bytes); the tile's heads sit at column
                         // (hc * HPC) % sc_heads of it
    int heads_seg;       // query heads per segment (HPC * G)
    int scratch_stride;  // floats per (subtile, pair) merge region
    float scale_log2;    // softmax scale * log2(e)
    // Pipeline fault injection (the wait time-out test; -1 = off): the producer of CTA
    // stall_cta never arrives on, nor loads into, the stage of its second tile (its first
    // when it has only one), and that CTA's waits give up after stall_limit_ns.
    int stall_cta;
    unsigned long long stall_limit_ns;
    SmemLayout lay;
};

// Wait limit of this CTA's pipeline waits.
__device__ __forceinline__ unsigned long long wait_limit(const DecodeParams &p)
{
    return (int)blockIdx.x == p.stall_cta ? p.stall_limit_ns : kWaitLimitNs;
}

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

// Row of q / out that query row hg of KV head kvh of sequence b maps to. The nq query
// tokens of a sequence share its KV tiles, so a KV head's rows are its Gq query heads for
// each of the nq tokens: row hg is token hg / Gq, head kvh * Gq + hg % Gq, and q, out are
// [B][nq][Hq][128]. With one token per sequence this is b * Hq + kvh * Gq + hg.
__device__ __forceinline__ long long q_row(const DecodeParams &p, int b, int kvh, int hg)
{
    const int i = hg / p.Gq, gq = hg - i * p.Gq;
    return ((long long)b * p.nq + i) * p.Hq + (long long)kvh * p.Gq + gq;
}

// CTA owning flat tile x: the largest i with cstart[i] <= x, where cstart[i] = i * N / g
// (the table every CTA builds once, so no 64-bit division runs after the prologue).
__device__ __forceinline__ int cta_of_tile(const int *cstart, int g, int x)
{
    int lo = 0, hi = g - 1;
#pragma unroll 1
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (cstart[mid] <= x)
            lo = mid;
        else
            hi = mid - 1;
    }
    return lo;
}

// Per-sequence prefixes of (tiles, has tokens), packed in 64 bits for one scan:
// prefix[b + 1] = sum over b' <= b of nhc * ceil(L_b' / TT); nseq[b + 1] (when nseq is
// given) = number of sequences b' <= b with L_b' > 0.
__device__ __forceinline__ unsigned long long prefix_item(const DecodeParams &p, int b)
{
    const int cap = p.mbps * p.bs;
    int L = __ldcg(p.seq_lens + b);
    if (L < 0 || L > cap) {
        atomicOr(p.errors, kErrSeqLen);
        L = L < 0 ? 0 : cap;
    }
    return ((unsigned long long)(((L + p.TT - 1) / p.TT) * p.nhc) << 32) | (L > 0 ? 1u : 0u);
}

// The prefixes of a batch of at most 32 sequences, by one warp (no block-wide step).
__device__ void scan_one_warp(const DecodeParams &p, int *prefix, int *nseq, int lane)
{
    unsigned long long v = lane < p.B ? prefix_item(p, lane) : 0ull;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const unsigned long long t = __shfl_up_sync(kFullMask, v, o);
        if (lane >= o)
            v += t;
    }
    if (lane < p.B) {
        prefix[lane + 1] = (int)(v >> 32);
        if (nseq)
            nseq[lane + 1] = (int)(v & 0xffffffffu);
    }
    if (lane == 0) {
        prefix[0] = 0;
        if (nseq)
            nseq[0] = 0;
    }
}

// The prefixes of any batch, by the consumer warps (ctid < kConsumerThreads); batches up
// to 32 take one warp. The caller synchronises the consumers afterwards.
__device__ void build_prefix(const DecodeParams &p, int *prefix, int *nseq,
                             volatile unsigned long long *wsum, int ctid, int warp, int lane)
{
    if (p.B <= 32) {
        if (warp == 0)
            scan_one_warp(p, prefix, nseq, lane);
        return;
    }
    unsigned long long carry = 0;
#pragma unroll 1
    for (int base = 0; base < p.B; base += kConsumerThreads) {
        const int b = base + ctid;
        unsigned long long v = b < p.B ? prefix_item(p, b) : 0ull;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const unsigned long long t = __shfl_up_sync(kFullMask, v, o);
            if (lane >= o)
                v += t;
        }
        if (lane == 31)
            wsum[warp] = v;
        consumer_bar();
        unsigned long long off = carry, total = 0;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) {
            const unsigned long long ws = wsum[w];
            if (w < warp)
                off += ws;
            total += ws;
        }
        if (b < p.B) {
            prefix[b + 1] = (int)((off + v) >> 32);
            if (nseq)
                nseq[b + 1] = (int)((off + v) & 0xffffffffu);
        }
        carry += total;
        consumer_bar();
    }
    if (ctid == 0) {
        prefix[0] = 0;
        if (nseq)
            nseq[0] = 0;
    }
}

// First tile of CTA i (of g) in the work split. Plain split: floor(i * N / g). Penalised
// split (pseg > 0): the virtual list puts pseg = P * nhc units before every sequence with
// tokens (P before each of its nhc segments); CTA i starts at virtual unit
// floor(i * V / g) and takes the tile it lands on, or the segment's first tile when it
// lands in the segment's penalty. All quantities fit 32 bits (V < 2^31 is checked on the
// host side through the tile count).
__device__ int cta_start(const DecodeParams &p, const int *prefix, const int *nseq, int pseg,
                         int V, int g, int i)
{
    const int N = prefix[p.B];
    if (i >= g)
        return N;
    const int qv = V / g, rv = V - qv * g;
    const int vi = i * qv + (i * rv) / g; // floor(i * V / g) without 64-bit division
    if (pseg == 0)
        return vi;
    const int P = pseg / p.nhc;
    int lo = 0, hi = p.B - 1; // largest b with vprefix(b) <= vi
#pragma unroll 1
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (prefix[mid] + pseg * nseq[mid] <= vi)
            lo = mid;
        else
            hi = mid - 1;
    }
    const int ntb = (prefix[lo + 1] - prefix[lo]) / p.nhc;
    if (ntb == 0)
        return prefix[lo];
    const int off = vi - (prefix[lo] + pseg * nseq[lo]);
    const int hc = off / (ntb + P);
    const int r = off - hc * (ntb + P);
    const int x = prefix[lo] + (hc < p.nhc ? hc * ntb + (r > P ? r - P : 0) : p.nhc * ntb);
    return x < N ? x : N;
}

// Work split of the flat tile list (see kSegPenaltyTiles): penalised when the sequence
// counts are at hand and every CTA's share is at least 2 penalties, so that no CTA's share
// can fall inside one segment's penalty (an empty CTA in the middle of a split segment would
// break the contributor numbering). The producer and the consumers compute it separately
// from the same prefixes, so they agree.
struct Split {
    int N;    // tiles
    int gcta; // CTAs with tiles
    int pseg; // penalty units before each sequence with tokens (0: plain split)
    int V;    // units of the virtual list
};

__device__ __forceinline__ Split split_of(const DecodeParams &p, const int *prefix,
                                          const int *nseq, int grid)
{
    Split sp;
    sp.N = prefix[p.B];
    sp.gcta = sp.N < grid ? sp.N : grid;
    const int nseg_units = nseq ? kSegPenaltyTiles * p.nhc * nseq[p.B] : 0;
    const bool pen = nseq && sp.gcta > 0 && (sp.N + nseg_units) / sp.gcta >= 2 * kSegPenaltyTiles;
    sp.pseg = pen ? kSegPenaltyTiles * p.nhc : 0;
    sp.V = sp.N + (pen ? nseg_units : 0);
    return sp;
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
    // Every loop here stays rolled: the producer issues a handful of instructions per stage,
    // and its code must not crowd the consumers' out of the instruction cache.
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + p.lay.off_full);
    uint64_t *empty = reinterpret_cast<uint64_t *>(smem + p.lay.off_empty);
    int *mask = reinterpret_cast<int *>(smem + p.lay.off_mask);
    const uint64_t pol = l2_policy_evict_first();
    const int cap = p.mbps * p.bs;
    const uint32_t kv_box = (uint32_t)(p.box_tok * p.HPC * kD);
    const uint32_t sc_box = (uint32_t)(p.box_tok * p.sc_heads * 4);
    int stage = 0;
    uint32_t phase = 0, issued = 0, issued_par = 0;
    bool aborted = false;
    const unsigned long long limit = wait_limit(p);
    // fault injection: the tile whose stage is never filled (-1: none)
    const int x_stall = (int)blockIdx.x == p.stall_cta ? (t1 - t0 > 1 ? t0 + 1 : t0) : -1;

    int *ptab = reinterpret_cast<int *>(smem + p.lay.off_ptab);
#pragma unroll 1
    for (int xb = t0; xb < t1 && !aborted; xb += 32) {
        // lane l resolves tile xb + l: its head chunk and the physical slot of every box
        const int x = xb + lane;
        int hc = 0;
        if (x < t1) {
            int lo = 0, hi = p.B - 1; // largest b with prefix[b] <= x
#pragma unroll 1
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
            const int32_t *bt_row = p.block_table + (long long)b * p.mbps;
            // the tile's first block-table entry is loaded together with the sequence length
            // (one round trip instead of two: tok0 < L <= mbps * bs, so it is in the row)
            const int ph0 = __ldg(bt_row + tok0 / p.bs);
            const int L = clamp_len(__ldg(p.seq_lens + b), cap);
#pragma unroll 1
            for (int bx = 0; bx < p.n_boxes; ++bx) {
                const int tk = tok0 + bx * p.box_tok;
                int sl = -1;
                if (tk < L) {
                    const int ph = bx == 0 ? ph0 : __ldg(bt_row + tk / p.bs);
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
#pragma unroll 1
        for (int i = 0; i < n; ++i) {
            const int hci = __shfl_sync(kFullMask, hc, i);
            int ok = 1;
            if (lane == 0) {
                if (!mbar_wait(&empty[stage], phase ^ 1u, limit)) {
                    ok = 0;
                    atomicOr(p.errors, kErrTimeout);
                } else if (xb + i == x_stall) {
                    // injected fault: no arrive and no copies, so this stage's phase never
                    // completes (nothing is in flight for it)
                } else {
                    const int *sl = ptab + i * kMaxBoxes;
                    uint32_t bytes = 0;
                    int loaded = 0;
#pragma unroll 1
                    for (int bx = 0; bx < p.n_boxes; ++bx)
                        if (sl[bx] >= 0) {
                            bytes += 2 * (kv_box + sc_box);
                            loaded |= 1 << bx;
                        }
                    // which boxes hold data; published by the release of the arrive below
                    mask[stage] = loaded;
                    mbar_arrive_expect_tx(&full[stage], bytes);
                    uint8_t *sb = smem + (size_t)stage * p.lay.stage_bytes;
#pragma unroll 1
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
                            const int h0 = (hci * p.HPC / p.sc_heads) * p.sc_heads;
                            tma_load_2d(sb + p.lay.off_ks + bx * sc_box, tmKs, &full[stage], h0,
                                        slot, pol);
                            tma_load_2d(sb + p.lay.off_vs + bx * sc_box, tmVs, &full[stage], h0,
                                        slot, pol);
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
#pragma unroll 1
        for (int s = 0; s < p.n_stages; ++s)
            if ((issued >> s) & 1u)
                mbar_wait(&full[s], (issued_par >> s) & 1u, limit);
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
        const float *qrow = p.q + (valid ? q_row(p, b, hc * p.HPC + kl, hg) : 0) * kD;
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

// The second-segment query buffer holds, per (KV head, slice) pair, the quantised rows of
// this warp's query tile in lane-fragment order: row r, word (j * 4 + c) * 2 + half is the
// code word that lane (g = row, c) puts into qa[j][half ? 2 : 0] (or [3] / [1] for the rows
// 8-15 of a two-tile warp), followed by the row's 4 block scales.
template <int NT, bool kPack>
__device__ __forceinline__ void store_query(uint32_t buf, const QueryFrag<NT> &qf, int g, int c)
{
#pragma unroll
    for (int r = 0; r < NT; ++r) {
        if (kPack && g >= 4)
            continue; // rows 4-7 repeat rows 0-3
        const uint32_t row = buf + (uint32_t)(r * 8 + g) * kQRowBytes;
#pragma unroll
        for (int j = 0; j < kNB; ++j) {
            sts64(row + ((j * 4 + c) * 2) * 4, qf.qa[j][r == 0 ? 0 : 1], qf.qa[j][r == 0 ? 2 : 3]);
            if (c == 0)
                sts_f32(row + 128 + 4 * j, qf.qs[r][j]);
        }
    }
}

template <int NT, bool kPack>
__device__ __forceinline__ QueryFrag<NT> load_query_smem(uint32_t buf, int g, int c)
{
    QueryFrag<NT> qf;
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        if (r >= NT) {
#pragma unroll
            for (int j = 0; j < kNB; ++j) {
                qf.qa[j][1] = 0u;
                qf.qa[j][3] = 0u;
            }
            continue;
        }
        const uint32_t row = buf + (uint32_t)(r * 8 + (kPack ? (g & 3) : g)) * kQRowBytes;
#pragma unroll
        for (int j = 0; j < kNB; ++j) {
            const uint2 w = lds64(row + ((j * 4 + c) * 2) * 4);
            qf.qa[j][r == 0 ? 0 : 1] = w.x;
            qf.qa[j][r == 0 ? 2 : 3] = w.y;
            qf.qs[r][j] = lds_f32(row + 128 + 4 * j);
        }
    }
    return qf;
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

// Per-thread shared-memory byte offsets within a stage (the stage's shared address is added
// once per stage; every fragment load then uses one register plus an immediate). Subtile u
// of a warp covers stage tokens ts * 16 * kSub + 16 * u + [0, 16), which lie in one TMA box
// (boxes hold at least 16 tokens), so the second 8-token half of a subtile is 8 rows
// (1024 bytes) further on and has the same 128-byte swizzle phase.
struct ThreadOffsets {
    uint32_t k[kSub][kNB]; // K fragment (subtile u, quant block j) of tokens 0-7; 8-15: +1024
    uint32_t s[kSub][2][2]; // K scale of token (u, nt, e) at column kl (add the segment's
                            // column offset); its V scale is sc_gap further
};

__device__ __forceinline__ ThreadOffsets make_offsets(const DecodeParams &p, int kl, int ts, int g,
                                                      int c)
{
    ThreadOffsets o;
    const int lb = p.log2_box, bt = p.box_tok, H = p.HPC;
    auto row_kv = [&](int tok) { return ((tok >> lb) * H + kl) * bt + (tok & (bt - 1)); };
#pragma unroll
    for (int u = 0; u < kSub; ++u) {
        const int t0 = (ts * kSub + u) * 16;
        const int rk = row_kv(t0 + g); // row & 7 == g
#pragma unroll
        for (int j = 0; j < kNB; ++j)
            o.k[u][j] = p.lay.off_k + rk * 128 + ((((2 * j) | (c >> 1)) ^ g) << 4) +
                        ((c & 1) << 3);
        // scales sit token-major ([token][head]) in stage token order
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e)
                o.s[u][nt][e] = p.lay.off_ks + 4 * ((t0 + nt * 8 + 2 * c + e) * p.sc_heads + kl);
    }
    return o;
}

// ------------------------------------------------------------------ packed path (group <= 4)
//
// With at most 4 query heads per KV head, rows 4-7 of the QK tile repeat rows 0-3. The
// packed path uses the repeat to halve the softmax work: lanes of rows 0-3 ("lower" lanes)
// take the first 16 tokens of the warp's 32, lanes of rows 4-7 the last 16, and the row
// reductions add one xor-16 step. PV then runs on the int8 tensor cores:
//  * A = V^T straight from the TMA-swizzled tile through ldmatrix .trans (no conversion),
//    rows = channels 16m + g (and + 8), k = tokens in the order tau(k) below;
//  * B = the exact integer P = round(w * vs * 2^(M - A) * 2^8) < 2^23 (an FFMA against
//    2^23 leaves it in the low mantissa bits) split into its three bytes: n-tile 0 holds
//    byte 0 of heads 0-3 in columns 0-3 and byte 1 in columns 4-7, n-tile 1 byte 2;
//  * the int32 accumulators run over up to 4 stages (128 tokens: |sum| < 2^22, so the
//    biased fp32 view stays exact) and are folded into the fp32 accumulator when that limit
//    is reached, when A rises, and at the end of a segment.
// k -> token within a 16-token subtile: k = 4c + i holds token 2c + (i & 1) + 8 (i >> 1),
// i.e. the tokens whose scores lane (g, c) holds after the QK MMAs.
constexpr int kPackFoldEvery = 4;
constexpr float kTwo23 = 8388608.0f;

struct PackedOffsets {
    uint32_t k[kSub][kNB]; // K fragments, as ThreadOffsets::k
    uint32_t s[2][2];      // K scale of this lane's kept token (nt, e); V scale sc_gap on
    uint32_t v;            // ldmatrix row address of this lane; XOR (16 m) selects chunk m
};

__device__ __forceinline__ PackedOffsets make_packed_offsets(const DecodeParams &p, int kl,
                                                             int ts, int g, int c, int lane)
{
    PackedOffsets o;
    const int lb = p.log2_box, bt = p.box_tok, H = p.HPC;
    auto row_kv = [&](int tok) { return ((tok >> lb) * H + kl) * bt + (tok & (bt - 1)); };
#pragma unroll
    for (int u = 0; u < kSub; ++u) {
        const int rk = row_kv((ts * kSub + u) * 16 + g);
#pragma unroll
        for (int j = 0; j < kNB; ++j)
            o.k[u][j] = p.lay.off_k + rk * 128 + ((((2 * j) | (c >> 1)) ^ g) << 4) +
                        ((c & 1) << 3);
    }
    const int uk = g >> 2; // subtile whose tokens this lane keeps
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e)
            o.s[nt][e] =
                p.lay.off_ks +
                4 * (((ts * kSub + uk) * 16 + nt * 8 + 2 * c + e) * p.sc_heads + kl);
    // ldmatrix: lanes 0-15 give the rows of matrix 0 (subtile 0), lanes 16-31 of matrix 1
    const int kk = lane & 15;
    const int tau = 2 * (kk >> 2) + (kk & 1) + 8 * ((kk >> 1) & 1);
    const int tok = (ts * kSub + (lane >> 4)) * 16 + tau;
    o.v = p.lay.off_v + row_kv(tok) * 128 + ((tok & 7) << 4);
    return o;
}

struct PackedAcc {
    int D[8][2][4]; // int32 PV accumulators (m-tile, n-tile), biased by 1.5 * 2^23
    int n;          // stages accumulated since the last fold
};

// acc = (acc + D) * f per column: D's digits recombined (k0, k1: weights of n-tiles 0 and 1
// in this lane's columns), f = 2^(A_old - A_new) of the column's head.
template <int NT>
__device__ __forceinline__ void packed_fold(WarpState<NT> &st, const PackedAcc &pa, float k0,
                                            float k1, float f0, float f1)
{
    const float kb = -kDotBiasF * (k0 + k1);
#pragma unroll
    for (int m = 0; m < 8; ++m)
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float v = fmaf(__int_as_float(pa.D[m][0][k]), k0,
                                 fmaf(__int_as_float(pa.D[m][1][k]), k1, kb));
            st.acc[0][m][k] = (st.acc[0][m][k] + v) * ((k & 1) ? f1 : f0);
        }
}

template <int NT>
__device__ __forceinline__ void packed_rescale(WarpState<NT> &st, float f0, float f1)
{
#pragma unroll
    for (int m = 0; m < 8; ++m)
#pragma unroll
        for (int k = 0; k < 4; ++k)
            st.acc[0][m][k] *= (k & 1) ? f1 : f0;
}

template <int NT, bool kDump>
__device__ __forceinline__ void process_stage_packed(const DecodeParams &p, WarpState<NT> &st,
                                                     PackedAcc &pa, const PackedOffsets &o,
                                                     uint32_t sb, uint32_t sbs, int tl0,
                                                     uint32_t vmask, bool causal, int lim,
                                                     float scale_log2,
                                                     int b, int hc, int kl, int tok0, int g,
                                                     int c, float k0, float k1)
{
    const bool lower = g < 4;
    const int uk = lower ? 0 : 1;
    // ---- scores of this lane's 16-token half (see process_stage for the exact chain)
    float s[2][2];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
        int p0[4] = {kDotBias, kDotBias, kDotBias, kDotBias};
        int p1[4] = {kDotBias, kDotBias, kDotBias, kDotBias};
        float prev[2] = {kDotBiasF, kDotBiasF};
        s[nt][0] = s[nt][1] = 0.f;
#pragma unroll
        for (int j = 0; j < kNB; ++j) {
            const uint2 kk0 = lds64(sb + o.k[0][j] + nt * 1024);
            const uint2 kk1 = lds64(sb + o.k[1][j] + nt * 1024);
            int d0[4], d1[4];
            mma_s8_16832_acc(d0, st.qa[j][0], 0u, st.qa[j][2], 0u, kk0.x, kk0.y, p0);
            mma_s8_16832_acc(d1, st.qa[j][0], 0u, st.qa[j][2], 0u, kk1.x, kk1.y, p1);
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const float cur = __int_as_float(lower ? d0[e] : d1[e]);
                if constexpr (kDump) {
                    const int tl = tl0 + uk * 16 + nt * 8 + e;
                    const int hg = g & 3;
                    if (hg < p.G && ((vmask >> (uk * 16 + nt * 8 + 2 * c + e)) & 1u)) {
                        const long long h = (long long)(hc * p.HPC + kl) * p.G + hg;
                        p.dbg_dots[(((long long)b * p.Hq + h) * p.dbg_max_len + tok0 + tl) *
                                       kNB +
                                   j] = __float_as_int(cur) - __float_as_int(prev[e]);
                    }
                }
                s[nt][e] += (cur - prev[e]) * st.qs[0][j];
                prev[e] = cur;
            }
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                p0[q] = d0[q];
                p1[q] = d1[q];
            }
        }
    }
    // ---- scales of the kept tokens; masked tokens get score -inf and V scale 0
    float kss[2][2], vsv[2][2];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            kss[nt][e] = lds_f32(sbs + o.s[nt][e]) * scale_log2;
            vsv[nt][e] = lds_f32(sbs + o.s[nt][e] + p.lay.sc_gap);
        }
    if (vmask != 0xffffffffu || causal) {
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int j = uk * 16 + nt * 8 + 2 * c + e;
                if (!((vmask >> j) & 1u)) {
                    s[nt][e] = -INFINITY;
                    kss[nt][e] = 1.f;
                    vsv[nt][e] = 0.f;
                } else if (j >= lim) {
                    s[nt][e] = -INFINITY; // after this row's own position
                }
            }
    }
    // ---- online softmax (base 2) over the stage's 32 tokens (M, S, A as in process_stage)
    float m = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const float v = s[nt][e] * kss[nt][e];
            s[nt][e] = v;
            m = fmaxf(m, v);
        }
    m = fmaxf(m, __shfl_xor_sync(kFullMask, m, 1));
    m = fmaxf(m, __shfl_xor_sync(kFullMask, m, 2));
    m = fmaxf(m, __shfl_xor_sync(kFullMask, m, 16));
    const float mn = fmaxf(st.M[0], m);
    const float ms = (mn == -INFINITY) ? 0.f : mn;
    const float alpha_s = fast_exp2(st.M[0] - ms);
    st.M[0] = mn;
    float ws = 0.f, pmax = 0.f, w[2][2];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const float x = fast_exp2(s[nt][e] - ms);
            ws += x;
            w[nt][e] = x * vsv[nt][e];
            pmax = fmaxf(pmax, w[nt][e]);
        }
    st.S[0] = st.S[0] * alpha_s + ws;
    pmax = fmaxf(pmax, __shfl_xor_sync(kFullMask, pmax, 1));
    pmax = fmaxf(pmax, __shfl_xor_sync(kFullMask, pmax, 2));
    pmax = fmaxf(pmax, __shfl_xor_sync(kFullMask, pmax, 16));
    const float an_stage = ms + exponent_as_float(pmax) - 14.f;
    const float an = (mn == -INFINITY) ? -INFINITY : fmaxf(fmaxf(st.A[0], an_stage), mn - 114.f);
    const float as = (an == -INFINITY) ? 0.f : an;
    const bool rose = an != st.A[0];
    const float alpha_a = rose ? fast_exp2(st.A[0] - as) : 1.f;
    st.A[0] = an;
    // ---- fold the int32 accumulators (scale of the old A) before this stage's products
    if (__any_sync(kFullMask, rose) || pa.n == kPackFoldEvery) {
        // columns 2c, 2c + 1 hold heads (2c) & 3, (2c + 1) & 3: rows 2c, 2c + 1 (or the
        // repeats 2c + 4, 2c + 5), i.e. lanes 8c and 8c + 4
        const float f0 = __shfl_sync(kFullMask, alpha_a, 8 * c);
        const float f1 = __shfl_sync(kFullMask, alpha_a, 8 * c + 4);
        if (pa.n > 0)
            packed_fold(st, pa, k0, k1, f0, f1);
        else
            packed_rescale(st, f0, f1);
        pa.n = 0;
    }
    // ---- P as exact integers, split into byte planes for the B operands
    const float cvs8 = fast_exp2(ms - as + 8.f); // 2^(M - A + 8)
    uint32_t X[2][2];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e)
            X[nt][e] = __float_as_uint(fmaf(w[nt][e], cvs8, kTwo23));
    const uint32_t x01 = prmt(X[0][0], X[0][1], 0x5140u), x23 = prmt(X[1][0], X[1][1], 0x5140u);
    const uint32_t y01 = prmt(X[0][0], X[0][1], 0x7362u), y23 = prmt(X[1][0], X[1][1], 0x7362u);
    const uint32_t pl0 = prmt(x01, x23, 0x5410u), pl1 = prmt(x01, x23, 0x7632u);
    const uint32_t pl2 = prmt(y01, y23, 0x5410u);
    // partner lane (row g ^ 4) holds the other 16 tokens of the same head
    const uint32_t r1 = __shfl_xor_sync(kFullMask, lower ? pl1 : pl0, 16);
    const uint32_t r2 = __shfl_xor_sync(kFullMask, pl2, 16);
    const uint32_t bA0 = lower ? pl0 : r1, bA1 = lower ? r1 : pl1; // n-tile 0: bytes 0 | 1
    const uint32_t bB0 = pl2, bB1 = r2;                            // n-tile 1: byte 2
    // ---- PV: V^T fragments by ldmatrix .trans, two u8 n-tiles per 16-channel m-tile
    const uint32_t vrow = sb + o.v;
    if (pa.n == 0) {
        const int z[4] = {kDotBias, kDotBias, kDotBias, kDotBias};
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
            uint32_t a0, a1, a2, a3;
            ldsm_x2_trans_b8(a0, a1, a2, a3, vrow ^ (uint32_t)(mt << 4));
            mma_s8u8_16832_acc(pa.D[mt][0], a0, a1, a2, a3, bA0, bA1, z);
            mma_s8u8_16832_acc(pa.D[mt][1], a0, a1, a2, a3, bB0, bB1, z);
        }
    } else {
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
            uint32_t a0, a1, a2, a3;
            ldsm_x2_trans_b8(a0, a1, a2, a3, vrow ^ (uint32_t)(mt << 4));
            mma_s8u8_16832_acc(pa.D[mt][0], a0, a1, a2, a3, bA0, bA1, pa.D[mt][0]);
            mma_s8u8_16832_acc(pa.D[mt][1], a0, a1, a2, a3, bB0, bB1, pa.D[mt][1]);
        }
    }
    ++pa.n;
}

// Packed layout: lane (g, c) holds channels 16 m + g (k = 0, 1) and 16 m + g + 8 (k = 2, 3)
// of columns 2c + (k & 1).
// ------------------------------------------------------------------ int8 PV, 5-16 rows
//
// One or two 8-row query tiles (5 to 16 query rows per KV head: a group of 5-16, or several
// query tokens of a smaller group) take the packed path's int8 PV without its row repeat: lane
// (g, c) keeps the scores of rows g (and g + 8) for tokens 2c, 2c + 1, 8 + 2c, 9 + 2c of
// each 16-token subtile, which are exactly the k positions 4c..4c+3 (and 16 + 4c..) of the
// B operand under the token order tau of the V^T ldmatrix load, so P needs no shuffle:
// each of its three bytes is one n-tile of 8 head columns (three u8 MMAs per 16-channel
// m-tile and row tile, no int8 -> f16 conversion of V). The stage's
// int32 sums are folded into the fp32 accumulator at once (exact: |sum| < 2^22).
template <int NT, bool kDump>
__device__ __forceinline__ void process_stage_i8(const DecodeParams &p, WarpState<NT> &st,
                                                 const ThreadOffsets &o, uint32_t vrow_off,
                                                 uint32_t sb, uint32_t sbs, int tl0,
                                                 uint32_t vmask, bool causal,
                                                 const int (&lim)[NT], float scale_log2, int b,
                                                 int hc, int kl, int slice, int tok0, int g,
                                                 int c)
{
    // ---- scores: the exact int32 block dots of process_stage
    float s[NT][kSub][2][2];
#pragma unroll
    for (int u = 0; u < kSub; ++u)
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
            for (int r = 0; r < NT; ++r)
                s[r][u][nt][0] = s[r][u][nt][1] = 0.f;
            int prev[4] = {kDotBias, kDotBias, kDotBias, kDotBias};
#pragma unroll
            for (int j = 0; j < kNB; ++j) {
                const uint2 kk = lds64(sb + o.k[u][j] + nt * 1024);
                int d[4];
                mma_s8_16832_acc(d, st.qa[j][0], NT == 2 ? st.qa[j][1] : 0u, st.qa[j][2],
                                 NT == 2 ? st.qa[j][3] : 0u, kk.x, kk.y, prev);
                if constexpr (kDump) {
#pragma unroll
                    for (int q = 0; q < 2 * NT; ++q) {
                        const int r = q >> 1, e = q & 1;
                        const int hg = slice * 16 + r * 8 + g;
                        const int tl = tl0 + u * 16 + nt * 8 + e;
                        if (hg < p.G && ((vmask >> (tl - tl0 + 2 * c)) & 1u)) {
                            const long long h = (long long)(hc * p.HPC + kl) * p.G + hg;
                            p.dbg_dots[(((long long)b * p.Hq + h) * p.dbg_max_len + tok0 + tl) *
                                           kNB +
                                       j] = d[q] - prev[q];
                        }
                    }
                }
#pragma unroll
                for (int r = 0; r < NT; ++r) {
                    s[r][u][nt][0] +=
                        (__int_as_float(d[2 * r]) - __int_as_float(prev[2 * r])) * st.qs[r][j];
                    s[r][u][nt][1] += (__int_as_float(d[2 * r + 1]) -
                                       __int_as_float(prev[2 * r + 1])) * st.qs[r][j];
                }
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    prev[q] = d[q];
            }
        }
    float kss[kSub][2][2], vsv[kSub][2][2];
#pragma unroll
    for (int u = 0; u < kSub; ++u)
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                kss[u][nt][e] = lds_f32(sbs + o.s[u][nt][e]) * scale_log2;
                vsv[u][nt][e] = lds_f32(sbs + o.s[u][nt][e] + p.lay.sc_gap);
            }
    if (vmask != 0xffffffffu || causal) {
#pragma unroll
        for (int u = 0; u < kSub; ++u)
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int j = u * 16 + nt * 8 + 2 * c + e;
                    if (!((vmask >> j) & 1u)) {
#pragma unroll
                        for (int r = 0; r < NT; ++r)
                            s[r][u][nt][e] = -INFINITY;
                        kss[u][nt][e] = 1.f;
                        vsv[u][nt][e] = 0.f;
                    } else {
#pragma unroll
                        for (int r = 0; r < NT; ++r)
                            if (j >= lim[r])
                                s[r][u][nt][e] = -INFINITY;
                    }
                }
    }
    // ---- online softmax of rows g (and g + 8) over the stage's 32 tokens; P as exact
    // integers < 2^23, split in bytes (k order 4c + i <-> token 2c + (i & 1) + 8 (i >> 1))
    float alpha_a[NT];
    uint32_t pl[NT][3][kSub];
#pragma unroll
    for (int r = 0; r < NT; ++r) {
        float m = -INFINITY;
#pragma unroll
        for (int u = 0; u < kSub; ++u)
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const float v = s[r][u][nt][e] * kss[u][nt][e];
                    s[r][u][nt][e] = v;
                    m = fmaxf(m, v);
                }
        m = fmaxf(m, __shfl_xor_sync(kFullMask, m, 1));
        m = fmaxf(m, __shfl_xor_sync(kFullMask, m, 2));
        const float mn = fmaxf(st.M[r], m);
        const float ms = (mn == -INFINITY) ? 0.f : mn;
        const float alpha_s = fast_exp2(st.M[r] - ms);
        st.M[r] = mn;
        float ws = 0.f, pmax = 0.f;
#pragma unroll
        for (int u = 0; u < kSub; ++u)
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const float x = fast_exp2(s[r][u][nt][e] - ms);
                    ws += x;
                    s[r][u][nt][e] = x * vsv[u][nt][e]; // the weight w * vs
                    pmax = fmaxf(pmax, s[r][u][nt][e]);
                }
        st.S[r] = st.S[r] * alpha_s + ws;
        pmax = fmaxf(pmax, __shfl_xor_sync(kFullMask, pmax, 1));
        pmax = fmaxf(pmax, __shfl_xor_sync(kFullMask, pmax, 2));
        const float an_stage = ms + exponent_as_float(pmax) - 14.f;
        const float an =
            (mn == -INFINITY) ? -INFINITY : fmaxf(fmaxf(st.A[r], an_stage), mn - 114.f);
        const float as = (an == -INFINITY) ? 0.f : an;
        alpha_a[r] = fast_exp2(st.A[r] - as);
        st.A[r] = an;
        const float cvs8 = fast_exp2(ms - as + 8.f); // 2^(M - A + 8)
#pragma unroll
        for (int u = 0; u < kSub; ++u) {
            uint32_t X[2][2];
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e)
                    X[nt][e] = __float_as_uint(fmaf(s[r][u][nt][e], cvs8, kTwo23));
            const uint32_t x01 = prmt(X[0][0], X[0][1], 0x5140u);
            const uint32_t x23 = prmt(X[1][0], X[1][1], 0x5140u);
            const uint32_t y01 = prmt(X[0][0], X[0][1], 0x7362u);
            const uint32_t y23 = prmt(X[1][0], X[1][1], 0x7362u);
            pl[r][0][u] = prmt(x01, x23, 0x5410u);
            pl[r][1][u] = prmt(x01, x23, 0x7632u);
            pl[r][2][u] = prmt(y01, y23, 0x5410u);
        }
    }
    // ---- rescale factors of the accumulator columns (heads 2c, 2c + 1 of each row tile:
    // the rows of lanes 8c, 8c + 4)
    float f0[NT], f1[NT];
#pragma unroll
    for (int r = 0; r < NT; ++r) {
        f0[r] = __shfl_sync(kFullMask, alpha_a[r], 8 * c);
        f1[r] = __shfl_sync(kFullMask, alpha_a[r], 8 * c + 4);
    }
    // ---- PV: V^T by ldmatrix .trans (k = the 32 tokens in tau order), one u8 n-tile per
    // byte of P and row tile; acc = acc * f + (S0 / 2^8 + S1 + S2 * 2^8), S_i the exact sums
    const uint32_t vrow = sb + vrow_off;
    const int z[4] = {kDotBias, kDotBias, kDotBias, kDotBias};
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
        uint32_t a0, a1, a2, a3;
        ldsm_x2_trans_b8(a0, a1, a2, a3, vrow ^ (uint32_t)(mt << 4));
#pragma unroll
        for (int r = 0; r < NT; ++r) {
            int d0[4], d1[4], d2[4];
            mma_s8u8_16832_acc(d0, a0, a1, a2, a3, pl[r][0][0], pl[r][0][1], z);
            mma_s8u8_16832_acc(d1, a0, a1, a2, a3, pl[r][1][0], pl[r][1][1], z);
            mma_s8u8_16832_acc(d2, a0, a1, a2, a3, pl[r][2][0], pl[r][2][1], z);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                // the biased fp32 views minus the bias are the exact sums; recombine them
                // with one rounding per step, smallest first
                const float s0 = __int_as_float(d0[k]) - kDotBiasF;
                const float s1 = __int_as_float(d1[k]) - kDotBiasF;
                const float s2 = __int_as_float(d2[k]) - kDotBiasF;
                const float v = fmaf(s2, 256.f, fmaf(s0, 0.00390625f, s1));
                st.acc[r][mt][k] = fmaf(st.acc[r][mt][k], (k & 1) ? f1[r] : f0[r], v);
            }
        }
    }
}

// Write channels 16m + g and 16m + g + 8 (m = 0..7) of column q's head scaled by f: the
// channel order of the ldmatrix-fed int8 PV (the packed path and the one-tile int8 PV).
template <int NT>
__device__ __forceinline__ void store_packed(float *dst, const WarpState<NT> &st, int pv, int q,
                                             float f)
{
#pragma unroll
    for (int m = 0; m < 8; ++m) {
        dst[16 * m] = st.acc[pv][m][q] * f;
        dst[16 * m + 8] = st.acc[pv][m][q + 2] * f;
    }
}

// End of a segment (all of this CTA's tiles of sequence b, head chunk hc).
template <int NT, bool kPack>
__device__ __forceinline__ void finalize_segment(const DecodeParams &p, WarpState<NT> &st,
                                                 uint8_t *smem, int b,
                                 int hc, int kl, int slice, int pair, int ts, int g, int c,
                                 const int *prefix, int t0, int t1)
{
    // complete this lane's row sums
#pragma unroll
    for (int r = 0; r < NT; ++r) {
        st.S[r] += __shfl_xor_sync(kFullMask, st.S[r], 1);
        st.S[r] += __shfl_xor_sync(kFullMask, st.S[r], 2);
        if constexpr (kPack) // rows g and g ^ 4 summed different tokens of one head
            st.S[r] += __shfl_xor_sync(kFullMask, st.S[r], 16);
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
#pragma unroll 1
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
                        const float f = sc > 0.f ? exp2f(ac - mc) / sc : 0.f;
                        float *dst = p.out + q_row(p, b, hc * p.HPC + kl, hg) * kD;
                        store_packed(dst + g, st, pv, q, f); // ldmatrix channel order
                    }
                }
        }
        return;
    }

    // partial: this CTA's share of the segment goes to its workspace slot (0: the segment
    // this CTA's range starts in, 1: the one it ends in); the combine kernel finds the
    // split segments and their contributors from the same work split
    const int which = (seg0 <= t0) ? 0 : 1;
    const int H = p.heads_seg;
    if (ts == 0) {
        float *slotp = p.partials + (size_t)(2 * blockIdx.x + which) * H * kSlotRow;
#pragma unroll
        for (int pv = 0; pv < NT; ++pv)
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                const int hg = slice * 16 + pv * 8 + 2 * c + q;
                if (col_lane && hg < p.G) {
                    float *dst = slotp + (size_t)(kl * p.G + hg) * kSlotRow;
                    store_packed(dst + g, st, pv, q, 1.0f);
                }
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
#pragma unroll 1
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

// Does this CTA's range [t0, t1) reach into a second segment whose query fits the buffer?
__device__ __forceinline__ bool has_second_query(const DecodeParams &p, const int *prefix, int t0,
                                                 int t1)
{
    return p.lay.qbuf_rows != 0 && cursor_at(p, prefix, t0).seg1 < t1;
}

// Warp 9: the quantised query rows of the CTA's second segment, for every (KV head, slice)
// pair, in the buffer's lane-fragment order (what the consumers' load_query would produce).
template <int NT, bool kPack>
__device__ void prepare_second_query(const DecodeParams &p, uint8_t *smem, const int *prefix,
                                     int t0, int lane)
{
    const SegCursor c1 = cursor_at(p, prefix, cursor_at(p, prefix, t0).seg1);
    const int g = lane >> 2, c = lane & 3;
#pragma unroll 1
    for (int pair = 0; pair < p.pairs; ++pair) {
        const int kl = pair / p.slices, slice = pair % p.slices;
        const QueryFrag<NT> qf = load_query<NT, kPack>(p, c1.b, c1.hc, kl, slice, g, c);
        store_query<NT, kPack>(smem_addr(smem) + p.lay.off_qbuf +
                                   (uint32_t)pair * p.lay.qbuf_rows * kQRowBytes,
                               qf, g, c);
    }
}

template <int NT, bool kPack, bool kDump>
__device__ void consume(const DecodeParams &p, uint8_t *smem, const int *prefix,
                        int t0, int t1, int warp, int lane)
{
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + p.lay.off_full);
    uint64_t *empty = reinterpret_cast<uint64_t *>(smem + p.lay.off_empty);
    const int pair = warp % p.pairs, ts = warp / p.pairs;
    const int kl = pair / p.slices, slice = pair % p.slices;
    const int g = lane >> 2, c = lane & 3;
    const ThreadOffsets o = make_offsets(p, kl, ts, g, c);
    const PackedOffsets po = make_packed_offsets(p, kl, ts, g, c, lane);
    PackedAcc pa;
    pa.n = 0;
    // weights of this lane's two n-tile columns in the packed PV (bytes 0 | 2, or byte 1)
    const float k0 = c < 2 ? 0.00390625f : 1.f, k1 = c < 2 ? 256.f : 0.f;
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

    // With nq query tokens per sequence, query row hg (token hg / Gq) may not see the last
    // fut = nq - 1 - hg / Gq tokens of the sequence (they come after its own position).
    int fut[NT];
#pragma unroll
    for (int r = 0; r < NT; ++r) {
        const int hg = kPack ? (g & 3) : slice * 16 + r * 8 + g;
        fut[r] = hg < p.G ? p.nq - 1 - hg / p.Gq : 0;
    }
    bool dead = false; // set when a pipeline wait timed out: skip work, keep the barriers
    const unsigned long long limit = wait_limit(p);
    int stage = 0;
    uint32_t phase = 0;
    const uint32_t smem_base = smem_addr(smem);
    const uint32_t stage_bytes = p.lay.stage_bytes;
    const float scale_log2 = p.scale_log2;
    const int tl0 = ts * kSub * 16 + 2 * c;
    const int all_boxes = (1 << p.n_boxes) - 1;
    const uint32_t qbuf = smem_base + p.lay.off_qbuf +
                          (uint32_t)pair * p.lay.qbuf_rows * kQRowBytes;
    // The quantised query of the CTA's second segment is prepared by warp 9 (otherwise idle)
    // while the first segment streams and kept in shared memory, so that switching segments
    // in the middle of the stream costs neither a global round trip nor the quantisation
    // code, and the first stage is not held up by it; the consumers take it at the switch
    // after named barrier 4.
    const bool prefetch_q = has_second_query(p, prefix, t0, t1);
    int seg_index = 0;
    // Outer loop: one segment (this CTA's tiles of one sequence and head chunk) per pass.
    for (int x = t0; x < t1;) {
        const SegCursor cu = cursor_at(p, prefix, x);
        const int x_end = cu.seg1 < t1 ? cu.seg1 : t1;
        const uint32_t scol4 = 4u * (uint32_t)((cu.hc * p.HPC) % p.sc_heads);
        {
            if (prefetch_q && seg_index == 1) // warp 9 has written the buffer
                asm volatile("bar.sync 4, %0;" ::"n"(kConsumerThreads + 32) : "memory");
            const QueryFrag<NT> qf = (prefetch_q && seg_index == 1)
                                         ? load_query_smem<NT, kPack>(qbuf, g, c)
                                         : load_query<NT, kPack>(p, cu.b, cu.hc, kl, slice, g, c);
            ++seg_index;
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
            pa.n = 0;
        }
        for (; x < x_end; ++x) {
            const int tok0 = (x - cu.seg0) * p.TT;
            const int nvalid = min(p.TT, cu.L - tok0);
            if (!dead && !mbar_wait(&full[stage], phase, limit)) {
                dead = true;
                atomicOr(p.errors, kErrTimeout);
            }
            if (!dead) {
                const int loaded = (int)lds_u32(smem_base + p.lay.off_mask + 4u * stage);
                const uint32_t sb = smem_base + (uint32_t)stage * stage_bytes;
                // bit k: token k of this warp's 32-token window holds data
                uint32_t vmask = 0xffffffffu;
                if (nvalid != p.TT || loaded != all_boxes) {
                    const int tk = ts * kSub * 16 + lane;
                    vmask = __ballot_sync(kFullMask,
                                          tk < nvalid && ((loaded >> (tk >> p.log2_box)) & 1));
                }
                // rows may see window tokens [0, lim): only in the last nq - 1 tokens of a
                // sequence does that differ between rows (never with one query per sequence)
                const int win0 = tok0 + ts * kSub * 16;
                const bool causal = p.nq > 1 && cu.L - (p.nq - 1) - win0 < 32;
                int lim[NT];
#pragma unroll
                for (int r = 0; r < NT; ++r)
                    lim[r] = cu.L - fut[r] - win0;
                const uint32_t sbs = sb + scol4; // this segment's scale column
                if constexpr (kPack)
                    process_stage_packed<NT, kDump>(p, st, pa, po, sb, sbs, tl0, vmask, causal,
                                                    lim[0], scale_log2, cu.b, cu.hc, kl, tok0, g,
                                                    c, k0, k1);
                else
                    process_stage_i8<NT, kDump>(p, st, o, po.v, sb, sbs, tl0, vmask, causal, lim,
                                                scale_log2, cu.b, cu.hc, kl, slice, tok0, g, c);
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(&empty[stage]);
            }
            if (++stage == p.n_stages) {
                stage = 0;
                phase ^= 1u;
            }
        }
        if constexpr (kPack) {
            if (pa.n > 0)
                packed_fold(st, pa, k0, k1, 1.f, 1.f);
        }
        finalize_segment<NT, kPack>(p, st, smem, cu.b, cu.hc, kl, slice, pair, ts, g, c,
                                    prefix, t0, t1);
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

    if (tid == 0) {
        for (int s = 0; s < p.n_stages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kConsumerWarps);
        }
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
    __syncthreads(); // the barrier initialisation is visible to every warp
    // Everything above touches only shared memory and kernel parameters; from here on the
    // previous kernel on the stream (another call's combine, which reads the workspace, or
    // a producer of the inputs) must be complete.
    grid_dep_wait();
    grid_dep_launch();
    int *nseq = p.lay.off_nseq ? reinterpret_cast<int *>(smem + p.lay.off_nseq) : nullptr;
    int *cstart = reinterpret_cast<int *>(smem + p.lay.off_cstart);
    // Warp specialisation: the producer warpgroup hands most of its registers to the two
    // consumer warpgroups (the sums match the launch allocation, checked by static_assert).
    // From here on the roles synchronise separately (named barriers), so the producer does
    // not wait for the consumers' prologue: for a batch of up to 32 sequences it scans the
    // sequence lengths and computes its CTA's range itself and starts loading at once.
    if (warp >= kConsumerWarps) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(RegSplit<NT, kPack>::producer));
        if (warp == kProducerWarp + 1) {
            // the second segment's query, once the consumers have published the split
            asm volatile("bar.sync 3, %0;" ::"n"(kConsumerThreads + 32) : "memory");
            const Split sp = split_of(p, prefix, nseq, (int)gridDim.x);
            if (sp.gcta == 0 || (int)blockIdx.x >= sp.gcta)
                return;
            const int t0 = cstart[blockIdx.x], t1 = cstart[blockIdx.x + 1];
            if (has_second_query(p, prefix, t0, t1)) {
                prepare_second_query<NT, kPack>(p, smem, prefix, t0, lane);
                asm volatile("bar.arrive 4, %0;" ::"n"(kConsumerThreads + 32) : "memory");
            }
            return;
        }
        if (warp != kProducerWarp)
            return;
        const int *pre = prefix;
        const int *pns = nseq;
        if (p.B <= 32) {
            int *pp = reinterpret_cast<int *>(smem + p.lay.off_pscan);
            scan_one_warp(p, pp, pp + kPscanLen, lane);
            __syncwarp();
            pre = pp;
            pns = pp + kPscanLen;
        } else {
            // the consumers publish the prefixes and this CTA's range
            asm volatile("bar.sync 2, %0;" ::"n"(kConsumerThreads + 32) : "memory");
        }
        const Split sp = split_of(p, pre, pns, (int)gridDim.x);
        if (sp.gcta == 0 || (int)blockIdx.x >= sp.gcta)
            return;
        int t0, t1;
        if (p.B <= 32) {
            const int v = lane < 2 ? cta_start(p, pre, pns, sp.pseg, sp.V, sp.gcta,
                                               (int)blockIdx.x + lane)
                                   : 0;
            t0 = __shfl_sync(kFullMask, v, 0);
            t1 = __shfl_sync(kFullMask, v, 1);
        } else {
            t0 = cstart[blockIdx.x];
            t1 = cstart[blockIdx.x + 1];
        }
        produce(p, &tmK, &tmV, &tmKs, &tmVs, smem, pre, t0, t1, lane);
        return;
    }
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(RegSplit<NT, kPack>::consumer));
    const int ctid = warp * 32 + lane;
    build_prefix(p, prefix, nseq,
                 reinterpret_cast<volatile unsigned long long *>(smem + p.lay.off_misc), ctid,
                 warp, lane);
    consumer_bar();
    const Split sp = split_of(p, prefix, nseq, (int)gridDim.x);
    const int gcta = sp.gcta;
    if (gcta > 0 && ctid < 2 && (int)blockIdx.x + ctid <= gcta)
        cstart[blockIdx.x + ctid] =
            cta_start(p, prefix, nseq, sp.pseg, sp.V, gcta, (int)blockIdx.x + ctid);
    consumer_bar();
    if (p.B > 32) // release the producer (it waits for the prefixes and the range)
        asm volatile("bar.arrive 2, %0;" ::"n"(kConsumerThreads + 32) : "memory");
    // and warp 9 (the second segment's query)
    asm volatile("bar.arrive 3, %0;" ::"n"(kConsumerThreads + 32) : "memory");
    if (gcta == 0) { // no sequence has tokens: every row is zero
#pragma unroll 1
        for (int b = blockIdx.x; b < p.B; b += gridDim.x) {
            float4 *row = reinterpret_cast<float4 *>(p.out + (long long)b * p.nq * p.Hq * kD);
#pragma unroll 1
            for (int i = ctid; i < p.nq * p.Hq * kD / 4; i += kConsumerThreads)
                row[i] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        return;
    }
    if ((int)blockIdx.x >= gcta)
        return;
    const int t0 = cstart[blockIdx.x], t1 = cstart[blockIdx.x + 1];
    // rows of empty sequences are zero (spread over the CTAs that have tiles)
#pragma unroll 1
    for (int b = blockIdx.x; b < p.B; b += gcta) {
        if (prefix[b + 1] != prefix[b])
            continue;
        float4 *row = reinterpret_cast<float4 *>(p.out + (long long)b * p.nq * p.Hq * kD);
#pragma unroll 1
        for (int i = ctid; i < p.nq * p.Hq * kD / 4; i += kConsumerThreads)
            row[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    consumer_bar();
    consume<NT, kPack, kDump>(p, smem, prefix, t0, t1, warp, lane);
}

} // namespace q8kv
