// q8kv_mq_tc.cuh -- decode attention for 9 to 32 query rows per KV head (several new query
// tokens per sequence) on the fifth-generation tensor cores: tcgen05.mma with int32
// accumulators in tensor memory (TMEM).
//
// What it computes is the single-query decode of q8kv_decode.cuh (Kestrel-LLM walk-through
// "flash_attn_single_q_q8_neon", trdm.cn/news/511694, section 2 parts 1-3) for every query
// row: int8 block dots per 32-channel block scaled by the Q block scale and the
// per-(token, KV head) K scale, an online softmax in base 2, int8 V weighted by the softmax
// weight times the per-(token, KV head) V scale, one division by the sum at the end. With
// several query tokens per sequence (the TILE idea of the llama.cpp SYCL FlashAttention
// change) a row sees only the tokens up to its own position.
//
// How:
//  * The work split, the producer warp and the partial-result format are those of
//    q8kv_decode.cuh (persistent CTAs over the flat tile list, combine kernel after). A tile
//    here is 128 tokens of one KV head: its K and V boxes land as 128 contiguous 128-byte
//    rows, 128-byte swizzled, which is the canonical K-major layout of a UMMA operand with
//    M = 128.
//  * QK per 32-channel block j: S_j^T = K_j . Q_j^T, M = 128 tokens, N = R rows, K = 32
//    channels, each block in TMEM columns of its own (tokens on TMEM lanes, two buffers so
//    that tile k + 1's QK runs while tile k's scores are read). The columns are seeded with
//    the bit pattern of 1.5 * 2^23 (tcgen05.st), so an int32 dot read as fp32 minus
//    1.5 * 2^23 is the exact dot.
//  * Softmax: thread t of a consumer warpgroup owns token t (TMEM lane t); warpgroup w of
//    the four owns rows [w R/4, (w + 1) R/4). Each thread forms its token's scores for its
//    rows; the tile maxima per row come from fp32 redux.sync and one exchange across the
//    warpgroup's 4 warps (one named barrier per tile). The row state (running max M of the
//    scores, running max A of score + log2 V scale) is kept by lane r of every warp of the
//    warpgroup, each computing it from the same exchanged maxima, and broadcast with
//    shuffles.
//  * PV: the weight w * vs * 2^(M - A + 19) of (token, row) is an exact integer P below
//    2^23 (A: the largest score + log2 vs, moved only when exceeded by 3); the fp32 bits
//    of P + 2^23 hold it in their low three bytes. Those 32-bit words are the B operand as
//    they are: O^T = V^T . W with M = 128 channels (V^T read straight from the swizzled
//    tile: MN-major int8), N = 4 R columns (row, byte), K = 32 tokens, int32 accumulators in
//    TMEM; byte k of a row's column group is plane k of P, the fourth (the constant exponent
//    byte) is never read. A warpgroup recombines its rows' planes in fp32 into per-thread
//    accumulators (thread t owns channel t) when A rises, every 256 tiles (int32 headroom)
//    and at segment end, and zeroes those columns again.
//  * Warp 17 issues the QK MMAs, warp 18 the PV MMAs (one thread each, in fixed orders with
//    hardware-suspended waits), warp 19 quantises the query rows of each later segment
//    (the consumers do the first), warp 16 is the TMA producer.
#pragma once

#include "q8kv_decode.cuh"

namespace q8kv {

constexpr int kTcTT = 128;           // tokens per tile: the QK MMA's M, the TMEM lanes
constexpr uint32_t kTcCols = 512;    // TMEM columns allocated: [S buffer 0 | S buffer 1 | O]
                                     // = [4 R | 4 R | 4 R]
constexpr int kTcFoldEvery = 256;    // tiles between forced folds: 256*128*255*127 < 2^31
constexpr float kTwo23F = 8388608.0f;
// Headroom of the weights' reference A (log2 units): a weight is w vs 2^(M - A + 22 - h), at
// most 2^(22 - h) for the largest (score + log2 vs) seen when A was set and below 2^22
// (< 2^23, the range of the byte planes) until a score + log2 vs exceeds A + h. A moves
// (and the accumulated planes are folded) only then, not on every new maximum.
constexpr float kTcAHead = 3.f;

// 4 consumer warpgroups (warps 0-15; warpgroup w owns rows [w R/4, (w + 1) R/4) of every
// tile) and one of helpers: the TMA producer, the two MMA issuers, the query quantiser.
constexpr int kTcWGs = 4;
constexpr int kTcConsumerWarps = 4 * kTcWGs;
constexpr int kTcConsumerThreads = 32 * kTcConsumerWarps;
constexpr int kTcThreads = kTcConsumerThreads + 128;
constexpr int kTcLaunchRegs = 96;    // per-thread registers at launch (65536 / 640, rounded)
constexpr int kTcConsumerRegs = 104; // after setmaxnreg
constexpr int kTcHelperRegs = 56;
static_assert(kTcConsumerThreads * kTcConsumerRegs + 128 * kTcHelperRegs <=
                  kTcThreads * kTcLaunchRegs,
              "register split exceeds the launch allocation");
constexpr int kTcProducerWarp = kTcConsumerWarps;
constexpr int kTcQkWarp = kTcConsumerWarps + 1; // also allocates and releases TMEM
constexpr int kTcPvWarp = kTcConsumerWarps + 2;
constexpr int kTcPrepWarp = kTcConsumerWarps + 3;

// Named barriers: 1 = consumer warps 0-7 (the prefix scan, as in the single-query kernel),
// 2 = warps 0-7 -> producer (batches over 32 sequences).
constexpr int kTcBarHelpers = 3;     // consumers -> warps 17-19: prefixes and range published
constexpr int kTcHelperThreads = kTcConsumerThreads + 96;
constexpr int kTcBarAll = 4;         // all consumer warps
constexpr int kTcBarWg = 5;          // 5 + w: one consumer warpgroup (5-8)
constexpr int kTcBarTeardown = 9;    // consumers -> warp 17: TMEM may be released
constexpr int kTcTeardownThreads = kTcConsumerThreads + 32;

// ------------------------------------------------------------------ tcgen05 wrappers

__device__ __forceinline__ void tc_alloc(uint32_t dst_smem, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     dst_smem),
                 "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tc_relinquish()
{
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tc_dealloc(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr),
                 "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before()
{
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after()
{
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Arrive on bar once every tcgen05.mma this thread issued before has completed.
__device__ __forceinline__ void tc_commit(uint64_t *bar)
{
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
            smem_addr(bar))
        : "memory");
}

// D (TMEM) = A . B (+ D when acc != 0), A and B described by shared-memory descriptors.
__device__ __forceinline__ void tc_mma_i8(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc,
                                          uint32_t acc)
{
    asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}\n"
                 ::"r"(d), "l"(a), "l"(b), "r"(idesc), "r"(acc), "r"(0), "r"(0), "r"(0), "r"(0)
                 : "memory");
}

__device__ __forceinline__ void tc_wait_ld()
{
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tc_wait_st()
{
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// N consecutive 32-bit columns of this thread's TMEM lane (warp-wide, 32x32b shape).
template <int N>
__device__ __forceinline__ void tc_ld(uint32_t taddr, uint32_t *v)
{
    static_assert(N == 4 || N == 8 || N == 16 || N == 32, "4, 8, 16 or 32 columns");
    if constexpr (N == 32) {
        tc_ld<16>(taddr, v);
        tc_ld<16>(taddr + 16, v + 16);
    } else if constexpr (N == 4)
        asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];"
                     : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3])
                     : "r"(taddr));
    else if constexpr (N == 16)
        asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,"
                     "%10,%11,%12,%13,%14,%15}, [%16];"
                     : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]),
                       "=r"(v[6]), "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]),
                       "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
                     : "r"(taddr));
    else
        asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                     : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]),
                       "=r"(v[6]), "=r"(v[7])
                     : "r"(taddr));
}

// Fill N consecutive columns of this thread's lane with x.
template <int N>
__device__ __forceinline__ void tc_fill(uint32_t taddr, uint32_t x)
{
    static_assert(N == 4 || N == 8 || N == 16 || N == 32, "4, 8, 16 or 32 columns");
    if constexpr (N == 32) {
        tc_fill<16>(taddr, x);
        tc_fill<16>(taddr + 16, x);
    } else if constexpr (N == 4)
        asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1,%1,%1,%1};" ::"r"(taddr),
                     "r"(x)
                     : "memory");
    else if constexpr (N == 16)
        asm volatile("tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%1,%1,%1,%1,%1,%1,%1,"
                     "%1,%1,%1,%1,%1,%1,%1,%1};" ::"r"(taddr),
                     "r"(x)
                     : "memory");
    else
        asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%1,%1,%1,%1,%1,%1,%1};" ::
                         "r"(taddr),
                     "r"(x)
                     : "memory");
}

// Shared-memory matrix descriptor: start address, leading / stride byte offsets, layout
// (0: no swizzle, 2: 128-byte swizzle), descriptor version 1.
__device__ __forceinline__ uint64_t umma_desc(uint32_t addr, uint32_t lbo, uint32_t sbo,
                                              uint32_t layout)
{
    return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | ((uint64_t)layout << 61);
}

constexpr uint32_t kSw128 = 2u, kNoSwizzle = 0u;

// Instruction descriptors (kind::i8, int32 accumulate, M = 128).
// QK: A = K (signed, K-major), B = Q (signed, K-major), N = R.
__host__ __device__ constexpr uint32_t idesc_qk(int R)
{
    return (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(R >> 3) << 17) | (8u << 24);
}
// PV: A = V^T (signed, MN-major), B = weight words (unsigned bytes, MN-major), N = 4 R.
__host__ __device__ constexpr uint32_t idesc_pv(int R)
{
    return (2u << 4) | (1u << 7) | (1u << 15) | (1u << 16) | ((uint32_t)((4 * R) >> 3) << 17) |
           (8u << 24);
}

// Maximum of v over the warp's 32 lanes (fp32 redux, sm_100a).
__device__ __forceinline__ float warp_max(float v)
{
    float r;
    asm("redux.sync.max.f32 %0, %1, %2;" : "=f"(r) : "f"(v), "r"(kFullMask));
    return r;
}


__device__ __forceinline__ void sts128(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                       uint32_t d)
{
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
                 "r"(d)
                 : "memory");
}


__device__ __forceinline__ void wg_bar(int w)
{
    asm volatile("bar.sync %0, %1;" ::"r"(kTcBarWg + w), "n"(128) : "memory");
}

// ------------------------------------------------------------------ shared memory

// Bytes of a query slot's operand (4 blocks of R rows x 32 codes in 8-row core matrices)
// and of one 32-token K-step of a weight buffer (R / 4 groups of 16 byte columns).
__host__ __device__ constexpr uint32_t tc_q_bytes(int R)
{
    return 4u * (uint32_t)R * 32u;
}
__host__ __device__ constexpr uint32_t tc_p_kstep_bytes(int R)
{
    return ((uint32_t)R / 4u) * 512u;
}

struct TcLayout {
    uint32_t off_tmem;   // TMEM base address written by tcgen05.alloc
    uint32_t off_bar;    // mbarriers, see TcBar
    uint32_t off_flag;   // (unused, 16 bytes)
    uint32_t off_q;      // Q operands [slot 2]
    uint32_t off_qs;     // Q block scales x softmax scale x log2 e [slot][block][row]
    uint32_t off_p;      // weight words [buffer 2][K-step 4]
    uint32_t off_xch;    // per-warp row maxima [tile parity 2][warpgroup 4][warp 4][row]
                         // float2 (and the row sums at segment end)
    uint32_t off_row;    // output factor per row at segment end [warpgroup][row] (float4
                         // stride)
    uint32_t total;
};

enum TcBar { kSFull = 0, kSFree = 2, kPReady = 4, kPvDone = 6, kQReady = 8, kQFree = 10,
             kFinal = 12, kNumTcBars = 13 };

__host__ __device__ inline TcLayout tc_layout(uint32_t base_total, int R)
{
    TcLayout L;
    uint32_t o = align_up(base_total, 16);
    L.off_tmem = o;
    o += 16;
    L.off_bar = o;
    o += 8 * 16;
    L.off_flag = o;
    o += 16;
    L.off_q = align_up(o, 128);
    o = L.off_q + 2u * tc_q_bytes(R);
    L.off_qs = o;
    o += 2u * 4u * (uint32_t)R * 4u;
    L.off_p = align_up(o, 128);
    o = L.off_p + 2u * 4u * tc_p_kstep_bytes(R);
    L.off_xch = o;
    o += 2u * 4u * (uint32_t)R * 8u; // 2 x 4 warpgroups x 4 warps x R/4 rows
    L.off_row = align_up(o, 16);
    o = L.off_row + (uint32_t)R * 16u;
    L.total = o;
    return L;
}

// ------------------------------------------------------------------ query quantisation

// Quantise segment cu's R query rows (rows >= G are zero) into query slot `slot`:
// quads of lanes take 32-element blocks, n_threads threads (a multiple of 32, every lane
// of their warps calling) stride over the 4 R (row, block) pairs.
template <int R>
__device__ void tc_quantize_query(const DecodeParams &p, uint8_t *smem, const TcLayout &L,
                                  const SegCursor &cu, int slot, int tid, int n_threads)
{
    const uint32_t sbase = smem_addr(smem);
    const int part = tid & 3;
#pragma unroll 1
    for (int base = 0; base < 4 * R; base += n_threads / 4) {
        const int bi = base + (tid >> 2);
        const int r = bi >> 2, j = bi & 3;
        const bool live = bi < 4 * R && r < p.G;
        float v[8];
        if (live) {
            const float4 *src = reinterpret_cast<const float4 *>(
                p.q + q_row(p, cu.b, cu.hc, r) * kD + 32 * j + 8 * part);
            const float4 a = __ldg(src), b = __ldg(src + 1);
            v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
            v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i)
                v[i] = 0.f;
        }
        uint32_t lo, hi;
        float qsc;
        quantize_block_quad(v, lo, hi, qsc);
        if (bi < 4 * R) {
            sts64(sbase + L.off_q + (uint32_t)slot * tc_q_bytes(R) + (uint32_t)j * R * 32u +
                      (uint32_t)(r >> 3) * 256u + (uint32_t)(part >> 1) * 128u +
                      (uint32_t)(r & 7) * 16u + (uint32_t)(part & 1) * 8u,
                  lo, hi);
            if (part == 0)
                sts_f32(sbase + L.off_qs + 4u * (uint32_t)((slot * 4 + j) * R + r),
                        live ? __fmul_rn(qsc, p.scale_log2) : 0.f);
        }
    }
}

// Warp 19: the query rows of the CTA's segments after the first, into slot (index & 1)
// once every warpgroup has finished the slot's previous segment.
template <int R>
__device__ void tc_prepare_queries(const DecodeParams &p, uint8_t *smem, const TcLayout &L,
                                   const int *prefix, int t0, int t1, int lane)
{
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L.off_bar);
    const unsigned long long limit = wait_limit(p);
    int sn = 0;
#pragma unroll 1
    for (int x = t0; x < t1; ++sn) {
        const SegCursor cu = cursor_at(p, prefix, x);
        x = cu.seg1 < t1 ? cu.seg1 : t1;
        if (sn == 0)
            continue; // the consumers quantise the first segment's rows
        const int slot = sn & 1;
        if (sn >= 2) {
            int ok = 1;
            if (lane == 0 && !mbar_wait(&bars[kQFree + slot], ((sn >> 1) - 1) & 1, limit)) {
                atomicOr(p.errors, kErrTimeout);
                ok = 0;
            }
            if (!__shfl_sync(kFullMask, ok, 0))
                return;
        }
        tc_quantize_query<R>(p, smem, L, cu, slot, lane, 32);
        fence_proxy_async_smem(); // generic writes -> the tensor core's reads
        __syncwarp();
        if (lane == 0)
            mbar_arrive(&bars[kQReady + slot]);
    }
}

// ------------------------------------------------------------------ MMA issuers

// Warp 17, lane 0: QK of tile k into score buffer k & 1, once the stage has landed, the
// segment's query slot is ready and every warpgroup has read that buffer's previous
// scores (tile k - 2).
template <int R>
__device__ void tc_issue_qk(const DecodeParams &p, uint8_t *smem, const TcLayout &L,
                            uint32_t tbase, const int *prefix, int t0, int t1)
{
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + p.lay.off_full);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L.off_bar);
    const uint32_t sbase = smem_addr(smem);
    const unsigned long long limit = wait_limit(p);
    constexpr uint32_t kId = idesc_qk(R);
    int qend = t0, qseg = -1;
#pragma unroll 1
    for (int k = 0; k < t1 - t0; ++k) {
        const int x = t0 + k;
        if (x == qend) { // first tile of a segment
            const SegCursor cu = cursor_at(p, prefix, x);
            qend = cu.seg1 < t1 ? cu.seg1 : t1;
            ++qseg;
        }
        const int qslot = qseg & 1, slot = k % p.n_stages, buf = k & 1;
        if (!mbar_wait(&bars[kQReady + qslot], (uint32_t)(qseg >> 1) & 1u, limit) ||
            !mbar_wait(&full[slot], (uint32_t)(k / p.n_stages) & 1u, limit) ||
            !mbar_wait(&bars[kSFree + buf], (uint32_t)(k >> 1) & 1u, limit)) {
            atomicOr(p.errors, kErrTimeout);
            break;
        }
        tc_fence_after();
        const uint32_t kt = sbase + (uint32_t)slot * p.lay.stage_bytes + p.lay.off_k;
        const uint32_t qb = sbase + L.off_q + (uint32_t)qslot * tc_q_bytes(R);
        const uint32_t d = tbase + (uint32_t)(buf * 4 * R);
#pragma unroll
        for (int j = 0; j < 4; ++j)
            tc_mma_i8(d + (uint32_t)(j * R), umma_desc(kt + 32u * j, 16u, 1024u, kSw128),
                      umma_desc(qb + (uint32_t)j * R * 32u, 128u, 256u, kNoSwizzle), kId, 1u);
        tc_commit(&bars[kSFull + buf]);
    }
    tc_commit(&bars[kFinal]);
}

// Warp 18, lane 0: PV of tile k once every warpgroup has written its weight words into
// weight buffer k & 1; its completion frees the stage and the weight buffer.
template <int R>
__device__ void tc_issue_pv(const DecodeParams &p, uint8_t *smem, const TcLayout &L,
                            uint32_t tbase, int n)
{
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + p.lay.off_full);
    uint64_t *empty = reinterpret_cast<uint64_t *>(smem + p.lay.off_empty);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L.off_bar);
    const uint32_t sbase = smem_addr(smem);
    const unsigned long long limit = wait_limit(p);
    constexpr uint32_t kId = idesc_pv(R);
    const uint32_t d = tbase + (uint32_t)(8 * R);
#pragma unroll 1
    for (int k = 0; k < n; ++k) {
        const int slot = k % p.n_stages, buf = k & 1;
        // (the stage has landed once the weights are written; the wait on it makes the TMA
        // writes visible to this thread's MMAs directly)
        if (!mbar_wait(&bars[kPReady + buf], (uint32_t)(k >> 1) & 1u, limit) ||
            !mbar_wait(&full[slot], (uint32_t)(k / p.n_stages) & 1u, limit)) {
            atomicOr(p.errors, kErrTimeout);
            break;
        }
        tc_fence_after();
        const uint32_t vt = sbase + (uint32_t)slot * p.lay.stage_bytes + p.lay.off_v;
        const uint32_t pb = sbase + L.off_p + (uint32_t)buf * 4u * tc_p_kstep_bytes(R);
#pragma unroll
        for (int s = 0; s < 4; ++s)
            tc_mma_i8(d, umma_desc(vt + 4096u * s, 16384u, 1024u, kSw128),
                      umma_desc(pb + tc_p_kstep_bytes(R) * s, 128u, 512u, kNoSwizzle), kId, 1u);
        tc_commit(&bars[kPvDone + buf]);
        tc_commit(&empty[slot]);
    }
    tc_commit(&bars[kFinal]);
}

// ------------------------------------------------------------------ consumer warpgroups

// Sum of v[i] over the 32 lanes, for row i = lane % N, by a transposing butterfly.
template <int N>
__device__ __forceinline__ float tc_row_sums(float (&v)[N], int lane)
{
#pragma unroll
    for (int o = 16; o >= N; o >>= 1)
#pragma unroll
        for (int i = 0; i < N; ++i)
            v[i] += __shfl_xor_sync(kFullMask, v[i], o);
#pragma unroll
    for (int o = N / 2, n = N; o >= 1; o >>= 1, n >>= 1) {
        const bool up = lane & o;
#pragma unroll
        for (int i = 0; i < n / 2; ++i) {
            const float send = up ? v[i] : v[i + n / 2];
            const float keep = up ? v[i + n / 2] : v[i];
            v[i] = keep + __shfl_xor_sync(kFullMask, send, o);
        }
    }
    return v[0];
}

// This warpgroup's columns of the PV accumulators: byte plane k of row i at tOw + 4 i + k.
// Fold them into acc (units of 2^A: the weights carry 2^(22 - h)) when add_o, scale every
// row by its fold factor (lane i holds row i's) when rescale, and zero the columns (the next
// PV starts from zero).
template <int R>
__device__ __forceinline__ void tc_fold(float (&acc)[R / kTcWGs], uint32_t tOw, float fa_lane,
                                        bool add_o, bool rescale)
{
    constexpr int RH = R / kTcWGs;
    if (add_o) {
        uint32_t o[4 * RH];
        tc_ld<4 * RH>(tOw, o);
        tc_wait_ld();
#pragma unroll
        for (int i = 0; i < RH; ++i) {
            const float c = fmaf((float)(int)o[4 * i + 2], 65536.f,
                                 fmaf((float)(int)o[4 * i + 1], 256.f, (float)(int)o[4 * i]));
            acc[i] = fmaf(c, 1.f / 524288.f, acc[i]); // 2^-(22 - kTcAHead)
        }
    }
    if (rescale) {
#pragma unroll
        for (int i = 0; i < RH; ++i)
            acc[i] *= __shfl_sync(kFullMask, fa_lane, i);
    }
    tc_fill<4 * RH>(tOw, 0u);
}

template <int R>
__device__ void tc_consume(const DecodeParams &p, uint8_t *smem, const TcLayout &L, uint32_t tbase,
                           const int *prefix, int t0, int t1, int warp, int lane)
{
    constexpr int RH = R / kTcWGs;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + p.lay.off_full);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L.off_bar);
    const int w = warp >> 2, q4 = warp & 3, tt = q4 * 32 + lane;
    const int r0 = w * RH; // this warpgroup's first row
    const bool owner = q4 == 0 && lane < RH; // writes the row's results at segment end
    const uint32_t sbase = smem_addr(smem);
    const uint32_t tlane = tbase + ((uint32_t)(q4 * 32) << 16);
    const uint32_t tOw = tlane + (uint32_t)(8 * R + 4 * r0);
    const uint32_t pofs = L.off_p + (uint32_t)q4 * tc_p_kstep_bytes(R) +
                          (uint32_t)(lane >> 3) * 128u + (uint32_t)(lane & 7) * 16u +
                          (uint32_t)(r0 / 4) * 512u;
    static_assert(RH == 4 || RH == 8 || RH == 16, "rows per warpgroup: 4, 8 or 16");
    const uint32_t xch = sbase + L.off_xch + (uint32_t)w * 4u * RH * 8u;
    const uint32_t rowi = sbase + L.off_row + (uint32_t)w * RH * 16u;
    // the tables read in the per-tile loop, as plain shared-memory pointers (ordinary loads
    // the compiler can batch; the named barriers order them against the writers)
    const float2 *xcht = reinterpret_cast<const float2 *>(smem + L.off_xch + w * 4 * RH * 8);
    constexpr int kXchParity = kTcWGs * 4 * RH; // float2 entries per tile parity
    const unsigned long long limit = wait_limit(p);
    bool dead = false;

    // both score buffers start from the bias pattern and this warpgroup's PV columns from
    // zero; then the first two QKs may go ahead
#pragma unroll
    for (int bj = 0; bj < 8; ++bj)
        tc_fill<RH>(tlane + (uint32_t)(bj * R + r0), (uint32_t)kDotBias);
    tc_fill<4 * RH>(tOw, 0u);
    tc_wait_st();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) {
        mbar_arrive(&bars[kSFree + 0]);
        mbar_arrive(&bars[kSFree + 1]);
    }

    float Spart[RH], acc[RH];
    float Mrow = -INFINITY, Arow = -INFINITY; // row `lane`'s state (lanes < RH, every warp)
    bool seed_pending = false; // this tile's score columns re-seeded, sfree not yet signalled
    int seed_buf = 0;
    int stage = 0;
    uint32_t phase = 0, kst = 0;
    int sn = 0;
#pragma unroll 1
    for (int x = t0; x < t1; ++sn) {
        const SegCursor cu = cursor_at(p, prefix, x);
        const int x_end = cu.seg1 < t1 ? cu.seg1 : t1;
        const int qslot = sn & 1;
        const float *qst = reinterpret_cast<const float *>(smem + L.off_qs) + qslot * 4 * R + r0;
        const int scol = cu.hc % p.sc_heads;
#pragma unroll
        for (int i = 0; i < RH; ++i) {
            Spart[i] = 0.f;
            acc[i] = 0.f;
        }
        Mrow = -INFINITY;
        Arow = -INFINITY;
        bool ofresh = true, had = false;
        int since_fold = 0;
#pragma unroll 1
        for (; x < x_end; ++x) {
            const int tok0 = (x - cu.seg0) * kTcTT;
            const int nvalid = min(kTcTT, cu.L - tok0);
            const int buf = (int)(kst & 1u);
            if (!dead && (!mbar_wait(&full[stage], phase, limit) ||
                          !mbar_wait(&bars[kSFull + buf], (kst >> 1) & 1u, limit))) {
                dead = true;
                atomicOr(p.errors, kErrTimeout);
            }
            float s[RH];
            float lvs = -INFINITY, vsv = 0.f;
            if (!dead) {
                tc_fence_after();
                const uint8_t *sb = smem + (size_t)stage * p.lay.stage_bytes;
                const int loaded = reinterpret_cast<const int *>(smem + p.lay.off_mask)[stage];
                const bool valid = tt < nvalid && ((loaded >> (tt >> p.log2_box)) & 1);
                // a box that was not loaded holds whatever shared memory held before: its
                // scales must not reach the maxima or the weights
                const int sci = tt * p.sc_heads + scol;
                const float kss = reinterpret_cast<const float *>(sb + p.lay.off_ks)[sci];
                vsv = valid ? reinterpret_cast<const float *>(sb + p.lay.off_vs)[sci] : 0.f;
                lvs = __log2f(vsv);
                const float pen = valid ? 0.f : -INFINITY; // masks the token in one FFMA
                const uint32_t tS = tlane + (uint32_t)(buf * 4 * R + r0);
                uint32_t F[4 * RH];
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    tc_ld<RH>(tS + (uint32_t)(j * R), F + j * RH);
                tc_wait_ld();
#pragma unroll
                for (int i = 0; i < RH; ++i)
                    s[i] = 0.f;
#pragma unroll
                for (int j = 0; j < 4; ++j)
#pragma unroll
                    for (int i4 = 0; i4 < RH / 4; ++i4) {
                        const float4 qv = *reinterpret_cast<const float4 *>(qst + j * R + 4 * i4);
                        const uint32_t *f = F + j * RH + 4 * i4;
                        s[4 * i4 + 0] = fmaf(qv.x, __uint_as_float(f[0]) - kDotBiasF, s[4 * i4 + 0]);
                        s[4 * i4 + 1] = fmaf(qv.y, __uint_as_float(f[1]) - kDotBiasF, s[4 * i4 + 1]);
                        s[4 * i4 + 2] = fmaf(qv.z, __uint_as_float(f[2]) - kDotBiasF, s[4 * i4 + 2]);
                        s[4 * i4 + 3] = fmaf(qv.w, __uint_as_float(f[3]) - kDotBiasF, s[4 * i4 + 3]);
                    }
                // re-seed this warpgroup's score columns for tile k + 2; they are released
                // (sfree) at the end of the tile, once the stores have completed
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    tc_fill<RH>(tS + (uint32_t)(j * R), (uint32_t)kDotBias);
                seed_pending = true;
                seed_buf = buf;
#pragma unroll
                for (int i = 0; i < RH; ++i)
                    s[i] = fmaf(s[i], kss, pen);
                if (R > p.G) { // padding rows
#pragma unroll
                    for (int i = 0; i < RH; ++i)
                        if (r0 + i >= p.G)
                            s[i] = -INFINITY;
                }
                // with several query tokens, row r sees tokens before L - (nq - 1 - r / Gq)
                if (tok0 + kTcTT > cu.L - (p.nq - 1)) {
                    const int tok = tok0 + tt;
#pragma unroll
                    for (int i = 0; i < RH; ++i)
                        if (r0 + i < p.G && tok >= cu.L - (p.nq - 1 - (r0 + i) / p.Gq))
                            s[i] = -INFINITY;
                }
            } else {
#pragma unroll
                for (int i = 0; i < RH; ++i)
                    s[i] = -INFINITY;
            }
            // tile maxima of s and s + log2 vs per row (warp-uniform results, stored by lane 0)
            float km[RH], ka[RH];
#pragma unroll
            for (int i = 0; i < RH; ++i) {
                km[i] = warp_max(s[i]);
                ka[i] = warp_max(s[i] + lvs);
            }
            const int xp = buf * kXchParity; // tile parity: a warp is at most one tile ahead
            if (lane == 0) {
                float2 *xw = reinterpret_cast<float2 *>(smem + L.off_xch) + xp + (w * 4 + q4) * RH;
#pragma unroll
                for (int i = 0; i < RH; ++i)
                    xw[i] = make_float2(km[i], ka[i]);
            }
            wg_bar(w);
            // every warp updates the row state from the same maxima (lane i: row i)
            float Ms = 0.f, cM = 1.f, g = 0.f, fa = 1.f;
            bool rose = false;
            {
                if (lane < RH) {
                    float mst = -INFINITY, ast = -INFINITY;
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const float2 v = xcht[xp + q * RH + lane];
                        mst = fmaxf(mst, v.x);
                        ast = fmaxf(ast, v.y);
                    }
                    const float Mn = fmaxf(Mrow, mst);
                    // the reference moves when this tile's largest score + log2 vs exceeds
                    // it by more than the headroom
                    float An = (Arow == -INFINITY || ast > Arow + kTcAHead) ? ast : Arow;
                    // 2^(M - A + 19) must stay finite: with V scales more than 2^104 below
                    // the weight of the top-scoring token the reference A is raised to
                    // M - 104 (the weights of that row then keep fewer significant bits)
                    if (An != -INFINITY && Mn - An > 104.f)
                        An = Mn - 104.f;
                    cM = Mrow == -INFINITY ? 1.f : fast_exp2(Mrow - Mn);
                    fa = Arow == -INFINITY ? 1.f : fast_exp2(Arow - An);
                    g = An == -INFINITY ? 0.f : fast_exp2(Mn - An + (22.f - kTcAHead));
                    Ms = Mn == -INFINITY ? 0.f : Mn;
                    rose = An != Arow && Arow != -INFINITY;
                    Mrow = Mn;
                    Arow = An;
                }
            }
            const bool fold = __any_sync(kFullMask, rose) || since_fold >= kTcFoldEvery;

            // weights: w = 2^(s - M) into the row sums, P = w vs 2^(M - A + 19) < 2^23 as an
            // integer in the low mantissa bits of P + 2^23
            uint32_t bits[RH];
#pragma unroll
            for (int i = 0; i < RH; ++i) {
                const float wv = fast_exp2(s[i] - __shfl_sync(kFullMask, Ms, i));
                Spart[i] = fmaf(Spart[i], __shfl_sync(kFullMask, cM, i), wv);
                bits[i] = __float_as_uint(fmaf(wv * vsv, __shfl_sync(kFullMask, g, i), kTwo23F));
            }
            // weight buffer k & 1 was read by tile k - 2's PV; a fold also needs tile k - 1's
            if (!dead && kst >= 2 &&
                !mbar_wait(&bars[kPvDone + buf], ((kst >> 1) - 1u) & 1u, limit)) {
                dead = true;
                atomicOr(p.errors, kErrTimeout);
            }
            if (fold && !dead) {
                if (kst >= 1 &&
                    !mbar_wait(&bars[kPvDone + (buf ^ 1)], ((kst - 1u) >> 1) & 1u, limit)) {
                    dead = true;
                    atomicOr(p.errors, kErrTimeout);
                } else {
                    tc_fence_after();
                    tc_fold<R>(acc, tOw, fa, !ofresh, true);
                    ofresh = true;
                    since_fold = 0;
                }
            }
            // the weight words of this warpgroup's rows: 4 rows (16 byte columns) per 16-byte
            // store (MN-major, 8-token core rows)
            const uint32_t pb = sbase + pofs + (uint32_t)buf * 4u * tc_p_kstep_bytes(R);
#pragma unroll
            for (int c = 0; c < RH / 4; ++c)
                sts128(pb + (uint32_t)c * 512u, bits[4 * c], bits[4 * c + 1], bits[4 * c + 2],
                       bits[4 * c + 3]);
            ofresh = false;
            ++since_fold;
            fence_proxy_async_smem();
            tc_wait_st(); // the score re-seed (and a fold's zeroing) has landed
            tc_fence_before();
            __syncwarp();
            if (!dead && lane == 0) {
                if (seed_pending)
                    mbar_arrive(&bars[kSFree + seed_buf]);
                mbar_arrive(&bars[kPReady + buf]);
            }
            seed_pending = false;
            ++kst;
            had = true;
            if (++stage == p.n_stages) {
                stage = 0;
                phase ^= 1u;
            }
        }

        // segment end: the last PV folded in (columns zeroed), row sums completed, rows
        // written (or the partial)
        if (had && !dead) {
            if (!mbar_wait(&bars[kPvDone + ((kst - 1u) & 1u)], ((kst - 1u) >> 1) & 1u,
                           limit)) {
                dead = true;
                atomicOr(p.errors, kErrTimeout);
            } else if (!ofresh) {
                tc_fence_after();
                tc_fold<R>(acc, tOw, 1.f, true, false);
                tc_wait_st();
                tc_fence_before();
            }
        }
        const float ssum = tc_row_sums<RH>(Spart, lane);
        wg_bar(w); // the last tile's maxima have been read
        if (lane < RH)
            sts_f32(xch + 8u * (uint32_t)(q4 * RH + lane), ssum);
        wg_bar(w);
        const int pre = prefix[cu.b];
        const int ntb = (prefix[cu.b + 1] - pre) / p.nhc;
        const int seg0 = pre + cu.hc * ntb, seg1 = seg0 + ntb;
        const bool complete = seg0 >= t0 && seg1 <= t1;
        float *slotp =
            p.partials + (size_t)(2 * blockIdx.x + ((seg0 <= t0) ? 0 : 1)) * p.heads_seg * kSlotRow;
        if (owner) {
            float S = 0.f;
#pragma unroll
            for (int q = 0; q < 4; ++q)
                S += lds_f32(xch + 8u * (uint32_t)(q * RH + lane));
            float f = 1.f;
            if (complete)
                f = (S > 0.f && Arow != -INFINITY) ? exp2f(Arow - Mrow) / S : 0.f;
            else if (r0 + lane < p.G)
                *reinterpret_cast<float4 *>(slotp + (size_t)(r0 + lane) * kSlotRow + kD) =
                    make_float4(Mrow, S, Arow, 0.f);
            sts_f32(rowi + 16u * lane, f);
        }
        wg_bar(w);
        if (!dead) {
#pragma unroll
            for (int i = 0; i < RH; ++i) {
                if (r0 + i < p.G) {
                    if (complete)
                        p.out[q_row(p, cu.b, cu.hc, r0 + i) * kD + tt] =
                            acc[i] * lds_f32(rowi + 16u * i);
                    else
                        slotp[(size_t)(r0 + i) * kSlotRow + tt] = acc[i];
                }
            }
        }
        wg_bar(w); // the sums and the row table are rewritten at the next segment end
        __syncwarp();
        if (lane == 0)
            mbar_arrive(&bars[kQFree + qslot]);
    }
}

// ------------------------------------------------------------------ the kernel

template <int R>
__global__ void __launch_bounds__(kTcThreads, 1)
    mq_tc_kernel(const __grid_constant__ DecodeParams p, const __grid_constant__ CUtensorMap tmK,
                 const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmKs,
                 const __grid_constant__ CUtensorMap tmVs)
{
    static_assert(R == 16 || R == 32, "rows per KV head: 16 or 32");
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte aligned base, kept as an offset from the shared array so that loads through
    // it stay shared-memory loads
    uint8_t *smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const TcLayout L = tc_layout(p.lay.total, R);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + p.lay.off_full);
    uint64_t *empty = reinterpret_cast<uint64_t *>(smem + p.lay.off_empty);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L.off_bar);
    int *prefix = reinterpret_cast<int *>(smem + p.lay.off_prefix);

    if (tid == 0) {
        for (int s = 0; s < p.n_stages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1); // the tile's PV commit
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bars[kSFull + b], 1);
            mbar_init(&bars[kSFree + b], kTcConsumerWarps);
            mbar_init(&bars[kPReady + b], kTcConsumerWarps);
            mbar_init(&bars[kPvDone + b], 1);
            mbar_init(&bars[kQReady + b], 1);
            mbar_init(&bars[kQFree + b], kTcConsumerWarps);
        }
        mbar_init(&bars[kFinal], 2);
        fence_mbar_init();
    }
    if (warp == kTcProducerWarp && lane == 0) {
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
        if (!p.scale_bulk) {
            tma_prefetch_desc(&tmKs);
            tma_prefetch_desc(&tmVs);
        }
    }
    if (warp == kTcQkWarp) { // one CTA per SM (shared memory), so this never waits
        tc_alloc(smem_addr(smem + L.off_tmem), kTcCols);
        tc_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *reinterpret_cast<volatile uint32_t *>(smem + L.off_tmem);
    grid_dep_wait();
    grid_dep_launch();
    int *nseq = p.lay.off_nseq ? reinterpret_cast<int *>(smem + p.lay.off_nseq) : nullptr;
    int *cstart = reinterpret_cast<int *>(smem + p.lay.off_cstart);

    if (warp >= kTcConsumerWarps) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kTcHelperRegs));
        if (warp == kTcProducerWarp) {
            const int *pre = prefix;
            const int *pns = nseq;
            if (p.B <= 32) {
                int *pp = reinterpret_cast<int *>(smem + p.lay.off_pscan);
                scan_one_warp(p, pp, pp + kPscanLen, lane);
                __syncwarp();
                pre = pp;
                pns = pp + kPscanLen;
            } else {
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
        // warps 17-19: the consumers publish the prefixes and this CTA's range
        asm volatile("bar.sync %0, %1;" ::"n"(kTcBarHelpers), "n"(kTcHelperThreads) : "memory");
        const Split sp = split_of(p, prefix, nseq, (int)gridDim.x);
        const bool has = sp.gcta > 0 && (int)blockIdx.x < sp.gcta;
        const int t0 = has ? cstart[blockIdx.x] : 0, t1 = has ? cstart[blockIdx.x + 1] : 0;
        if (warp == kTcQkWarp) {
            if (lane == 0)
                tc_issue_qk<R>(p, smem, L, tbase, prefix, t0, t1);
            __syncwarp();
            // both issuers' MMAs have completed (kFinal), and the consumers are done
            if (lane == 0 && !mbar_wait(&bars[kFinal], 0, wait_limit(p)))
                atomicOr(p.errors, kErrTimeout);
            __syncwarp();
            asm volatile("bar.sync %0, %1;" ::"n"(kTcBarTeardown), "n"(kTcTeardownThreads)
                         : "memory");
            tc_fence_after();
            tc_dealloc(tbase, kTcCols);
        } else if (warp == kTcPvWarp) {
            if (lane == 0)
                tc_issue_pv<R>(p, smem, L, tbase, t1 - t0);
        } else if (warp == kTcPrepWarp && has) {
            tc_prepare_queries<R>(p, smem, L, prefix, t0, t1, lane);
        }
        return;
    }
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kTcConsumerRegs));
    const int ctid = warp * 32 + lane;
    // warps 0-7 scan the sequence lengths and publish this CTA's range (the prefix code of
    // the single-query kernel, written for its 8 consumer warps)
    if (warp < kConsumerWarps) {
        build_prefix(p, prefix, nseq,
                     reinterpret_cast<volatile unsigned long long *>(smem + p.lay.off_misc),
                     ctid, warp, lane);
        consumer_bar();
        const Split sp = split_of(p, prefix, nseq, (int)gridDim.x);
        if (sp.gcta > 0 && ctid < 2 && (int)blockIdx.x + ctid <= sp.gcta)
            cstart[blockIdx.x + ctid] =
                cta_start(p, prefix, nseq, sp.pseg, sp.V, sp.gcta, (int)blockIdx.x + ctid);
        consumer_bar();
        if (p.B > 32)
            asm volatile("bar.arrive 2, %0;" ::"n"(kConsumerThreads + 32) : "memory");
    }
    asm volatile("bar.sync %0, %1;" ::"n"(kTcBarAll), "n"(kTcConsumerThreads) : "memory");
    asm volatile("bar.arrive %0, %1;" ::"n"(kTcBarHelpers), "n"(kTcHelperThreads) : "memory");
    const Split sp = split_of(p, prefix, nseq, (int)gridDim.x);
    const int gcta = sp.gcta;
    if (gcta > 0 && (int)blockIdx.x < gcta) {
        const int t0 = cstart[blockIdx.x], t1 = cstart[blockIdx.x + 1];
        // the first segment's query rows (later ones: warp 19)
        tc_quantize_query<R>(p, smem, L, cursor_at(p, prefix, t0), 0, ctid, kTcConsumerThreads);
        fence_proxy_async_smem();
        asm volatile("bar.sync %0, %1;" ::"n"(kTcBarAll), "n"(kTcConsumerThreads) : "memory");
        if (ctid == 0)
            mbar_arrive(&bars[kQReady + 0]);
        // rows of empty sequences are zero (spread over the CTAs that have tiles)
#pragma unroll 1
        for (int b = blockIdx.x; b < p.B; b += gcta) {
            if (prefix[b + 1] != prefix[b])
                continue;
            float4 *row = reinterpret_cast<float4 *>(p.out + (long long)b * p.nq * p.Hq * kD);
#pragma unroll 1
            for (int i = ctid; i < p.nq * p.Hq * kD / 4; i += kTcConsumerThreads)
                row[i] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        tc_consume<R>(p, smem, L, tbase, prefix, t0, t1, warp, lane);
    } else if (gcta == 0) {
#pragma unroll 1
        for (int b = blockIdx.x; b < p.B; b += gridDim.x) {
            float4 *row = reinterpret_cast<float4 *>(p.out + (long long)b * p.nq * p.Hq * kD);
#pragma unroll 1
            for (int i = ctid; i < p.nq * p.Hq * kD / 4; i += kTcConsumerThreads)
                row[i] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }
    tc_fence_before();
    asm volatile("bar.arrive %0, %1;" ::"n"(kTcBarTeardown), "n"(kTcTeardownThreads)
                 : "memory");
}

} // namespace q8kv
