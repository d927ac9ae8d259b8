// q8kv_qquant.cuh -- the Q quantisation step, shared by the decode kernel's prologue and
// the debug entry point.
//
// Kestrel-LLM walk-through "flash_attn_single_q_q8_neon" (trdm.cn/news/511694), section 2
// part 1: each 32-element block of q gets qm = max|q| (qm = 1 when qm < 1e-6, so an
// all-zero block quantises to zeros), a scale qsc = qm * (1/127) and codes
// q * (127 / qm), which this library rounds half-to-even and clamps to [-127, 127].
// Every operation is an explicitly rounded IEEE fp32 operation (no fast-math, no FMA
// contraction), so the codes are a deterministic function of q.
#pragma once

#include <cstdint>

namespace q8kv {

constexpr unsigned kFullMask = 0xffffffffu;

// A quad of 4 consecutive lanes (lane bits 0-1) holds one 32-element block, 8 values per
// lane. Returns this lane's 8 codes packed little-endian into two words and the block's
// scale (same value in all 4 lanes). All 32 lanes of the warp must call it.
__device__ __forceinline__ void quantize_block_quad(const float (&v)[8], uint32_t &lo,
                                                    uint32_t &hi, float &qsc)
{
    float qm = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i)
        qm = fmaxf(qm, fabsf(v[i]));
    qm = fmaxf(qm, __shfl_xor_sync(kFullMask, qm, 1));
    qm = fmaxf(qm, __shfl_xor_sync(kFullMask, qm, 2));
    if (qm < 1e-6f)
        qm = 1.0f;
    qsc = __fmul_rn(qm, 1.0f / 127.0f);
    const float iq = __fdiv_rn(127.0f, qm);
    uint32_t w[2] = {0u, 0u};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        int r = __float2int_rn(__fmul_rn(v[i], iq));
        r = max(-127, min(127, r));
        w[i >> 2] |= (uint32_t)(r & 0xff) << (8 * (i & 3));
    }
    lo = w[0];
    hi = w[1];
}

// Debug kernel: quantise n_blocks consecutive 32-element blocks of q.
// Thread t handles values [8 * (t % 4), 8 * (t % 4) + 8) of block t / 4.
__global__ void qquant_debug_kernel(int8_t *__restrict__ qi, float *__restrict__ qsc,
                                    const float *__restrict__ q, long long n_blocks)
{
    const long long tid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const long long blk = tid >> 2;
    const int part = (int)(tid & 3);
    const bool live = blk < n_blocks;
    float v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
        v[i] = live ? q[blk * 32 + part * 8 + i] : 0.0f;
    uint32_t lo, hi;
    float s;
    quantize_block_quad(v, lo, hi, s);
    if (live) {
        uint2 packed = make_uint2(lo, hi);
        *reinterpret_cast<uint2 *>(qi + blk * 32 + part * 8) = packed;
        if (part == 0)
            qsc[blk] = s;
    }
}

} // namespace q8kv
