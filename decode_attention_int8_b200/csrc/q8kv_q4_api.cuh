// q8kv_q4_api.cuh -- host side of q8kv_decode_attn_q4 (include/q8kv.h): argument checks,
// the chunk workspace and the launches of q4_decode_kernel and q4_combine_kernel.
// Included at the end of q8kv_api.cu, whose device bookkeeping it uses.
#pragma once

#include "q8kv_q4.cuh"

namespace {

using namespace q8kv;

struct Q4Workspace {
    void *ptr = nullptr;
    size_t bytes = 0;
    bool attr_set = false;
};

Q4Workspace g_q4[kMaxDevices];

template <int GT>
cudaError_t q4_set_smem()
{
    return cudaFuncSetAttribute(q4_decode_kernel<GT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)q4_smem_bytes<GT>());
}

// The instantiation for groups up to GT (a power of two): heads G..GT-1 are padding.
template <int GT>
cudaError_t q4_launch(cudaLaunchConfig_t cfg, const Q4Params &p)
{
    cfg.dynamicSmemBytes = q4_smem_bytes<GT>();
    return cudaLaunchKernelEx(&cfg, q4_decode_kernel<GT>, p);
}

} // namespace

extern "C" {

q8kv_status q8kv_decode_attn_q4(float *out, const float *q, const uint8_t *k4_blocks,
                                const uint8_t *v4_blocks, const uint16_t *kd,
                                const uint16_t *vd, const int32_t *block_table,
                                const int32_t *seq_lens, int B, int n_q_heads, int n_kv_heads,
                                int head_dim, int kv_block_size, int max_blocks_per_seq,
                                int num_kv_blocks, float scale, cudaStream_t stream)
{
    if (!out || !q || !k4_blocks || !v4_blocks || !kd || !vd || !block_table || !seq_lens)
        return Q8KV_ERR_INVALID_ARG;
    if (B <= 0 || n_q_heads <= 0 || n_kv_heads <= 0 || head_dim <= 0 || head_dim % 32 != 0 ||
        kv_block_size <= 0 || max_blocks_per_seq <= 0 || num_kv_blocks <= 0 ||
        n_q_heads % n_kv_heads != 0 || !std::isfinite(scale))
        return Q8KV_ERR_INVALID_ARG;
    if (!aligned16(out) || !aligned16(q) || !aligned16(k4_blocks) || !aligned16(v4_blocks) ||
        (reinterpret_cast<uintptr_t>(kd) & 7u) != 0 || (reinterpret_cast<uintptr_t>(vd) & 7u) != 0)
        return Q8KV_ERR_INVALID_ARG;
    const int G = n_q_heads / n_kv_heads;
    if (head_dim != kD || G > kQ4MaxG || (long long)B * n_kv_heads > 65535 ||
        (long long)max_blocks_per_seq * kv_block_size >= (1LL << 31) ||
        (long long)num_kv_blocks * kv_block_size >= (1LL << 31))
        return Q8KV_ERR_UNSUPPORTED;
    const long long n_chunks = ((long long)max_blocks_per_seq * kv_block_size + kQ4Chunk - 1) /
                               kQ4Chunk;
    const size_t ws_need =
        sizeof(float) * (size_t)B * n_kv_heads * (size_t)n_chunks * G * kQ4SlotRow;
    DeviceInfo *dev = nullptr;
    q8kv_status st;
    Q4Workspace *ws = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_mutex);
        st = device_info(&dev);
        if (st != Q8KV_OK)
            return st;
        int d = 0;
        Q8KV_CUDA(cudaGetDevice(&d));
        ws = &g_q4[d];
        if (ws->bytes < ws_need) {
            if (ws->ptr) {
                Q8KV_CUDA(cudaFree(ws->ptr));
                ws->ptr = nullptr;
                ws->bytes = 0;
            }
            Q8KV_CUDA(cudaMalloc(&ws->ptr, ws_need));
            ws->bytes = ws_need;
        }
        if (!ws->attr_set) {
            Q8KV_CUDA(q4_set_smem<1>());
            Q8KV_CUDA(q4_set_smem<2>());
            Q8KV_CUDA(q4_set_smem<4>());
            Q8KV_CUDA(q4_set_smem<8>());
            Q8KV_CUDA(q4_set_smem<16>());
            ws->attr_set = true;
        }
    }
    Q4Params p;
    p.out = out;
    p.q = q;
    p.k4 = k4_blocks;
    p.v4 = v4_blocks;
    p.kd = kd;
    p.vd = vd;
    p.block_table = block_table;
    p.seq_lens = seq_lens;
    p.partials = static_cast<float *>(ws->ptr);
    p.errors = dev->errors;
    p.B = B;
    p.Hq = n_q_heads;
    p.Hk = n_kv_heads;
    p.G = G;
    p.bs = kv_block_size;
    p.log2_bs = -1;
    if ((kv_block_size & (kv_block_size - 1)) == 0)
        for (p.log2_bs = 0; (1 << p.log2_bs) < kv_block_size; ++p.log2_bs) {
        }
    p.mbps = max_blocks_per_seq;
    p.num_blocks = num_kv_blocks;
    p.n_chunks = (int)n_chunks;
    p.scale_log2 = (float)((double)scale * 1.4426950408889634);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)n_chunks, (unsigned)(B * n_kv_heads));
    cfg.blockDim = dim3(kQ4Threads);
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (G <= 1)
        Q8KV_CUDA(q4_launch<1>(cfg, p));
    else if (G <= 2)
        Q8KV_CUDA(q4_launch<2>(cfg, p));
    else if (G <= 4)
        Q8KV_CUDA(q4_launch<4>(cfg, p));
    else if (G <= 8)
        Q8KV_CUDA(q4_launch<8>(cfg, p));
    else
        Q8KV_CUDA(q4_launch<16>(cfg, p));
    cudaLaunchConfig_t cc = cfg;
    cc.gridDim = dim3((unsigned)(((long long)B * n_q_heads + 7) / 8));
    cc.blockDim = dim3(256);
    cc.dynamicSmemBytes = 0;
    Q8KV_CUDA(cudaLaunchKernelEx(&cc, q4_combine_kernel, p));
    return Q8KV_OK;
}

} // extern "C"
