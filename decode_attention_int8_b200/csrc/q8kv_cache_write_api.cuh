// q8kv_cache_write_api.cuh -- host side of q8kv_cache_write (include/q8kv.h): argument
// checks and the launch of cache_write_kernel. Included at the end of q8kv_api.cu, whose
// device bookkeeping (device_info, the error word, the CUDA error helpers) it uses.
#pragma once

#include "q8kv_cache_write.cuh"

namespace {

using namespace q8kv;

static_assert(kErrSlot == Q8KV_DEVERR_SLOT && kErrNonFinite == Q8KV_DEVERR_NONFINITE,
              "device error bits differ from the header");

template <int D>
q8kv_status launch_cache_write(const CacheWriteParams &p, int sms, cudaStream_t stream)
{
    // one full wave of resident blocks, striding over the (token, head) pairs
    const long long per_block = (long long)kWriteWarps * write_pairs_per_warp(D);
    const long long want = (p.n_tokens * p.Hk + per_block - 1) / per_block;
    const long long cap = (long long)write_blocks_per_sm(D) * sms;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(want < cap ? want : cap));
    cfg.blockDim = dim3(kWriteThreads);
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    Q8KV_CUDA(cudaLaunchKernelEx(&cfg, cache_write_kernel<D>, p));
    return Q8KV_OK;
}

template <int D>
q8kv_status launch_cache_write_q4(const CacheWriteQ4Params &p, int sms, cudaStream_t stream)
{
    const long long per_block = (long long)kWriteWarps * write_pairs_per_warp(D);
    const long long want = (p.n_tokens * p.Hk + per_block - 1) / per_block;
    const long long cap = (long long)write_blocks_per_sm(D) * sms;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(want < cap ? want : cap));
    cfg.blockDim = dim3(kWriteThreads);
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    Q8KV_CUDA(cudaLaunchKernelEx(&cfg, cache_write_q4_kernel<D>, p));
    return Q8KV_OK;
}

} // namespace

extern "C" {

q8kv_status q8kv_cache_write(int8_t *k_blocks, int8_t *v_blocks, float *kscale, float *vscale,
                             const float *k_new, const float *v_new,
                             const int64_t *slot_mapping, int n_tokens, int n_kv_heads,
                             int head_dim, int kv_block_size, int num_kv_blocks,
                             long long token_stride, cudaStream_t stream)
{
    if (!k_blocks || !v_blocks || !kscale || !vscale)
        return Q8KV_ERR_INVALID_ARG;
    if (n_tokens < 0 || n_kv_heads <= 0 || head_dim <= 0 || head_dim % 32 != 0 ||
        kv_block_size <= 0 || num_kv_blocks <= 0)
        return Q8KV_ERR_INVALID_ARG;
    const long long row = (long long)n_kv_heads * head_dim;
    if (token_stride == 0)
        token_stride = row;
    if (token_stride < row || token_stride % 4 != 0)
        return Q8KV_ERR_INVALID_ARG;
    if (!aligned16(k_blocks) || !aligned16(v_blocks) ||
        (reinterpret_cast<uintptr_t>(kscale) & 3u) != 0 ||
        (reinterpret_cast<uintptr_t>(vscale) & 3u) != 0)
        return Q8KV_ERR_INVALID_ARG;
    if (head_dim != 64 && head_dim != 128 && head_dim != 256)
        return Q8KV_ERR_UNSUPPORTED;
    if (n_tokens == 0) // nothing to write (the row pointers may be null)
        return Q8KV_OK;
    if (!k_new || !v_new || !slot_mapping || !aligned16(k_new) || !aligned16(v_new) ||
        (reinterpret_cast<uintptr_t>(slot_mapping) & 7u) != 0)
        return Q8KV_ERR_INVALID_ARG;
    DeviceInfo *dev = nullptr;
    q8kv_status st;
    {
        std::lock_guard<std::mutex> lock(g_mutex);
        st = device_info(&dev);
    }
    if (st != Q8KV_OK)
        return st;
    CacheWriteParams p;
    p.k = k_blocks;
    p.v = v_blocks;
    p.ks = kscale;
    p.vs = vscale;
    p.k_new = k_new;
    p.v_new = v_new;
    p.slots = slot_mapping;
    p.n_tokens = n_tokens;
    p.token_stride = token_stride;
    p.n_slots = (long long)num_kv_blocks * kv_block_size;
    p.Hk = n_kv_heads;
    p.errors = dev->errors;
    if (head_dim == 64)
        return launch_cache_write<64>(p, dev->sms, stream);
    if (head_dim == 128)
        return launch_cache_write<128>(p, dev->sms, stream);
    return launch_cache_write<256>(p, dev->sms, stream);
}

q8kv_status q8kv_cache_write_q4(uint8_t *k4_blocks, uint8_t *v4_blocks, uint16_t *kd,
                                uint16_t *vd, const float *k_new, const float *v_new,
                                const int64_t *slot_mapping, int n_tokens, int n_kv_heads,
                                int head_dim, int kv_block_size, int num_kv_blocks,
                                long long token_stride, cudaStream_t stream)
{
    if (!k4_blocks || !v4_blocks || !kd || !vd)
        return Q8KV_ERR_INVALID_ARG;
    if (n_tokens < 0 || n_kv_heads <= 0 || head_dim <= 0 || head_dim % 32 != 0 ||
        kv_block_size <= 0 || num_kv_blocks <= 0)
        return Q8KV_ERR_INVALID_ARG;
    const long long row = (long long)n_kv_heads * head_dim;
    if (token_stride == 0)
        token_stride = row;
    if (token_stride < row || token_stride % 4 != 0)
        return Q8KV_ERR_INVALID_ARG;
    // code rows are head_dim / 2 bytes, scale rows head_dim / 16 bytes: 2-byte stores
    if ((reinterpret_cast<uintptr_t>(k4_blocks) & 15u) != 0 ||
        (reinterpret_cast<uintptr_t>(v4_blocks) & 15u) != 0 ||
        (reinterpret_cast<uintptr_t>(kd) & 7u) != 0 ||
        (reinterpret_cast<uintptr_t>(vd) & 7u) != 0)
        return Q8KV_ERR_INVALID_ARG;
    if (head_dim != 64 && head_dim != 128 && head_dim != 256)
        return Q8KV_ERR_UNSUPPORTED;
    if (n_tokens == 0)
        return Q8KV_OK;
    if (!k_new || !v_new || !slot_mapping || !aligned16(k_new) || !aligned16(v_new) ||
        (reinterpret_cast<uintptr_t>(slot_mapping) & 7u) != 0)
        return Q8KV_ERR_INVALID_ARG;
    DeviceInfo *dev = nullptr;
    q8kv_status st;
    {
        std::lock_guard<std::mutex> lock(g_mutex);
        st = device_info(&dev);
    }
    if (st != Q8KV_OK)
        return st;
    CacheWriteQ4Params p;
    p.k4 = k4_blocks;
    p.v4 = v4_blocks;
    p.kd = kd;
    p.vd = vd;
    p.k_new = k_new;
    p.v_new = v_new;
    p.slots = slot_mapping;
    p.n_tokens = n_tokens;
    p.token_stride = token_stride;
    p.n_slots = (long long)num_kv_blocks * kv_block_size;
    p.Hk = n_kv_heads;
    p.errors = dev->errors;
    if (head_dim == 64)
        return launch_cache_write_q4<64>(p, dev->sms, stream);
    if (head_dim == 128)
        return launch_cache_write_q4<128>(p, dev->sms, stream);
    return launch_cache_write_q4<256>(p, dev->sms, stream);
}

} // extern "C"
