// q8kv_quest_api.cuh -- host side of q8kv_quest_metadata (include/q8kv.h): argument checks
// and the launch of quest_metadata_kernel. Included at the end of q8kv_api.cu, whose device
// bookkeeping (device_info, the error word, the CUDA error helpers) it uses.
#pragma once

#include "q8kv_quest.cuh"

namespace {

using namespace q8kv;

static_assert(kErrMeta == Q8KV_DEVERR_META, "device error bits differ from the header");

} // namespace

extern "C" {

q8kv_status q8kv_quest_metadata(float *maxblocks, float *minblocks, const int8_t *k_blocks,
                                const float *kscale, const int32_t *block_table,
                                const int32_t *seq_lens, const int32_t *meta_block_table, int B,
                                int n_kv_heads, int head_dim, int kv_block_size,
                                int max_blocks_per_seq, int max_meta_blocks_per_seq,
                                int num_kv_blocks, int num_meta_blocks, cudaStream_t stream)
{
    if (!maxblocks || !minblocks || !k_blocks || !kscale || !block_table || !seq_lens ||
        !meta_block_table)
        return Q8KV_ERR_INVALID_ARG;
    if (B <= 0 || n_kv_heads <= 0 || head_dim <= 0 || kv_block_size <= 0 ||
        max_blocks_per_seq <= 0 || max_meta_blocks_per_seq <= 0 || num_kv_blocks <= 0 ||
        num_meta_blocks <= 0)
        return Q8KV_ERR_INVALID_ARG;
    if (!aligned16(maxblocks) || !aligned16(minblocks) || !aligned16(k_blocks) ||
        (reinterpret_cast<uintptr_t>(kscale) & 3u) != 0)
        return Q8KV_ERR_INVALID_ARG;
    if (head_dim != 128)
        return Q8KV_ERR_UNSUPPORTED;
    if ((long long)max_blocks_per_seq * kv_block_size >= (1LL << 31) ||
        (long long)num_kv_blocks * kv_block_size >= (1LL << 31) ||
        (long long)num_meta_blocks * kv_block_size >= (1LL << 31) ||
        (long long)max_meta_blocks_per_seq * kv_block_size >= (1LL << 31))
        return Q8KV_ERR_UNSUPPORTED;
    DeviceInfo *dev = nullptr;
    q8kv_status st;
    {
        std::lock_guard<std::mutex> lock(g_mutex);
        st = device_info(&dev);
    }
    if (st != Q8KV_OK)
        return st;
    QuestParams p;
    p.maxb = maxblocks;
    p.minb = minblocks;
    p.k = k_blocks;
    p.ks = kscale;
    p.block_table = block_table;
    p.seq_lens = seq_lens;
    p.meta_table = meta_block_table;
    p.B = B;
    p.Hk = n_kv_heads;
    p.bs = kv_block_size;
    p.mbps = max_blocks_per_seq;
    p.mmbpr = max_meta_blocks_per_seq;
    p.num_blocks = num_kv_blocks;
    p.num_meta = num_meta_blocks;
    p.errors = dev->errors;
    // one warp per (request, metadata row, head); one wave of resident blocks strides them
    const long long items = (long long)B * max_meta_blocks_per_seq * kv_block_size * n_kv_heads;
    const long long want = (items + kQuestWarps - 1) / kQuestWarps;
    const long long cap = (long long)kQuestBlocksPerSM * dev->sms;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(want < cap ? want : cap));
    cfg.blockDim = dim3(kQuestThreads);
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    switch (n_kv_heads) { // head counts whose batch offsets compile to immediates
    case 1: Q8KV_CUDA(cudaLaunchKernelEx(&cfg, quest_metadata_kernel<1>, p)); break;
    case 2: Q8KV_CUDA(cudaLaunchKernelEx(&cfg, quest_metadata_kernel<2>, p)); break;
    case 4: Q8KV_CUDA(cudaLaunchKernelEx(&cfg, quest_metadata_kernel<4>, p)); break;
    case 8: Q8KV_CUDA(cudaLaunchKernelEx(&cfg, quest_metadata_kernel<8>, p)); break;
    case 16: Q8KV_CUDA(cudaLaunchKernelEx(&cfg, quest_metadata_kernel<16>, p)); break;
    case 32: Q8KV_CUDA(cudaLaunchKernelEx(&cfg, quest_metadata_kernel<32>, p)); break;
    default: Q8KV_CUDA(cudaLaunchKernelEx(&cfg, quest_metadata_kernel<0>, p)); break;
    }
    return Q8KV_OK;
}

} // extern "C"
