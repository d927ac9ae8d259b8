// q8kv_api.cu -- the C ABI of include/q8kv.h: host-side argument checks, the tiling plan,
// TMA descriptors, workspace management and kernel launches.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "q8kv.h"
#include "q8kv_combine.cuh" // (includes the decode kernel)
#include "q8kv_mq_tc.cuh"
#include "q8kv_qquant.cuh"

namespace {

using namespace q8kv;

static_assert(kErrSeqLen == Q8KV_DEVERR_SEQ_LEN && kErrBlockTable == Q8KV_DEVERR_BLOCK_TABLE &&
                  kErrTimeout == Q8KV_DEVERR_TIMEOUT,
              "device error bits differ from the header");

__device__ unsigned g_device_errors = 0;

thread_local int t_last_cuda_error = 0;

q8kv_status cuda_fail(cudaError_t e)
{
    t_last_cuda_error = static_cast<int>(e);
    return Q8KV_ERR_CUDA;
}

#define Q8KV_CUDA(call)                                                                            \
    do {                                                                                           \
        cudaError_t e_ = (call);                                                                   \
        if (e_ != cudaSuccess)                                                                     \
            return cuda_fail(e_);                                                                  \
    } while (0)

constexpr int kMaxDevices = 64;

struct DeviceInfo {
    bool ready = false;
    int sms = 0;
    int smem_optin = 0;
    unsigned *errors = nullptr;      // address of g_device_errors on this device
    bool attr_set[3][2] = {{false, false}, {false, false}, {false, false}};
    bool tc_attr[2] = {false, false}; // mq_tc_kernel<16>, <32>
    bool combine_attr = false;
    void *ws = nullptr;              // library-managed workspace
    size_t ws_bytes = 0;
};

std::mutex g_mutex;
DeviceInfo g_dev[kMaxDevices];
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

q8kv_status device_info(DeviceInfo **out)
{
    int dev = 0;
    Q8KV_CUDA(cudaGetDevice(&dev));
    if (dev < 0 || dev >= kMaxDevices)
        return Q8KV_ERR_UNSUPPORTED;
    DeviceInfo &d = g_dev[dev];
    if (!d.ready) {
        Q8KV_CUDA(cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev));
        Q8KV_CUDA(cudaDeviceGetAttribute(&d.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev));
        void *addr = nullptr;
        Q8KV_CUDA(cudaGetSymbolAddress(&addr, g_device_errors));
        d.errors = static_cast<unsigned *>(addr);
        d.ready = true;
    }
    *out = &d;
    return Q8KV_OK;
}

q8kv_status encoder(PFN_cuTensorMapEncodeTiled_v12000 *fn)
{
    if (!g_encode) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        Q8KV_CUDA(cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000,
                                                   cudaEnableDefault, &q));
        if (q != cudaDriverEntryPointSuccess || !p)
            return Q8KV_ERR_CUDA;
        g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    *fn = g_encode;
    return Q8KV_OK;
}

struct Shape {
    int B, Hq, Hk, D, bs, mbps, P;
    int nq = 1; // query tokens per sequence
};

// How the work is tiled for one shape on one device.
struct Plan {
    int G, slices, NT, HPC, nhc, pairs, subtiles, TT, box_tok, log2_box, n_boxes, n_stages;
    int scale_bulk, sc_heads, heads_seg, scratch_stride, grid;
    int box_heads = 0; // KV heads per TMA box of the K / V tensor maps
    int tc_rows = 0;   // > 0: the tensor-memory kernel for this many rows per KV head
    SmemLayout lay;
    size_t smem_bytes;
    size_t ws_bytes;
};

bool is_pow2(int x)
{
    return x > 0 && (x & (x - 1)) == 0;
}

int ilog2(int x)
{
    int r = 0;
    while ((1 << (r + 1)) <= x)
        ++r;
    return r;
}

size_t align256(size_t x)
{
    return (x + 255) & ~static_cast<size_t>(255);
}

// Head tiling only (what the workspace size depends on).
q8kv_status plan_heads(int Hq, int Hk, int D, Plan &pl)
{
    if (Hq <= 0 || Hk <= 0 || D <= 0 || Hq % Hk != 0)
        return Q8KV_ERR_INVALID_ARG;
    if (D != kD)
        return Q8KV_ERR_UNSUPPORTED;
    pl.G = Hq / Hk;
    if (pl.G > 128)
        return Q8KV_ERR_UNSUPPORTED;
    pl.slices = 1;
    while (pl.slices * 16 < pl.G)
        pl.slices *= 2;
    pl.NT = (pl.G > 8) ? 2 : 1;
    const int max_hpc = kConsumerWarps / pl.slices;
    pl.HPC = 1;
    while (pl.HPC * 2 <= max_hpc && Hk % (pl.HPC * 2) == 0)
        pl.HPC *= 2;
    pl.scale_bulk = (pl.HPC == Hk) ? 1 : 0;
    // A tile with fewer heads than the cache loads its scales through a 2-D tensor map
    // whose rows (Hk * 4 bytes) and boxes (at least 4 heads: 16 bytes) must be 16-byte
    // multiples; a tile of 1 or 2 heads loads the aligned 4-head box around them.
    if (!pl.scale_bulk && Hk % 4 != 0)
        return Q8KV_ERR_UNSUPPORTED;
    pl.sc_heads = pl.scale_bulk ? pl.HPC : (pl.HPC < 4 ? 4 : pl.HPC);
    pl.nhc = Hk / pl.HPC;
    pl.pairs = pl.HPC * pl.slices;
    pl.subtiles = kConsumerWarps / pl.pairs;
    pl.TT = 16 * kSub * pl.subtiles;
    pl.heads_seg = pl.HPC * pl.G;
    pl.scratch_stride = 32 * 32 * pl.NT + 48; // acc fragments + M, S, A of 16 heads
    return Q8KV_OK;
}

// Workspace: the partial slots (2 per CTA). Every call writes the slots its combine reads
// (the combine derives which from the work split), so no part needs an initial value.
void plan_workspace(int grid, Plan &pl)
{
    pl.ws_bytes = align256(sizeof(float) * 2 * (size_t)grid * pl.heads_seg * kSlotRow);
}

q8kv_status make_plan(const Shape &s, const DeviceInfo &dev, Plan &pl)
{
    if (s.B <= 0 || s.bs <= 0 || s.mbps <= 0 || s.P <= 0 || s.nq <= 0)
        return Q8KV_ERR_INVALID_ARG;
    // the nq query tokens of a sequence share its KV tiles: the tiling sees nq * Hq rows
    if ((long long)s.nq * s.Hq > (1LL << 20))
        return Q8KV_ERR_UNSUPPORTED;
    q8kv_status st = plan_heads(s.nq * s.Hq, s.Hk, s.D, pl);
    if (st != Q8KV_OK)
        return st;
    if (!is_pow2(s.bs) || s.bs < 16 || s.bs > 256)
        return Q8KV_ERR_UNSUPPORTED;
    if (s.B > 16384 || (long long)s.P * s.bs >= (1LL << 31) ||
        (long long)s.mbps * s.bs >= (1LL << 31))
        return Q8KV_ERR_UNSUPPORTED;
    const long long tiles_per_seq = ((long long)s.mbps * s.bs + pl.TT - 1) / pl.TT;
    const long long tiles_max = (long long)s.B * pl.nhc * tiles_per_seq;
    if (tiles_max >= (1LL << 30))
        return Q8KV_ERR_UNSUPPORTED; // tile indices (and the penalised split) are 32-bit
    pl.grid = (int)(tiles_max < dev.sms ? tiles_max : dev.sms);
    // the combine kernel's dynamic shared memory (its static part is about 2 KB)
    if (combine_layout(s.B, pl.grid).total + kCombineStaticSmemMax > (uint32_t)dev.smem_optin)
        return Q8KV_ERR_UNSUPPORTED;
    pl.box_tok = pl.TT < s.bs ? pl.TT : s.bs;
    pl.log2_box = ilog2(pl.box_tok);
    pl.n_boxes = pl.TT / pl.box_tok;
    const int scratch_floats = (pl.subtiles - 1) * pl.pairs * pl.scratch_stride;
    pl.n_stages = 0;
    for (int n = kMaxStages; n >= 2; --n) {
        SmemLayout L = make_layout(pl.TT, pl.HPC, pl.sc_heads, n, s.B, scratch_floats, pl.grid);
        if ((size_t)L.total + 1024 <= (size_t)dev.smem_optin) {
            pl.n_stages = n;
            pl.lay = L;
            break;
        }
    }
    if (pl.n_stages == 0)
        return Q8KV_ERR_UNSUPPORTED;
    // The quantised query of each CTA's second segment is prepared in the prologue when the
    // buffer fits next to the stages (it never costs a stage).
    {
        const uint32_t rows = pl.G <= 4 ? 4u : 8u * (uint32_t)pl.NT;
        const uint32_t need = (uint32_t)pl.pairs * rows * kQRowBytes;
        if ((size_t)pl.lay.off_qbuf + need + 1024 <= (size_t)dev.smem_optin) {
            pl.lay.qbuf_rows = rows;
            pl.lay.total = pl.lay.off_qbuf + need;
        }
    }
    pl.smem_bytes = (size_t)pl.lay.total + 1024;
    pl.box_heads = pl.HPC;
    plan_workspace(dev.sms, pl); // sized for the full grid so one size fits all calls
    return Q8KV_OK;
}

// Rows per KV head the tensor-memory kernel (q8kv_mq_tc.cuh) takes this shape with: several
// query tokens per sequence, 9 to 32 rows (padded to 16 or 32), K / V scales that load as
// a bulk copy (one KV head) or 16-byte boxes (KV heads a multiple of 4). 0: not taken.
int tc_rows(const Shape &s)
{
    if (s.nq < 2 || s.D != kD || s.Hk <= 0 || s.Hq % s.Hk != 0)
        return 0;
    const long long rows = (long long)s.nq * (s.Hq / s.Hk);
    if (rows <= 8 || rows > 32)
        return 0;
    if (s.Hk != 1 && s.Hk % 4 != 0)
        return 0;
    return rows <= 16 ? 16 : 32;
}

// The tiling of the tensor-memory kernel: tiles of 128 tokens of one KV head, the same
// work split and partial-result slots as the single-query kernel.
q8kv_status make_plan_tc(const Shape &s, const DeviceInfo &dev, int R, Plan &pl)
{
    if (s.B <= 0 || s.bs <= 0 || s.mbps <= 0 || s.P <= 0)
        return Q8KV_ERR_INVALID_ARG;
    if (!is_pow2(s.bs) || s.bs < 16 || s.bs > 256)
        return Q8KV_ERR_UNSUPPORTED;
    if (s.B > 16384 || (long long)s.P * s.bs >= (1LL << 31) ||
        (long long)s.mbps * s.bs >= (1LL << 31))
        return Q8KV_ERR_UNSUPPORTED;
    pl.G = s.nq * (s.Hq / s.Hk);
    pl.slices = 1;
    pl.NT = 1;
    pl.HPC = 1;
    pl.nhc = s.Hk;
    pl.pairs = 1;
    pl.subtiles = 1;
    pl.TT = kTcTT;
    pl.heads_seg = pl.G;
    pl.scratch_stride = 0;
    pl.scale_bulk = (s.Hk == 1) ? 1 : 0;
    pl.sc_heads = pl.scale_bulk ? 1 : 4;
    pl.box_heads = 1;
    pl.tc_rows = R;
    const long long tiles_per_seq = ((long long)s.mbps * s.bs + pl.TT - 1) / pl.TT;
    const long long tiles_max = (long long)s.B * pl.nhc * tiles_per_seq;
    if (tiles_max >= (1LL << 30))
        return Q8KV_ERR_UNSUPPORTED;
    pl.grid = (int)(tiles_max < dev.sms ? tiles_max : dev.sms);
    if (combine_layout(s.B, pl.grid).total + kCombineStaticSmemMax > (uint32_t)dev.smem_optin)
        return Q8KV_ERR_UNSUPPORTED;
    pl.box_tok = pl.TT < s.bs ? pl.TT : s.bs;
    pl.log2_box = ilog2(pl.box_tok);
    pl.n_boxes = pl.TT / pl.box_tok;
    pl.n_stages = 0;
    for (int n = kMaxStages; n >= 2; --n) {
        SmemLayout Lb = make_layout(pl.TT, pl.HPC, pl.sc_heads, n, s.B, 0, pl.grid);
        const TcLayout Lt = tc_layout(Lb.total, R);
        if ((size_t)Lt.total + 1024 <= (size_t)dev.smem_optin) {
            pl.n_stages = n;
            pl.lay = Lb;
            pl.smem_bytes = (size_t)Lt.total + 1024;
            break;
        }
    }
    if (pl.n_stages == 0)
        return Q8KV_ERR_UNSUPPORTED;
    plan_workspace(dev.sms, pl);
    return Q8KV_OK;
}

bool aligned16(const void *p)
{
    return (reinterpret_cast<uintptr_t>(p) & 15u) == 0;
}

q8kv_status encode_maps_uncached(const Shape &s, const Plan &pl, const int8_t *k, const int8_t *v,
                        const float *ks, const float *vs, CUtensorMap *mk, CUtensorMap *mv,
                        CUtensorMap *mks, CUtensorMap *mvs)
{
    PFN_cuTensorMapEncodeTiled_v12000 enc;
    q8kv_status st = encoder(&enc);
    if (st != Q8KV_OK)
        return st;
    const cuuint64_t slots = (cuuint64_t)s.P * s.bs;
    // K/V pool viewed as (channel, slot, kv head): the box lands in shared memory as
    // [kv head][token][128 channels], 128-byte swizzled.
    cuuint64_t dims[3] = {(cuuint64_t)kD, slots, (cuuint64_t)s.Hk};
    cuuint64_t strides[2] = {(cuuint64_t)s.Hk * kD, (cuuint64_t)kD};
    cuuint32_t box[3] = {(cuuint32_t)kD, (cuuint32_t)pl.box_tok, (cuuint32_t)pl.box_heads};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(mk, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<int8_t *>(k), dims, strides,
                     box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS)
        return Q8KV_ERR_UNSUPPORTED;
    r = enc(mv, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<int8_t *>(v), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS)
        return Q8KV_ERR_UNSUPPORTED;
    std::memset(mks, 0, sizeof(*mks));
    std::memset(mvs, 0, sizeof(*mvs));
    if (!pl.scale_bulk) {
        cuuint64_t sd[2] = {(cuuint64_t)s.Hk, slots};
        cuuint64_t ss[1] = {(cuuint64_t)s.Hk * 4};
        cuuint32_t sb[2] = {(cuuint32_t)pl.sc_heads, (cuuint32_t)pl.box_tok};
        cuuint32_t se[2] = {1, 1};
        r = enc(mks, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float *>(ks), sd, ss, sb, se,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS)
            return Q8KV_ERR_UNSUPPORTED;
        r = enc(mvs, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float *>(vs), sd, ss, sb, se,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS)
            return Q8KV_ERR_UNSUPPORTED;
    }
    return Q8KV_OK;
}

// Tensor maps depend only on the pool pointers and the tiling; repeated calls on the same
// cache reuse them (a small round-robin cache, guarded by g_mutex).
struct MapKey {
    const void *k, *v, *ks, *vs;
    int Hk, bs, P, HPC, box_heads, box_tok, scale_bulk, sc_heads;
    bool operator==(const MapKey &o) const
    {
        return k == o.k && v == o.v && ks == o.ks && vs == o.vs && Hk == o.Hk && bs == o.bs &&
               P == o.P && HPC == o.HPC && box_heads == o.box_heads && box_tok == o.box_tok &&
               scale_bulk == o.scale_bulk && sc_heads == o.sc_heads;
    }
};

struct MapEntry {
    bool used = false;
    MapKey key{};
    CUtensorMap mk, mv, mks, mvs;
};

constexpr int kMapCache = 16;
MapEntry g_maps[kMapCache];
int g_map_next = 0;

q8kv_status encode_maps(const Shape &s, const Plan &pl, const int8_t *k, const int8_t *v,
                        const float *ks, const float *vs, CUtensorMap *mk, CUtensorMap *mv,
                        CUtensorMap *mks, CUtensorMap *mvs)
{
    const MapKey key{k, v, ks, vs, s.Hk, s.bs, s.P, pl.HPC, pl.box_heads, pl.box_tok,
                     pl.scale_bulk, pl.sc_heads};
    std::lock_guard<std::mutex> lock(g_mutex);
    for (auto &e : g_maps) {
        if (e.used && e.key == key) {
            *mk = e.mk;
            *mv = e.mv;
            *mks = e.mks;
            *mvs = e.mvs;
            return Q8KV_OK;
        }
    }
    q8kv_status st = encode_maps_uncached(s, pl, k, v, ks, vs, mk, mv, mks, mvs);
    if (st != Q8KV_OK)
        return st;
    MapEntry &e = g_maps[g_map_next];
    g_map_next = (g_map_next + 1) % kMapCache;
    e.used = true;
    e.key = key;
    e.mk = *mk;
    e.mv = *mv;
    e.mks = *mks;
    e.mvs = *mvs;
    return Q8KV_OK;
}

struct Call {
    float *out;
    const float *q;
    const int8_t *k, *v;
    const float *ks, *vs;
    const int32_t *bt, *lens;
    Shape s;
    float scale;
    int32_t *dots;
    int dots_max_len;
    int stall_cta = -1;                    // fault injection (q8kv_debug_stall_pipeline)
    unsigned long long stall_limit_ns = 0;
};

q8kv_status check_call(const Call &c)
{
    if (!c.out || !c.q || !c.k || !c.v || !c.ks || !c.vs || !c.bt || !c.lens)
        return Q8KV_ERR_INVALID_ARG;
    if (c.s.B <= 0 || c.s.Hq <= 0 || c.s.Hk <= 0 || c.s.D <= 0 || c.s.bs <= 0 || c.s.mbps <= 0 ||
        c.s.P <= 0 || c.s.Hq % c.s.Hk != 0 || c.s.D % 32 != 0 || c.s.nq <= 0)
        return Q8KV_ERR_INVALID_ARG;
    if (!std::isfinite(c.scale))
        return Q8KV_ERR_INVALID_ARG;
    if (!aligned16(c.out) || !aligned16(c.q) || !aligned16(c.k) || !aligned16(c.v) ||
        !aligned16(c.ks) || !aligned16(c.vs))
        return Q8KV_ERR_INVALID_ARG;
    return Q8KV_OK;
}

// The log-sum-exp combine after a decode kernel launched with cfg (same stream, programmatic
// dependent launch).
q8kv_status launch_combine(DeviceInfo &dev, const DecodeParams &p, const Plan &pl,
                           const cudaLaunchConfig_t &cfg)
{
    if (!dev.combine_attr) {
        // the dynamic part may use what the kernel's static shared memory leaves of the limit
        cudaFuncAttributes fa;
        Q8KV_CUDA(cudaFuncGetAttributes(&fa, combine_kernel));
        Q8KV_CUDA(cudaFuncSetAttribute(combine_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       dev.smem_optin - (int)fa.sharedSizeBytes));
        dev.combine_attr = true;
    }
    cudaLaunchConfig_t cc = cfg;
    cc.gridDim = dim3((unsigned)dev.sms);
    cc.blockDim = dim3(kCombineThreads);
    cc.dynamicSmemBytes = combine_layout(p.B, pl.grid).total;
    Q8KV_CUDA(cudaLaunchKernelEx(&cc, combine_kernel, p, pl.grid));
    return Q8KV_OK;
}

template <int NT, bool kPack, bool kDump>
q8kv_status launch_kernel(DeviceInfo &dev, const DecodeParams &p, const Plan &pl,
                          const CUtensorMap &mk, const CUtensorMap &mv, const CUtensorMap &mks,
                          const CUtensorMap &mvs, cudaStream_t stream)
{
    auto fn = decode_kernel<NT, kPack, kDump>;
    const int variant = kPack ? 2 : NT - 1;
    if (!dev.attr_set[variant][kDump ? 1 : 0]) {
        // the setmaxnreg split in the kernel assumes exactly kLaunchRegs registers per thread
        // at launch; anything else could leave a warpgroup waiting for registers forever
        cudaFuncAttributes attr;
        Q8KV_CUDA(cudaFuncGetAttributes(&attr, fn));
        if (attr.numRegs != kLaunchRegs)
            return Q8KV_ERR_UNSUPPORTED;
        Q8KV_CUDA(cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       dev.smem_optin));
        dev.attr_set[variant][kDump ? 1 : 0] = true;
    }
    // Both kernels allow programmatic dependent launch: each may be scheduled while the
    // kernel before it on the stream drains, and waits for it (griddepcontrol.wait) before
    // touching global memory.
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)pl.grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = pl.smem_bytes;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    Q8KV_CUDA(cudaLaunchKernelEx(&cfg, fn, p, mk, mv, mks, mvs));
    return launch_combine(dev, p, pl, cfg);
}

// The tensor-memory kernel for R rows per KV head, then the combine.
template <int R>
q8kv_status launch_tc(DeviceInfo &dev, const DecodeParams &p, const Plan &pl,
                      const CUtensorMap &mk, const CUtensorMap &mv, const CUtensorMap &mks,
                      const CUtensorMap &mvs, cudaStream_t stream)
{
    auto fn = mq_tc_kernel<R>;
    bool &set = dev.tc_attr[R == 16 ? 0 : 1];
    if (!set) {
        cudaFuncAttributes attr;
        Q8KV_CUDA(cudaFuncGetAttributes(&attr, fn));
        if (attr.numRegs != kTcLaunchRegs)
            return Q8KV_ERR_UNSUPPORTED;
        Q8KV_CUDA(cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       dev.smem_optin));
        set = true;
    }
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)pl.grid);
    cfg.blockDim = dim3(kTcThreads);
    cfg.dynamicSmemBytes = pl.smem_bytes;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    Q8KV_CUDA(cudaLaunchKernelEx(&cfg, fn, p, mk, mv, mks, mvs));
    return launch_combine(dev, p, pl, cfg);
}

q8kv_status run(const Call &c, void *ws, size_t ws_bytes, bool managed_ws, cudaStream_t stream)
{
    q8kv_status st = check_call(c);
    if (st != Q8KV_OK)
        return st;
    DeviceInfo *dev = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_mutex);
        st = device_info(&dev);
    }
    if (st != Q8KV_OK)
        return st;
    Plan pl;
    const int R = (c.dots || c.stall_cta >= 0) ? 0 : tc_rows(c.s);
    st = R ? make_plan_tc(c.s, *dev, R, pl) : make_plan(c.s, *dev, pl);
    if (st != Q8KV_OK)
        return st;
    if (managed_ws) {
        std::lock_guard<std::mutex> lock(g_mutex);
        if (dev->ws_bytes < pl.ws_bytes) {
            if (dev->ws) {
                Q8KV_CUDA(cudaFree(dev->ws));
                dev->ws = nullptr;
                dev->ws_bytes = 0;
            }
            Q8KV_CUDA(cudaMalloc(&dev->ws, pl.ws_bytes));
            dev->ws_bytes = pl.ws_bytes;
        }
        ws = dev->ws;
        ws_bytes = dev->ws_bytes;
    }
    if (!ws || ws_bytes < pl.ws_bytes || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0)
        return Q8KV_ERR_WORKSPACE;

    CUtensorMap mk, mv, mks, mvs;
    st = encode_maps(c.s, pl, c.k, c.v, c.ks, c.vs, &mk, &mv, &mks, &mvs);
    if (st != Q8KV_OK)
        return st;

    DecodeParams p;
    std::memset(&p, 0, sizeof(p));
    uint8_t *w = static_cast<uint8_t *>(ws);
    p.out = c.out;
    p.q = c.q;
    p.block_table = c.bt;
    p.seq_lens = c.lens;
    p.kscale = c.ks;
    p.vscale = c.vs;
    p.partials = reinterpret_cast<float *>(w);
    p.errors = dev->errors;
    p.dbg_dots = c.dots;
    p.dbg_max_len = c.dots_max_len;
    p.B = c.s.B;
    p.Hq = c.s.Hq;
    p.Hk = c.s.Hk;
    p.G = pl.G;
    p.nq = c.s.nq;
    p.Gq = c.s.Hq / c.s.Hk;
    p.bs = c.s.bs;
    p.mbps = c.s.mbps;
    p.num_blocks = c.s.P;
    p.HPC = pl.HPC;
    p.nhc = pl.nhc;
    p.slices = pl.slices;
    p.pairs = pl.pairs;
    p.subtiles = pl.subtiles;
    p.TT = pl.TT;
    p.box_tok = pl.box_tok;
    p.log2_box = pl.log2_box;
    p.n_boxes = pl.n_boxes;
    p.n_stages = pl.n_stages;
    p.scale_bulk = pl.scale_bulk;
    p.sc_heads = pl.sc_heads;
    p.heads_seg = pl.heads_seg;
    p.scratch_stride = pl.scratch_stride;
    p.scale_log2 = (float)((double)c.scale * 1.4426950408889634);
    p.stall_cta = c.stall_cta;
    p.stall_limit_ns = c.stall_limit_ns;
    p.lay = pl.lay;

    if (pl.tc_rows == 16)
        return launch_tc<16>(*dev, p, pl, mk, mv, mks, mvs, stream);
    if (pl.tc_rows == 32)
        return launch_tc<32>(*dev, p, pl, mk, mv, mks, mvs, stream);
    const bool dump = c.dots != nullptr;
    if (pl.G <= 4) // heads fill at most half of the 8 MMA columns: pack the split halves
        return dump ? launch_kernel<1, true, true>(*dev, p, pl, mk, mv, mks, mvs, stream)
                    : launch_kernel<1, true, false>(*dev, p, pl, mk, mv, mks, mvs, stream);
    if (pl.NT == 1)
        return dump ? launch_kernel<1, false, true>(*dev, p, pl, mk, mv, mks, mvs, stream)
                    : launch_kernel<1, false, false>(*dev, p, pl, mk, mv, mks, mvs, stream);
    return dump ? launch_kernel<2, false, true>(*dev, p, pl, mk, mv, mks, mvs, stream)
                : launch_kernel<2, false, false>(*dev, p, pl, mk, mv, mks, mvs, stream);
}

} // namespace

// Scratch of q8kv_decode_attn_static: the partial results of split sequences, at the same
// offsets as in a caller-owned workspace. A file-scope device array rather than an allocation,
// so that a call of that entry point never allocates: its callers are ones that must not
// allocate while serving (a pool allocator owns all device memory, or the step cannot take
// cudaMalloc's latency or cudaFree's device-wide synchronisation). One instance exists per
// device; calls that may overlap on the GPU share it and therefore race.
static __device__ __align__(256) unsigned char g_static_scratch[Q8KV_STATIC_SCRATCH_BYTES];

namespace {

struct StaticScratch {
    bool ready = false;
    void *ptr = nullptr;
};

StaticScratch g_static[kMaxDevices];

// Set-up, once per device, with that device current: look up the array's address on this
// device. No part of the scratch needs an initial value (every call's combine reads only
// the partial slots the same call's decode kernel wrote).
q8kv_status static_scratch(void **out)
{
    std::lock_guard<std::mutex> lock(g_mutex);
    DeviceInfo *dev = nullptr;
    q8kv_status st = device_info(&dev);
    if (st != Q8KV_OK)
        return st;
    int d = 0;
    Q8KV_CUDA(cudaGetDevice(&d));
    StaticScratch &sc = g_static[d];
    if (!sc.ready) {
        void *ptr = nullptr;
        Q8KV_CUDA(cudaGetSymbolAddress((void **)&ptr, g_static_scratch));
        if (!ptr || (reinterpret_cast<uintptr_t>(ptr) & 255u) != 0)
            return Q8KV_ERR_WORKSPACE;
        sc.ptr = ptr;
        sc.ready = true;
    }
    *out = sc.ptr;
    return Q8KV_OK;
}

} // namespace

extern "C" {

q8kv_status q8kv_decode_attn(float *out, const float *q, const int8_t *k_blocks,
                             const int8_t *v_blocks, const float *kscale, const float *vscale,
                             const int32_t *block_table, const int32_t *seq_lens, int B,
                             int n_q_heads, int n_kv_heads, int head_dim, int kv_block_size,
                             int max_blocks_per_seq, int num_kv_blocks, float scale,
                             cudaStream_t stream)
{
    Call c{out, q, k_blocks, v_blocks, kscale, vscale, block_table, seq_lens,
           Shape{B, n_q_heads, n_kv_heads, head_dim, kv_block_size, max_blocks_per_seq,
                 num_kv_blocks},
           scale, nullptr, 0};
    return run(c, nullptr, 0, true, stream);
}

q8kv_status q8kv_decode_attn_multi(float *out, const float *q, const int8_t *k_blocks,
                                   const int8_t *v_blocks, const float *kscale,
                                   const float *vscale, const int32_t *block_table,
                                   const int32_t *seq_lens, int B, int n_queries, int n_q_heads,
                                   int n_kv_heads, int head_dim, int kv_block_size,
                                   int max_blocks_per_seq, int num_kv_blocks, float scale,
                                   cudaStream_t stream)
{
    if (n_queries <= 0)
        return Q8KV_ERR_INVALID_ARG;
    Shape sh{B, n_q_heads, n_kv_heads, head_dim, kv_block_size, max_blocks_per_seq,
             num_kv_blocks};
    sh.nq = n_queries;
    Call c{out, q, k_blocks, v_blocks, kscale, vscale, block_table, seq_lens, sh, scale, nullptr,
           0};
    return run(c, nullptr, 0, true, stream);
}

size_t q8kv_workspace_bytes(int B, int n_q_heads, int n_kv_heads, int head_dim)
{
    if (B <= 0)
        return 0;
    Plan pl;
    if (plan_heads(n_q_heads, n_kv_heads, head_dim, pl) != Q8KV_OK)
        return 0;
    DeviceInfo *dev = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_mutex);
        if (device_info(&dev) != Q8KV_OK)
            return 0;
    }
    plan_workspace(dev->sms, pl);
    return pl.ws_bytes;
}

q8kv_status q8kv_workspace_init(void *workspace, size_t workspace_bytes, cudaStream_t stream)
{
    if (!workspace || workspace_bytes == 0)
        return Q8KV_ERR_INVALID_ARG;
    Q8KV_CUDA(cudaMemsetAsync(workspace, 0, workspace_bytes, stream));
    return Q8KV_OK;
}

q8kv_status q8kv_decode_attn_ws(float *out, const float *q, const int8_t *k_blocks,
                                const int8_t *v_blocks, const float *kscale,
                                const float *vscale, const int32_t *block_table,
                                const int32_t *seq_lens, int B, int n_q_heads, int n_kv_heads,
                                int head_dim, int kv_block_size, int max_blocks_per_seq,
                                int num_kv_blocks, float scale, void *workspace,
                                size_t workspace_bytes, cudaStream_t stream)
{
    Call c{out, q, k_blocks, v_blocks, kscale, vscale, block_table, seq_lens,
           Shape{B, n_q_heads, n_kv_heads, head_dim, kv_block_size, max_blocks_per_seq,
                 num_kv_blocks},
           scale, nullptr, 0};
    return run(c, workspace, workspace_bytes, false, stream);
}

q8kv_status q8kv_decode_attn_static(float *out, const float *q, const int8_t *k_blocks,
                                    const int8_t *v_blocks, const float *kscale,
                                    const float *vscale, const int32_t *block_table,
                                    const int32_t *seq_lens, int B, int n_q_heads,
                                    int n_kv_heads, int head_dim, int kv_block_size,
                                    int max_blocks_per_seq, int num_kv_blocks, float scale,
                                    cudaStream_t stream)
{
    Call c{out, q, k_blocks, v_blocks, kscale, vscale, block_table, seq_lens,
           Shape{B, n_q_heads, n_kv_heads, head_dim, kv_block_size, max_blocks_per_seq,
                 num_kv_blocks},
           scale, nullptr, 0};
    q8kv_status st = check_call(c); // argument errors before any CUDA call
    if (st != Q8KV_OK)
        return st;
    // Unsupported shapes, and shapes whose workspace exceeds the array, are rejected here,
    // before set-up enqueues anything.
    {
        DeviceInfo *dev = nullptr;
        {
            std::lock_guard<std::mutex> lock(g_mutex);
            st = device_info(&dev);
        }
        if (st != Q8KV_OK)
            return st;
        Plan pl;
        st = make_plan(c.s, *dev, pl);
        if (st != Q8KV_OK)
            return st;
        if (pl.ws_bytes > Q8KV_STATIC_SCRATCH_BYTES)
            return Q8KV_ERR_WORKSPACE;
    }
    void *scratch = nullptr;
    st = static_scratch(&scratch);
    if (st != Q8KV_OK)
        return st;
    return run(c, scratch, Q8KV_STATIC_SCRATCH_BYTES, false, stream);
}

q8kv_status q8kv_debug_quantize_q(int8_t *qi, float *qsc, const float *q, int n_rows,
                                  int head_dim, cudaStream_t stream)
{
    if (!qi || !qsc || !q || n_rows <= 0 || head_dim <= 0 || head_dim % 32 != 0)
        return Q8KV_ERR_INVALID_ARG;
    if (!aligned16(q) || (reinterpret_cast<uintptr_t>(qi) & 7u) != 0)
        return Q8KV_ERR_INVALID_ARG;
    const long long n_blocks = (long long)n_rows * (head_dim / 32);
    const long long threads = n_blocks * 4;
    const int tpb = 256;
    const long long grid = (threads + tpb - 1) / tpb;
    if (grid > 0x7fffffffLL)
        return Q8KV_ERR_UNSUPPORTED;
    qquant_debug_kernel<<<(unsigned)grid, tpb, 0, stream>>>(qi, qsc, q, n_blocks);
    Q8KV_CUDA(cudaGetLastError());
    return Q8KV_OK;
}

q8kv_status q8kv_debug_block_dots(int32_t *dots, int max_seq_len, float *out, const float *q,
                                  const int8_t *k_blocks, const int8_t *v_blocks,
                                  const float *kscale, const float *vscale,
                                  const int32_t *block_table, const int32_t *seq_lens, int B,
                                  int n_q_heads, int n_kv_heads, int head_dim,
                                  int kv_block_size, int max_blocks_per_seq, int num_kv_blocks,
                                  float scale, cudaStream_t stream)
{
    if (!dots || max_seq_len <= 0)
        return Q8KV_ERR_INVALID_ARG;
    if ((long long)max_seq_len < (long long)max_blocks_per_seq * kv_block_size)
        return Q8KV_ERR_INVALID_ARG; // a valid seq_len could exceed the dots buffer
    Call c{out, q, k_blocks, v_blocks, kscale, vscale, block_table, seq_lens,
           Shape{B, n_q_heads, n_kv_heads, head_dim, kv_block_size, max_blocks_per_seq,
                 num_kv_blocks},
           scale, dots, max_seq_len};
    return run(c, nullptr, 0, true, stream);
}

q8kv_status q8kv_debug_stall_pipeline(float *out, const float *q, const int8_t *k_blocks,
                                      const int8_t *v_blocks, const float *kscale,
                                      const float *vscale, const int32_t *block_table,
                                      const int32_t *seq_lens, int B, int n_q_heads,
                                      int n_kv_heads, int head_dim, int kv_block_size,
                                      int max_blocks_per_seq, int num_kv_blocks, float scale,
                                      int stall_cta, unsigned long long limit_ns,
                                      cudaStream_t stream)
{
    if (stall_cta < 0 || limit_ns < 1000ull || limit_ns > 1000000000ull)
        return Q8KV_ERR_INVALID_ARG;
    Call c{out, q, k_blocks, v_blocks, kscale, vscale, block_table, seq_lens,
           Shape{B, n_q_heads, n_kv_heads, head_dim, kv_block_size, max_blocks_per_seq,
                 num_kv_blocks},
           scale, nullptr, 0};
    c.stall_cta = stall_cta;
    c.stall_limit_ns = limit_ns;
    return run(c, nullptr, 0, true, stream);
}

q8kv_status q8kv_device_errors(unsigned *flags, int clear)
{
    if (!flags)
        return Q8KV_ERR_INVALID_ARG;
    DeviceInfo *dev = nullptr;
    q8kv_status st;
    {
        std::lock_guard<std::mutex> lock(g_mutex);
        st = device_info(&dev);
    }
    if (st != Q8KV_OK)
        return st;
    Q8KV_CUDA(cudaDeviceSynchronize());
    Q8KV_CUDA(cudaMemcpy(flags, dev->errors, sizeof(unsigned), cudaMemcpyDeviceToHost));
    if (clear)
        Q8KV_CUDA(cudaMemset(dev->errors, 0, sizeof(unsigned)));
    return Q8KV_OK;
}

const char *q8kv_status_string(q8kv_status status)
{
    switch (status) {
    case Q8KV_OK:
        return "ok";
    case Q8KV_ERR_INVALID_ARG:
        return "invalid argument";
    case Q8KV_ERR_UNSUPPORTED:
        return "unsupported shape";
    case Q8KV_ERR_CUDA:
        return "CUDA error";
    case Q8KV_ERR_WORKSPACE:
        return "workspace missing or too small";
    }
    return "unknown status";
}

int q8kv_last_cuda_error(void)
{
    return t_last_cuda_error;
}

int q8kv_version(void)
{
    return 103;
}

} // extern "C"

// The KV-cache write entry point (uses the device bookkeeping above).
#include "q8kv_cache_write_api.cuh"

// The QUEST block-metadata entry point.
#include "q8kv_quest_api.cuh"

// The q4_0-cache decode entry point.
#include "q8kv_q4_api.cuh"
