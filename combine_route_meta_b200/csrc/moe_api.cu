// C ABI of the MoE dispatch / combine library: host-side validation and
// launches.  The declarations and their contracts are in
// include/moe_dispatch_combine.h.
#include <algorithm>
#include <cstdint>
#include <cstring>
#include <atomic>
#include <mutex>

#include <cuda_runtime.h>

#include "moe_dispatch_combine.h"

#include "combine.cuh"
#include "combine_partial.cuh"
#include "common.cuh"
#include "dispatch_fused.cuh"
#include "dispatch_multi.cuh"
#include "ep.cuh"
#include "meta.cuh"
#include "router.cuh"
#include "scatter.cuh"
#include "silu_quant.cuh"

// Scratch of moe_dispatch_no_alloc: a fixed array in device memory, allocated
// by the CUDA runtime when the library's module is loaded on a device and held
// there until the process exits.  Host code must not use this name as a device
// address; it resolves the address with cudaGetSymbolAddress (below).
static __device__ __align__(256) int32_t g_no_alloc_scratch[MOE_NO_ALLOC_SCRATCH_BYTES / sizeof(int32_t)];

namespace moe {

// Diagnostic: waits on an mbarrier that nothing completes, with the same bounded
// wait the bulk kernels use, and reports MOE_DEV_TIMEOUT when it gives up.
__global__ void __launch_bounds__(kWarp) wait_selftest(int32_t *err, uint64_t limit_ns)
{
    stream_order_begin();
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(smem_addr(&bar), 1);
        fence_mbar_init();
    }
    __syncwarp();
    if (threadIdx.x == 0 && !mbar_wait(smem_addr(&bar), 0, limit_ns))
        raise_error(err, MOE_DEV_TIMEOUT);
}

namespace {

constexpr int kMaxDevices = 64;
constexpr int kVersion = 100; // 0.1.0

// Per-device launch facts, read once per device.
struct DeviceInfo {
    std::atomic<bool> ready{false};
    int sms = 0;
    // resident CTAs per SM of the kernels whose grid is one wave
    int silu_per_sm[2] = {1, 1}; // silu_quant_rows<1>, <kSiluWideCtas>
    int router_per_sm[4] = {1, 1, 1, 1}; // 4, 8, 16, 32 logits per lane
    int send_per_sm[2] = {1, 1};         // combine_partial_send<false>, <true>
    int recv_per_sm = 1;
};

template <typename K>
int resident_per_sm(K kernel, int block, size_t smem)
{
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, block, smem) != cudaSuccess)
        return 0;
    return n > 0 ? n : 1;
}
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mutex; // the first call on a device fills its entry; later calls read it

int device_info(DeviceInfo **out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return MOE_ERR_CUDA;
    DeviceInfo &d = g_dev[dev];
    if (d.ready.load(std::memory_order_acquire)) {
        *out = &d;
        return MOE_OK;
    }
    std::lock_guard<std::mutex> lock(g_dev_mutex);
    if (!d.ready.load(std::memory_order_relaxed)) {
        if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return MOE_ERR_CUDA;
        const size_t big = meta_single_smem(MOE_MAX_EXPERTS);
        if (cudaFuncSetAttribute(meta_single_block, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)big) != cudaSuccess ||
            cudaFuncSetAttribute(scatter_bulk_fp8<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)kBulkMaxSmem) != cudaSuccess ||
            cudaFuncSetAttribute(scatter_bulk_fp8<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)kBulkMaxSmem) != cudaSuccess ||
            cudaFuncSetAttribute(meta_tile_assign, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)meta_assign_smem(MOE_MAX_EXPERTS)) != cudaSuccess ||
            cudaFuncSetAttribute(scatter_bulk_bf16, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)kBulkMaxSmem) != cudaSuccess)
            return MOE_ERR_CUDA;
        const int rb = kRouterWarps * kWarp;
        if (!(d.silu_per_sm[0] = resident_per_sm(silu_quant_rows<1>, kSiluThreads, 0)) ||
            !(d.silu_per_sm[1] = resident_per_sm(silu_quant_rows<kSiluWideCtas>, kSiluThreads, 0)) ||
            !(d.router_per_sm[0] = resident_per_sm(router_topk<4>, rb, 0)) ||
            !(d.router_per_sm[1] = resident_per_sm(router_topk<8>, rb, 0)) ||
            !(d.router_per_sm[2] = resident_per_sm(router_topk<16>, rb, 0)) ||
            !(d.router_per_sm[3] = resident_per_sm(router_topk<kRouterMaxE / kWarp>, rb, 0)) ||
            !(d.send_per_sm[0] = resident_per_sm(combine_partial_send<false>, kPartialThreads, 0)) ||
            !(d.send_per_sm[1] = resident_per_sm(combine_partial_send<true>, kPartialThreads, 0)) ||
            !(d.recv_per_sm = resident_per_sm(combine_partial_recv, kPartialThreads, 0)))
            return MOE_ERR_CUDA;
        d.ready.store(true, std::memory_order_release);
    }
    *out = &d;
    return MOE_OK;
}

// Device address of g_no_alloc_scratch on the current device, looked up once
// per device (with that device current) and cached.
void *g_no_alloc_addr[kMaxDevices];
std::mutex g_no_alloc_mutex;

int no_alloc_scratch(void **out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return MOE_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_no_alloc_mutex);
    if (g_no_alloc_addr[dev] == nullptr) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_no_alloc_scratch) != cudaSuccess || p == nullptr)
            return MOE_ERR_CUDA;
        g_no_alloc_addr[dev] = p;
    }
    *out = g_no_alloc_addr[dev];
    return MOE_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Launches a kernel that may begin while the previous kernel in the stream is
// finishing (programmatic stream serialization); each kernel starts with
// stream_order_begin(), which waits for that kernel before touching memory.
template <typename... Params, typename... Args>
cudaError_t launch(void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                   Args... args)
{
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

int check_config(const moe_config *c)
{
    if (c == nullptr)
        return MOE_ERR_INVALID_ARG;
    if (c->H <= 0 || c->k <= 0 || c->E <= 0 || c->R <= 0 || c->E % c->R != 0)
        return MOE_ERR_INVALID_ARG;
    if ((c->flags & ~(MOE_FP8 | MOE_PAD128 | MOE_INPUTS_READY)) != 0)
        return MOE_ERR_INVALID_ARG;
    if (c->H % 8 != 0 || c->E > MOE_MAX_EXPERTS || c->k > MOE_MAX_TOPK)
        return MOE_ERR_UNSUPPORTED;
    if ((c->flags & MOE_FP8) && c->H % 128 != 0)
        return MOE_ERR_UNSUPPORTED;
    return MOE_OK;
}

int64_t rows_capacity(const moe_config *c, int32_t T)
{
    const int64_t S = (int64_t)T * c->k;
    if (!(c->flags & MOE_PAD128))
        return S;
    // At most min(E, S) non-empty experts, each adding at most 127 pad rows;
    // the total is a whole number of 128-row blocks, and the bound
    // floor((S + 127*m) / 128) blocks is reached with m-1 single-entry experts.
    const int64_t m = S < c->E ? S : c->E;
    return (S + 127 * m) / 128 * 128;
}

bool use_single_block(int64_t S) { return S <= kSingleBlockEntries; }

// Chunks per warp of the one-token-per-CTA dispatch (1, 2 or 4: the fewest that
// fit the row in one CTA), or 0 if those kernels do not apply.
int fused_chunks(const moe_config *c, int32_t T)
{
    const int64_t S = (int64_t)T * c->k;
    const int32_t chunks = (c->H + chunk_cols<kFusedLaneCols>() - 1) / chunk_cols<kFusedLaneCols>();
    if (T <= 0 || S > kFusedMaxEntries || c->k > kFusedMaxK)
        return 0;
    const int max_warps = kFusedMaxThreads / kWarp;
    for (int per = 1; per <= kFusedMaxChunks; per *= 2)
        if (chunks <= max_warps * per)
            return per;
    return 0;
}

using SmallKernel = void (*)(FusedArgs);

// The one-token-per-CTA dispatch kernel for a shape: the direct-rank form
// without padding, the histogram form with it.
SmallKernel small_kernel(bool fp8, bool pad, bool big_k, int per)
{
    const int i = per == 1 ? 0 : (per == 2 ? 1 : 2);
    if (pad) {
        static const SmallKernel t[2][3] = {
            {dispatch_fused<1, false>, dispatch_fused<2, false>, dispatch_fused<4, false>},
            {dispatch_fused<1, true>, dispatch_fused<2, true>, dispatch_fused<4, true>}};
        return t[fp8][i];
    }
    static const SmallKernel t[2][2][3] = {
        {{dispatch_direct<1, false, 8>, dispatch_direct<2, false, 8>, dispatch_direct<4, false, 8>},
         {dispatch_direct<1, false, kFusedMaxK>, dispatch_direct<2, false, kFusedMaxK>,
          dispatch_direct<4, false, kFusedMaxK>}},
        {{dispatch_direct<1, true, 8>, dispatch_direct<2, true, 8>, dispatch_direct<4, true, 8>},
         {dispatch_direct<1, true, kFusedMaxK>, dispatch_direct<2, true, kFusedMaxK>,
          dispatch_direct<4, true, kFusedMaxK>}}};
    return t[fp8][big_k][i];
}

// Resident CTAs per SM of a kernel at a block size, cached per device.
int cached_per_sm(const void *fn, int block, size_t smem)
{
    struct Entry {
        const void *fn;
        int block, dev, n;
        size_t smem;
    };
    static Entry cache[256];
    static int used = 0;
    static std::mutex m;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return 0;
    std::lock_guard<std::mutex> lock(m);
    for (int i = 0; i < used; ++i)
        if (cache[i].fn == fn && cache[i].block == block && cache[i].smem == smem && cache[i].dev == dev)
            return cache[i].n;
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, fn, block, smem) != cudaSuccess || n <= 0)
        return 0;
    if (used < 256)
        cache[used++] = Entry{fn, block, dev, n, smem};
    return n;
}

// Launches the one-token-per-CTA dispatch with `per` chunks per warp (the
// fewest that fit the row in one CTA).  It runs only for T below the SM count
// (larger small batches take dispatch_multi), so its T (+1) CTAs of at most
// 1024 threads are resident in one wave.
// after_router: the previous kernel in the stream is the router of the same
// moe_route_dispatch call, so the direct-rank kernel may load x before waiting.
// inputs_ready: the caller's MOE_INPUTS_READY (x and the routing were complete
// before the previous kernel began), so it may read everything before waiting.
cudaError_t launch_small(bool fp8, int per, int32_t T, cudaStream_t s, const FusedArgs &f, bool after_router,
                         bool inputs_ready)
{
    const bool pad = f.pad128 != 0;
    const unsigned grid = pad ? (unsigned)T : (unsigned)T + 1;
    const int32_t chunks = (f.H + chunk_cols<kFusedLaneCols>() - 1) / chunk_cols<kFusedLaneCols>();
    const unsigned block = (unsigned)((chunks + per - 1) / per * kWarp);
    if (inputs_ready && !pad) {
        const int i = per == 1 ? 0 : (per == 2 ? 1 : 2);
        static const SmallKernel t[2][2][3] = {
            {{dispatch_direct_ready<1, false, 8>, dispatch_direct_ready<2, false, 8>,
              dispatch_direct_ready<4, false, 8>},
             {dispatch_direct_ready<1, false, kFusedMaxK>, dispatch_direct_ready<2, false, kFusedMaxK>,
              dispatch_direct_ready<4, false, kFusedMaxK>}},
            {{dispatch_direct_ready<1, true, 8>, dispatch_direct_ready<2, true, 8>,
              dispatch_direct_ready<4, true, 8>},
             {dispatch_direct_ready<1, true, kFusedMaxK>, dispatch_direct_ready<2, true, kFusedMaxK>,
              dispatch_direct_ready<4, true, kFusedMaxK>}}};
        return launch(t[fp8][f.k > 8][i], grid, block, fused_smem(f.E), s, f);
    }
    if (after_router && !pad && f.k <= 8) {
        const int i = per == 1 ? 0 : (per == 2 ? 1 : 2);
        static const SmallKernel t[2][3] = {
            {dispatch_direct_after_router<1, false, 8>, dispatch_direct_after_router<2, false, 8>,
             dispatch_direct_after_router<4, false, 8>},
            {dispatch_direct_after_router<1, true, 8>, dispatch_direct_after_router<2, true, 8>,
             dispatch_direct_after_router<4, true, 8>}};
        return launch(t[fp8][i], grid, block, fused_smem(f.E), s, f);
    }
    return launch(small_kernel(fp8, pad, f.k > 8, per), grid, block, fused_smem(f.E), s, f);
}

// The mid-size one-launch dispatch applies past the one-token-per-CTA kernels
// up to kMultiMaxEntries entries, for fp8 payloads and for bf16 rows too narrow
// for the bulk scatter (wider bf16 rows keep the bulk stores, whose write
// stream is worth more than the metadata launches at these sizes).
// It also takes the small batches the one-token-per-CTA kernels do not: T at or
// above the SM count (one CTA per SM owning a few tokens beats two waves or two
// half-size CTAs per SM) and k > kFusedMaxK.
bool use_multi(const moe_config *c, int32_t T)
{
    const int64_t S = (int64_t)T * c->k;
    const bool fp8 = c->flags & MOE_FP8;
    if (S <= kFusedMaxEntries)
        return T > 0;
    return S <= kMultiMaxEntries && (fp8 || !use_bulk_scatter(c->H, false));
}

cudaError_t launch_multi(bool fp8, int32_t T, int sms, cudaStream_t s, const FusedArgs &f)
{
    // one CTA per SM at most (one wave), each owning a contiguous run of tokens
    void (*k)(FusedArgs, int32_t) = fp8 ? dispatch_multi<true> : dispatch_multi<false>;
    const int32_t G = T < sms ? T : sms;
    const int32_t n_ent = (T + G - 1) / G * f.k;
    const size_t smem = multi_smem(f.E, n_ent);
    if (cached_per_sm((const void *)k, kMultiThreads, smem) == 0)
        return cudaErrorInvalidConfiguration;
    return launch(k, (unsigned)G, (unsigned)kMultiThreads, smem, s, f, n_ent);
}

size_t workspace_bytes(const moe_config *c, int32_t T)
{
    const int64_t S = (int64_t)T * c->k;
    if (use_single_block(S))
        return 0;
    const size_t raw = (size_t)meta_tiles(S) * (size_t)c->E * sizeof(int32_t);
    return (raw + 255) / 256 * 256;
}

int launched(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

// Grid for `units` work units of a 128-thread kernel: enough CTAs to fill every
// SM at full occupancy, fewer if there are fewer units.
unsigned grid_for(int64_t units, int sms, int ctas_per_sm)
{
    int64_t cap = (int64_t)sms * ctas_per_sm;
    int64_t g = units < cap ? units : cap;
    return (unsigned)(g > 0 ? g : 1);
}

// Argument checks of the layout phase (shared by moe_dispatch).
int check_layout_args(const moe_config *cfg, int32_t T, const int32_t *topk_idx,
                      const moe_dispatch_out *out, const int32_t *slot, const void *workspace,
                      size_t workspace_bytes_given, const int32_t *dev_err)
{
    if (T < 0 || out == nullptr || dev_err == nullptr)
        return MOE_ERR_INVALID_ARG;
    const int64_t S = (int64_t)T * cfg->k;
    const int64_t rows_cap = out->rows_cap;
    if (rows_cap < 0 || rows_cap > INT32_MAX || S > INT32_MAX)
        return MOE_ERR_INVALID_ARG;
    if (rows_capacity(cfg, T) > INT32_MAX)
        return MOE_ERR_UNSUPPORTED;
    if (out->expert_count == nullptr || out->expert_offset == nullptr ||
        out->rank_offset == nullptr || (rows_cap > 0 && out->recv_src == nullptr))
        return MOE_ERR_INVALID_ARG;
    if (T > 0 && (topk_idx == nullptr || slot == nullptr))
        return MOE_ERR_INVALID_ARG;
    const size_t need_ws = workspace_bytes(cfg, T);
    if (need_ws > 0 && (workspace == nullptr || workspace_bytes_given < need_ws))
        return MOE_ERR_INVALID_ARG;
    return MOE_OK;
}

// Argument checks of the payload phase (shared by moe_dispatch).
int check_payload_args(const moe_config *cfg, int32_t T, const void *x, const int32_t *slot,
                       const moe_dispatch_out *out)
{
    const bool fp8 = cfg->flags & MOE_FP8;
    if (T < 0 || out == nullptr)
        return MOE_ERR_INVALID_ARG;
    if (T > 0 && (x == nullptr || slot == nullptr))
        return MOE_ERR_INVALID_ARG;
    if (out->rows_cap > 0 && (out->recv_x == nullptr || (fp8 && out->recv_scale == nullptr)))
        return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(out->recv_x) || (fp8 && !aligned16(out->recv_scale)))
        return MOE_ERR_INVALID_ARG;
    return MOE_OK;
}

// Routing metadata without payload: one CTA for small batches, tiled otherwise.
int launch_layout(const moe_config *cfg, int32_t T, const int32_t *topk_idx,
                  const moe_dispatch_out *out, int32_t *slot, void *workspace, int32_t *dev_err,
                  cudaStream_t s)
{
    MetaArgs m;
    m.topk_idx = topk_idx;
    m.S = (int64_t)T * cfg->k;
    m.k = cfg->k;
    m.E = cfg->E;
    m.R = cfg->R;
    m.pad128 = (cfg->flags & MOE_PAD128) ? 1 : 0;
    m.rows_cap = out->rows_cap;
    m.expert_count = out->expert_count;
    m.expert_offset = out->expert_offset;
    m.rank_offset = out->rank_offset;
    m.slot = slot;
    m.recv_src = out->recv_src;
    m.err = dev_err;
    if (use_single_block(m.S))
        return launched(launch(meta_single_block, 1, kMetaThreads, meta_single_smem(cfg->E), s, m));
    const int64_t ntiles = meta_tiles(m.S);
    int32_t *tile_hist = static_cast<int32_t *>(workspace);
    const int32_t *tile_prefix = tile_hist;
    int st;
    if ((st = launched(launch(meta_tile_count, (unsigned)ntiles, kMetaThreads, meta_count_smem(cfg->E),
                              s, m, tile_hist))) != MOE_OK ||
        (st = launched(launch(meta_tile_scan, (unsigned)((cfg->E + kWarp - 1) / kWarp), kScanThreads,
                              0, s, m, tile_hist, (int32_t)ntiles))) != MOE_OK ||
        (st = launched(launch(meta_tile_assign, (unsigned)ntiles, kMetaThreads,
                              meta_assign_smem(cfg->E), s, m, tile_prefix))) != MOE_OK)
        return st;
    return MOE_OK;
}

// Payload rows to the slots: bulk copies for bf16 rows of at least 1 KB,
// register stores (and the fp8 quantiser) otherwise.
int launch_payload(const moe_config *cfg, int32_t T, const void *x, const int32_t *slot,
                   const moe_dispatch_out *out, int32_t *dev_err, const DeviceInfo *dev,
                   cudaStream_t s, bool after_layout)
{
    if (T == 0)
        return MOE_OK;
    const bool fp8 = cfg->flags & MOE_FP8;
    ScatterArgs a;
    a.x = static_cast<const uint16_t *>(x);
    a.slot = slot;
    a.T = T;
    a.H = cfg->H;
    a.k = cfg->k;
    a.rows_cap = out->rows_cap;
    a.recv_x = out->recv_x;
    a.recv_scale = out->recv_scale;
    a.err = dev_err;
    cudaError_t e;
    if (use_bulk_scatter(cfg->H, fp8)) {
        const unsigned grid = grid_for(T, dev->sms, kBulkCtasPerSm);
        const size_t smem = (size_t)kBulkStages * bulk_stage_bytes(cfg->H);
        e = launch(scatter_bulk_bf16, grid, kWarp, smem, s, a);
    } else if (fp8 && use_bulk_fp8(cfg->H, cfg->k)) {
        void (*k)(ScatterArgs) = after_layout ? scatter_bulk_fp8<true> : scatter_bulk_fp8<false>;
        const unsigned block = (unsigned)((cfg->H / 512 + 1) * kWarp); // quantiser warps + store warp
        const size_t smem = (size_t)kFp8Stages * fp8_stage_bytes(cfg->H);
        const int per_sm = cached_per_sm((const void *)k, (int)block, smem);
        if (per_sm == 0)
            return MOE_ERR_CUDA;
        e = launch(k, grid_for(T, dev->sms, per_sm), block, smem, s, a);
    } else {
        constexpr int kCols = chunk_cols<kScatterLaneCols>();
        const int64_t warp_units = (int64_t)T * ((cfg->H + kCols - 1) / kCols);
        const int warps_per_cta = kScatterThreads / kWarp;
        const unsigned grid = grid_for((warp_units + warps_per_cta - 1) / warps_per_cta, dev->sms,
                                       2048 / kScatterThreads);
        if (after_layout)
            e = fp8 ? launch(scatter_rows<true, true>, grid, kScatterThreads, 0, s, a)
                    : launch(scatter_rows<false, true>, grid, kScatterThreads, 0, s, a);
        else
            e = fp8 ? launch(scatter_rows<true, false>, grid, kScatterThreads, 0, s, a)
                    : launch(scatter_rows<false, false>, grid, kScatterThreads, 0, s, a);
    }
    return launched(e);
}

} // namespace
} // namespace moe

using namespace moe;

extern "C" {

int moe_version(void) { return kVersion; }

const char *moe_status_string(int status)
{
    switch (status) {
    case MOE_OK:
        return "ok";
    case MOE_ERR_INVALID_ARG:
        return "invalid argument";
    case MOE_ERR_UNSUPPORTED:
        return "unsupported configuration";
    case MOE_ERR_CUDA:
        return "CUDA error";
    case MOE_ERR_DEVICE:
        return "device reported an error";
    case MOE_ERR_TOO_LARGE:
        return "problem needs more scratch than the fixed no-allocation buffer holds";
    default:
        return "unknown status";
    }
}

int64_t moe_rows_capacity(const moe_config *cfg, int32_t T)
{
    if (check_config(cfg) != MOE_OK || T < 0)
        return -1;
    return rows_capacity(cfg, T);
}

size_t moe_workspace_bytes(const moe_config *cfg, int32_t T)
{
    if (check_config(cfg) != MOE_OK || T < 0)
        return 0;
    return workspace_bytes(cfg, T);
}

int moe_dispatch_sizes_for(const moe_config *cfg, int32_t T, int64_t rows_cap,
                           moe_dispatch_sizes *sizes)
{
    int st = check_config(cfg);
    if (st != MOE_OK)
        return st;
    if (sizes == nullptr || T < 0 || rows_cap < 0)
        return MOE_ERR_INVALID_ARG;
    const bool fp8 = cfg->flags & MOE_FP8;
    sizes->recv_x = (size_t)rows_cap * cfg->H * (fp8 ? 1 : 2);
    sizes->recv_scale = fp8 ? (size_t)rows_cap * (cfg->H / 128) * sizeof(float) : 0;
    sizes->expert_count = (size_t)cfg->E * sizeof(int32_t);
    sizes->expert_offset = (size_t)(cfg->E + 1) * sizeof(int32_t);
    sizes->rank_offset = (size_t)(cfg->R + 1) * sizeof(int32_t);
    sizes->recv_src = (size_t)rows_cap * sizeof(int32_t);
    sizes->slot = (size_t)T * cfg->k * sizeof(int32_t);
    return MOE_OK;
}

namespace {

int check_dispatch_args(const moe_config *cfg, int32_t T, const void *x, const int32_t *topk_idx,
                        const float *topk_w, const moe_dispatch_out *out, int32_t *slot,
                        void *workspace, size_t workspace_bytes_given, int32_t *dev_err,
                        moe_handle *handle)
{
    int st = check_config(cfg);
    if (st != MOE_OK)
        return st;
    if (handle == nullptr || (T > 0 && topk_w == nullptr))
        return MOE_ERR_INVALID_ARG;
    if ((st = check_layout_args(cfg, T, topk_idx, out, slot, workspace, workspace_bytes_given,
                                dev_err)) != MOE_OK ||
        (st = check_payload_args(cfg, T, x, slot, out)) != MOE_OK)
        return st;
    return MOE_OK;
}

// Checks of moe_router_topk's arguments (T == 0 passes).
int check_router_args(int32_t T, int32_t E, int32_t k, const float *logits, int32_t score_fn,
                      int32_t n_group, int32_t topk_group, const int32_t *topk_idx,
                      const float *topk_w)
{
    if (T < 0 || E <= 0 || k <= 0 || n_group <= 0 || topk_group <= 0 || topk_group > n_group ||
        (score_fn != MOE_SCORE_SOFTMAX && score_fn != MOE_SCORE_SIGMOID) || E % n_group != 0)
        return MOE_ERR_INVALID_ARG;
    if ((int64_t)k > (int64_t)topk_group * (E / n_group))
        return MOE_ERR_INVALID_ARG;
    if (E > kRouterMaxE || k > kRouterMaxK || n_group > kRouterMaxGroups)
        return MOE_ERR_UNSUPPORTED;
    if (T > 0 && (logits == nullptr || topk_idx == nullptr || topk_w == nullptr))
        return MOE_ERR_INVALID_ARG;
    return MOE_OK;
}

int launch_router(int32_t T, int32_t E, int32_t k, const float *logits, int32_t score_fn,
                  int32_t n_group, int32_t topk_group, int32_t renormalize, int32_t *topk_idx,
                  float *topk_w, const DeviceInfo *dev, cudaStream_t s)
{
    RouterArgs a;
    a.logits = logits;
    a.T = T;
    a.E = E;
    a.k = k;
    a.score_fn = score_fn;
    a.n_group = n_group;
    a.topk_group = topk_group;
    a.renormalize = renormalize ? 1 : 0;
    a.topk_idx = topk_idx;
    a.topk_w = topk_w;
    const unsigned block = kRouterWarps * kWarp;
    const int64_t units = (T + kRouterWarps - 1) / kRouterWarps;
    // logits per lane, rounded up to a power of two; at most one wave of CTAs
    if (E <= 4 * kWarp)
        return launched(launch(router_topk<4>, grid_for(units, dev->sms, dev->router_per_sm[0]),
                               block, 0, s, a));
    if (E <= 8 * kWarp)
        return launched(launch(router_topk<8>, grid_for(units, dev->sms, dev->router_per_sm[1]),
                               block, 0, s, a));
    if (E <= 16 * kWarp)
        return launched(launch(router_topk<16>, grid_for(units, dev->sms, dev->router_per_sm[2]),
                               block, 0, s, a));
    return launched(launch(router_topk<kRouterMaxE / kWarp>,
                           grid_for(units, dev->sms, dev->router_per_sm[3]), block, 0, s, a));
}

int run_dispatch(const moe_config *cfg, int32_t T, const void *x, const int32_t *topk_idx,
                 const float *topk_w, const moe_dispatch_out *out, int32_t *slot,
                 void *workspace, int32_t *dev_err, DeviceInfo *dev, cudaStream_t s,
                 moe_handle *handle, bool after_router = false);

} // namespace

int moe_dispatch(const moe_config *cfg, int32_t T, const void *x, const int32_t *topk_idx,
                 const float *topk_w, const moe_dispatch_out *out, int32_t *slot,
                 void *workspace, size_t workspace_bytes_given, int32_t *dev_err, void *stream,
                 moe_handle *handle)
{
    int st = check_dispatch_args(cfg, T, x, topk_idx, topk_w, out, slot, workspace,
                                 workspace_bytes_given, dev_err, handle);
    if (st != MOE_OK)
        return st;
    DeviceInfo *dev = nullptr;
    if ((st = device_info(&dev)) != MOE_OK)
        return st;
    return run_dispatch(cfg, T, x, topk_idx, topk_w, out, slot, workspace, dev_err, dev,
                        static_cast<cudaStream_t>(stream), handle);
}

namespace {

} // namespace

int moe_route_dispatch(const moe_config *cfg, int32_t T, const void *x, const float *logits,
                       int32_t score_fn, int32_t n_group, int32_t topk_group, int32_t renormalize,
                       int32_t *topk_idx, float *topk_w, const moe_dispatch_out *out,
                       int32_t *slot, void *workspace, size_t workspace_bytes_given,
                       int32_t *dev_err, void *stream, moe_handle *handle)
{
    int st = check_config(cfg);
    if (st != MOE_OK)
        return st;
    if ((st = check_router_args(T, cfg->E, cfg->k, logits, score_fn, n_group, topk_group, topk_idx,
                                topk_w)) != MOE_OK ||
        (st = check_dispatch_args(cfg, T, x, topk_idx, topk_w, out, slot, workspace,
                                  workspace_bytes_given, dev_err, handle)) != MOE_OK)
        return st;
    DeviceInfo *dev = nullptr;
    if ((st = device_info(&dev)) != MOE_OK)
        return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (T > 0 && (st = launch_router(T, cfg->E, cfg->k, logits, score_fn, n_group, topk_group,
                                     renormalize, topk_idx, topk_w, dev, s)) != MOE_OK)
        return st;
    return run_dispatch(cfg, T, x, topk_idx, topk_w, out, slot, workspace, dev_err, dev, s, handle,
                        true);
}

namespace {

int run_dispatch(const moe_config *cfg, int32_t T, const void *x, const int32_t *topk_idx,
                 const float *topk_w, const moe_dispatch_out *out, int32_t *slot,
                 void *workspace, int32_t *dev_err, DeviceInfo *dev, cudaStream_t s,
                 moe_handle *handle, bool after_router)
{
    int st;
    const bool fp8 = cfg->flags & MOE_FP8;

    const int per = T < dev->sms ? fused_chunks(cfg, T) : 0;
    if (per != 0) {
        FusedArgs f;
        f.x = static_cast<const uint16_t *>(x);
        f.topk_idx = topk_idx;
        f.T = T;
        f.H = cfg->H;
        f.k = cfg->k;
        f.E = cfg->E;
        f.R = cfg->R;
        f.pad128 = (cfg->flags & MOE_PAD128) ? 1 : 0;
        f.rows_cap = out->rows_cap;
        f.recv_x = out->recv_x;
        f.recv_scale = out->recv_scale;
        f.expert_count = out->expert_count;
        f.expert_offset = out->expert_offset;
        f.rank_offset = out->rank_offset;
        f.recv_src = out->recv_src;
        f.slot = slot;
        f.err = dev_err;
        const cudaError_t e = launch_small(fp8, per, T, s, f, after_router,
                                           !after_router && (cfg->flags & MOE_INPUTS_READY));
        if ((st = launched(e)) != MOE_OK)
            return st;
    } else if (use_multi(cfg, T)) {
        FusedArgs f;
        f.x = static_cast<const uint16_t *>(x);
        f.topk_idx = topk_idx;
        f.T = T;
        f.H = cfg->H;
        f.k = cfg->k;
        f.E = cfg->E;
        f.R = cfg->R;
        f.pad128 = (cfg->flags & MOE_PAD128) ? 1 : 0;
        f.rows_cap = out->rows_cap;
        f.recv_x = out->recv_x;
        f.recv_scale = out->recv_scale;
        f.expert_count = out->expert_count;
        f.expert_offset = out->expert_offset;
        f.rank_offset = out->rank_offset;
        f.recv_src = out->recv_src;
        f.slot = slot;
        f.err = dev_err;
        if ((st = launched(launch_multi(fp8, T, dev->sms, s, f))) != MOE_OK)
            return st;
    } else {
        if ((st = launch_layout(cfg, T, topk_idx, out, slot, workspace, dev_err, s)) != MOE_OK ||
            (st = launch_payload(cfg, T, x, slot, out, dev_err, dev, s, true)) != MOE_OK)
            return st;
    }
    handle->cfg = *cfg;
    handle->T = T;
    handle->slot = slot;
    handle->topk_w = topk_w;
    handle->rows_cap = out->rows_cap;
    return MOE_OK;
}

} // namespace

int moe_dispatch_layout(const moe_config *cfg, int32_t T, const int32_t *topk_idx,
                        const moe_dispatch_out *out, int32_t *slot, void *workspace,
                        size_t workspace_bytes_given, int32_t *dev_err, void *stream)
{
    int st = check_config(cfg);
    if (st != MOE_OK)
        return st;
    if ((st = check_layout_args(cfg, T, topk_idx, out, slot, workspace, workspace_bytes_given,
                                dev_err)) != MOE_OK)
        return st;
    DeviceInfo *dev = nullptr;
    if ((st = device_info(&dev)) != MOE_OK)
        return st;
    return launch_layout(cfg, T, topk_idx, out, slot, workspace, dev_err,
                         static_cast<cudaStream_t>(stream));
}

int moe_dispatch_payload(const moe_config *cfg, int32_t T, const void *x, const int32_t *slot,
                         const moe_dispatch_out *out, int32_t *dev_err, void *stream)
{
    int st = check_config(cfg);
    if (st != MOE_OK)
        return st;
    if (dev_err == nullptr || out == nullptr || out->rows_cap < 0 || out->rows_cap > INT32_MAX)
        return MOE_ERR_INVALID_ARG;
    if ((st = check_payload_args(cfg, T, x, slot, out)) != MOE_OK)
        return st;
    DeviceInfo *dev = nullptr;
    if ((st = device_info(&dev)) != MOE_OK)
        return st;
    return launch_payload(cfg, T, x, slot, out, dev_err, dev, static_cast<cudaStream_t>(stream),
                          false);
}

int moe_combine(const moe_handle *handle, const void *expert_out, void *y, int32_t *dev_err,
                void *stream)
{
    if (handle == nullptr)
        return MOE_ERR_INVALID_ARG;
    int st = check_config(&handle->cfg);
    if (st != MOE_OK)
        return st;
    const moe_config &c = handle->cfg;
    if (handle->T < 0 || handle->rows_cap < 0)
        return MOE_ERR_INVALID_ARG;
    if (handle->T == 0)
        return MOE_OK;
    if (handle->slot == nullptr || handle->topk_w == nullptr || y == nullptr ||
        (handle->rows_cap > 0 && expert_out == nullptr))
        return MOE_ERR_INVALID_ARG;
    if (!aligned16(expert_out) || !aligned16(y))
        return MOE_ERR_INVALID_ARG;
    DeviceInfo *dev = nullptr;
    if ((st = device_info(&dev)) != MOE_OK)
        return st;
    CombineArgs a;
    a.expert_out = static_cast<const uint16_t *>(expert_out);
    a.slot = handle->slot;
    a.w = handle->topk_w;
    a.T = handle->T;
    a.H = c.H;
    a.k = c.k;
    a.parts = (c.H / 8 + kCombineThreads - 1) / kCombineThreads;
    a.rows_cap = handle->rows_cap;
    a.y = static_cast<uint16_t *>(y);
    a.err = dev_err;
    const unsigned grid = grid_for((int64_t)a.T * a.parts, dev->sms, 16);
    return launched(launch(combine_rows, grid, kCombineThreads, 0, static_cast<cudaStream_t>(stream), a));
}

int moe_dispatch_no_alloc(const moe_config *cfg, int32_t T, const void *x,
                          const int32_t *topk_idx, const float *topk_w,
                          const moe_dispatch_out *out, int32_t *slot, int32_t *dev_err,
                          void *stream, moe_handle *handle)
{
    int st = check_config(cfg);
    if (st != MOE_OK)
        return st;
    if (T < 0)
        return MOE_ERR_INVALID_ARG;
    const size_t need = workspace_bytes(cfg, T);
    if (need > MOE_NO_ALLOC_SCRATCH_BYTES)
        return MOE_ERR_TOO_LARGE;
    void *scratch = nullptr;
    if ((st = no_alloc_scratch(&scratch)) != MOE_OK)
        return st;
    // The tiled metadata kernels write every scratch word they later read, so
    // the array needs no clearing between calls.
    return moe_dispatch(cfg, T, x, topk_idx, topk_w, out, slot, need > 0 ? scratch : nullptr, need,
                        dev_err, stream, handle);
}

int moe_selftest_bounded_wait(int32_t *dev_err, uint64_t limit_ns, void *stream)
{
    if (dev_err == nullptr || limit_ns == 0 || limit_ns > kWaitLimitNs)
        return MOE_ERR_INVALID_ARG;
    return launched(launch(wait_selftest, 1, kWarp, 0, static_cast<cudaStream_t>(stream), dev_err,
                           limit_ns));
}

int moe_combine_rank_partial(const moe_handle *handle, const int32_t *rank_offset,
                             const void *expert_out, void *partial, int32_t *partial_rank,
                             int32_t *npart, void *y, int32_t *dev_err, void *stream)
{
    if (handle == nullptr)
        return MOE_ERR_INVALID_ARG;
    int st = check_config(&handle->cfg);
    if (st != MOE_OK)
        return st;
    const moe_config &c = handle->cfg;
    if (handle->T < 0 || handle->rows_cap < 0)
        return MOE_ERR_INVALID_ARG;
    if (handle->T == 0)
        return MOE_OK;
    if (handle->slot == nullptr || handle->topk_w == nullptr || rank_offset == nullptr ||
        partial == nullptr || partial_rank == nullptr || npart == nullptr || y == nullptr ||
        (handle->rows_cap > 0 && expert_out == nullptr))
        return MOE_ERR_INVALID_ARG;
    if (!aligned16(expert_out) || !aligned16(partial) || !aligned16(y))
        return MOE_ERR_INVALID_ARG;
    DeviceInfo *dev = nullptr;
    if ((st = device_info(&dev)) != MOE_OK)
        return st;
    PartialArgs a;
    a.expert_out = static_cast<const uint16_t *>(expert_out);
    a.slot = handle->slot;
    a.w = handle->topk_w;
    a.rank_offset = rank_offset;
    a.T = handle->T;
    a.H = c.H;
    a.k = c.k;
    a.R = c.R;
    a.parts = (c.H / 8 + kPartialThreads - 1) / kPartialThreads;
    a.rows_cap = handle->rows_cap;
    a.partial = static_cast<uint16_t *>(partial);
    a.partial_rank = partial_rank;
    a.npart = npart;
    a.y = static_cast<uint16_t *>(y);
    a.err = dev_err;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // one resident wave of CTAs each
    const int64_t units = (int64_t)a.T * a.parts;
    const bool all_rows = a.k <= kCombineBatch;
    const unsigned send_grid = grid_for(units, dev->sms, dev->send_per_sm[all_rows ? 1 : 0]);
    const cudaError_t e = all_rows
                              ? launch(combine_partial_send<true>, send_grid, kPartialThreads, 0, s, a)
                              : launch(combine_partial_send<false>, send_grid, kPartialThreads, 0, s, a);
    if ((st = launched(e)) != MOE_OK)
        return st;
    return launched(launch(combine_partial_recv, grid_for(units, dev->sms, dev->recv_per_sm),
                           kPartialThreads, 0, s, a));
}

int moe_silu_quant(int64_t rows_cap, int32_t I, const void *gate_up, const int32_t *recv_src,
                   const int32_t *rows_in_use, void *act, float *act_scale,
                   int32_t scale_col_major, void *stream)
{
    if (rows_cap < 0 || rows_cap > INT32_MAX || I <= 0)
        return MOE_ERR_INVALID_ARG;
    if (I % 128 != 0)
        return MOE_ERR_UNSUPPORTED;
    if (rows_cap == 0)
        return MOE_OK;
    if (gate_up == nullptr || recv_src == nullptr || rows_in_use == nullptr || act == nullptr ||
        act_scale == nullptr)
        return MOE_ERR_INVALID_ARG;
    if (!aligned16(gate_up) || !aligned16(act))
        return MOE_ERR_INVALID_ARG;
    DeviceInfo *dev = nullptr;
    int st;
    if ((st = device_info(&dev)) != MOE_OK)
        return st;
    SiluQuantArgs a;
    a.gate_up = static_cast<const uint16_t *>(gate_up);
    a.recv_src = recv_src;
    a.rows_in_use = rows_in_use;
    a.rows_cap = rows_cap;
    a.I = I;
    a.act = static_cast<uint8_t *>(act);
    a.scale = act_scale;
    a.col_major = scale_col_major ? 1 : 0;
    // A fixed grid, whatever the routing (the kernel reads how many rows are in
    // use); the build and the grid follow the buffer's capacity in 512-column units.
    const int64_t units_cap = rows_cap * ((I + 511) / 512);
    const int64_t wide = (int64_t)dev->sms * dev->silu_per_sm[1];
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (units_cap >= wide * (kSiluThreads / kWarp) * kSiluUnitsPerWarpWide)
        return launched(launch(silu_quant_rows<kSiluWideCtas>, (unsigned)wide, kSiluThreads, 0, s, a));
    const unsigned grid = (unsigned)(dev->sms * std::min(dev->silu_per_sm[0], kSiluNarrowCtas));
    return launched(launch(silu_quant_rows<1>, grid, kSiluThreads, 0, s, a));
}

int moe_silu_mul(int64_t n, const void *gate, const void *up, float *act, double *fast_value,
                 int32_t exact_only, void *stream)
{
    if (n < 0)
        return MOE_ERR_INVALID_ARG;
    if (n == 0)
        return MOE_OK;
    if (gate == nullptr || up == nullptr || act == nullptr)
        return MOE_ERR_INVALID_ARG;
    DeviceInfo *dev = nullptr;
    int st;
    if ((st = device_info(&dev)) != MOE_OK)
        return st;
    SiluMulArgs a;
    a.gate = static_cast<const uint16_t *>(gate);
    a.up = static_cast<const uint16_t *>(up);
    a.n = n;
    a.act = act;
    a.fast_value = fast_value;
    a.exact_only = exact_only ? 1 : 0;
    const unsigned grid = grid_for((n + kSiluThreads - 1) / kSiluThreads, dev->sms, 8);
    return launched(launch(silu_mul_values, grid, kSiluThreads, 0, static_cast<cudaStream_t>(stream), a));
}

int moe_router_topk(int32_t T, int32_t E, int32_t k, const float *logits, int32_t score_fn,
                    int32_t n_group, int32_t topk_group, int32_t renormalize, int32_t *topk_idx,
                    float *topk_w, void *stream)
{
    int st = check_router_args(T, E, k, logits, score_fn, n_group, topk_group, topk_idx, topk_w);
    if (st != MOE_OK || T == 0)
        return st;
    DeviceInfo *dev = nullptr;
    if ((st = device_info(&dev)) != MOE_OK)
        return st;
    return launch_router(T, E, k, logits, score_fn, n_group, topk_group, renormalize, topk_idx,
                         topk_w, dev, static_cast<cudaStream_t>(stream));
}

namespace {

// Checks shared by the expert-parallel calls: cfg->R is the number of ranks.
int check_ep(const moe_config *cfg, int32_t T, int64_t rows_cap)
{
    int st = check_config(cfg);
    if (st != MOE_OK)
        return st;
    if (T < 0 || rows_cap < 0 || rows_cap > INT32_MAX)
        return MOE_ERR_INVALID_ARG;
    if (cfg->R > kEpMaxRanks)
        return MOE_ERR_UNSUPPORTED;
    return MOE_OK;
}

int fill_peers(EpPeers *t, const void *const *peers, int32_t W, bool need)
{
    for (int32_t r = 0; r < kEpMaxRanks; ++r)
        t->p[r] = nullptr;
    if (!need)
        return MOE_OK;
    if (peers == nullptr)
        return MOE_ERR_INVALID_ARG;
    for (int32_t r = 0; r < W; ++r) {
        if (peers[r] == nullptr || !aligned16(peers[r]))
            return MOE_ERR_INVALID_ARG;
        t->p[r] = const_cast<void *>(peers[r]);
    }
    return MOE_OK;
}

} // namespace

int64_t moe_ep_rows_capacity(const moe_config *cfg, int32_t T)
{
    if (check_config(cfg) != MOE_OK || T < 0 || cfg->R > kEpMaxRanks)
        return -1;
    const int64_t S = (int64_t)cfg->R * T * cfg->k; // every rank's entries to one rank
    if (!(cfg->flags & MOE_PAD128))
        return S;
    const int64_t el = cfg->E / cfg->R;
    const int64_t m = S < el ? S : el;
    return (S + 127 * m) / 128 * 128;
}

int moe_ep_layout(const moe_config *cfg, int32_t rank, int32_t T, const int32_t *topk_idx,
                  const int32_t *local_slot, const int32_t *local_offset, const int32_t *counts_all,
                  int64_t rows_cap, int32_t *dst_row, int32_t *recv_count, int32_t *recv_offset,
                  int32_t *dev_err, void *stream)
{
    int st = check_ep(cfg, T, rows_cap);
    if (st != MOE_OK)
        return st;
    if (rank < 0 || rank >= cfg->R || counts_all == nullptr || recv_count == nullptr ||
        recv_offset == nullptr || dev_err == nullptr)
        return MOE_ERR_INVALID_ARG;
    if (T > 0 && (topk_idx == nullptr || local_slot == nullptr || local_offset == nullptr ||
                  dst_row == nullptr))
        return MOE_ERR_INVALID_ARG;
    DeviceInfo *dev = nullptr;
    if ((st = device_info(&dev)) != MOE_OK)
        return st;
    EpRowsArgs a;
    a.topk_idx = topk_idx;
    a.local_slot = local_slot;
    a.local_offset = local_offset;
    a.counts_all = counts_all;
    a.T = T;
    a.k = cfg->k;
    a.E = cfg->E;
    a.W = cfg->R;
    a.rank = rank;
    a.pad128 = (cfg->flags & MOE_PAD128) ? 1 : 0;
    a.rows_cap = rows_cap;
    a.dst_row = dst_row;
    a.recv_count = recv_count;
    a.recv_offset = recv_offset;
    a.err = dev_err;
    const int64_t S = (int64_t)T * cfg->k;
    const unsigned grid = grid_for((S + kEpThreads - 1) / kEpThreads, dev->sms, 4);
    return launched(launch(ep_rows, grid, kEpThreads, ep_rows_smem(cfg->E),
                           static_cast<cudaStream_t>(stream), a));
}

int moe_ep_dispatch_payload(const moe_config *cfg, int32_t T, const void *x, const int32_t *topk_idx,
                            const int32_t *dst_row, void *const *peer_recv_x,
                            float *const *peer_recv_scale, int64_t rows_cap, int32_t rank,
                            int32_t *const *peer_flags, int32_t *epoch, int32_t *done_count,
                            int32_t *dev_err, void *stream)
{
    int st = check_ep(cfg, T, rows_cap);
    if (st != MOE_OK)
        return st;
    const bool fp8 = cfg->flags & MOE_FP8;
    const bool signal = peer_flags != nullptr;
    if (dev_err == nullptr)
        return MOE_ERR_INVALID_ARG;
    if (signal && (rank < 0 || rank >= cfg->R || epoch == nullptr || done_count == nullptr))
        return MOE_ERR_INVALID_ARG;
    if (T == 0 && !signal)
        return MOE_OK;
    if (T > 0 && (x == nullptr || !aligned16(x) || topk_idx == nullptr || dst_row == nullptr))
        return MOE_ERR_INVALID_ARG;
    EpPayloadArgs a;
    if ((st = fill_peers(&a.recv_x, (const void *const *)peer_recv_x, cfg->R, T > 0)) != MOE_OK ||
        (st = fill_peers(&a.recv_scale, (const void *const *)peer_recv_scale, cfg->R, T > 0 && fp8)) != MOE_OK)
        return st;
    a.sig.enabled = signal ? 1 : 0;
    a.sig.rank = rank;
    a.sig.W = cfg->R;
    a.sig.epoch = epoch;
    a.sig.done = done_count;
    for (int32_t r = 0; r < kEpMaxRanks; ++r)
        a.sig.flags.p[r] = nullptr;
    if (signal)
        for (int32_t r = 0; r < cfg->R; ++r) {
            if (peer_flags[r] == nullptr)
                return MOE_ERR_INVALID_ARG;
            a.sig.flags.p[r] = peer_flags[r];
        }
    DeviceInfo *dev = nullptr;
    if ((st = device_info(&dev)) != MOE_OK)
        return st;
    a.x = static_cast<const uint16_t *>(x);
    a.topk_idx = topk_idx;
    a.dst_row = dst_row;
    a.T = T;
    a.H = cfg->H;
    a.k = cfg->k;
    a.E = cfg->E;
    a.W = cfg->R;
    a.rows_cap = rows_cap;
    a.err = dev_err;
    const int64_t units = (int64_t)T * ((cfg->H + chunk_cols<kScatterLaneCols>() - 1) /
                                        chunk_cols<kScatterLaneCols>());
    const int64_t ctas = (units + kScatterThreads / kWarp - 1) / (kScatterThreads / kWarp);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // with T == 0 one CTA still runs, to signal
    const unsigned grid = grid_for(ctas, dev->sms, 8);
    const cudaError_t e = fp8 ? launch(ep_payload<true>, grid, kScatterThreads, 0, s, a)
                              : launch(ep_payload<false>, grid, kScatterThreads, 0, s, a);
    return launched(e);
}

int moe_ep_signal(int32_t W, int32_t rank, int32_t *const *peer_flags, int32_t *epoch, void *stream)
{
    if (W <= 0 || W > kEpMaxRanks || rank < 0 || rank >= W || peer_flags == nullptr || epoch == nullptr)
        return MOE_ERR_INVALID_ARG;
    EpSignal sig;
    for (int32_t r = 0; r < kEpMaxRanks; ++r)
        sig.flags.p[r] = nullptr;
    for (int32_t r = 0; r < W; ++r) {
        if (peer_flags[r] == nullptr)
            return MOE_ERR_INVALID_ARG;
        sig.flags.p[r] = peer_flags[r];
    }
    sig.epoch = epoch;
    sig.done = nullptr;
    sig.rank = rank;
    sig.W = W;
    sig.enabled = 1;
    return launched(launch(ep_signal, 1, kWarp, 0, static_cast<cudaStream_t>(stream), sig));
}

int moe_ep_wait(int32_t W, const int32_t *flags, const int32_t *epoch, uint64_t limit_ns,
                int32_t *dev_err, void *stream)
{
    if (W <= 0 || W > kEpMaxRanks || flags == nullptr || epoch == nullptr || dev_err == nullptr ||
        limit_ns == 0 || limit_ns > MOE_EP_MAX_WAIT_NS)
        return MOE_ERR_INVALID_ARG;
    return launched(launch(ep_wait, 1, kEpThreads, 0, static_cast<cudaStream_t>(stream), flags, epoch, W,
                           limit_ns, dev_err));
}

int moe_ep_combine(const moe_config *cfg, int32_t T, const int32_t *topk_idx, const int32_t *dst_row,
                   const float *topk_w, const void *const *peer_expert_out, int64_t rows_cap, void *y,
                   int32_t *dev_err, void *stream)
{
    int st = check_ep(cfg, T, rows_cap);
    if (st != MOE_OK)
        return st;
    if (dev_err == nullptr)
        return MOE_ERR_INVALID_ARG;
    if (T == 0)
        return MOE_OK;
    if (topk_idx == nullptr || dst_row == nullptr || topk_w == nullptr || y == nullptr || !aligned16(y))
        return MOE_ERR_INVALID_ARG;
    EpCombineArgs a;
    if ((st = fill_peers(&a.expert_out, peer_expert_out, cfg->R, true)) != MOE_OK)
        return st;
    DeviceInfo *dev = nullptr;
    if ((st = device_info(&dev)) != MOE_OK)
        return st;
    a.topk_idx = topk_idx;
    a.dst_row = dst_row;
    a.w = topk_w;
    a.T = T;
    a.H = cfg->H;
    a.k = cfg->k;
    a.E = cfg->E;
    a.W = cfg->R;
    a.parts = (cfg->H / 8 + kCombineThreads - 1) / kCombineThreads;
    a.rows_cap = rows_cap;
    a.y = static_cast<uint16_t *>(y);
    a.err = dev_err;
    const unsigned grid = grid_for((int64_t)T * a.parts, dev->sms, 16);
    return launched(launch(ep_combine, grid, kCombineThreads, 0, static_cast<cudaStream_t>(stream), a));
}

int moe_check(int32_t *dev_err, void *stream, int32_t *bits_out)
{
    if (dev_err == nullptr)
        return MOE_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int32_t bits = 0;
    if (cudaMemcpyAsync(&bits, dev_err, sizeof bits, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess ||
        cudaMemsetAsync(dev_err, 0, sizeof(int32_t), s) != cudaSuccess)
        return MOE_ERR_CUDA;
    if (bits_out != nullptr)
        *bits_out = bits;
    return bits ? MOE_ERR_DEVICE : MOE_OK;
}

} // extern "C"
