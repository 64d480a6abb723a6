// Dispatch of a small batch in one launch: routing metadata and payload fused.
//
// Same results as the metadata kernels followed by the scatter (counts, offsets,
// (token, k)-ordered slots, bf16 rows or e4m3 codes with per-128 scales; the
// steps of "Enabling trillion-parameter models on AWS EFA", section "Despacho e
// Combinação"), shaped for decode batches where one launch and one DRAM round
// trip cost more than the bytes.
//
// One CTA per token t; its warps own 256-column chunks of x[t] (the scatter's
// layout with 8 columns per lane, so a decode row gets up to 32 warps).  The CTA first issues the loads of x[t] (they do not
// depend on the routing), then reads all S = T*k expert ids (a few KB, served
// from L2 after the first CTA) and builds in shared memory the histogram of all
// entries and, in the same pass, the histogram of the entries that come before
// token t (shared-memory atomics).  With the exclusive scan of the (padded) counts, the slot of (t, j)
// with expert e is
//   offset[e] + before_t[e] + #{j' < j : topk_idx[t, j'] == e},
// which is the stable (token, k) order.  The CTA then stores (or quantises and
// stores) its row to its k slots.  CTA 0 also writes the per-expert counts and
// offsets; the padding rows' recv_src = -1 is split over all CTAs.  The
// redundant histogram per CTA is a few hundred instructions per warp at decode
// sizes, which is why this path is limited to S <= kFusedMaxEntries.
#pragma once

#include "common.cuh"
#include "meta.cuh"
#include "router.cuh"
#include "scatter.cuh"

namespace moe {

constexpr int kFusedMaxEntries = 2048;
constexpr int kFusedMaxK = 16;
constexpr int kFusedMaxThreads = 1024;
constexpr int kFusedLaneCols = 8;   // 256-column chunks: twice the warps per row of the scatter
constexpr int kFusedMaxChunks = 4;  // chunks per warp: rows up to 32 warps x 4 x 256 columns
constexpr int kFusedLoadRounds = 4; // expert ids loaded together per thread

struct FusedArgs {
    const uint16_t *x;
    const int32_t *topk_idx;
    int32_t T, H, k, E, R, pad128;
    int64_t rows_cap;
    void *recv_x;
    float *recv_scale;
    int32_t *expert_count, *expert_offset, *rank_offset, *recv_src, *slot;
    int32_t *err;
};

// Shared memory: hist[E], before[E], off[E+1].
inline size_t fused_smem(int32_t E) { return sizeof(int32_t) * ((size_t)3 * E + 1); }

template <int kChunks, bool kFp8>
__global__ void __launch_bounds__(kFusedMaxThreads, 1) dispatch_fused(FusedArgs a)
{
    stream_order_begin();
    extern __shared__ int32_t sm[];
    int32_t *hist = sm, *before = sm + a.E, *off = sm + 2 * a.E;
    __shared__ int32_t s_slot[kFusedMaxK];
    __shared__ int32_t s_own[kFusedMaxK];

    const int32_t t = blockIdx.x;
    const int nt = blockDim.x;
    const int nwarps = nt / kWarp;
    const int warp = threadIdx.x / kWarp;
    const unsigned lane = lane_id();
    constexpr int L = kFusedLaneCols;
    const int32_t chunks = (a.H + chunk_cols<L>() - 1) / chunk_cols<L>();

    // 1. The row's loads go out first: warp w owns chunks w, w + nwarps, ...
    const uint16_t *xr = a.x + (int64_t)t * a.H;
    LaneData<L> d[kChunks];
#pragma unroll
    for (int i = 0; i < kChunks; ++i) {
        const int32_t c = warp + i * nwarps;
        if (c < chunks)
            load_chunk<L, kFp8>(xr, a.H, c, d[i]);
    }

    // 2. Histograms of all entries and of the entries before token t; the
    //    token's own ids are kept in shared memory.
    for (int32_t e = threadIdx.x; e < a.E; e += nt) {
        hist[e] = 0;
        before[e] = 0;
    }
    __syncthreads();
    const int64_t S = (int64_t)a.T * a.k;
    const int64_t mine = (int64_t)t * a.k;
    for (int64_t base = 0; base < S; base += (int64_t)nt * kFusedLoadRounds) {
        int32_t ev[kFusedLoadRounds];
#pragma unroll
        for (int r = 0; r < kFusedLoadRounds; ++r) {
            const int64_t i = base + (int64_t)r * nt + threadIdx.x;
            ev[r] = i < S ? __ldg(a.topk_idx + i) : -1;
        }
#pragma unroll
        for (int r = 0; r < kFusedLoadRounds; ++r) {
            const int64_t i = base + (int64_t)r * nt + threadIdx.x;
            int32_t e = ev[r];
            if (i >= mine && i < mine + a.k)
                s_own[i - mine] = e;
            if (i < S && (e < 0 || e >= a.E)) {
                if (t == 0)
                    raise_error(a.err, MOE_DEV_BAD_INDEX);
                e = -1;
            }
            // Plain shared-memory atomics: at S <= kFusedMaxEntries a hot expert
            // costs little, and grouping lanes first (match_any) cost more than
            // it saved at decode sizes.
            if (e >= 0) {
                atomicAdd(&hist[e], 1);
                if (i < mine)
                    atomicAdd(&before[e], 1);
            }
        }
    }
    __syncthreads();

    // 3. Offsets (exclusive scan of the padded counts).
    block_offsets(hist, off, a.E, a.pad128);

    // 4. This token's slots.
    if (threadIdx.x < a.k) {
        const int j = threadIdx.x;
        const int32_t e = s_own[j];
        int32_t s = -1;
        if (e >= 0 && e < a.E) {
            int32_t dup = 0;
            for (int jj = 0; jj < j; ++jj)
                dup += s_own[jj] == e;
            const int64_t row = (int64_t)off[e] + before[e] + dup;
            if (row < a.rows_cap) {
                s = (int32_t)row;
                a.recv_src[row] = (int32_t)(mine + j);
            } else {
                raise_error(a.err, MOE_DEV_CAPACITY);
            }
        }
        a.slot[mine + j] = s;
        s_slot[j] = s;
    }
    if (t == 0) {
        for (int32_t e = threadIdx.x; e < a.E; e += nt) {
            a.expert_count[e] = hist[e];
            a.expert_offset[e] = off[e];
        }
        if (threadIdx.x == 0)
            a.expert_offset[a.E] = off[a.E];
        for (int32_t r = threadIdx.x; r <= a.R; r += nt)
            a.rank_offset[r] = off[(int64_t)r * (a.E / a.R)];
    }
    block_fill_unused(a.rows_cap, a.E, a.recv_src, hist, off, t, gridDim.x);
    __syncthreads();

    // 5. Payload to the k slots.
#pragma unroll
    for (int i = 0; i < kChunks; ++i) {
        const int32_t c = warp + i * nwarps;
        if (c < chunks)
            store_chunk<L, kFp8>(a.recv_x, a.recv_scale, a.H, c, a.k, s_slot, a.rows_cap, a.err, d[i]);
    }
}

// ---- direct-rank variant (no padding) -----------------------------------------
// Without padding the stable (token, k) order gives each entry a closed-form
// slot: for entry (t, j) with expert e,
//   slot = #{entries with expert < e} + #{entries (t', j') before (t, j) with expert e},
// the first term being the unpadded offset of e and the second its rank within
// e.  A token's CTA counts both terms for its own k experts while its row is in
// flight: each thread compares its share of the S expert ids with the k own ids,
// the two counts of entry j travel packed in one 32-bit word (low and high
// halves, S <= kFusedMaxEntries < 2^16), and a warp reduction plus one barrier
// finish them, so no per-expert histogram or scan sits on the token's path.
// One extra CTA (blockIdx.x == T) writes the per-expert counts and offsets, the
// rank offsets and the unused rows' recv_src, and flags bad expert ids.
// An expert id: from global memory through the read-only path (dispatch_direct,
// whose ids another kernel wrote), or from this CTA's shared memory (the fused
// router, which routes every token into it).
template <bool kShared>
__device__ __forceinline__ int32_t load_id(const int32_t *p)
{
    if constexpr (kShared)
        return *p;
    else
        return __ldg(p);
}

// The metadata CTA of the direct-rank dispatch: histogram, scan, offsets, and
// recv_src = -1 past the last segment (without padding there are no gaps
// between segments).  It runs beside the token CTAs and is about as long, so
// it is kept lean.  sm: E + 1 + E int32 of shared memory.
// With kDeferWrites the CTA reads and computes before waiting for the
// previous kernel in the stream (stream_order_begin) and writes only after it.
template <bool kIdsShared, bool kDeferWrites = false>
__device__ __forceinline__ void direct_meta_cta(const FusedArgs &a, const int32_t *ids, int32_t *sm)
{
    bool bad = false;
    const int nt = blockDim.x;
    const int64_t S = (int64_t)a.T * a.k;
    int32_t *hist = sm, *off = sm + a.E;
    for (int32_t e = threadIdx.x; e < a.E; e += nt)
        hist[e] = 0;
    __syncthreads();
    const int32_t S32 = (int32_t)S; // S <= kFusedMaxEntries
    for (int32_t base = 0; base < S32; base += nt * kFusedLoadRounds) {
        int32_t ev[kFusedLoadRounds];
#pragma unroll
        for (int r = 0; r < kFusedLoadRounds; ++r) {
            const int32_t i = base + r * nt + (int32_t)threadIdx.x;
            ev[r] = i < S32 ? load_id<kIdsShared>(ids + i) : 0;
        }
#pragma unroll
        for (int r = 0; r < kFusedLoadRounds; ++r) {
            if (base + r * nt + (int32_t)threadIdx.x >= S32)
                break;
            if ((uint32_t)ev[r] < (uint32_t)a.E)
                atomicAdd(&hist[ev[r]], 1);
            else
                bad = true;
        }
    }
    __syncthreads();
    block_offsets(hist, off, a.E, 0);
    if constexpr (kDeferWrites)
        stream_order_begin();
    if (bad)
        raise_error(a.err, MOE_DEV_BAD_INDEX);
    for (int32_t e = threadIdx.x; e < a.E; e += nt) {
        a.expert_count[e] = hist[e];
        a.expert_offset[e] = off[e];
    }
    if (threadIdx.x == 0)
        a.expert_offset[a.E] = off[a.E];
    for (int32_t r = threadIdx.x; r <= a.R; r += nt)
        a.rank_offset[r] = off[r * (a.E / a.R)];
    block_fill_tail(a.rows_cap, a.E, a.recv_src, off, 0, 1);
}

// Loads the token's row: warp w owns chunks w, w + nwarps, ...
template <int kChunks, bool kFp8>
__device__ __forceinline__ void direct_load_row(const FusedArgs &a, int32_t t, LaneData<kFusedLaneCols> (&d)[kChunks])
{
    constexpr int L = kFusedLaneCols;
    const int nwarps = blockDim.x / kWarp;
    const int warp = threadIdx.x / kWarp;
    const int32_t chunks = (a.H + chunk_cols<L>() - 1) / chunk_cols<L>();
    const uint16_t *xr = a.x + (int64_t)t * a.H;
#pragma unroll
    for (int i = 0; i < kChunks; ++i) {
        const int32_t c = warp + i * nwarps;
        if (c < chunks)
            load_chunk<L, kFp8>(xr, a.H, c, d[i]);
    }
}

// Shared memory of a direct-rank token CTA.
template <int kK>
struct DirectShared {
    uint32_t part[kFusedMaxThreads / kWarp][kK];
    int32_t slot[kK];
    int32_t own[kK];
};

// fp8 rows of the direct-rank dispatch leave as whole-row bulk stores (one per
// slot for the codes, one for the scales) from a shared-memory copy of the row,
// when the row fits it and both stores are whole 16-byte units (H % 512 == 0
// makes the H/32 scale bytes one).  One contiguous multi-kilobyte write per
// receive row is what the HBM write stream favours; the register path writes
// every slot's row in 256-byte pieces from all warps.
constexpr int32_t kDirectBulkMaxH = 8192;

__host__ __device__ inline bool direct_bulk_rows(int32_t H) { return H % 512 == 0 && H <= kDirectBulkMaxH; }

struct __align__(128) DirectRow {
    uint8_t b[kDirectBulkMaxH + kDirectBulkMaxH / 32]; // codes, then the H/128 fp32 scales
};

// The CTA's shared-memory row (allocated only in kernels that use it).
__device__ __forceinline__ DirectRow &sh_row()
{
    __shared__ DirectRow row;
    return row;
}

// A token CTA of the direct-rank dispatch, from the expert ids on; with
// kRowLoaded the row is already in d (else it is loaded after the ids go out).
template <int kChunks, bool kFp8, int kK, bool kRowLoaded, bool kIdsShared, bool kDeferWrites = false>
__device__ __forceinline__ void direct_token_cta(const FusedArgs &a, const int32_t *ids, int32_t t,
                                                 LaneData<kFusedLaneCols> (&d)[kChunks],
                                                 LaneCodes<kFusedLaneCols> (&q)[kFp8 ? kChunks : 1],
                                                 bool quantised, DirectShared<kK> &sh)
{
    const int nt = blockDim.x;
    const int nwarps = nt / kWarp;
    const int warp = threadIdx.x / kWarp;
    const unsigned lane = lane_id();
    const int64_t S = (int64_t)a.T * a.k;
    constexpr int L = kFusedLaneCols;
    const int32_t chunks = (a.H + chunk_cols<L>() - 1) / chunk_cols<L>();
    const int64_t mine = (int64_t)t * a.k;
    constexpr int32_t kNone = 0x7fffffff; // never below or equal to a valid id
    const int32_t S32 = (int32_t)S, mine32 = (int32_t)mine; // S <= kFusedMaxEntries

    // 1. The expert ids go out first (the own ids as broadcast loads, then this
    //    thread's first round of all ids), ahead of the row, whose kilobytes
    //    would otherwise queue in front of them.
    constexpr bool kOwnInRegs = kK <= 8; // more own ids are read from shared memory
    int32_t own[kOwnInRegs ? kK : 1];
    if constexpr (kOwnInRegs) {
#pragma unroll
        for (int j = 0; j < kK; ++j) {
            const int32_t e = j < a.k ? load_id<kIdsShared>(ids + mine + j) : -1;
            own[j] = (uint32_t)e < (uint32_t)a.E ? e : -1;
        }
    }
    int32_t ev[kFusedLoadRounds];
#pragma unroll
    for (int r = 0; r < kFusedLoadRounds; ++r) {
        const int32_t i = r * nt + (int32_t)threadIdx.x;
        ev[r] = i < S32 ? load_id<kIdsShared>(ids + i) : kNone;
    }

    // 2. The row: warp w owns chunks w, w + nwarps, ...
    if constexpr (!kRowLoaded)
        direct_load_row<kChunks, kFp8>(a, t, d);
    if ((int)threadIdx.x < kK) {
        const int32_t e = (int)threadIdx.x < a.k ? load_id<kIdsShared>(ids + mine + threadIdx.x) : -1;
        sh.own[threadIdx.x] = (e >= 0 && e < a.E) ? e : -1;
    }
    if constexpr (!kOwnInRegs)
        __syncthreads();

    // 3. Counts of this thread's entries against the own ids, round by round;
    //    a warp whose entries of a round all lie past S stops there.
    uint32_t cnt[kK];
#pragma unroll
    for (int j = 0; j < kK; ++j)
        cnt[j] = 0;
    for (int32_t base = 0; base < S32; base += nt * kFusedLoadRounds) {
        if (base > 0) {
#pragma unroll
            for (int r = 0; r < kFusedLoadRounds; ++r) {
                const int32_t i = base + r * nt + (int32_t)threadIdx.x;
                ev[r] = i < S32 ? load_id<kIdsShared>(ids + i) : kNone;
            }
        }
#pragma unroll
        for (int r = 0; r < kFusedLoadRounds; ++r) {
            const int32_t i = base + r * nt + (int32_t)threadIdx.x;
            if (__all_sync(kFullMask, i >= S32))
                break; // later rounds start further out
            // Compared as unsigned, an id outside [0, E) is above every valid own
            // id, so bad ids count in neither term without a separate check.
            const uint32_t e = (uint32_t)ev[r];
            const int32_t before = i - mine32; // entry i precedes (t, j) when before < j
#pragma unroll
            for (int j = 0; j < kK; ++j) {
                const uint32_t o = (uint32_t)(kOwnInRegs ? own[kOwnInRegs ? j : 0] : sh.own[j]);
                cnt[j] += e < o ? 1u : 0u;
                cnt[j] += (e == o && before < j) ? 0x10000u : 0u;
            }
        }
    }
#pragma unroll
    for (int j = 0; j < kK; ++j) {
        const uint32_t w = __reduce_add_sync(kFullMask, cnt[j]);
        if (lane == 0)
            sh.part[warp][j] = w;
    }
    __syncthreads();

    // 4. This token's slots: warp j adds the per-warp counts of entry j.
    //    (With kDeferWrites they are written in 5b.)
    for (int j = warp; j < a.k; j += nwarps) {
        const uint32_t v = (int)lane < nwarps ? sh.part[lane][j] : 0u;
        const uint32_t tot = __reduce_add_sync(kFullMask, v);
        if (lane == 0) {
            int32_t s = -1;
            if (sh.own[j] >= 0) {
                const int64_t row = (int64_t)(tot & 0xffffu) + (tot >> 16);
                if (row < a.rows_cap) {
                    s = (int32_t)row;
                    if constexpr (!kDeferWrites)
                        a.recv_src[row] = (int32_t)(mine + j);
                } else if constexpr (!kDeferWrites) {
                    raise_error(a.err, MOE_DEV_CAPACITY);
                } else {
                    s = -2; // over capacity: flagged in 5b
                }
            }
            if constexpr (!kDeferWrites)
                a.slot[mine + j] = s;
            sh.slot[j] = s;
        }
    }

    // 5. The row's codes (unless already made), while the slot sums above
    //    complete; for the bulk stores they go to the shared-memory row.
    const bool bulk_rows = kFp8 && direct_bulk_rows(a.H);
    if constexpr (kFp8) {
        if (!quantised) {
#pragma unroll
            for (int i = 0; i < kChunks; ++i)
                if (warp + i * nwarps < chunks)
                    quantise_lane<L>(d[i], q[i].codes, q[i].scale);
        }
        if (bulk_rows) {
            static_assert(L == 8, "two code words per lane");
            uint8_t *row = sh_row().b;
#pragma unroll
            for (int i = 0; i < kChunks; ++i) {
                const int32_t c = warp + i * nwarps;
                const int32_t col = c * chunk_cols<L>() + (int32_t)lane * L;
                if (c < chunks) { // H % 512 == 0: every column of the chunk is in the row
                    *reinterpret_cast<uint2 *>(row + col) = make_uint2(q[i].codes[0], q[i].codes[1]);
                    if ((lane & 15) == 0) // the first lane of each 128-column block
                        reinterpret_cast<float *>(row + a.H)[col / 128] = q[i].scale;
                }
            }
            fence_async_shared(); // the bulk stores read what the generic proxy wrote
        }
    }
    __syncthreads();

    // 5b. With kDeferWrites: wait for the previous kernel, then write the slots.
    if constexpr (kDeferWrites) {
        stream_order_begin();
        if ((int)threadIdx.x < a.k) {
            const int j = threadIdx.x;
            int32_t s = sh.slot[j];
            if (s == -2) {
                raise_error(a.err, MOE_DEV_CAPACITY);
                s = -1;
                sh.slot[j] = -1;
            } else if (s >= 0) {
                a.recv_src[s] = (int32_t)(mine + j);
            }
            a.slot[mine + j] = s;
        }
        __syncthreads();
    }

    // 6. Payload to the k slots: thread j issues slot j's two bulk stores and
    //    waits until they have read the row (the writes complete with the grid),
    //    or every warp stores its chunks from registers.
    if constexpr (kFp8) {
        if (bulk_rows) {
            if ((int)threadIdx.x < a.k) {
                const int32_t s = sh.slot[threadIdx.x]; // -1 or a row below rows_cap
                const uint8_t *row = sh_row().b;
                if (s >= 0) {
                    bulk_store(static_cast<uint8_t *>(a.recv_x) + (int64_t)s * a.H, smem_addr(row),
                               (uint32_t)a.H);
                    bulk_store(a.recv_scale + (int64_t)s * (a.H / 128), smem_addr(row + a.H),
                               (uint32_t)(a.H / 32));
                }
                bulk_commit();
                bulk_wait_read<0>();
            }
            return;
        }
    }
#pragma unroll
    for (int i = 0; i < kChunks; ++i) {
        const int32_t c = warp + i * nwarps;
        if (c >= chunks)
            continue;
        if constexpr (kFp8)
            store_codes<L>(a.recv_x, a.recv_scale, a.H, c, a.k, sh.slot, a.rows_cap, a.err, q[i]);
        else
            store_chunk<L, false>(a.recv_x, a.recv_scale, a.H, c, a.k, sh.slot, a.rows_cap, a.err, d[i]);
    }
}

template <int kChunks, bool kFp8, int kK>
__global__ void __launch_bounds__(kFusedMaxThreads, 1) dispatch_direct(FusedArgs a)
{
    stream_order_begin();
    extern __shared__ int32_t sm[];
    __shared__ DirectShared<kK> sh;
    const int32_t t = blockIdx.x;
    if (t == a.T) {
        direct_meta_cta<false>(a, a.topk_idx, sm);
        return;
    }
    LaneData<kFusedLaneCols> d[kChunks];
    LaneCodes<kFusedLaneCols> q[kFp8 ? kChunks : 1];
    direct_token_cta<kChunks, kFp8, kK, false, false>(a, a.topk_idx, t, d, q, false, sh);
}

// dispatch_direct when the caller states (MOE_INPUTS_READY) that x and the
// routing were complete before the previous kernel in the stream began: all
// the reading and computing (ids, row, codes, counts, slots, the histogram and
// scan) happens before waiting for that kernel, so it overlaps that kernel's
// tail, and only the writes follow the wait (the previous kernel may still be
// reading the buffers this one writes).
template <int kChunks, bool kFp8, int kK>
__global__ void __launch_bounds__(kFusedMaxThreads, 1) dispatch_direct_ready(FusedArgs a)
{
    extern __shared__ int32_t sm[];
    __shared__ DirectShared<kK> sh;
    const int32_t t = blockIdx.x;
    if (t == a.T) {
        direct_meta_cta<false, true>(a, a.topk_idx, sm);
        return;
    }
    LaneData<kFusedLaneCols> d[kChunks];
    LaneCodes<kFusedLaneCols> q[kFp8 ? kChunks : 1];
    direct_token_cta<kChunks, kFp8, kK, false, false, true>(a, a.topk_idx, t, d, q, false, sh);
}

// ---- after the router (decode) ----------------------------------------------------
// dispatch_direct for moe_route_dispatch, launched right after the router in
// the same stream.  The row of x and (fp8) its codes do not depend on the
// routing, and the router writes neither x nor anything x depends on; it
// waited for every earlier kernel before it let this one launch, so x is
// complete when this kernel starts.  Each token CTA therefore loads and
// quantises its row while the router is still running, and waits for the
// router (griddepcontrol.wait) only before it reads the expert ids.  (The x
// loads do not allocate in L1, so no stale line can exist.)
template <int kChunks, bool kFp8, int kK>
__global__ void __launch_bounds__(kFusedMaxThreads, 1) dispatch_direct_after_router(FusedArgs a)
{
    extern __shared__ int32_t sm[];
    __shared__ DirectShared<kK> sh;
    const int32_t t = blockIdx.x;
    LaneData<kFusedLaneCols> d[kChunks];
    LaneCodes<kFusedLaneCols> q[kFp8 ? kChunks : 1];
    if (t < a.T) {
        direct_load_row<kChunks, kFp8>(a, t, d);
        if constexpr (kFp8) {
            const int nwarps = blockDim.x / kWarp, warp = threadIdx.x / kWarp;
            const int32_t chunks = (a.H + chunk_cols<kFusedLaneCols>() - 1) / chunk_cols<kFusedLaneCols>();
#pragma unroll
            for (int i = 0; i < kChunks; ++i)
                if (warp + i * nwarps < chunks)
                    quantise_lane<kFusedLaneCols>(d[i], q[i].codes, q[i].scale);
        }
    }
    stream_order_begin();
    if (t == a.T) {
        direct_meta_cta<false>(a, a.topk_idx, sm);
        return;
    }
    direct_token_cta<kChunks, kFp8, kK, true, false>(a, a.topk_idx, t, d, q, kFp8, sh);
}

} // namespace moe
