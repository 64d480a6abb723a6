// Routing metadata: per-expert counts, offsets and deterministic slots.
//
// "Enabling trillion-parameter models on AWS EFA", section "Despacho e
// Combinação": the dispatch first counts the tokens routed to each expert
// (atomic accumulation in shared memory), then takes the cumulative sum of the
// counts to find where each expert's tokens are packed contiguously; section
// "Buffers de Envio e Recebimento" asks for contiguous packing so that no
// private per-sender space is needed.  The order inside an expert's segment is
// fixed here as (token, k) ascending, which makes slot assignment a stable
// counting sort of the S = T*k routing entries by expert id.
//
// GPU design.  Entries are processed in rounds of one entry per thread.  The
// counts are plain shared-memory atomics.  For the slots, lanes of a warp
// holding the same expert find each other with __match_any_sync: the lowest
// such lane does one shared-memory update for the whole group, and a lane's
// rank inside the group is the population count of the group's lanes below
// it.  A lane's slot is then
//   cursor[e]                          (rows handed out to e by earlier rounds)
// + sum over lower warps of their group sizes for e   (this round)
// + rank inside its own warp's group.
// That is exactly the stable order, with no sort and no global atomics.
//
// Launch shapes (moe_dispatch takes the one-launch kernels of dispatch_fused.cuh
// and dispatch_multi.cuh where they apply; moe_dispatch_layout always uses these):
//  - S <= kSingleBlockEntries: one CTA does counts, scan and slots in shared
//    memory (one launch, no scratch);
//  - larger batches: tiles of kTileEntries entries.  (1) each CTA counts its
//    tile into scratch tile_hist[tile][E]; (2) CTAs of 32 experts turn each
//    expert's column into an exclusive prefix over tiles and write the counts;
//    (3) each CTA takes the scan of the counts for the offsets and assigns its
//    tile's slots from offset[e] + tile prefix.
// Every CTA loads the expert ids of all its rounds before the first round, so
// it pays one memory latency, not one per round.
#pragma once

#include "common.cuh"

namespace moe {

constexpr int kMetaThreads = 512;
constexpr int kMetaWarps = kMetaThreads / kWarp;
constexpr int kTileEntries = 1024;
constexpr int kSingleBlockEntries = 4096;

struct MetaArgs {
    const int32_t *topk_idx;
    int64_t S; // T*k routing entries
    int32_t k, E, R, pad128;
    int64_t rows_cap;
    int32_t *expert_count;  // [E]
    int32_t *expert_offset; // [E+1]
    int32_t *rank_offset;   // [R+1]
    int32_t *slot;          // [S]
    int32_t *recv_src;      // [rows_cap]
    int32_t *err;
};

// Expert id of entry i, or -1 for no entry (past the end, or out of range).
__device__ __forceinline__ int32_t entry_expert(const MetaArgs &a, int64_t i, bool flag_bad)
{
    if (i >= a.S)
        return -1;
    int32_t e = __ldg(a.topk_idx + i);
    if (e < 0 || e >= a.E) {
        if (flag_bad)
            raise_error(a.err, MOE_DEV_BAD_INDEX);
        return -1;
    }
    return e;
}

// Expert ids of entries begin + r*kMetaThreads + threadIdx.x for r < kRounds
// (-1 where there is no entry), loaded together.
template <int kRounds>
__device__ __forceinline__ void load_entries(const MetaArgs &a, int64_t begin, int64_t end,
                                             bool flag_bad, int32_t (&e)[kRounds])
{
#pragma unroll
    for (int r = 0; r < kRounds; ++r) {
        const int64_t i = begin + (int64_t)r * kMetaThreads + threadIdx.x;
        e[r] = i < end ? entry_expert(a, i, flag_bad) : -1;
    }
}

// Adds the entries [begin, end) into hist[E] (shared memory);
// end - begin <= kRounds * kMetaThreads.  Plain shared-memory atomics: equal
// ids in a warp serialise only as far as they repeat, and grouping them first
// with __match_any_sync cost more on sm_100 than it saved, even for a Zipf-hot
// expert.
template <int kRounds>
__device__ __forceinline__ void block_count(const MetaArgs &a, int64_t begin, int64_t end,
                                            int32_t *hist)
{
    int32_t e[kRounds];
    load_entries<kRounds>(a, begin, end, true, e);
#pragma unroll
    for (int r = 0; r < kRounds; ++r)
        if (e[r] >= 0)
            atomicAdd(&hist[e[r]], 1);
}

// Exclusive scan of the (optionally 128-padded) counts in shared memory:
// off[e] = sum_{e' < e} seg(e'), off[E] = total.  `cnt` and `off` may not alias.
// Any block size that is a multiple of 32 (up to 1024); uses the whole block
// and ends with a barrier.
__device__ void block_offsets(const int32_t *cnt, int32_t *off, int32_t E, int32_t pad128)
{
    // Each round scans blockDim.x counts: shuffle scan inside every warp, then
    // every warp scans the warp totals itself (shuffles again, no serial walk).
    __shared__ int32_t warp_sums[32];
    const unsigned lane = lane_id(), warp = threadIdx.x / kWarp;
    const int nt = blockDim.x;
    const int nwarps = nt / kWarp;
    int32_t carry = 0; // identical in every thread
    for (int32_t base = 0; base < E; base += nt) {
        const int32_t e = base + threadIdx.x;
        int32_t v = 0;
        if (e < E) {
            v = cnt[e];
            if (pad128)
                v = (v + 127) / 128 * 128;
        }
        int32_t incl = v;
#pragma unroll
        for (int d = 1; d < kWarp; d <<= 1) {
            const int32_t n = __shfl_up_sync(kFullMask, incl, d);
            if (lane >= (unsigned)d)
                incl += n;
        }
        if (lane == kWarp - 1)
            warp_sums[warp] = incl;
        __syncthreads();
        const int32_t ws = (int)lane < nwarps ? warp_sums[lane] : 0;
        int32_t wincl = ws;
#pragma unroll
        for (int d = 1; d < kWarp; d <<= 1) {
            const int32_t n = __shfl_up_sync(kFullMask, wincl, d);
            if (lane >= (unsigned)d)
                wincl += n;
        }
        const int32_t before = __shfl_sync(kFullMask, wincl - ws, warp); // exclusive, this warp
        const int32_t total = __shfl_sync(kFullMask, wincl, kWarp - 1);
        if (e < E)
            off[e] = carry + before + incl - v;
        carry += total;
        __syncthreads(); // warp_sums is rewritten by the next round
    }
    if (threadIdx.x == 0)
        off[E] = carry;
    __syncthreads();
}

// Assigns slots to entries [begin, end) in order; end - begin <= kRounds *
// kMetaThreads.  cursor[e] (shared) holds the first free row of expert e for
// this range and is advanced; wcnt is [kMetaWarps][E] shared scratch that must
// be zero on entry and is zero on exit.
template <int kRounds>
__device__ __forceinline__ void block_assign(const MetaArgs &a, int64_t begin, int64_t end,
                                             int32_t *cursor, int32_t *wcnt)
{
    int32_t ev[kRounds];
    load_entries<kRounds>(a, begin, end, false, ev);
    const unsigned lane = lane_id(), warp = threadIdx.x / kWarp;
#pragma unroll
    for (int r = 0; r < kRounds; ++r) {
        const int64_t base = begin + (int64_t)r * kMetaThreads;
        if (base >= end)
            break;
        const int64_t i = base + threadIdx.x;
        const int32_t e = ev[r];
        const unsigned peers = __match_any_sync(kFullMask, e);
        const unsigned leader = __ffs(peers) - 1;
        const int32_t rank = __popc(peers & lanemask_lt());
        const int32_t group = __popc(peers);
        const bool lead = e >= 0 && lane == leader;
        if (lead)
            wcnt[warp * a.E + e] = group;
        __syncthreads();
        int32_t first = 0;
        if (lead) {
            first = cursor[e];
            for (unsigned w = 0; w < warp; ++w)
                first += wcnt[w * a.E + e];
        }
        first = __shfl_sync(kFullMask, first, leader);
        __syncthreads();
        if (lead) {
            atomicAdd(&cursor[e], group);
            wcnt[warp * a.E + e] = 0;
        }
        if (i < end) {
            int32_t s = -1;
            if (e >= 0) {
                const int64_t row = (int64_t)first + rank;
                if (row < a.rows_cap) {
                    s = (int32_t)row;
                    a.recv_src[row] = (int32_t)i;
                } else {
                    raise_error(a.err, MOE_DEV_CAPACITY);
                }
            }
            a.slot[i] = s;
        }
        __syncthreads();
    }
}

// recv_src = -1 on rows that hold no entry: each expert's padding, and the rows
// from expert_offset[E] to rows_cap.  Work is split over `nblk` blocks; inside
// a block, one warp clears one expert's padding (at most 127 rows).
// recv_src = -1 on the rows past the last segment, [off[E], rows_cap).
__device__ __forceinline__ void block_fill_tail(int64_t rows_cap, int32_t E, int32_t *recv_src,
                                                const int32_t *off, int blk, int nblk)
{
    for (int64_t r = (int64_t)off[E] + (int64_t)blk * blockDim.x + threadIdx.x; r < rows_cap;
         r += (int64_t)nblk * blockDim.x)
        recv_src[r] = -1;
}

// recv_src = -1 on every row no entry fills: the padding at the end of each
// expert's segment and the rows past the last segment.
__device__ __forceinline__ void block_fill_unused(int64_t rows_cap, int32_t E, int32_t *recv_src,
                                                  const int32_t *cnt, const int32_t *off, int blk,
                                                  int nblk)
{
    const int nwarps = blockDim.x / kWarp;
    const int warp = threadIdx.x / kWarp, lane = lane_id();
    for (int32_t e = blk * nwarps + warp; e < E; e += nblk * nwarps) {
        int64_t lo = (int64_t)off[e] + cnt[e];
        int64_t hi = off[e + 1] < rows_cap ? off[e + 1] : rows_cap;
        for (int64_t r = lo + lane; r < hi; r += kWarp)
            recv_src[r] = -1;
    }
    block_fill_tail(rows_cap, E, recv_src, off, blk, nblk);
}

// Writes expert_count, expert_offset and rank_offset from shared cnt/off.
__device__ __forceinline__ void write_offsets(const MetaArgs &a, const int32_t *cnt,
                                              const int32_t *off)
{
    for (int32_t e = threadIdx.x; e < a.E; e += blockDim.x) {
        a.expert_count[e] = cnt[e];
        a.expert_offset[e] = off[e];
    }
    if (threadIdx.x == 0)
        a.expert_offset[a.E] = off[a.E];
    for (int32_t r = threadIdx.x; r <= a.R; r += blockDim.x)
        a.rank_offset[r] = off[(int64_t)r * (a.E / a.R)];
}

// ---- one-CTA path -------------------------------------------------------------
constexpr int kSingleRounds = kSingleBlockEntries / kMetaThreads;

// Shared memory: cnt[E], off[E+1], cursor[E], wcnt[kMetaWarps*E].
__global__ void __launch_bounds__(kMetaThreads) meta_single_block(MetaArgs a)
{
    stream_order_begin();
    extern __shared__ int32_t sm[];
    int32_t *cnt = sm, *off = sm + a.E, *cursor = off + a.E + 1, *wcnt = cursor + a.E;
    for (int32_t e = threadIdx.x; e < a.E; e += kMetaThreads)
        cnt[e] = 0;
    for (int32_t i = threadIdx.x; i < kMetaWarps * a.E; i += kMetaThreads)
        wcnt[i] = 0;
    __syncthreads();
    block_count<kSingleRounds>(a, 0, a.S, cnt);
    __syncthreads();
    block_offsets(cnt, off, a.E, a.pad128);
    write_offsets(a, cnt, off);
    for (int32_t e = threadIdx.x; e < a.E; e += kMetaThreads)
        cursor[e] = off[e];
    __syncthreads();
    block_assign<kSingleRounds>(a, 0, a.S, cursor, wcnt);
    block_fill_unused(a.rows_cap, a.E, a.recv_src, cnt, off, 0, 1);
}

// ---- tiled path ----------------------------------------------------------------
constexpr int kTileRounds = kTileEntries / kMetaThreads;

// (1) tile_hist[tile][e] = entries of tile `tile` routed to e.
__global__ void __launch_bounds__(kMetaThreads) meta_tile_count(MetaArgs a, int32_t *tile_hist)
{
    stream_order_begin();
    extern __shared__ int32_t hist[];
    for (int32_t e = threadIdx.x; e < a.E; e += kMetaThreads)
        hist[e] = 0;
    __syncthreads();
    const int64_t begin = (int64_t)blockIdx.x * kTileEntries;
    const int64_t end = begin + kTileEntries < a.S ? begin + kTileEntries : a.S;
    block_count<kTileRounds>(a, begin, end, hist);
    __syncthreads();
    for (int32_t e = threadIdx.x; e < a.E; e += kMetaThreads)
        tile_hist[(int64_t)blockIdx.x * a.E + e] = hist[e];
}

// (2) Per-expert exclusive prefix over tiles, in place, and the counts.
// A CTA owns 32 experts (one per lane); its 8 warps split the tiles, add their
// share, combine the shares through shared memory, then rewrite their tiles
// with running prefixes.  Loads are issued 8 tiles at a time.
constexpr int kScanThreads = 256;
constexpr int kScanWarps = kScanThreads / kWarp;

__global__ void __launch_bounds__(kScanThreads) meta_tile_scan(MetaArgs a, int32_t *tile_hist,
                                                               int32_t ntiles)
{
    stream_order_begin();
    __shared__ int32_t part[kScanWarps][kWarp];
    const int warp = threadIdx.x / kWarp, lane = lane_id();
    const int32_t e = blockIdx.x * kWarp + lane;
    const bool valid = e < a.E;
    const int32_t per = (ntiles + kScanWarps - 1) / kScanWarps;
    const int32_t t_lo = warp * per;
    const int32_t t_hi = t_lo + per < ntiles ? t_lo + per : ntiles;
    int32_t sum = 0;
    for (int32_t t0 = t_lo; t0 < t_hi; t0 += 8) {
        int32_t c[8];
#pragma unroll
        for (int u = 0; u < 8; ++u)
            c[u] = (valid && t0 + u < t_hi) ? tile_hist[(int64_t)(t0 + u) * a.E + e] : 0;
#pragma unroll
        for (int u = 0; u < 8; ++u)
            sum += c[u];
    }
    part[warp][lane] = sum;
    __syncthreads();
    int32_t run = 0, total = 0;
    for (int w = 0; w < kScanWarps; ++w) {
        if (w < warp)
            run += part[w][lane];
        total += part[w][lane];
    }
    for (int32_t t0 = t_lo; t0 < t_hi; t0 += 8) {
        int32_t c[8];
#pragma unroll
        for (int u = 0; u < 8; ++u)
            c[u] = (valid && t0 + u < t_hi) ? tile_hist[(int64_t)(t0 + u) * a.E + e] : 0;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            if (valid && t0 + u < t_hi)
                tile_hist[(int64_t)(t0 + u) * a.E + e] = run;
            run += c[u];
        }
    }
    if (valid && warp == 0)
        a.expert_count[e] = total;
}

// (3) Slots of one tile.  Every CTA scans the counts for the offsets (E values,
// cheaper than another launch), starts each expert's cursor at offset[e] + the
// tile's prefix, and assigns its entries; CTA 0 writes the offsets, and all
// CTAs share clearing the unused rows' recv_src.
// Shared memory: cnt[E], off[E+1], cursor[E], wcnt[kMetaWarps*E].
__global__ void __launch_bounds__(kMetaThreads) meta_tile_assign(MetaArgs a,
                                                                 const int32_t *tile_prefix)
{
    stream_order_begin();
    extern __shared__ int32_t sm[];
    int32_t *cnt = sm, *off = sm + a.E, *cursor = off + a.E + 1, *wcnt = cursor + a.E;
    for (int32_t e = threadIdx.x; e < a.E; e += kMetaThreads) {
        cnt[e] = a.expert_count[e];
        cursor[e] = tile_prefix[(int64_t)blockIdx.x * a.E + e];
    }
    for (int32_t i = threadIdx.x; i < kMetaWarps * a.E; i += kMetaThreads)
        wcnt[i] = 0;
    __syncthreads();
    block_offsets(cnt, off, a.E, a.pad128);
    if (blockIdx.x == 0)
        write_offsets(a, cnt, off);
    for (int32_t e = threadIdx.x; e < a.E; e += kMetaThreads)
        cursor[e] += off[e];
    __syncthreads();
    const int64_t begin = (int64_t)blockIdx.x * kTileEntries;
    const int64_t end = begin + kTileEntries < a.S ? begin + kTileEntries : a.S;
    block_assign<kTileRounds>(a, begin, end, cursor, wcnt);
    block_fill_unused(a.rows_cap, a.E, a.recv_src, cnt, off, blockIdx.x, gridDim.x);
}

inline size_t meta_single_smem(int32_t E) { return sizeof(int32_t) * ((size_t)3 * E + 1 + (size_t)kMetaWarps * E); }
inline size_t meta_count_smem(int32_t E) { return sizeof(int32_t) * (size_t)E; }
inline size_t meta_assign_smem(int32_t E) { return meta_single_smem(E); }

inline int64_t meta_tiles(int64_t S) { return (S + kTileEntries - 1) / kTileEntries; }

} // namespace moe
