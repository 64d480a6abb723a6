// Dispatch of a mid-size batch in one launch: routing metadata and payload fused.
//
// Same results as the metadata kernels followed by the scatter (counts, offsets,
// (token, k)-ordered slots, bf16 rows or e4m3 codes with per-128 scales; the
// steps of "Enabling trillion-parameter models on AWS EFA", section "Despacho e
// Combinação"), for batches past the one-token-per-CTA kernels, where the
// three-launch tiled metadata would cost more than the counting it saves.
//
// One CTA per SM; CTA b owns the contiguous tokens [t0, t1) of a balanced split.
//   1. It issues the loads of row t0 (they do not depend on the routing).
//   2. It reads all S expert ids (served from L2 after the first CTA) and builds
//      in shared memory the histogram of all entries and of the entries before
//      its first one with plain shared-memory atomics.  Every CTA counts all S
//      entries, so the per-entry cost decides: grouping equal ids first
//      (__match_any_sync) cost several times more than the atomics it saved,
//      and equal ids within one warp serialise only as far as they repeat.
//   3. The exclusive scan of the (padded) counts gives every expert's offset.
//   4. The slot of its entry i (expert e) is offset[e] + before[e] + the number
//      of its own earlier entries with expert e: the stable (token, k) order.
//   5. Its warps walk the CTA's (token, 512-column chunk) units, the scatter's
//      layout of 16 columns per lane, each quantising (fp8) and storing one
//      unit while the loads of its next unit are in flight.
// CTA 0 writes the per-expert arrays; every CTA writes its share of the unused
// rows' recv_src = -1.
#pragma once

#include "common.cuh"
#include "dispatch_fused.cuh"
#include "meta.cuh"
#include "scatter.cuh"

namespace moe {

// Every CTA counts all S ids, which grows with S while the tiled metadata's
// cost barely does: measured on sweep batches (fp8, H = 7168), this kernel's
// dispatch took 20.0 us at S = 8192 against about 31 us for metadata + scatter,
// and 75 us at S = 32768 against 67 us; the two meet near S = 16384.
constexpr int64_t kMultiMaxEntries = 16384;
constexpr int kMultiLoadRounds = 4;
constexpr int kMultiThreads = 1024; // counting S ids and the payload both want many warps

// Shared memory: hist[E], before[E], off[E+1], ids[n_ent], slots[n_ent] with
// n_ent = the most entries one CTA owns.
inline size_t multi_smem(int32_t E, int32_t n_ent)
{
    return sizeof(int32_t) * ((size_t)3 * E + 1 + 2 * (size_t)n_ent);
}

template <bool kFp8>
__global__ void __launch_bounds__(kMultiThreads, 1) dispatch_multi(FusedArgs a, int32_t n_ent_max)
{
    stream_order_begin();
    extern __shared__ int32_t sm[];
    const int32_t E = a.E;
    int32_t *hist = sm, *before = sm + E, *off = sm + 2 * E;
    int32_t *s_ids = off + E + 1; // this CTA's entries' expert ids (-1: bad id)
    int32_t *s_slot = s_ids + n_ent_max;

    const int nt = blockDim.x;
    const int nwarps = nt / kWarp;
    const int warp = threadIdx.x / kWarp;
    constexpr int L = kScatterLaneCols;
    const int32_t chunks = (a.H + chunk_cols<L>() - 1) / chunk_cols<L>();
    const int32_t G = gridDim.x;
    const int32_t t0 = (int32_t)((int64_t)a.T * blockIdx.x / G);
    const int32_t t1 = (int32_t)((int64_t)a.T * (blockIdx.x + 1) / G);
    const int32_t S = a.T * a.k; // <= kMultiMaxEntries
    const int32_t e0 = t0 * a.k, e1 = t1 * a.k;

    // 1. The first payload unit of each warp: unit u is chunk u % chunks of
    //    token t0 + u / chunks; warp w owns units w, w + nwarps, ...
    const int32_t units = (t1 - t0) * chunks;
    LaneData<L> cur;
    if (warp < units)
        load_chunk<L, kFp8>(a.x + (int64_t)(t0 + warp / chunks) * a.H, a.H, warp % chunks, cur);

    // 2. Histograms of all entries and of the entries before e0.
    for (int32_t e = threadIdx.x; e < E; e += nt) {
        hist[e] = 0;
        before[e] = 0;
    }
    __syncthreads();
    for (int32_t base = 0; base < S; base += nt * kMultiLoadRounds) {
        int32_t ev[kMultiLoadRounds];
#pragma unroll
        for (int r = 0; r < kMultiLoadRounds; ++r) {
            const int32_t i = base + r * nt + (int32_t)threadIdx.x;
            ev[r] = i < S ? __ldg(a.topk_idx + i) : -1;
        }
#pragma unroll
        for (int r = 0; r < kMultiLoadRounds; ++r) {
            if (base + r * nt >= S)
                break; // the same for the whole CTA
            const int32_t i = base + r * nt + (int32_t)threadIdx.x;
            const bool valid = (uint32_t)ev[r] < (uint32_t)E;
            if (!valid && i < S && blockIdx.x == 0)
                raise_error(a.err, MOE_DEV_BAD_INDEX);
            const int32_t key = valid ? ev[r] : -1;
            if (key >= 0) {
                atomicAdd(&hist[key], 1);
                if (i < e0)
                    atomicAdd(&before[key], 1);
            }
            if (i >= e0 && i < e1)
                s_ids[i - e0] = key;
        }
    }
    __syncthreads();

    // 3. Offsets (exclusive scan of the padded counts); ends with a barrier.
    block_offsets(hist, off, E, a.pad128);

    // 4. This CTA's slots.
    for (int32_t i = threadIdx.x; i < e1 - e0; i += nt) {
        const int32_t e = s_ids[i];
        int32_t s = -1;
        if (e >= 0) {
            int32_t rank = 0;
            for (int32_t p = 0; p < i; ++p)
                rank += s_ids[p] == e;
            const int64_t row = (int64_t)off[e] + before[e] + rank;
            if (row < a.rows_cap) {
                s = (int32_t)row;
                a.recv_src[row] = e0 + i;
            } else {
                raise_error(a.err, MOE_DEV_CAPACITY);
            }
        }
        a.slot[e0 + i] = s;
        s_slot[i] = s;
    }
    if (blockIdx.x == 0) {
        for (int32_t e = threadIdx.x; e < E; e += nt) {
            a.expert_count[e] = hist[e];
            a.expert_offset[e] = off[e];
        }
        if (threadIdx.x == 0)
            a.expert_offset[E] = off[E];
        for (int32_t r = threadIdx.x; r <= a.R; r += nt)
            a.rank_offset[r] = off[r * (E / a.R)];
    }
    block_fill_unused(a.rows_cap, E, a.recv_src, hist, off, blockIdx.x, G);
    __syncthreads();

    // 5. Payload: quantise and store unit u while unit u + nwarps loads.
    for (int32_t u = warp; u < units; u += nwarps) {
        const int32_t un = u + nwarps;
        LaneData<L> nxt;
        if (un < units)
            load_chunk<L, kFp8>(a.x + (int64_t)(t0 + un / chunks) * a.H, a.H, un % chunks, nxt);
        store_chunk<L, kFp8>(a.recv_x, a.recv_scale, a.H, u % chunks, a.k, s_slot + (u / chunks) * a.k,
                             a.rows_cap, a.err, cur);
        if (un < units)
            cur = nxt;
    }
}

} // namespace moe
