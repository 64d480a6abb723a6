// Expert parallelism across GPUs: every rank dispatches its own tokens straight
// into the receive buffers of the ranks that host their experts, and gathers
// the experts' output rows back for its own combine.
//
// "Enabling trillion-parameter models on AWS EFA", sections "Buffers de Envio e
// Recebimento" and "Despacho e Combinação": the ranks first share their
// per-expert counts; from them every sender knows, for each peer, the
// contiguous range its rows take in that peer's receive buffer, so one
// receive buffer per rank suffices and each sender writes its rows straight
// into it.  Inside a node the writes are NVLink stores to peer-mapped memory
// (section "MoE all-to-all sobre EFA").
//
// Layout.  W ranks; rank d hosts experts [d E_l, (d+1) E_l), E_l = E / W.  With
// cnt[s][e] the number of rank s's entries routed to expert e (gathered from
// all ranks), rank d's receive buffer holds, expert by expert, the rows of rank
// 0, then rank 1, ..., each in (token, k) order; with MOE_PAD128 every expert's
// segment is padded to a multiple of 128 rows.  The row of rank s's entry
// (t, j) with expert e in rank d's buffer is therefore
//   off_d(e) + sum_{s' < s} cnt[s'][e] + (its rank among s's entries with e),
// off_d(e) = sum over d's experts e' < e of the (padded) totals over ranks.
// That is the single-GPU layout of all ranks' batches concatenated in rank
// order, rank d's part starting at its rank offset, so the single-GPU oracle
// fixes it.  A rank's own rank among its entries is slot - offset[e] of its
// local, unpadded, one-rank layout (moe_dispatch_layout with R = 1).
//
// Peer buffers are reached through a table of W base pointers (peer mappings
// of the other GPUs' buffers, this rank's own at its index).  Stores and loads
// are plain 16-byte accesses; nothing here uses TMA or multicast, so the same
// kernels are correct on peer memory.
//
// Completion (section "Despacho e Combinação": a receiver reads its buffers
// once the senders have signalled that their writes are complete).  Every rank
// holds, in its own memory, one int32 flag per sender for each of two events:
// "the sender's rows are in my receive buffer" and "the sender's expert
// outputs are ready to be read".  A rank counts its own signals of each event
// in a device epoch.  To signal, it fences at system scope, increments the
// epoch and stores it into its slot of every peer's flags (a release pattern);
// the payload kernel does this from its last CTA, after every CTA has fenced
// its stores at system scope and counted itself done.  To wait, a rank polls
// its own flags until each reaches its own epoch of the event, then fences (an
// acquire pattern)
// (every rank signals each event once per layer, so the epochs agree), for a
// bounded time; on expiry it sets MOE_DEV_TIMEOUT and returns.  The host never
// blocks, so a layer's exchange can be captured in a CUDA graph.
#pragma once

#include "combine.cuh"
#include "common.cuh"
#include "meta.cuh"
#include "scatter.cuh"

namespace moe {

constexpr int kEpMaxRanks = 64;
constexpr int kEpThreads = 256;

struct EpPeers {
    void *p[kEpMaxRanks];
};

struct EpRowsArgs {
    const int32_t *topk_idx;     // [T, k] this rank's routing
    const int32_t *local_slot;   // [T, k] its one-rank unpadded layout
    const int32_t *local_offset; // [E + 1] of that layout
    const int32_t *counts_all;   // [W, E] every rank's per-expert counts
    int32_t T, k, E, W, rank, pad128;
    int64_t rows_cap; // rows of every rank's receive buffer
    int32_t *dst_row;     // [T, k] row in the destination rank's buffer, -1 if dropped
    int32_t *recv_count;  // [E_l] this rank's experts' totals over ranks
    int32_t *recv_offset; // [E_l + 1] their offsets in this rank's buffer
    int32_t *err;
};

// Shared memory: tot[E], base[E], goff[E + 1].
inline size_t ep_rows_smem(int32_t E) { return sizeof(int32_t) * ((size_t)3 * E + 1); }

__global__ void __launch_bounds__(kEpThreads) ep_rows(EpRowsArgs a)
{
    stream_order_begin();
    extern __shared__ int32_t sm[];
    const int32_t E = a.E, El = a.E / a.W;
    int32_t *tot = sm, *base = sm + E, *goff = sm + 2 * E;
    for (int32_t e = threadIdx.x; e < E; e += blockDim.x) {
        int32_t t = 0, b = 0;
        for (int32_t s = 0; s < a.W; ++s) {
            const int32_t c = __ldg(a.counts_all + (int64_t)s * E + e);
            t += c;
            if (s < a.rank)
                b += c;
        }
        tot[e] = t;
        base[e] = b;
    }
    __syncthreads();
    // offsets over all experts; an expert's offset in its rank's buffer is the
    // difference from the offset of that rank's first expert
    block_offsets(tot, goff, E, a.pad128);
    for (int32_t e = threadIdx.x; e < E; e += blockDim.x)
        base[e] += goff[e] - goff[e / El * El];
    __syncthreads();
    if (blockIdx.x == 0) {
        const int32_t e0 = a.rank * El;
        for (int32_t i = threadIdx.x; i < El; i += blockDim.x) {
            a.recv_count[i] = tot[e0 + i];
            a.recv_offset[i] = goff[e0 + i] - goff[e0];
        }
        if (threadIdx.x == 0)
            a.recv_offset[El] = goff[e0 + El] - goff[e0];
    }
    const int64_t S = (int64_t)a.T * a.k;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < S;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int32_t e = __ldg(a.topk_idx + i);
        const int32_t s = __ldg(a.local_slot + i);
        int32_t row = -1;
        if ((uint32_t)e < (uint32_t)E && s >= 0) {
            const int64_t r = (int64_t)base[e] + (s - __ldg(a.local_offset + e));
            if (r < a.rows_cap)
                row = (int32_t)r;
            else
                raise_error(a.err, MOE_DEV_CAPACITY);
        }
        a.dst_row[i] = row;
    }
}

// ---- completion flags ---------------------------------------------------------

struct EpFlagPeers {
    int32_t *p[kEpMaxRanks]; // [W] each rank's flags of one event, W int32 each
};

// A sender's side of one event: its slot `rank` in every peer's flags, its
// epoch of the event, and (payload kernel only) the count of CTAs done.
struct EpSignal {
    EpFlagPeers flags;
    int32_t *epoch;
    int32_t *done;
    int32_t rank, W;
    int32_t enabled;
};

// Relaxed system-scope accesses: with one fence before the stores (a release
// pattern) and one after the loads (an acquire pattern), a signal costs one
// system-scope fence however many peers it reaches or polls.
__device__ __forceinline__ void st_relaxed_sys(int32_t *p, int32_t v)
{
    asm volatile("st.relaxed.sys.global.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ int32_t ld_relaxed_sys(const int32_t *p)
{
    int32_t v;
    asm volatile("ld.relaxed.sys.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// One thread: makes this grid's earlier writes visible at system scope, then
// publishes the next epoch in every peer's slot of this sender.
__device__ __forceinline__ void ep_publish(const EpSignal &s)
{
    __threadfence_system();
    const int32_t e = *s.epoch + 1;
    *s.epoch = e;
    for (int32_t d = 0; d < s.W; ++d)
        st_relaxed_sys(s.flags.p[d] + s.rank, e);
}

// End of a grid whose writes the signal covers: the CTA's barrier orders its
// threads' writes before thread 0, whose system-scope fence (cumulative over
// what the barrier ordered before it) precedes its count of the CTA as done;
// the last CTA to count publishes.  The count is reset for the next launch,
// which stream order puts after this one.
__device__ __forceinline__ void ep_signal_grid(const EpSignal &s)
{
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence_system();
        const int32_t prev = atomicAdd(s.done, 1);
        if (prev == (int32_t)gridDim.x - 1) {
            *s.done = 0;
            ep_publish(s);
        }
    }
}

// moe_ep_signal: publishes after the previous kernel in the stream completed.
__global__ void __launch_bounds__(kWarp) ep_signal(EpSignal s)
{
    stream_order_begin();
    if (threadIdx.x == 0)
        ep_publish(s);
}

// moe_ep_wait: until flags[s] reaches *epoch for every sender s (wrap-safe
// comparison), each polled by one thread, for at most limit_ns in all; then a
// system-scope fence.
__global__ void __launch_bounds__(kEpThreads) ep_wait(const int32_t *flags, const int32_t *epoch, int32_t W,
                                                      uint64_t limit_ns, int32_t *err)
{
    stream_order_begin();
    const int32_t target = *epoch;
    const uint64_t t0 = global_ns();
    for (int32_t s = threadIdx.x; s < W; s += blockDim.x) {
        // the difference is taken in unsigned arithmetic, which wraps
        while ((int32_t)((uint32_t)ld_relaxed_sys(flags + s) - (uint32_t)target) < 0) {
            if (global_ns() - t0 > limit_ns) {
                raise_error(err, MOE_DEV_TIMEOUT);
                break;
            }
            __nanosleep(100);
        }
    }
    __threadfence_system(); // the peers' writes before their signals are seen after this kernel
}

struct EpPayloadArgs {
    const uint16_t *x;
    const int32_t *topk_idx, *dst_row;
    int32_t T, H, k, E, W;
    int64_t rows_cap;
    EpPeers recv_x;     // [W] receive buffers [rows_cap, H]
    EpPeers recv_scale; // [W] fp8 scales [rows_cap, H/128]
    EpSignal sig;       // "rows in place", when enabled
    int32_t *err;
};

// The destination row of entry j of a token (the same for the whole warp) and
// its rank in d, or -1 when the entry is dropped; a row outside [-1, rows_cap)
// is flagged and skipped, so no store or load leaves a buffer.
__device__ __forceinline__ int64_t ep_entry(const int32_t *idx_t, const int32_t *row_t, int32_t j,
                                            int32_t E, int32_t El, int64_t rows_cap, int32_t *err,
                                            int32_t &d)
{
    const int32_t e = __ldg(idx_t + j);
    const int32_t r = __ldg(row_t + j);
    if (r == -1 || (uint32_t)e >= (uint32_t)E)
        return -1;
    if (r < 0 || r >= rows_cap) {
        raise_error(err, MOE_DEV_BAD_SLOT);
        return -1;
    }
    d = e / El;
    return r;
}

// Warps walk (token, chunk) units as scatter_rows does; the k rows of a token
// go to the buffers of the ranks hosting their experts.
template <bool kFp8>
__global__ void __launch_bounds__(kScatterThreads) ep_payload(EpPayloadArgs a)
{
    stream_order_begin();
    constexpr int L = kScatterLaneCols;
    const unsigned lane = lane_id();
    const int32_t El = a.E / a.W;
    const int64_t nwarps = (int64_t)gridDim.x * (kScatterThreads / kWarp);
    const int32_t chunks = (a.H + chunk_cols<L>() - 1) / chunk_cols<L>();
    const int64_t units = (int64_t)a.T * chunks;
    const int32_t nb = a.H / 128;
    for (int64_t u = (int64_t)blockIdx.x * (kScatterThreads / kWarp) + threadIdx.x / kWarp; u < units;
         u += nwarps) {
        const int32_t t = (int32_t)(u / chunks);
        const int32_t c = (int32_t)(u % chunks);
        LaneData<L> dl;
        load_chunk<L, kFp8>(a.x + (int64_t)t * a.H, a.H, c, dl);
        const int32_t *idx_t = a.topk_idx + (int64_t)t * a.k;
        const int32_t *row_t = a.dst_row + (int64_t)t * a.k;
        if constexpr (kFp8) {
            LaneCodes<L> q;
            quantise_lane<L>(dl, q.codes, q.scale);
            const int32_t col = lane_col<L, true>(c, 0);
            const bool active = col < a.H; // H % 128 == 0: whole blocks are in or out
            for (int32_t j = 0; j < a.k; ++j) {
                int32_t d = 0;
                const int64_t r = ep_entry(idx_t, row_t, j, a.E, El, a.rows_cap, a.err, d);
                if (r < 0)
                    continue;
                if (active) {
                    uint8_t *dst = static_cast<uint8_t *>(a.recv_x.p[d]) + r * a.H + col;
                    st_v4(dst, make_uint4(q.codes[0], q.codes[1], q.codes[2], q.codes[3]));
                    if ((lane & (128 / L - 1)) == 0)
                        static_cast<float *>(a.recv_scale.p[d])[r * nb + col / 128] = q.scale;
                }
            }
        } else {
            for (int32_t j = 0; j < a.k; ++j) {
                int32_t d = 0;
                const int64_t r = ep_entry(idx_t, row_t, j, a.E, El, a.rows_cap, a.err, d);
                if (r < 0)
                    continue;
                uint16_t *dst = static_cast<uint16_t *>(a.recv_x.p[d]) + r * a.H;
#pragma unroll
                for (int i = 0; i < L / 8; ++i) {
                    const int32_t col = lane_col<L, false>(c, i);
                    if (col < a.H)
                        st_v4(dst + col, dl.v[i]);
                }
            }
        }
    }
    if (a.sig.enabled)
        ep_signal_grid(a.sig);
}

struct EpCombineArgs {
    const int32_t *topk_idx, *dst_row;
    const float *w;
    int32_t T, H, k, E, W;
    int32_t parts;
    int64_t rows_cap;
    EpPeers expert_out; // [W] expert outputs [rows_cap, H] bf16, receive layout
    uint16_t *y;
    int32_t *err;
};

// combine_rows with each entry's row read from the buffer of the rank that
// hosts its expert: the same fp32 chain in ascending j, the same bf16 result.
__global__ void __launch_bounds__(kCombineThreads) ep_combine(EpCombineArgs a)
{
    stream_order_begin();
    const int32_t nvec = a.H / 8;
    const int32_t El = a.E / a.W;
    const int64_t units = (int64_t)a.T * a.parts;
    for (int64_t u = blockIdx.x; u < units; u += gridDim.x) {
        const int32_t t = (int32_t)(u / a.parts);
        const int32_t v = (int32_t)(u % a.parts) * kCombineThreads + threadIdx.x;
        if (v >= nvec)
            continue;
        const int32_t *idx_t = a.topk_idx + (int64_t)t * a.k;
        const int32_t *row_t = a.dst_row + (int64_t)t * a.k;
        const float *ws = a.w + (int64_t)t * a.k;
        float acc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i)
            acc[i] = 0.0f;
        for (int32_t j0 = 0; j0 < a.k; j0 += kCombineBatch) {
            uint4 r[kCombineBatch];
            bool use[kCombineBatch];
#pragma unroll
            for (int jj = 0; jj < kCombineBatch; ++jj) {
                use[jj] = false;
                r[jj] = make_uint4(0u, 0u, 0u, 0u);
                if (j0 + jj < a.k) {
                    int32_t d = 0;
                    const int64_t row = ep_entry(idx_t, row_t, j0 + jj, a.E, El, a.rows_cap, a.err, d);
                    if (row >= 0) {
                        use[jj] = true;
                        r[jj] = ld_stream_v4(static_cast<const uint16_t *>(a.expert_out.p[d]) +
                                             row * a.H + (int64_t)v * 8);
                    }
                }
            }
#pragma unroll
            for (int jj = 0; jj < kCombineBatch; ++jj) {
                if (!use[jj])
                    continue;
                const float wj = __ldg(ws + j0 + jj);
                acc[0] = fmaf(wj, bf16_lo(r[jj].x), acc[0]);
                acc[1] = fmaf(wj, bf16_hi(r[jj].x), acc[1]);
                acc[2] = fmaf(wj, bf16_lo(r[jj].y), acc[2]);
                acc[3] = fmaf(wj, bf16_hi(r[jj].y), acc[3]);
                acc[4] = fmaf(wj, bf16_lo(r[jj].z), acc[4]);
                acc[5] = fmaf(wj, bf16_hi(r[jj].z), acc[5]);
                acc[6] = fmaf(wj, bf16_lo(r[jj].w), acc[6]);
                acc[7] = fmaf(wj, bf16_hi(r[jj].w), acc[7]);
            }
        }
        uint4 out;
        out.x = pack_bf16x2(acc[0], acc[1]);
        out.y = pack_bf16x2(acc[2], acc[3]);
        out.z = pack_bf16x2(acc[4], acc[5]);
        out.w = pack_bf16x2(acc[6], acc[7]);
        st_v4(a.y + (int64_t)t * a.H + (int64_t)v * 8, out);
    }
}

} // namespace moe
