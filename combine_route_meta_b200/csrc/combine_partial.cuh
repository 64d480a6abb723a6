// Combine with sender-side (per-rank) partial accumulation.
//
// "Enabling trillion-parameter models on AWS EFA", section "Avaliação": DeepEP
// accumulates on the sending side of the combine to move less data, and the
// page notes this may change precision; the page's own kernels accumulate only
// on the receiver.  Here every virtual rank r sums, for each token t, the
// weighted rows of t's entries whose experts r hosts, and emits that sum as
// one bf16 row (what the rank would send); the token's home then adds the at
// most min(k, R) partial rows (what it would receive).
//
//   stage 1 (send):  partial[t, q] = bf16( sum over t's entries j with rank r_q,
//                                          ascending j, of fma(w_j, row_j) ),
//                    r_q = the q-th distinct rank among t's kept entries in
//                    order of first appearance;
//   stage 2 (recv):  y[t] = bf16( sum_q float(partial[t, q]) ), ascending q.
//
// A slot's rank is found from rank_offset (rank r owns receive rows
// [rank_offset[r], rank_offset[r+1])), so the handle needs no expert ids.
// Layout: partial [T, k, H] bf16 (rows q >= npart[t] untouched),
// partial_rank [T, k], npart [T].  Both stages are one CTA per (token, part)
// with one 16-byte vector per thread, like combine_rows; the send stage works
// out the token's partials afresh in every unit (a warp-wide step for k <= 32).
#pragma once

#include "common.cuh"
#include "combine.cuh"

namespace moe {

constexpr int kPartialThreads = 128;
constexpr int kPartialMaxK = MOE_MAX_TOPK;

struct PartialArgs {
    const uint16_t *expert_out; // [rows_cap, H] bf16
    const int32_t *slot;        // [T, k]
    const float *w;             // [T, k]
    const int32_t *rank_offset; // [R+1]
    int32_t T, H, k, R;
    int32_t parts;
    int64_t rows_cap;
    uint16_t *partial;     // [T, k, H] bf16
    int32_t *partial_rank; // [T, k]
    int32_t *npart;        // [T]
    uint16_t *y;           // [T, H] bf16
    int32_t *err;
};

// Rank owning receive row s: the largest r with rank_offset[r] <= s.
__device__ __forceinline__ int32_t rank_of_row(const int32_t *rank_offset, int32_t R, int32_t s)
{
    int32_t lo = 0, hi = R;
    while (hi - lo > 1) {
        const int32_t mid = (lo + hi) / 2;
        if (__ldg(rank_offset + mid) <= s)
            lo = mid;
        else
            hi = mid;
    }
    return lo;
}

__device__ __forceinline__ void fma_row(float (&acc)[8], float wj, uint4 r)
{
    acc[0] = fmaf(wj, bf16_lo(r.x), acc[0]);
    acc[1] = fmaf(wj, bf16_hi(r.x), acc[1]);
    acc[2] = fmaf(wj, bf16_lo(r.y), acc[2]);
    acc[3] = fmaf(wj, bf16_hi(r.y), acc[3]);
    acc[4] = fmaf(wj, bf16_lo(r.z), acc[4]);
    acc[5] = fmaf(wj, bf16_hi(r.z), acc[5]);
    acc[6] = fmaf(wj, bf16_lo(r.w), acc[6]);
    acc[7] = fmaf(wj, bf16_hi(r.w), acc[7]);
}

__device__ __forceinline__ uint4 pack_row(const float (&acc)[8])
{
    return make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]),
                      pack_bf16x2(acc[4], acc[5]), pack_bf16x2(acc[6], acc[7]));
}

// Entry j's slot, and the partial it belongs to (-1 if dropped), into shared
// memory; *n = the token's number of partials.  Part 0 also writes the token's
// partial ranks and count.  For k <= 32, warp 0 does it with one lane per entry:
// lanes holding the same rank find each other (match_any), the first of them
// opens a partial, and an entry's partial is the number of partials opened
// before its rank's first entry.  Larger k takes one thread, in order.
__device__ __forceinline__ void partial_layout(const PartialArgs &a, int32_t t, int32_t part,
                                               int32_t *s_slot, int32_t *s_q, int32_t *s_rank,
                                               int32_t *n_out)
{
    const int64_t base = (int64_t)t * a.k;
    if (a.k <= kWarp) {
        if (threadIdx.x >= kWarp)
            return;
        const int32_t j = (int32_t)lane_id();
        int32_t s = -1, r = -1 - j; // dropped entries get ranks nobody shares
        bool valid = false;
        if (j < a.k) {
            s = __ldg(a.slot + base + j);
            if (s >= 0 && s < a.rows_cap) {
                valid = true;
                r = rank_of_row(a.rank_offset, a.R, s);
            } else {
                if (s != -1)
                    raise_error(a.err, MOE_DEV_BAD_SLOT);
                s = -1;
            }
        }
        const unsigned same = __match_any_sync(kFullMask, r);
        const int32_t first = __ffs(same) - 1;
        const unsigned opens = __ballot_sync(kFullMask, valid && first == j);
        const int32_t q = valid ? __popc(opens & ((1u << first) - 1u)) : -1;
        if (j < a.k) {
            s_slot[j] = s;
            s_q[j] = q;
        }
        if (part == 0 && valid && first == j)
            a.partial_rank[base + q] = r;
        if (j == 0) {
            *n_out = __popc(opens);
            if (part == 0)
                a.npart[t] = __popc(opens);
        }
        return;
    }
    if (threadIdx.x != 0)
        return;
    int32_t n = 0;
    for (int32_t j = 0; j < a.k; ++j) {
        int32_t s = __ldg(a.slot + base + j);
        if (!(s >= 0 && s < a.rows_cap)) {
            if (s != -1)
                raise_error(a.err, MOE_DEV_BAD_SLOT);
            s_slot[j] = -1;
            s_q[j] = -1;
            continue;
        }
        const int32_t r = rank_of_row(a.rank_offset, a.R, s);
        int32_t q = 0;
        while (q < n && s_rank[q] != r)
            ++q;
        if (q == n) {
            s_rank[n++] = r;
            if (part == 0)
                a.partial_rank[base + q] = r;
        }
        s_slot[j] = s;
        s_q[j] = q;
    }
    *n_out = n;
    if (part == 0)
        a.npart[t] = n;
}

// kAllRows (k <= kCombineBatch): every receive row of the token is loaded at
// once, then the partials are formed from registers one after another.
// Otherwise each partial loads its own rows, kCombineBatch at a time.
template <bool kAllRows>
__global__ void __launch_bounds__(kPartialThreads) combine_partial_send(PartialArgs a)
{
    stream_order_begin();
    __shared__ int32_t s_slot[kPartialMaxK];
    __shared__ int32_t s_q[kPartialMaxK]; // partial index of entry j, -1 if dropped
    __shared__ int32_t s_rank[kPartialMaxK];
    __shared__ int32_t s_n;
    const int32_t nvec = a.H / 8;
    const int64_t units = (int64_t)a.T * a.parts;
    for (int64_t u = blockIdx.x; u < units; u += gridDim.x) {
        const int32_t t = (int32_t)(u / a.parts);
        const int32_t part = (int32_t)(u % a.parts);
        __syncthreads(); // the previous unit is done with the shared arrays
        partial_layout(a, t, part, s_slot, s_q, s_rank, &s_n);
        __syncthreads();
        const int32_t v = part * kPartialThreads + (int32_t)threadIdx.x;
        if (v >= nvec)
            continue;
        const int32_t n = s_n;
        const float *ws = a.w + (int64_t)t * a.k;
        uint16_t *out = a.partial + (int64_t)t * a.k * a.H + (int64_t)v * 8;
        if constexpr (kAllRows) {
            uint4 r[kCombineBatch];
            float wv[kCombineBatch];
            int32_t qv[kCombineBatch];
#pragma unroll
            for (int j = 0; j < kCombineBatch; ++j) {
                const bool use = j < a.k && s_q[j] >= 0;
                qv[j] = use ? s_q[j] : -1;
                r[j] = use ? ld_stream_v4(a.expert_out + (int64_t)s_slot[j] * a.H + (int64_t)v * 8)
                           : make_uint4(0u, 0u, 0u, 0u);
                wv[j] = use ? __ldg(ws + j) : 0.0f;
            }
            for (int32_t q = 0; q < n; ++q) {
                float acc[8];
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    acc[i] = 0.0f;
#pragma unroll
                for (int j = 0; j < kCombineBatch; ++j)
                    if (qv[j] == q)
                        fma_row(acc, wv[j], r[j]);
                st_v4(out + (int64_t)q * a.H, pack_row(acc));
            }
        } else {
            for (int32_t q = 0; q < n; ++q) {
                float acc[8];
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    acc[i] = 0.0f;
                for (int32_t j0 = 0; j0 < a.k; j0 += kCombineBatch) {
                    uint4 r[kCombineBatch];
                    bool use[kCombineBatch];
#pragma unroll
                    for (int jj = 0; jj < kCombineBatch; ++jj) {
                        const int32_t j = j0 + jj;
                        use[jj] = j < a.k && s_q[j] == q;
                        r[jj] = use[jj] ? ld_stream_v4(a.expert_out + (int64_t)s_slot[j] * a.H + (int64_t)v * 8)
                                        : make_uint4(0u, 0u, 0u, 0u);
                    }
#pragma unroll
                    for (int jj = 0; jj < kCombineBatch; ++jj)
                        if (use[jj])
                            fma_row(acc, __ldg(ws + j0 + jj), r[jj]);
                }
                st_v4(out + (int64_t)q * a.H, pack_row(acc));
            }
        }
    }
}

__global__ void __launch_bounds__(kPartialThreads) combine_partial_recv(PartialArgs a)
{
    stream_order_begin();
    const int32_t nvec = a.H / 8;
    const int64_t units = (int64_t)a.T * a.parts;
    for (int64_t u = blockIdx.x; u < units; u += gridDim.x) {
        const int32_t t = (int32_t)(u / a.parts);
        const int32_t v = (int32_t)(u % a.parts) * kPartialThreads + (int32_t)threadIdx.x;
        if (v >= nvec)
            continue;
        const int32_t n = __ldg(a.npart + t);
        float acc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i)
            acc[i] = 0.0f;
        for (int32_t q0 = 0; q0 < n; q0 += kCombineBatch) {
            uint4 r[kCombineBatch];
#pragma unroll
            for (int qq = 0; qq < kCombineBatch; ++qq)
                r[qq] = q0 + qq < n ? ld_stream_v4(a.partial + ((int64_t)t * a.k + q0 + qq) * a.H + (int64_t)v * 8)
                                    : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
            for (int qq = 0; qq < kCombineBatch; ++qq)
                if (q0 + qq < n)
                    fma_row(acc, 1.0f, r[qq]);
        }
        st_v4(a.y + (int64_t)t * a.H + (int64_t)v * 8, pack_row(acc));
    }
}

} // namespace moe
