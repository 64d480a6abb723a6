// Router top-k: the per-token expert choice that feeds dispatch.
//
// "Lower latency and higher throughput with multi-node DeepSeek deployment",
// section "Roteador MoE": one top-k with index tracking serves every MoE model,
// plain top-k being group-limited top-k with a single group.  For a token's
// logits l[0..E):
//   - experts form n_group contiguous groups; a group's score is its largest
//     logit; the topk_group best groups are kept (ties: lower group id);
//   - the k largest logits among the kept groups' experts are chosen, best
//     first (ties: lower expert id);
//   - weights: softmax (exp(l_j - m) over the chosen k when renormalising, else
//     over all E) or sigmoid (1/(1+exp(-l_j)), divided by their sum when
//     renormalising).
// Softmax and sigmoid are increasing, so the choice compares logits only and
// is exact; the weights use expf and IEEE division.
//
// One warp per token: the logits go to shared memory, the lanes fold them into
// per-group maxima with shared-memory atomics, and each pick is a warp-wide
// argmax of (value, id) pairs (larger value, then smaller id) over each lane's
// best remaining candidate; lane e % 32 owns expert e and keeps a bitmask of
// its experts already taken.
#pragma once

#include "common.cuh"

namespace moe {

constexpr int kRouterMaxE = 1024;
constexpr int kRouterMaxK = 32;
constexpr int kRouterMaxGroups = 32;
constexpr int kRouterWarps = 4;

struct RouterArgs {
    const float *logits; // [T, E]
    int32_t T, E, k, score_fn, n_group, topk_group, renormalize;
    int32_t *topk_idx; // [T, k]
    float *topk_w;     // [T, k]
};

// Warp-wide best (value, id): larger value wins, equal values go to the smaller id.
__device__ __forceinline__ void warp_argmax(float &v, int32_t &id)
{
#pragma unroll
    for (int d = 16; d >= 1; d >>= 1) {
        const float ov = __shfl_xor_sync(kFullMask, v, d);
        const int32_t oid = __shfl_xor_sync(kFullMask, id, d);
        if (ov > v || (ov == v && oid < id)) {
            v = ov;
            id = oid;
        }
    }
}

// A signed integer that orders like the float it comes from (finite values).
__device__ __forceinline__ int32_t ordered_key(float f)
{
    const int32_t i = __float_as_int(f);
    return i >= 0 ? i : (int32_t)(0x80000000u - (uint32_t)i);
}

__device__ __forceinline__ float key_value(int32_t k)
{
    return __int_as_float(k >= 0 ? k : (int32_t)(0x80000000u - (uint32_t)k));
}

__device__ __forceinline__ float warp_sum(float v)
{
#pragma unroll
    for (int d = 16; d >= 1; d >>= 1)
        v += __shfl_xor_sync(kFullMask, v, d);
    return v;
}

__global__ void __launch_bounds__(kRouterWarps * kWarp) router_topk(RouterArgs a)
{
    stream_order_begin();
    __shared__ float s_l[kRouterWarps][kRouterMaxE];
    __shared__ int32_t s_g[kRouterWarps][kRouterMaxGroups];
    const int warp = threadIdx.x / kWarp;
    const int32_t lane = (int32_t)lane_id();
    float *sl = s_l[warp];
    int32_t *sg = s_g[warp];
    const int32_t gsize = a.E / a.n_group;
    const int32_t per_lane = (a.E + kWarp - 1) / kWarp;
    const float neg_inf = -__int_as_float(0x7f800000);
    const int64_t nwarps = (int64_t)gridDim.x * kRouterWarps;
    for (int64_t t = (int64_t)blockIdx.x * kRouterWarps + warp; t < a.T; t += nwarps) {
        const float *l = a.logits + t * a.E;
        for (int32_t e = lane; e < a.E; e += kWarp)
            sl[e] = __ldg(l + e);
        __syncwarp();

        // groups: every lane folds its own experts into the group maxima (order-
        // preserving integer keys, shared-memory atomics), then lane g reads group g
        uint32_t kept = 0xffffffffu;
        if (a.n_group > 1) {
            if (lane < a.n_group)
                sg[lane] = INT32_MIN;
            __syncwarp();
            for (int32_t e = lane; e < a.E; e += kWarp)
                atomicMax(&sg[e / gsize], ordered_key(sl[e]));
            __syncwarp();
            const float gscore = lane < a.n_group ? key_value(sg[lane]) : neg_inf;
            kept = 0;
            for (int32_t p = 0; p < a.topk_group; ++p) {
                float v = (lane < a.n_group && !((kept >> lane) & 1u)) ? gscore : neg_inf;
                int32_t id = lane < a.n_group ? lane : INT32_MAX;
                warp_argmax(v, id);
                kept |= 1u << id;
            }
        }

        // experts: lane owns e = lane + 32 i
        uint32_t taken = 0;
        int32_t my_idx = -1;  // lane j < k ends holding the j-th pick
        float my_logit = 0.0f;
        for (int32_t j = 0; j < a.k; ++j) {
            float v = neg_inf;
            int32_t id = INT32_MAX;
            for (int32_t i = 0; i < per_lane; ++i) {
                const int32_t e = lane + kWarp * i;
                if (e >= a.E || ((taken >> i) & 1u) || !((kept >> (e / gsize)) & 1u))
                    continue;
                const float le = sl[e];
                if (le > v) { // e increases with i, so ties keep the smaller id
                    v = le;
                    id = e;
                }
            }
            warp_argmax(v, id);
            if (id != INT32_MAX && id % kWarp == lane)
                taken |= 1u << (id / kWarp);
            if (lane == j) {
                my_idx = id;
                my_logit = v;
            }
        }

        // weights
        float wj = 0.0f;
        if (a.score_fn == 0) {
            float m = __shfl_sync(kFullMask, my_logit, 0); // the best chosen logit
            float denom;
            if (a.renormalize) {
                wj = lane < a.k ? expf(my_logit - m) : 0.0f;
                denom = warp_sum(wj);
            } else {
                float mm = neg_inf;
                for (int32_t e = lane; e < a.E; e += kWarp)
                    mm = fmaxf(mm, sl[e]);
#pragma unroll
                for (int d = 16; d >= 1; d >>= 1)
                    mm = fmaxf(mm, __shfl_xor_sync(kFullMask, mm, d));
                m = mm;
                float part = 0.0f;
                for (int32_t e = lane; e < a.E; e += kWarp)
                    part += expf(sl[e] - m);
                denom = warp_sum(part);
                wj = lane < a.k ? expf(my_logit - m) : 0.0f;
            }
            wj = __fdiv_rn(wj, denom);
        } else {
            wj = lane < a.k ? __fdiv_rn(1.0f, 1.0f + expf(-my_logit)) : 0.0f;
            if (a.renormalize)
                wj = __fdiv_rn(wj, warp_sum(wj));
        }
        if (lane < a.k) {
            a.topk_idx[t * a.k + lane] = my_idx;
            a.topk_w[t * a.k + lane] = wj;
        }
        __syncwarp(); // the next token may overwrite the logits
    }
}

} // namespace moe
