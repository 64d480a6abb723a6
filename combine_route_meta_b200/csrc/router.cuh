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
// One warp per token.  Lane e % 32 keeps the logits of experts e = lane + 32 i
// in registers, as integers that order like the floats (finite or infinite
// logits), so every comparison is an integer one.  A pick is two warp
// reductions (redux.sync): the largest key among the lanes' best remaining
// candidates, then the smallest expert id holding that key.  Group maxima are
// folded with shared-memory atomics; the topk_group picks over them use the
// same two reductions.
#pragma once

#include "common.cuh"

namespace moe {

constexpr int kRouterMaxE = 1024;
constexpr int kRouterMaxK = 32;
constexpr int kRouterMaxGroups = 32;
constexpr int kRouterWarps = 8;
constexpr int32_t kNoKey = INT32_MIN; // below every logit's key

struct RouterArgs {
    const float *logits; // [T, E]
    int32_t T, E, k, score_fn, n_group, topk_group, renormalize;
    int32_t *topk_idx; // [T, k]
    float *topk_w;     // [T, k]
};

// A signed integer that orders like the float it comes from (not NaN).
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

// The warp's best (key, id): largest key, then smallest id.  Lanes without a
// candidate pass kNoKey.
__device__ __forceinline__ int32_t warp_pick(int32_t key, int32_t id, int32_t &best_key)
{
    best_key = __reduce_max_sync(kFullMask, key);
    return __reduce_min_sync(kFullMask, key == best_key ? id : INT32_MAX);
}

// The routing of token t by the calling warp (all 32 lanes): lane j < k ends
// holding the j-th pick in my_idx and its logit in my_logit.  lv keeps the
// token's logits (lane + 32 i) for the weights.  sg is the warp's scratch of
// kRouterMaxGroups int32 in shared memory.
template <int kPer>
__device__ __forceinline__ void route_pick(const RouterArgs &a, int64_t t, int32_t *sg, float (&lv)[kPer],
                                           int32_t &my_idx, float &my_logit)
{
    const int32_t lane = (int32_t)lane_id();
    const int32_t gsize = a.E / a.n_group;
    const float neg_inf = -__int_as_float(0x7f800000);
    const float *l = a.logits + t * a.E;
    int32_t key[kPer];
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
        const int32_t e = lane + kWarp * i;
        lv[i] = e < a.E ? __ldg(l + e) : neg_inf;
        key[i] = e < a.E ? ordered_key(lv[i]) : kNoKey;
    }

    // groups: drop the experts of the groups that are not kept
    if (a.n_group > 1) {
        if (lane < a.n_group)
            sg[lane] = kNoKey;
        __syncwarp();
#pragma unroll
        for (int i = 0; i < kPer; ++i) {
            const int32_t e = lane + kWarp * i;
            if (e < a.E)
                atomicMax(&sg[e / gsize], key[i]);
        }
        __syncwarp();
        const int32_t gkey = lane < a.n_group ? sg[lane] : kNoKey;
        uint32_t kept = 0;
        for (int32_t p = 0; p < a.topk_group; ++p) {
            int32_t best;
            const int32_t g = warp_pick((kept >> lane) & 1u ? kNoKey : gkey,
                                        lane < a.n_group ? lane : INT32_MAX, best);
            kept |= 1u << g;
        }
#pragma unroll
        for (int i = 0; i < kPer; ++i) {
            const int32_t e = lane + kWarp * i;
            if (e < a.E && !((kept >> (e / gsize)) & 1u))
                key[i] = kNoKey;
        }
        __syncwarp(); // sg is rewritten by the next token
    }

    // experts: each pick marks the chosen expert taken in its lane
    my_idx = -1;
    my_logit = 0.0f;
    uint32_t taken = 0; // bit i: expert lane + 32 i already chosen
    for (int32_t j = 0; j < a.k; ++j) {
        int32_t cand = kNoKey, ci = 0;
#pragma unroll
        for (int i = 0; i < kPer; ++i) {
            const int32_t ki = (taken >> i) & 1u ? kNoKey : key[i];
            if (ki > cand) { // i ascending: ties keep the smaller id
                cand = ki;
                ci = i;
            }
        }
        int32_t best;
        const int32_t id = warp_pick(cand, cand == kNoKey ? INT32_MAX : lane + kWarp * ci, best);
        if (id % kWarp == lane)
            taken |= 1u << (id / kWarp);
        if (lane == j) {
            my_idx = id;
            my_logit = key_value(best);
        }
    }
}

// The weights of token t's picks (route_pick's outputs), then topk_idx[t, :]
// and topk_w[t, :].
template <int kPer>
__device__ __forceinline__ void route_finish(const RouterArgs &a, int64_t t, const float (&lv)[kPer],
                                             int32_t my_idx, float my_logit)
{
    const int32_t lane = (int32_t)lane_id();
    float wj = 0.0f;
    if (a.score_fn == 0) {
        float m = __shfl_sync(kFullMask, my_logit, 0); // the best chosen logit
        float denom;
        if (a.renormalize) {
            wj = lane < a.k ? expf(my_logit - m) : 0.0f;
            denom = warp_sum(wj);
        } else {
            int32_t mk = kNoKey;
#pragma unroll
            for (int i = 0; i < kPer; ++i)
                if (lane + kWarp * i < a.E)
                    mk = max(mk, ordered_key(lv[i]));
            m = key_value(__reduce_max_sync(kFullMask, mk));
            float part = 0.0f;
#pragma unroll
            for (int i = 0; i < kPer; ++i)
                if (lane + kWarp * i < a.E)
                    part += expf(lv[i] - m);
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
}

// Routes token t with the calling warp: writes topk_idx[t, :] and topk_w[t, :].
template <int kPer>
__device__ __forceinline__ void route_token(const RouterArgs &a, int64_t t, int32_t *sg)
{
    float lv[kPer];
    int32_t my_idx;
    float my_logit;
    route_pick<kPer>(a, t, sg, lv, my_idx, my_logit);
    route_finish<kPer>(a, t, lv, my_idx, my_logit);
}

template <int kPer>
__global__ void __launch_bounds__(kRouterWarps * kWarp) router_topk(RouterArgs a)
{
    stream_order_begin();
    __shared__ int32_t s_g[kRouterWarps][kRouterMaxGroups];
    const int warp = threadIdx.x / kWarp;
    const int64_t nwarps = (int64_t)gridDim.x * kRouterWarps;
    for (int64_t t = (int64_t)blockIdx.x * kRouterWarps + warp; t < a.T; t += nwarps)
        route_token<kPer>(a, t, s_g[warp]);
}

} // namespace moe
