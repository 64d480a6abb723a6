// Combine: each token's routing-weighted sum of its experts' output rows.
//
// "Enabling trillion-parameter models on AWS EFA", section "Despacho e
// Combinação": before returning, the combine accumulates the tokens from the
// receive buffers into the output tensors; sections "Introdução" and "Buffers
// de Envio e Recebimento": the result is each token's weighted combination of
// its processed rows.  "Lower latency and higher throughput with multi-node
// DeepSeek deployment", section "Paralelismo de Especialistas": the 8 routed
// results of a token are summed with their weights.
//
// GPU design.  A work unit is (token t, part p), one 16-byte vector (8 bf16
// columns) per thread, as in the scatter.  A thread first issues the loads of
// its vector from up to 8 receive rows at once (8 independent 16-byte loads in
// flight), then folds them into 8 fp32 accumulators with one fused
// multiply-add per row in ascending j, and finally stores 8 bf16 values
// rounded to nearest-even.  For k > 8 the rows are taken 8 at a time, still in
// ascending j, so the result does not depend on the launch shape.
#pragma once

#include "common.cuh"

namespace moe {

constexpr int kCombineThreads = 128;
constexpr int kCombineBatch = 8; // receive rows whose loads are in flight together

struct CombineArgs {
    const uint16_t *expert_out; // [rows_cap, H] bf16
    const int32_t *slot;        // [T, k]
    const float *w;             // [T, k]
    int32_t T, H, k;
    int32_t parts;
    int64_t rows_cap;
    uint16_t *y; // [T, H] bf16
    int32_t *err;
};

__global__ void __launch_bounds__(kCombineThreads) combine_rows(CombineArgs a)
{
    stream_order_begin();
    const int32_t nvec = a.H / 8;
    const int64_t units = (int64_t)a.T * a.parts;
    for (int64_t u = blockIdx.x; u < units; u += gridDim.x) {
        const int32_t t = (int32_t)(u / a.parts);
        const int32_t v = (int32_t)(u % a.parts) * kCombineThreads + threadIdx.x;
        if (v >= nvec)
            continue;
        const int32_t *slots = a.slot + (int64_t)t * a.k;
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
                    int32_t s = __ldg(slots + j0 + jj);
                    if (s >= 0 && s < a.rows_cap) {
                        use[jj] = true;
                        r[jj] = ld_stream_v4(a.expert_out + (int64_t)s * a.H + (int64_t)v * 8);
                    } else if (s != -1) {
                        raise_error(a.err, MOE_DEV_BAD_SLOT);
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
