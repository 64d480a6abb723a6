// Dispatch payload: copy (bf16) or block-quantise (fp8) each token's row into
// the receive rows of all its routing entries.
//
// "Enabling trillion-parameter models on AWS EFA", section "Despacho e
// Combinação": once the offsets are known, the tokens are packed into the
// contiguous per-peer buffers; section "Avaliação": the dispatch payload is
// block-scaled fp8.  "Lower latency and higher throughput with multi-node
// DeepSeek deployment", section "Quantização": activations get one scale per
// 128-element vector, computed on the fly.
//
// GPU design (register path).  A work unit is (token t, part p): part p covers
// kScatterThreads consecutive 16-byte vectors of x[t] (8 bf16 each), one per
// thread.  Each thread loads its vector once and stores it (or its 8 e4m3
// codes) to all k receive rows of the token, so x is read from HBM once and
// every store of a warp is a contiguous 512-byte (bf16) or 256-byte (fp8) run.
// For fp8 the 16 lanes holding one 128-column block reduce |x| with
// butterfly shuffles; the block's scale is amax/448 and each code is
// e4m3(x/scale), with IEEE round-to-nearest divisions and a saturating
// round-to-nearest-even conversion.
#pragma once

#include "common.cuh"

namespace moe {

constexpr int kScatterThreads = 128;

struct ScatterArgs {
    const uint16_t *x; // [T, H] bf16
    const int32_t *slot; // [T, k]
    int32_t T, H, k;
    int32_t parts; // per row: ceil((H/8) / kScatterThreads)
    void *recv_x; // [rows_cap, H] bf16 or e4m3
    float *recv_scale; // [rows_cap, H/128] (fp8)
};

// Quantises the 8 values of one vector; the 16 lanes of a 128-column block
// must all call this together (inactive lanes pass zeros).  Returns the codes
// packed little-endian (element 0 in the low byte) and the block scale.
__device__ __forceinline__ uint2 quantise_vec_e4m3(uint4 v, float &scale_out)
{
    float f[8] = {bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y),
                  bf16_lo(v.z), bf16_hi(v.z), bf16_lo(v.w), bf16_hi(v.w)};
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i)
        amax = fmaxf(amax, fabsf(f[i]));
#pragma unroll
    for (int d = 8; d >= 1; d >>= 1)
        amax = fmaxf(amax, __shfl_xor_sync(kFullMask, amax, d));
    uint2 codes = make_uint2(0u, 0u);
    float scale = 0.0f;
    if (amax > 0.0f) {
        scale = __fdiv_rn(amax, 448.0f);
        float q[8];
#pragma unroll
        for (int i = 0; i < 8; ++i)
            q[i] = __fdiv_rn(f[i], scale);
        codes.x = pack_e4m3x2(q[0], q[1]) | (pack_e4m3x2(q[2], q[3]) << 16);
        codes.y = pack_e4m3x2(q[4], q[5]) | (pack_e4m3x2(q[6], q[7]) << 16);
    }
    scale_out = scale;
    return codes;
}

template <bool kFp8>
__global__ void __launch_bounds__(kScatterThreads) scatter_rows(ScatterArgs a)
{
    const int32_t nvec = a.H / 8;
    const int64_t units = (int64_t)a.T * a.parts;
    for (int64_t u = blockIdx.x; u < units; u += gridDim.x) {
        const int32_t t = (int32_t)(u / a.parts);
        const int32_t v = (int32_t)(u % a.parts) * kScatterThreads + threadIdx.x;
        const bool active = v < nvec;
        uint4 val = make_uint4(0u, 0u, 0u, 0u);
        if (active)
            val = ld_stream_v4(a.x + (int64_t)t * a.H + (int64_t)v * 8);
        const int32_t *slots = a.slot + (int64_t)t * a.k;
        if constexpr (kFp8) {
            float scale;
            uint2 codes = quantise_vec_e4m3(val, scale);
            const int32_t nb = a.H / 128;
            uint8_t *rx = static_cast<uint8_t *>(a.recv_x);
            for (int32_t j = 0; j < a.k; ++j) {
                int32_t s = __ldg(slots + j);
                if (s < 0 || !active)
                    continue;
                st_v2(rx + (int64_t)s * a.H + (int64_t)v * 8, codes);
                if ((threadIdx.x & 15) == 0)
                    a.recv_scale[(int64_t)s * nb + v / 16] = scale;
            }
        } else {
            uint16_t *rx = static_cast<uint16_t *>(a.recv_x);
            for (int32_t j = 0; j < a.k; ++j) {
                int32_t s = __ldg(slots + j);
                if (s < 0 || !active)
                    continue;
                st_v4(rx + (int64_t)s * a.H + (int64_t)v * 8, val);
            }
        }
    }
}

} // namespace moe
