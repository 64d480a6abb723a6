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
// GPU design (register path).  A work unit is (token t, chunk c): 512 columns
// of x[t], owned by one warp, so a unit moves 1 KB of bf16 in and k KB (bf16)
// or k/2 KB + k*16 B (fp8) out.  Warps walk the units grid-stride, so x is
// read from HBM once and every store instruction of a warp is one contiguous
// 512-byte run:
//  - bf16: lane l moves columns [8l, 8l+8) and [256+8l, 256+8l+8) of the chunk;
//  - fp8: lane l owns 16 consecutive columns, 8 lanes make one 128-column
//    block; the block's |x| maximum is reduced with butterfly shuffles inside
//    the 8 lanes, the scale is amax/448 and each code is e4m3(x/scale) (IEEE
//    round-to-nearest divisions, saturating round-to-nearest-even conversion).
//    A lane stores its 16 codes with one 16-byte store, and lane 0 stores the
//    warp's 4 block scales with one 16-byte store when the scale row allows.
// The token's k slots are read once per unit (lane j holds slot j) and
// broadcast with shuffles.
#pragma once

#include "common.cuh"

namespace moe {

constexpr int kScatterThreads = 256;
constexpr int kChunkCols = 512;

struct ScatterArgs {
    const uint16_t *x; // [T, H] bf16
    const int32_t *slot; // [T, k]
    int32_t T, H, k;
    void *recv_x; // [rows_cap, H] bf16 or e4m3
    float *recv_scale; // [rows_cap, H/128] (fp8)
};

// Quantises the 16 values of one lane (two 16-byte vectors of bf16); the 8 lanes
// of a 128-column block must call this together (inactive lanes pass zeros).
// Returns the 16 codes, element 0 in the low byte, and the block scale.
__device__ __forceinline__ uint4 quantise16_e4m3(uint4 a, uint4 b, float &scale_out)
{
    float f[16] = {bf16_lo(a.x), bf16_hi(a.x), bf16_lo(a.y), bf16_hi(a.y),
                   bf16_lo(a.z), bf16_hi(a.z), bf16_lo(a.w), bf16_hi(a.w),
                   bf16_lo(b.x), bf16_hi(b.x), bf16_lo(b.y), bf16_hi(b.y),
                   bf16_lo(b.z), bf16_hi(b.z), bf16_lo(b.w), bf16_hi(b.w)};
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i)
        amax = fmaxf(amax, fabsf(f[i]));
#pragma unroll
    for (int d = 4; d >= 1; d >>= 1)
        amax = fmaxf(amax, __shfl_xor_sync(kFullMask, amax, d));
    uint4 codes = make_uint4(0u, 0u, 0u, 0u);
    float scale = 0.0f;
    if (amax > 0.0f) {
        scale = __fdiv_rn(amax, 448.0f);
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float q0 = __fdiv_rn(f[4 * i + 0], scale), q1 = __fdiv_rn(f[4 * i + 1], scale);
            const float q2 = __fdiv_rn(f[4 * i + 2], scale), q3 = __fdiv_rn(f[4 * i + 3], scale);
            w[i] = pack_e4m3x2(q0, q1) | (pack_e4m3x2(q2, q3) << 16);
        }
        codes = make_uint4(w[0], w[1], w[2], w[3]);
    }
    scale_out = scale;
    return codes;
}

// Loads the lane's part of chunk c of row xr (see the layout above).
template <bool kFp8>
__device__ __forceinline__ void load_chunk(const uint16_t *xr, int32_t H, int32_t c, uint4 &v0,
                                           uint4 &v1)
{
    const unsigned lane = lane_id();
    v0 = make_uint4(0u, 0u, 0u, 0u);
    v1 = v0;
    if constexpr (kFp8) {
        const int32_t col = c * kChunkCols + (int32_t)lane * 16; // H % 128 == 0
        if (col < H) {
            v0 = ld_stream_v4(xr + col);
            v1 = ld_stream_v4(xr + col + 8);
        }
    } else {
        const int32_t col0 = c * kChunkCols + (int32_t)lane * 8; // H % 8 == 0
        if (col0 < H)
            v0 = ld_stream_v4(xr + col0);
        if (col0 + kChunkCols / 2 < H)
            v1 = ld_stream_v4(xr + col0 + kChunkCols / 2);
    }
}

// Stores chunk c (loaded by load_chunk) to the receive rows slots[0..k) of its
// token (-1 = no row); the whole warp calls this.  `slots` may point to global
// or shared memory.
template <bool kFp8>
__device__ __forceinline__ void store_chunk(void *recv_x, float *recv_scale, int32_t H, int32_t c,
                                            int32_t k, const int32_t *slots, uint4 v0, uint4 v1)
{
    const unsigned lane = lane_id();
    if constexpr (kFp8) {
        const int32_t nb = H / 128;
        const int32_t col = c * kChunkCols + (int32_t)lane * 16;
        const bool active = col < H;
        float scale;
        const uint4 codes = quantise16_e4m3(v0, v1, scale);
        const float s1 = __shfl_sync(kFullMask, scale, 8);
        const float s2 = __shfl_sync(kFullMask, scale, 16);
        const float s3 = __shfl_sync(kFullMask, scale, 24);
        const bool scale_vec = (nb % 4 == 0) && (c * 4 + 3 < nb);
        uint8_t *rx = static_cast<uint8_t *>(recv_x);
        for (int32_t j0 = 0; j0 < k; j0 += kWarp) {
            const int32_t my = j0 + (int32_t)lane < k ? slots[j0 + lane] : -1;
            const int32_t jn = k - j0 < kWarp ? k - j0 : kWarp;
            for (int32_t j = 0; j < jn; ++j) {
                const int32_t s = __shfl_sync(kFullMask, my, j);
                if (s < 0)
                    continue;
                if (active)
                    st_v4(rx + (int64_t)s * H + col, codes);
                float *sr = recv_scale + (int64_t)s * nb;
                if (scale_vec) {
                    if (lane == 0)
                        st_v4(sr + c * 4, make_uint4(__float_as_uint(scale), __float_as_uint(s1),
                                                     __float_as_uint(s2), __float_as_uint(s3)));
                } else if (active && (lane & 7) == 0) {
                    sr[col / 128] = scale;
                }
            }
        }
    } else {
        const int32_t col0 = c * kChunkCols + (int32_t)lane * 8;
        const int32_t col1 = col0 + kChunkCols / 2;
        const bool a0 = col0 < H, a1 = col1 < H;
        uint16_t *rx = static_cast<uint16_t *>(recv_x);
        for (int32_t j0 = 0; j0 < k; j0 += kWarp) {
            const int32_t my = j0 + (int32_t)lane < k ? slots[j0 + lane] : -1;
            const int32_t jn = k - j0 < kWarp ? k - j0 : kWarp;
            for (int32_t j = 0; j < jn; ++j) {
                const int32_t s = __shfl_sync(kFullMask, my, j);
                if (s < 0)
                    continue;
                uint16_t *row = rx + (int64_t)s * H;
                if (a0)
                    st_v4(row + col0, v0);
                if (a1)
                    st_v4(row + col1, v1);
            }
        }
    }
}

template <bool kFp8>
__global__ void __launch_bounds__(kScatterThreads) scatter_rows(ScatterArgs a)
{
    const int64_t nwarps = (int64_t)gridDim.x * (kScatterThreads / kWarp);
    const int32_t chunks = (a.H + kChunkCols - 1) / kChunkCols;
    const int64_t units = (int64_t)a.T * chunks;
    for (int64_t u = (int64_t)blockIdx.x * (kScatterThreads / kWarp) + threadIdx.x / kWarp;
         u < units; u += nwarps) {
        const int32_t t = (int32_t)(u / chunks);
        const int32_t c = (int32_t)(u % chunks);
        uint4 v0, v1;
        load_chunk<kFp8>(a.x + (int64_t)t * a.H, a.H, c, v0, v1);
        store_chunk<kFp8>(a.recv_x, a.recv_scale, a.H, c, a.k, a.slot + (int64_t)t * a.k, v0, v1);
    }
}

} // namespace moe
