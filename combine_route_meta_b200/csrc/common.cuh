// Device helpers shared by the dispatch / combine kernels (sm_100a).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "moe_dispatch_combine.h"

namespace moe {

constexpr int kWarp = 32;
constexpr unsigned kFullMask = 0xffffffffu;

__device__ __forceinline__ void raise_error(int32_t *err, int32_t bit)
{
    if (err != nullptr)
        atomicOr(err, bit);
}

__device__ __forceinline__ unsigned lane_id() { return threadIdx.x & (kWarp - 1); }

// Programmatic dependent launch.  Every kernel here is launched so that it may
// start while the previous kernel in the stream is still finishing.  Before its
// first global-memory access it waits for that kernel to complete and its
// writes to be visible (so stream order still holds for every buffer), then
// lets the next kernel start launching.  The next kernel's launch therefore
// overlaps this one's tail; the wait itself is done by the hardware.
__device__ __forceinline__ void stream_order_begin()
{
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ unsigned lanemask_lt()
{
    unsigned m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

// 16-byte global load through the read-only path, not kept in L1: every byte
// of the payloads is read once.
__device__ __forceinline__ uint4 ld_stream_v4(const void *p)
{
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ void st_v4(void *p, uint4 v)
{
    asm volatile("st.global.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
                 "r"(v.w)
                 : "memory");
}

__device__ __forceinline__ void st_v2(void *p, uint2 v)
{
    asm volatile("st.global.v2.u32 [%0], {%1,%2};" ::"l"(p), "r"(v.x), "r"(v.y) : "memory");
}

// bf16 bits -> float: the bits are the top half of a binary32.
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Two floats -> packed bf16x2 (round to nearest even); `lo` lands in the low half.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// Two floats -> packed e4m3x2, round to nearest even, saturating to +-448.
// `lo` lands in the low byte.
__device__ __forceinline__ uint32_t pack_e4m3x2(float lo, float hi)
{
    unsigned short r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

} // namespace moe
