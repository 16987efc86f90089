// common.cuh -- small device helpers shared by the library's kernels.
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

namespace sqz {

constexpr int kWarp = 32;

__device__ __forceinline__ float h2f(uint16_t h) { return __half2float(__ushort_as_half(h)); }

__device__ __forceinline__ uint16_t f2h_rn(float f) { return __half_as_ushort(__float2half_rn(f)); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    return v;
}

// Read-only, non-coherent global loads (the weights never change during a call).
__device__ __forceinline__ uint32_t ldg_u32(const uint32_t* p) { return __ldg(p); }

__device__ __forceinline__ uint4 ldg_u128(const void* p) { return __ldg(reinterpret_cast<const uint4*>(p)); }

// Streaming 128-bit load: data read exactly once, keep it out of L1.
__device__ __forceinline__ uint4 ldg_stream_u128(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

}  // namespace sqz
