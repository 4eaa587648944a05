// k_ycast.cuh -- bf16 copy of y for mpq_linear_typed(MPQ_Y_BF16): each fp32
// value of the finished product rounded to nearest-even bf16.
#pragma once
#include <cuda_bf16.h>

#include "common.cuh"

namespace mpq {

constexpr int YCAST_THREADS = 256;

__device__ __forceinline__ uint32_t bf16x2_bits(float lo, float hi) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&v);
}

__global__ void __launch_bounds__(YCAST_THREADS) k_y_to_bf16(const float* __restrict__ y32,
                                                            uint16_t* __restrict__ y16, size_t n) {
    pdl_launch_dependents();
    pdl_wait();   // y32 comes from the kernel before
    const size_t stride = (size_t)gridDim.x * YCAST_THREADS;
    const size_t i0 = (size_t)blockIdx.x * YCAST_THREADS + threadIdx.x;
    size_t done = 0;
    if ((((uintptr_t)y32) & 15) == 0 && (((uintptr_t)y16) & 7) == 0) {
        // four values per thread and step: one 16-byte load, one 8-byte store
        const size_t n4 = n / 4;
        for (size_t j = i0; j < n4; j += stride) {
            const float4 v = reinterpret_cast<const float4*>(y32)[j];
            reinterpret_cast<uint2*>(y16)[j] = make_uint2(bf16x2_bits(v.x, v.y), bf16x2_bits(v.z, v.w));
        }
        done = n4 * 4;
    }
    for (size_t j = done + i0; j < n; j += stride)
        y16[j] = __bfloat16_as_ushort(__float2bfloat16_rn(y32[j]));
}

}  // namespace mpq
