// Device helpers shared by the block-diffusion attention kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace bd {

// Device status word (one per device, in this library's module).  Kernels OR
// a code into it when a bounded wait runs out or a device-resident size is
// out of range; bd_attn_get_device_status reads and clears it.
__device__ unsigned int g_status_word;

enum DeviceCode : unsigned int {
    DEV_BAD_CACHE_LEN = 1u,
    DEV_WAIT_TIMEOUT = 2u,
    DEV_SCHED_OVERLAP = 4u, // two launches shared a work counter pair
};

__device__ __forceinline__ void raise_device_code(unsigned int code)
{
    atomicOr(&g_status_word, code);
}

__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
}

// 2^x on the special-function unit.
__device__ __forceinline__ float ex2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
    return y;
}

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

} // namespace bd
