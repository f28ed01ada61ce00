// common.cuh -- small device helpers shared by the GDN-2 kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace gdn2 {

// Bits of the device-side error word (read and cleared by gdn2_check_device_error).
enum : unsigned int {
    kErrTimeout = 1u,  // a bounded wait gave up
};

// The chunk kernels fold the decay into split factors e^{+x} and e^{-x},
// x = Gamma_t - Gamma_r, around a reference Gamma_r inside the chunk.  They
// use that fast form while every |x| of the chunk stays within this range, in
// which both factors are normal fp32 (and bf16) numbers with margin; a chunk
// whose decay is stronger takes a bounded form whose factors are all decays
// (<= 1).  The fp32 path uses a tighter range: the rounding of x (about
// |x| * 2^-24 per cumulated term) must stay far below its 1e-4 tolerance.
constexpr float kMidpointLogDecayRange = 80.0f;
constexpr float kMidpointLogDecayRangeF32 = 24.0f;

constexpr int kChunk = 64;  // tokens per chunk

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// Load 4 consecutive elements (16-byte aligned for float, 8-byte for bf16) as float4.
__device__ __forceinline__ float4 load4(const float *p) { return *reinterpret_cast<const float4 *>(p); }
__device__ __forceinline__ float4 load4(const __nv_bfloat16 *p) {
    const uint2 raw = *reinterpret_cast<const uint2 *>(p);
    const __nv_bfloat162 lo = *reinterpret_cast<const __nv_bfloat162 *>(&raw.x);
    const __nv_bfloat162 hi = *reinterpret_cast<const __nv_bfloat162 *>(&raw.y);
    const float2 a = __bfloat1622float2(lo), b = __bfloat1622float2(hi);
    return make_float4(a.x, a.y, b.x, b.y);
}

__device__ __forceinline__ void store4(float *p, float4 v) { *reinterpret_cast<float4 *>(p) = v; }
__device__ __forceinline__ void store4(__nv_bfloat16 *p, float4 v) {
    __nv_bfloat162 lo = __floats2bfloat162_rn(v.x, v.y);
    __nv_bfloat162 hi = __floats2bfloat162_rn(v.z, v.w);
    uint2 raw;
    raw.x = *reinterpret_cast<uint32_t *>(&lo);
    raw.y = *reinterpret_cast<uint32_t *>(&hi);
    *reinterpret_cast<uint2 *>(p) = raw;
}

}  // namespace gdn2
