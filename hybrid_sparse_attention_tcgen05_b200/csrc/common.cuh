// Shared device helpers for the hysparse kernels (not part of the C ABI).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "hysparse.h"

namespace hs {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// Workspace layout: [0, 256) status word and reserved, then per-call regions.
constexpr size_t kStatusBytes = 256;

__host__ __device__ inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Record a device-side error bit in the workspace status word.
__device__ inline void report(unsigned int *status, int code) {
    if (status) atomicOr(status, 1u << code);
}

template <typename T> struct Elem;
template <> struct Elem<float> {
    __device__ static inline float to_f(float x) { return x; }
    __device__ static inline float from_f(float x) { return x; }
};
template <> struct Elem<__nv_bfloat16> {
    __device__ static inline float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
    __device__ static inline __nv_bfloat16 from_f(float x) { return __float2bfloat16_rn(x); }
};

__device__ inline float warp_max(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
    return x;
}
__device__ inline float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// Load 8 consecutive elements (16 bytes for bf16, 32 for f32) as floats.
__device__ inline void load8(const __nv_bfloat16 *p, float *f) {
    uint4 u = *reinterpret_cast<const uint4 *>(p);
    const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
    for (int t = 0; t < 4; ++t) {
        float2 x = __bfloat1622float2(h[t]);
        f[2 * t] = x.x;
        f[2 * t + 1] = x.y;
    }
}
__device__ inline void load8(const float *p, float *f) {
    float4 a = *reinterpret_cast<const float4 *>(p);
    float4 b = *reinterpret_cast<const float4 *>(p + 4);
    f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
    f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}

}  // namespace hs
