// common.cuh -- shared device helpers of the Nystromformer attention library.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "nys_attn.h"

namespace nys {

constexpr int kTaps = NYS_CONV_TAPS;
constexpr int kHalfTaps = NYS_CONV_TAPS / 2;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// Device status word: bounded waits that run out record NYS_ERR_TIMEOUT here.
__device__ int g_status;

__device__ __forceinline__ void record_status(int code) { atomicCAS(&g_status, 0, code); }

// Element loads widened to float -------------------------------------------------

template <typename T> struct Elt;

template <> struct Elt<float> {
    static constexpr int kVec = 4;  // elements per 16-byte load
    __device__ __forceinline__ static void load16(const float* p, float* out) {
        float4 v = *reinterpret_cast<const float4*>(p);
        out[0] = v.x; out[1] = v.y; out[2] = v.z; out[3] = v.w;
    }
    __device__ __forceinline__ static float to_f(float x) { return x; }
    __device__ __forceinline__ static float from_f(float x) { return x; }
};

template <> struct Elt<__nv_bfloat16> {
    static constexpr int kVec = 8;
    __device__ __forceinline__ static void load16(const __nv_bfloat16* p, float* out) {
        uint4 raw = *reinterpret_cast<const uint4*>(p);
        const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float2 f = __bfloat1622float2(h[i]);
            out[2 * i] = f.x;
            out[2 * i + 1] = f.y;
        }
    }
    __device__ __forceinline__ static float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
    __device__ __forceinline__ static __nv_bfloat16 from_f(float x) { return __float2bfloat16_rn(x); }
};

__host__ __device__ __forceinline__ float split_scale(int d) {
    // d^-1/4: walkthrough 2.2 divides Q and K each by sqrt(sqrt(d)).
    return d == 64 ? 0.35355339059327373f : (d == 32 ? 0.42044820762685725f : 1.0f / sqrtf(sqrtf((float)d)));
}

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
    return x;
}
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

}  // namespace nys
