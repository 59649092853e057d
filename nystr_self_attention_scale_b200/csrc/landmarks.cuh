// landmarks.cuh -- fused d^-1/4 scale + segment means of Q and K.
//
// Walkthrough (blog.gitcode.com) 2.2 and 2.3: Q_l[j] = mean over the L = n/m
// consecutive rows j*L .. j*L+L-1 of d^-1/4 * Q; the same for K.
//
// One thread owns one 16-byte column slice (4 fp32 or 8 bf16 elements) of one
// landmark and walks the L rows of its segment; the d/kVec threads of a
// landmark read each row as one contiguous 64- or 128-byte run, so every load
// is a full 128-bit access and each warp touches whole 32-byte sectors only.
// The sum is accumulated in fp32 and multiplied once by fl(d^-1/4) / L.
#pragma once

#include "common.cuh"

namespace nys {

template <typename T>
__global__ void __launch_bounds__(256)
landmarks_kernel(const T* __restrict__ q, const T* __restrict__ k, float* __restrict__ ql,
                 float* __restrict__ kl, __nv_bfloat16* __restrict__ ql16,
                 __nv_bfloat16* __restrict__ kl16, int BH, int n, int d, int m) {
    constexpr int V = Elt<T>::kVec;
    const int slices = d / V;                                 // threads per landmark row
    const long long per_tensor = (long long)BH * m * slices;
    long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const int which = blockIdx.y;                             // 0: Q, 1: K
    if (gid >= per_tensor) return;
    const int slice = (int)(gid % slices);
    const long long lm = gid / slices;                        // (bh, j) flattened
    const int j = (int)(lm % m);
    const long long bh = lm / m;
    const int L = n / m;
    const T* src = (which == 0 ? q : k) + ((bh * n + (long long)j * L) * d) + slice * V;

    float acc[V];
#pragma unroll
    for (int e = 0; e < V; ++e) acc[e] = 0.f;
    int t = 0;
    for (; t + 8 <= L; t += 8) {   // eight independent 16-byte loads in flight per thread
        float x[8][V];
#pragma unroll
        for (int u = 0; u < 8; ++u) Elt<T>::load16(src + (long long)(t + u) * d, x[u]);
#pragma unroll
        for (int e = 0; e < V; ++e)
            acc[e] += ((x[0][e] + x[1][e]) + (x[2][e] + x[3][e])) + ((x[4][e] + x[5][e]) + (x[6][e] + x[7][e]));
    }
    for (; t + 4 <= L; t += 4) {
        float x0[V], x1[V], x2[V], x3[V];
        Elt<T>::load16(src + (long long)(t + 0) * d, x0);
        Elt<T>::load16(src + (long long)(t + 1) * d, x1);
        Elt<T>::load16(src + (long long)(t + 2) * d, x2);
        Elt<T>::load16(src + (long long)(t + 3) * d, x3);
#pragma unroll
        for (int e = 0; e < V; ++e) acc[e] += (x0[e] + x1[e]) + (x2[e] + x3[e]);
    }
    for (; t < L; ++t) {
        float x0[V];
        Elt<T>::load16(src + (long long)t * d, x0);
#pragma unroll
        for (int e = 0; e < V; ++e) acc[e] += x0[e];
    }
    const float scale = split_scale(d) / (float)L;
    float* dst = (which == 0 ? ql : kl) + lm * d + slice * V;
    __nv_bfloat16* dst16 = which == 0 ? ql16 : kl16;
#pragma unroll
    for (int e = 0; e < V; e += 4) {
        float4 o = make_float4(acc[e] * scale, acc[e + 1] * scale, acc[e + 2] * scale,
                               acc[e + 3] * scale);
        *reinterpret_cast<float4*>(dst + e) = o;
        if (dst16) {
            __nv_bfloat162 lo = __floats2bfloat162_rn(o.x, o.y);
            __nv_bfloat162 hi = __floats2bfloat162_rn(o.z, o.w);
            uint2 pk;
            pk.x = *reinterpret_cast<uint32_t*>(&lo);
            pk.y = *reinterpret_cast<uint32_t*>(&hi);
            *reinterpret_cast<uint2*>(dst16 + lm * d + slice * V + e) = pk;
        }
    }
}

// bf16, when one warp instruction covers whole rows (D = 64: 4 rows, D = 32: 8 rows) and
// L is a multiple of that: one warp per landmark (grid-stride over the 2 * BH * m landmarks
// of Q and K), reading the landmark's L contiguous rows as 512-byte warp instructions (lane l
// takes 16-byte slice l % (D / 8) of row l / (D / 8) of each instruction), eight loads in
// flight per lane (measured with L2 flushed by a read: 26.5 us at 8, 28.6 us at 16, and 28.7 us
// for a persistent CTA per SM streaming 16 KB bulk copies through an 8-stage ring); the lanes
// holding the same slice are summed with shuffles. Every warp
// reads contiguous 4 KB runs, and the landmarks are spread over all warps of all SMs.
template <int D>
__global__ void __launch_bounds__(256)
landmarks_warp_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                      float* __restrict__ ql, float* __restrict__ kl, __nv_bfloat16* __restrict__ ql16,
                      __nv_bfloat16* __restrict__ kl16, int BH, int n, int m) {
    constexpr int S = D / 8;        // 16-byte slices per row
    constexpr int R = 32 / S;       // rows per warp instruction
    constexpr int U = 8;            // loads in flight per lane
    const int lane = threadIdx.x & 31;
    const int slice = lane % S, rsub = lane / S;
    const long long per_tensor = (long long)BH * m;
    const long long units = 2 * per_tensor;
    const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
    const int L = n / m;
    const int instr = L / R;        // warp instructions per landmark
    const float scale = split_scale(D) / (float)L;
    for (long long u = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); u < units; u += warps) {
        const int which = u >= per_tensor;
        const long long lm = which ? u - per_tensor : u;   // (bh, j) flattened
        const __nv_bfloat16* src = (which ? k : q) + ((size_t)lm * L + rsub) * D + slice * 8;
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        for (int t = 0; t < instr; t += U) {
            // a batch of up to U loads, all issued before any is used (the last batch is predicated)
            uint4 raw[U];
#pragma unroll
            for (int e = 0; e < U; ++e)
                raw[e] = t + e < instr ? __ldg(reinterpret_cast<const uint4*>(src + (size_t)(t + e) * R * D))
                                       : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
            for (int e = 0; e < U; ++e) {
                const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw[e]);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float2 f = __bfloat1622float2(h2[i]);
                    acc[2 * i] += f.x;
                    acc[2 * i + 1] += f.y;
                }
            }
        }
#pragma unroll
        for (int off = S; off < 32; off <<= 1)
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], off);
        if (lane < S) {
            float* dst = (which ? kl : ql) + (size_t)lm * D + slice * 8;
            const float4 o0 = make_float4(acc[0] * scale, acc[1] * scale, acc[2] * scale, acc[3] * scale);
            const float4 o1 = make_float4(acc[4] * scale, acc[5] * scale, acc[6] * scale, acc[7] * scale);
            reinterpret_cast<float4*>(dst)[0] = o0;
            reinterpret_cast<float4*>(dst)[1] = o1;
            const __nv_bfloat162 b0 = __floats2bfloat162_rn(o0.x, o0.y), b1 = __floats2bfloat162_rn(o0.z, o0.w);
            const __nv_bfloat162 b2 = __floats2bfloat162_rn(o1.x, o1.y), b3 = __floats2bfloat162_rn(o1.z, o1.w);
            uint4 pk;
            pk.x = *reinterpret_cast<const uint32_t*>(&b0);
            pk.y = *reinterpret_cast<const uint32_t*>(&b1);
            pk.z = *reinterpret_cast<const uint32_t*>(&b2);
            pk.w = *reinterpret_cast<const uint32_t*>(&b3);
            *reinterpret_cast<uint4*>((which ? kl16 : ql16) + (size_t)lm * D + slice * 8) = pk;
        }
    }
}

}  // namespace nys
