// exact.cuh -- epilogue of the exact branch (walkthrough, blog.gitcode.com, 2.1, path A).
//
// When the number of landmarks equals the segment length the layer computes full
// softmax attention instead of the approximation:
//   out = softmax_row(Qs Ks^T + mask) V + dwconv65(V)      (2.1, 2.2, 2.6)
// The attention term runs through the kernel_3 V machinery with the raw query rows
// (an online softmax over key splits that leaves unnormalised partials O, running
// max M and running sum l per row and split). This kernel merges the splits in a
// fixed order (log-sum-exp, as the kernel_3 V combine does), divides by the row sum,
// adds the 65-tap depthwise conv of V (zero padding 32, tap t multiplies
// V[i + t - 32]) and writes the output in the input's element type.
#pragma once

#include "common.cuh"

namespace nys {

// CTA (64 query rows, one (batch, head)), 256 threads. V rows i0 - 32 .. i0 + 95 are
// staged in shared memory as float (zero outside [0, n)); each thread owns (row, 4
// columns) items.
template <typename T, int D>
__global__ void __launch_bounds__(256)
exact_finish_kernel(const float* __restrict__ part_o, const float* __restrict__ part_m,
                    const float* __restrict__ part_l, const T* __restrict__ v,
                    const float* __restrict__ conv_w, T* __restrict__ out, int H, int n, int splits) {
    __shared__ __align__(16) float sV[128][D + 4];
    __shared__ float sw[kTaps];
    const int bh = blockIdx.y, i0 = blockIdx.x * 64, h = bh % H;
    const int tid = threadIdx.x;
    const bool conv = conv_w != nullptr;
    if (conv) {
        const T* vb = v + (size_t)bh * n * D;
        for (int e = tid; e < 128 * D; e += 256) {
            const int r = e / D, c = e % D;
            const int src = i0 - kHalfTaps + r;
            sV[r][c] = (src >= 0 && src < n) ? Elt<T>::to_f(vb[(size_t)src * D + c]) : 0.f;
        }
        if (tid < kTaps) sw[tid] = conv_w[(size_t)h * kTaps + tid];
    }
    __syncthreads();
    constexpr int Q4 = D / 4;
    for (int e = tid; e < 64 * Q4; e += 256) {
        const int r = e / Q4, c4 = e % Q4;
        const int i = i0 + r;
        if (i >= n) continue;
        const size_t row0 = (size_t)bh * splits * n + i;   // split s adds s * n
        float M = -INFINITY;
        for (int s = 0; s < splits; ++s) M = fmaxf(M, __ldg(part_m + row0 + (size_t)s * n));
        float4 num = make_float4(0.f, 0.f, 0.f, 0.f);
        float den = 0.f;
        for (int s = 0; s < splits; ++s) {
            const size_t row = row0 + (size_t)s * n;
            const float ms = __ldg(part_m + row);
            if (ms == -INFINITY) continue;   // a split whose keys are all padded
            const float f = __expf(ms - M);
            const float4 o = __ldg(reinterpret_cast<const float4*>(part_o + row * D) + c4);
            num.x = fmaf(f, o.x, num.x);
            num.y = fmaf(f, o.y, num.y);
            num.z = fmaf(f, o.z, num.z);
            num.w = fmaf(f, o.w, num.w);
            den = fmaf(f, __ldg(part_l + row), den);
        }
        const float inv = 1.f / den;
        float o[4] = {num.x * inv, num.y * inv, num.z * inv, num.w * inv};
        if (conv) {
            for (int t = 0; t < kTaps; ++t) {
                const float wt = sw[t];
                const float4 vv = *reinterpret_cast<const float4*>(&sV[r + t][4 * c4]);
                o[0] = fmaf(wt, vv.x, o[0]);
                o[1] = fmaf(wt, vv.y, o[1]);
                o[2] = fmaf(wt, vv.z, o[2]);
                o[3] = fmaf(wt, vv.w, o[3]);
            }
        }
        T* dst = out + ((size_t)bh * n + i) * D + 4 * c4;
#pragma unroll
        for (int j = 0; j < 4; ++j) dst[j] = Elt<T>::from_f(o[j]);
    }
}

}  // namespace nys
