// probs.cuh -- the attention weights returned for output_attentions (walkthrough,
// blog.gitcode.com, 2.7): on the Nystrom path attention_probs = kernel_1 Z, an
// n x m matrix per (batch, head) (2.4: kernel_1 = softmax_row(Qs K_l^T), Z the
// iterative inverse of kernel_2); on the exact branch (2.1, path A) the full
// n x n softmax_row(Qs Ks^T + mask).
//
// These are optional outputs, float32, computed on CUDA cores from the layer's
// inputs and the float32 stages (K_l, Z) of the same call; they are written only
// when the caller passes a buffer and never feed the main output.
#pragma once

#include "common.cuh"

namespace nys {

// ------------------------------------------------------------------ Nystrom path: kernel_1 Z
// CTA (64 query rows, one (batch, head)), 256 threads: S = Qs K_l^T for all m landmarks in
// shared memory, exact row softmax, then probs = P Z in 64 x 64 output tiles (each thread
// a 4 x 4 block), Z staged 64 rows at a time.
template <int D>
struct ProbsSmem {
    static constexpr size_t bytes(int m) {
        return sizeof(float) * ((size_t)D * 68 * 2 + (size_t)64 * (m + 1) + (size_t)64 * 68);
    }
};

template <typename T, int D>
__global__ void __launch_bounds__(256)
nystrom_probs_kernel(const T* __restrict__ q, const float* __restrict__ kl, const float* __restrict__ z,
                     float* __restrict__ probs, int n, int m) {
    extern __shared__ float smem[];
    float (*sQ)[68] = reinterpret_cast<float (*)[68]>(smem);                    // [D][68]
    float (*sB)[68] = reinterpret_cast<float (*)[68]>(smem + D * 68);           // [D][68]
    float* sS = smem + 2 * D * 68;                                              // [64][m+1]
    float (*sZ)[68] = reinterpret_cast<float (*)[68]>(sS + 64 * (m + 1));       // [64][68]
    const int ldS = m + 1;
    const int bh = blockIdx.y, i0 = blockIdx.x * 64;
    const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4, lane = tid & 31, warp = tid >> 5;
    const float s = split_scale(D);
    const T* qb = q + (size_t)bh * n * D;
    for (int e = tid; e < 64 * D; e += 256) {
        const int r = e / D, c = e % D;
        sQ[c][r] = (i0 + r < n) ? s * Elt<T>::to_f(qb[(size_t)(i0 + r) * D + c]) : 0.f;
    }
    const float* klb = kl + (size_t)bh * m * D;
    for (int j0 = 0; j0 < m; j0 += 64) {
        __syncthreads();
        for (int e = tid; e < 64 * D; e += 256) {
            const int r = e / D, c = e % D;
            sB[c][r] = (j0 + r < m) ? klb[(size_t)(j0 + r) * D + c] : 0.f;
        }
        __syncthreads();
        float acc[4][4] = {};
        for (int e = 0; e < D; ++e) {
            const float4 av = *reinterpret_cast<const float4*>(&sQ[e][ty * 4]);
            const float4 bv = *reinterpret_cast<const float4*>(&sB[e][tx * 4]);
            const float a4[4] = {av.x, av.y, av.z, av.w}, b4[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a4[i], b4[j], acc[i][j]);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int c = j0 + tx * 4 + j;
                if (c < m) sS[(ty * 4 + i) * ldS + c] = acc[i][j];
            }
    }
    __syncthreads();
    for (int r = warp; r < 64; r += 8) {   // kernel_1: exact row softmax over the m landmarks
        float* row = sS + r * ldS;
        float mx = -INFINITY;
        for (int c = lane; c < m; c += 32) mx = fmaxf(mx, row[c]);
        mx = warp_max(mx);
        float sum = 0.f;
        for (int c = lane; c < m; c += 32) {
            const float e = __expf(row[c] - mx);
            row[c] = e;
            sum += e;
        }
        sum = warp_sum(sum);
        const float inv = 1.f / sum;
        for (int c = lane; c < m; c += 32) row[c] *= inv;
    }
    const float* zb = z + (size_t)bh * m * m;
    float* pb = probs + (size_t)bh * n * m;
    for (int c0 = 0; c0 < m; c0 += 64) {
        float acc[4][4] = {};
        for (int k0 = 0; k0 < m; k0 += 64) {
            __syncthreads();
            for (int e = tid; e < 64 * 64; e += 256) {
                const int r = e >> 6, c = e & 63;
                sZ[r][c] = (k0 + r < m && c0 + c < m) ? zb[(size_t)(k0 + r) * m + c0 + c] : 0.f;
            }
            __syncthreads();
            const int kn = min(64, m - k0);
            for (int kk = 0; kk < kn; ++kk) {
                float pv[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) pv[i] = sS[(ty * 4 + i) * ldS + k0 + kk];
                const float4 zv = *reinterpret_cast<const float4*>(&sZ[kk][tx * 4]);
                const float z4[4] = {zv.x, zv.y, zv.z, zv.w};
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(pv[i], z4[j], acc[i][j]);
            }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int r = i0 + ty * 4 + i;
            if (r >= n) continue;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int c = c0 + tx * 4 + j;
                if (c < m) pb[(size_t)r * m + c] = acc[i][j];
            }
        }
    }
}

// ------------------------------------------------------------------ exact branch: full softmax
// CTA (64 query rows, one (batch, head)), 256 threads, two passes over 64-key blocks:
// the first keeps each row's running max and sum (online softmax), the second recomputes
// the scores and writes exp(s - max) / sum (exactly 0 at padded keys).
template <typename T, int D>
__global__ void __launch_bounds__(256)
exact_probs_kernel(const T* __restrict__ q, const T* __restrict__ k, const uint8_t* __restrict__ mask,
                   float* __restrict__ probs, int H, int n) {
    __shared__ __align__(16) float sQ[D][68];
    __shared__ __align__(16) float sK[D][68];
    __shared__ float sM[64], sL[64];
    const int bh = blockIdx.y, i0 = blockIdx.x * 64, b = bh / H;
    const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
    const float s = split_scale(D);
    const T* qb = q + (size_t)bh * n * D;
    const T* kb = k + (size_t)bh * n * D;
    for (int e = tid; e < 64 * D; e += 256) {
        const int r = e / D, c = e % D;
        sQ[c][r] = (i0 + r < n) ? s * Elt<T>::to_f(qb[(size_t)(i0 + r) * D + c]) : 0.f;
    }
    float mrun[4], lrun[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) { mrun[i] = -INFINITY; lrun[i] = 0.f; }
    float* pb = probs + (size_t)bh * n * n;
    for (int pass = 0; pass < 2; ++pass) {
        for (int j0 = 0; j0 < n; j0 += 64) {
            __syncthreads();
            for (int e = tid; e < 64 * D; e += 256) {
                const int r = e / D, c = e % D;
                sK[c][r] = (j0 + r < n) ? s * Elt<T>::to_f(kb[(size_t)(j0 + r) * D + c]) : 0.f;
            }
            __syncthreads();
            float acc[4][4] = {};
            for (int e = 0; e < D; ++e) {
                const float4 av = *reinterpret_cast<const float4*>(&sQ[e][ty * 4]);
                const float4 bv = *reinterpret_cast<const float4*>(&sK[e][tx * 4]);
                const float a4[4] = {av.x, av.y, av.z, av.w}, b4[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a4[i], b4[j], acc[i][j]);
            }
            bool valid[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int key = j0 + tx * 4 + j;
                valid[j] = key < n && (mask == nullptr || mask[(size_t)b * n + key] != 0);
            }
            if (pass == 0) {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    float cm = -INFINITY;
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        if (valid[j]) cm = fmaxf(cm, acc[i][j]);
#pragma unroll
                    for (int off = 8; off > 0; off >>= 1) cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, off));
                    const float mnew = fmaxf(mrun[i], cm);
                    float rs = 0.f;
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        if (valid[j]) rs += __expf(acc[i][j] - mnew);
#pragma unroll
                    for (int off = 8; off > 0; off >>= 1) rs += __shfl_xor_sync(0xffffffffu, rs, off);
                    lrun[i] = (mrun[i] == -INFINITY ? 0.f : lrun[i] * __expf(mrun[i] - mnew)) + rs;
                    mrun[i] = mnew;
                }
            } else {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int r = i0 + ty * 4 + i;
                    if (r >= n) continue;
                    const float M = sM[ty * 4 + i], inv = 1.f / sL[ty * 4 + i];
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int key = j0 + tx * 4 + j;
                        if (key < n) pb[(size_t)r * n + key] = valid[j] ? __expf(acc[i][j] - M) * inv : 0.f;
                    }
                }
            }
        }
        if (pass == 0) {
            if (tx == 0) {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    sM[ty * 4 + i] = mrun[i];
                    sL[ty * 4 + i] = lrun[i];
                }
            }
        }
    }
}

}  // namespace nys
