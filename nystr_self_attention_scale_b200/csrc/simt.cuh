// simt.cuh -- float32 CUDA-core kernels of the Nystromformer attention forward.
//
// These carry the float32 path (fp32 in, fp32 out, FFMA arithmetic), where
// tensor-core precision (bf16 / tf32 operands) would not meet a 1e-4 relative
// error budget, and the m x m stages that are small for every shape.
// Walkthrough (blog.gitcode.com) section references are given per kernel.
#pragma once

#include "common.cuh"

namespace nys {

// ------------------------------------------------------------------ block GEMM
// C = alpha * (A . op(B)) + diag * I over a rows x cols output, by one CTA of
// 256 threads. A is rows x inner row-major (lda); B is inner x cols row-major
// (ldb) or, with TRANS_B, cols x inner row-major. 64 x 64 output tiles, each
// thread owns a 4 x 4 sub-block; the inner dimension is staged 16 at a time
// through shared memory. Callers synchronise the block around it.
struct GemmSmem {
    float a[16][64 + 4];
    float b[16][64 + 4];
};

template <bool TRANS_B>
__device__ void block_gemm(float* __restrict__ C, int ldc, const float* __restrict__ A, int lda,
                           const float* __restrict__ B, int ldb, int rows, int inner, int cols,
                           float alpha, float diag, GemmSmem& sm) {
    const int tid = threadIdx.x;
    const int tx = tid & 15, ty = tid >> 4;
    for (int r0 = 0; r0 < rows; r0 += 64) {
        for (int c0 = 0; c0 < cols; c0 += 64) {
            float acc[4][4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
            for (int k0 = 0; k0 < inner; k0 += 16) {
                // A tile: 64 rows x 16 k, stored k-major
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    int idx = tid + e * 256;
                    int r = idx >> 4, kk = idx & 15;
                    int gr = r0 + r, gk = k0 + kk;
                    sm.a[kk][r] = (gr < rows && gk < inner) ? A[(size_t)gr * lda + gk] : 0.f;
                }
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    int idx = tid + e * 256;
                    if (TRANS_B) {
                        int c = idx >> 4, kk = idx & 15;
                        int gc = c0 + c, gk = k0 + kk;
                        sm.b[kk][c] = (gc < cols && gk < inner) ? B[(size_t)gc * ldb + gk] : 0.f;
                    } else {
                        int kk = idx >> 6, c = idx & 63;
                        int gc = c0 + c, gk = k0 + kk;
                        sm.b[kk][c] = (gc < cols && gk < inner) ? B[(size_t)gk * ldb + gc] : 0.f;
                    }
                }
                __syncthreads();
#pragma unroll
                for (int kk = 0; kk < 16; ++kk) {
                    float4 av = *reinterpret_cast<const float4*>(&sm.a[kk][ty * 4]);
                    float4 bv = *reinterpret_cast<const float4*>(&sm.b[kk][tx * 4]);
                    float a4[4] = {av.x, av.y, av.z, av.w};
                    float b4[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
                    for (int i = 0; i < 4; ++i)
#pragma unroll
                        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a4[i], b4[j], acc[i][j]);
                }
                __syncthreads();
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                int gr = r0 + ty * 4 + i;
                if (gr >= rows) continue;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    int gc = c0 + tx * 4 + j;
                    if (gc >= cols) continue;
                    C[(size_t)gr * ldc + gc] = alpha * acc[i][j] + (gr == gc ? diag : 0.f);
                }
            }
        }
    }
}

// ------------------------------------------------------------------ kernel_2 + iterative inverse
// Walkthrough 2.4 (kernel_2 = softmax(Q_l K_l^T)) and 2.5 (iterative inverse):
//   Z_0 = c k2^T, c = 1 / (max column sum * max row sum) (or 1 / max column sum with
//   the exact-coefficient option, walkthrough 2.5 second bullet)
//   repeat: X = k2 Z; T = 7I - X; U = 15I - X T; T = 13I - X U; Z = Z T / 4
// One CTA per (batch, head); the m x m matrices live in global scratch
// (L2-resident), 5 per head: k2, X, T, U, and the second Z buffer.
__global__ void __launch_bounds__(256)
pinv_simt_kernel(const float* __restrict__ ql, const float* __restrict__ kl, float* __restrict__ z_out,
                 float* __restrict__ scratch, int m, int d, int n_iter, int inv_init) {
    __shared__ GemmSmem sm;
    __shared__ float red[2][8];
    const int bh = blockIdx.x;
    const size_t mm = (size_t)m * m;
    float* A = scratch + (size_t)bh * 5 * mm;
    float* X = A + mm;
    float* T = X + mm;
    float* U = T + mm;
    float* Zb = U + mm;
    float* Z = z_out + (size_t)bh * mm;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    block_gemm<true>(A, m, ql + (size_t)bh * m * d, d, kl + (size_t)bh * m * d, d, m, d, m, 1.f, 0.f, sm);
    __syncthreads();
    for (int r = warp; r < m; r += 8) {
        float* row = A + (size_t)r * m;
        float mx = -INFINITY;
        for (int c = lane; c < m; c += 32) mx = fmaxf(mx, row[c]);
        mx = warp_max(mx);
        float s = 0.f;
        for (int c = lane; c < m; c += 32) {
            float e = __expf(row[c] - mx);
            row[c] = e;
            s += e;
        }
        s = warp_sum(s);
        const float inv = 1.f / s;
        for (int c = lane; c < m; c += 32) row[c] *= inv;
    }
    __syncthreads();
    float mcol = -INFINITY, mrow = -INFINITY;
    for (int i = tid; i < m; i += 256) {
        float cs = 0.f, rs = 0.f;
        for (int j = 0; j < m; ++j) {
            cs += A[(size_t)j * m + i];
            rs += A[(size_t)i * m + j];
        }
        mcol = fmaxf(mcol, cs);
        mrow = fmaxf(mrow, rs);
    }
    mcol = warp_max(mcol);
    mrow = warp_max(mrow);
    if (lane == 0) { red[0][warp] = mcol; red[1][warp] = mrow; }
    __syncthreads();
    float c_mc = red[0][0], c_mr = red[1][0];
    for (int w = 1; w < 8; ++w) { c_mc = fmaxf(c_mc, red[0][w]); c_mr = fmaxf(c_mr, red[1][w]); }
    // default: 1 / (max column sum * max row sum); exact-coefficient option: 1 / max column sum
    const float coeff = inv_init == NYS_INV_INIT_EXACT ? 1.f / c_mc : 1.f / (c_mc * c_mr);
    for (size_t e = tid; e < mm; e += 256) {
        size_t r = e / m, c = e % m;
        Z[e] = coeff * A[c * m + r];
    }
    __syncthreads();
    float* zc = Z;
    float* zn = Zb;
    for (int it = 0; it < n_iter; ++it) {
        block_gemm<false>(X, m, A, m, zc, m, m, m, m, 1.f, 0.f, sm);       // X = A Z
        __syncthreads();
        for (size_t e = tid; e < mm; e += 256) {
            size_t r = e / m, c = e % m;
            T[e] = (r == c ? 7.f : 0.f) - X[e];                             // T = 7I - X
        }
        __syncthreads();
        block_gemm<false>(U, m, X, m, T, m, m, m, m, -1.f, 15.f, sm);      // U = 15I - X T
        __syncthreads();
        block_gemm<false>(T, m, X, m, U, m, m, m, m, -1.f, 13.f, sm);      // T = 13I - X U
        __syncthreads();
        block_gemm<false>(zn, m, zc, m, T, m, m, m, m, 0.25f, 0.f, sm);    // Z = Z T / 4
        __syncthreads();
        float* t = zc; zc = zn; zn = t;
    }
    if (zc != Z) {
        for (size_t e = tid; e < mm; e += 256) Z[e] = zc[e];
    }
}

// ------------------------------------------------------------------ kernel_2 + inverse, m <= 64
// The same computation as pinv_simt_kernel with every m x m matrix in shared memory (six
// 64 x 68 float buffers, 104 KB), for m <= 64: no operand goes through L2 between products.
// Each product C = alpha (L R) + diag I is computed by the 256 threads in 4 x 4 blocks
// (rows 4 ty .., columns 4 tx ..), the left factor read as scalars (the two row groups of a
// warp fall in different banks), the right factor as 16-byte rows; entries outside m x m stay
// zero, so the padding never contributes.
constexpr int kPinvSmemLd = 68;
constexpr size_t kPinvSmemBytes = sizeof(float) * 6 * 64 * kPinvSmemLd;

__device__ __forceinline__ void smem_gemm64(float* __restrict__ C, const float* __restrict__ Lm,
                                            const float* __restrict__ Rm, int inner, int m, float alpha,
                                            float diag) {
    constexpr int LD = kPinvSmemLd;
    const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
    float acc[4][4] = {};
#pragma unroll 4
    for (int k = 0; k < inner; ++k) {
        const float4 b = *reinterpret_cast<const float4*>(Rm + k * LD + 4 * tx);
        const float bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float a = Lm[(4 * ty + i) * LD + k];
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a, bv[j], acc[i][j]);
        }
    }
    __syncthreads();   // every thread has read its operands before any result is stored
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int r = 4 * ty + i;
        float4 o;
        float* ov = reinterpret_cast<float*>(&o);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int c = 4 * tx + j;
            ov[j] = (r < m && c < m) ? alpha * acc[i][j] + (r == c ? diag : 0.f) : 0.f;
        }
        *reinterpret_cast<float4*>(C + r * LD + 4 * tx) = o;
    }
    __syncthreads();
}

__global__ void __launch_bounds__(256)
pinv_simt_smem_kernel(const float* __restrict__ ql, const float* __restrict__ kl, float* __restrict__ z_out,
                      int m, int d, int n_iter, int inv_init) {
    constexpr int LD = kPinvSmemLd;
    extern __shared__ __align__(16) float psm[];
    float* A = psm;                 // k2
    float* Zc = A + 64 * LD;        // Z (current)
    float* Zn = Zc + 64 * LD;       // Z (next)
    float* X = Zn + 64 * LD;
    float* T = X + 64 * LD;
    float* U = T + 64 * LD;
    __shared__ float red[2][8];
    const int bh = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // landmarks: Q_l rows into X ([r][k]), K_l transposed into T ([k][c]), zero-padded to 64 x 64
    for (int e = tid; e < 64 * 64; e += 256) {
        const int r = e >> 6, c = e & 63;
        X[r * LD + c] = (r < m && c < d) ? ql[((size_t)bh * m + r) * d + c] : 0.f;
        T[c * LD + r] = (r < m && c < d) ? kl[((size_t)bh * m + r) * d + c] : 0.f;
    }
    __syncthreads();
    smem_gemm64(A, X, T, d, m, 1.f, 0.f);    // S2 = Q_l K_l^T (sum over the d columns)
    // walkthrough 2.4: k2 = softmax_row(S2), one warp per row
    for (int r = warp; r < m; r += 8) {
        float* row = A + r * LD;
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
    __syncthreads();
    // walkthrough 2.5: c = 1 / (max column sum * max row sum), or 1 / max column sum (exact option)
    float mcol = -INFINITY, mrow = -INFINITY;
    if (tid < m) {
        float cs = 0.f, rs = 0.f;
        for (int j = 0; j < m; ++j) {
            cs += A[j * LD + tid];
            rs += A[tid * LD + j];
        }
        mcol = cs;
        mrow = rs;
    }
    mcol = warp_max(mcol);
    mrow = warp_max(mrow);
    if (lane == 0) { red[0][warp] = mcol; red[1][warp] = mrow; }
    __syncthreads();
    float c_mc = red[0][0], c_mr = red[1][0];
    for (int w = 1; w < 8; ++w) { c_mc = fmaxf(c_mc, red[0][w]); c_mr = fmaxf(c_mr, red[1][w]); }
    const float coeff = inv_init == NYS_INV_INIT_EXACT ? 1.f / c_mc : 1.f / (c_mc * c_mr);
    for (int e = tid; e < 64 * 64; e += 256) {
        const int r = e >> 6, c = e & 63;
        Zc[r * LD + c] = (r < m && c < m) ? coeff * A[c * LD + r] : 0.f;   // Z_0 = c k2^T
    }
    __syncthreads();
    for (int it = 0; it < n_iter; ++it) {
        smem_gemm64(X, A, Zc, m, m, 1.f, 0.f);     // X = A Z
        for (int e = tid; e < 64 * 64; e += 256) {
            const int r = e >> 6, c = e & 63;
            T[r * LD + c] = (r < m && c < m) ? (r == c ? 7.f : 0.f) - X[r * LD + c] : 0.f;   // T = 7I - X
        }
        __syncthreads();
        smem_gemm64(U, X, T, m, m, -1.f, 15.f);    // U = 15I - X T
        smem_gemm64(T, X, U, m, m, -1.f, 13.f);    // T = 13I - X U
        smem_gemm64(Zn, Zc, T, m, m, 0.25f, 0.f);  // Z = Z T / 4
        float* t = Zc; Zc = Zn; Zn = t;
    }
    float* Z = z_out + (size_t)bh * m * m;
    for (int e = tid; e < m * m; e += 256) Z[e] = Zc[(e / m) * LD + (e % m)];
}

// ------------------------------------------------------------------ kernel_3 V, split over keys
// Walkthrough 2.4: k3 = softmax_row(Q_l Ks^T + mask), new_value = k3 V.
// CTA (bh, 64-landmark block, key split) runs an online softmax over its key
// range in 64-key chunks and writes unnormalised partials: O (64 x D), the
// running max M and the running sum l per landmark row. The rows are scaled by
// q_scale on load: 1 for the landmarks (already scaled by d^-1/4), d^-1/4 when
// the rows are the raw queries of the exact branch (walkthrough 2.1, path A),
// which runs the same online softmax over all n query rows.
template <int D>
constexpr size_t k3v_simt_smem_bytes() { return sizeof(float) * (2 * D * 68 + 64 * (D + 4) + 64 * 68); }

template <typename T, int D>
__global__ void __launch_bounds__(256)
k3v_partial_simt_kernel(const float* __restrict__ ql, const T* __restrict__ k, const T* __restrict__ v,
                        const uint8_t* __restrict__ mask, float* __restrict__ part_o,
                        float* __restrict__ part_m, float* __restrict__ part_l, int H, int n, int m,
                        int splits, int keys_per_split, float q_scale) {
    constexpr int CW = D / 16;  // output columns per thread
    extern __shared__ float smem[];
    float (*sQ)[68] = reinterpret_cast<float (*)[68]>(smem);                  // [D][68]
    float (*sK)[68] = reinterpret_cast<float (*)[68]>(smem + D * 68);         // [D][68]
    float (*sV)[D + 4] = reinterpret_cast<float (*)[D + 4]>(smem + 2 * D * 68);  // [64][D+4]
    float (*sP)[68] = reinterpret_cast<float (*)[68]>(smem + 2 * D * 68 + 64 * (D + 4));  // [64][68]
    const int bh = blockIdx.x, lb = blockIdx.y, sp = blockIdx.z;
    const int b = bh / H;
    const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
    const int j0 = lb * 64;
    const float s = split_scale(D);
    for (int e = tid; e < 64 * D; e += 256) {
        int r = e / D, c = e % D;
        sQ[c][r] = (j0 + r < m) ? q_scale * ql[((size_t)bh * m + j0 + r) * D + c] : 0.f;
    }
    float o[4][CW], mrun[4], lrun[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        mrun[i] = -INFINITY;
        lrun[i] = 0.f;
#pragma unroll
        for (int j = 0; j < CW; ++j) o[i][j] = 0.f;
    }
    const int kbeg = sp * keys_per_split;
    const int kend = min(n, kbeg + keys_per_split);
    const T* kb = k + (size_t)bh * n * D;
    const T* vb = v + (size_t)bh * n * D;
    for (int c0 = kbeg; c0 < kend; c0 += 64) {
        __syncthreads();
        for (int e = tid; e < 64 * D; e += 256) {
            int r = e / D, c = e % D;
            int key = c0 + r;
            bool ok = key < kend;
            sK[c][r] = ok ? s * Elt<T>::to_f(kb[(size_t)key * D + c]) : 0.f;
            sV[r][c] = ok ? Elt<T>::to_f(vb[(size_t)key * D + c]) : 0.f;
        }
        __syncthreads();
        float acc[4][4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
#pragma unroll 8
        for (int e = 0; e < D; ++e) {
            float4 av = *reinterpret_cast<const float4*>(&sQ[e][ty * 4]);
            float4 bv = *reinterpret_cast<const float4*>(&sK[e][tx * 4]);
            float a4[4] = {av.x, av.y, av.z, av.w};
            float b4[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a4[i], b4[j], acc[i][j]);
        }
        bool valid[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            int key = c0 + tx * 4 + j;
            valid[j] = key < kend && (mask == nullptr || mask[(size_t)b * n + key] != 0);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float cm = -INFINITY;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                if (!valid[j]) acc[i][j] = -INFINITY;
                cm = fmaxf(cm, acc[i][j]);
            }
#pragma unroll
            for (int off = 8; off > 0; off >>= 1) cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, off));
            const float mnew = fmaxf(mrun[i], cm);
            const float alpha = (mnew == -INFINITY) ? 1.f : __expf(mrun[i] - mnew);
            float rs = 0.f;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                float p = (mnew == -INFINITY) ? 0.f : __expf(acc[i][j] - mnew);
                sP[ty * 4 + i][tx * 4 + j] = p;
                rs += p;
            }
#pragma unroll
            for (int off = 8; off > 0; off >>= 1) rs += __shfl_xor_sync(0xffffffffu, rs, off);
            lrun[i] = lrun[i] * alpha + rs;
            mrun[i] = mnew;
#pragma unroll
            for (int j = 0; j < CW; ++j) o[i][j] *= alpha;
        }
        __syncthreads();
#pragma unroll 4
        for (int kk = 0; kk < 64; ++kk) {
            float pv[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) pv[i] = sP[ty * 4 + i][kk];
#pragma unroll
            for (int j = 0; j < CW; ++j) {
                float vv = sV[kk][tx * CW + j];
#pragma unroll
                for (int i = 0; i < 4; ++i) o[i][j] = fmaf(pv[i], vv, o[i][j]);
            }
        }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        int j = j0 + ty * 4 + i;
        if (j >= m) continue;
        size_t row = ((size_t)bh * splits + sp) * m + j;
#pragma unroll
        for (int c = 0; c < CW; ++c) part_o[row * D + tx * CW + c] = o[i][c];
        if (tx == 0) {
            part_m[row] = mrun[i];
            part_l[row] = lrun[i];
        }
    }
}

// Merge the key-split partials: k3v[j] = sum_s e^{M_s - M} O_s / sum_s e^{M_s - M} l_s.
// One thread per (head, landmark row, 4 columns), one pass: the splits are taken
// four at a time with all their loads in flight together, and the running sums
// are rescaled when a later group raises the maximum. The split order is fixed,
// so the result is deterministic. Four CTAs fit per SM, so the grid of the
// supported sizes runs in one wave. May be launched as a programmatic dependent of
// the kernel that writes the partials: it waits for that grid before reading them.
__global__ void __launch_bounds__(256, 4)
k3v_combine_kernel(const float* __restrict__ part_o, const float* __restrict__ part_m,
                   const float* __restrict__ part_l, float* __restrict__ k3v, int BH, int m, int d, int splits) {
    constexpr int G = 4;
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int q = d / 4;
    const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (gid >= (long long)BH * m * q) return;
    const int c4 = (int)(gid % q);
    const long long bj = gid / q;           // bh * m + j
    const int j = (int)(bj % m);
    const long long bh = bj / m;
    const size_t row0 = (size_t)bh * splits * m + j;   // row of split 0; split s adds s * m
    float M = -INFINITY, den = 0.f;
    float4 num = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s0 = 0; s0 < splits; s0 += G) {
        float ms[G], ls[G];
        float4 os[G];
#pragma unroll
        for (int e = 0; e < G; ++e) {
            const size_t row = row0 + (size_t)(s0 + e) * m;
            const bool ok = s0 + e < splits;
            ms[e] = ok ? __ldg(part_m + row) : -INFINITY;
            ls[e] = ok ? __ldg(part_l + row) : 0.f;
            os[e] = ok ? __ldg(reinterpret_cast<const float4*>(part_o + row * d) + c4) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        float gm = M;
#pragma unroll
        for (int e = 0; e < G; ++e) gm = fmaxf(gm, ms[e]);
        if (gm != -INFINITY && gm != M) {
            const float sc = M == -INFINITY ? 0.f : __expf(M - gm);
            num.x *= sc; num.y *= sc; num.z *= sc; num.w *= sc;
            den *= sc;
            M = gm;
        }
#pragma unroll
        for (int e = 0; e < G; ++e) {
            const float f = (ms[e] == -INFINITY) ? 0.f : __expf(ms[e] - M);
            num.x = fmaf(f, os[e].x, num.x);
            num.y = fmaf(f, os[e].y, num.y);
            num.z = fmaf(f, os[e].z, num.z);
            num.w = fmaf(f, os[e].w, num.w);
            den = fmaf(f, ls[e], den);
        }
    }
    const float inv = 1.f / den;
    reinterpret_cast<float4*>(k3v + (size_t)bj * d)[c4] =
        make_float4(num.x * inv, num.y * inv, num.z * inv, num.w * inv);
}

// W = Z (k3 V) (walkthrough 2.4, reassociated as k1 (Z (k3 V))): one CTA per
// 64-row tile of one head; the inner dimension is staged 64 at a time through
// shared memory with all of a thread's loads issued before its stores. The Z
// slice is stored transposed, so that a thread's four rows at one k are one
// 16-byte shared load, as are its columns of k3V: two loads per 4 x CW block of
// FMAs. Also writes W^T in bf16 ([d, m] per head) when wt16 is given.
template <int D>
__global__ void __launch_bounds__(256)
w_kernel(const float* __restrict__ z, const float* __restrict__ k3v, float* __restrict__ w,
         __nv_bfloat16* __restrict__ wt16, int m) {
    constexpr int CW = D / 16;                       // columns per thread
    __shared__ __align__(16) float sZ[64][64 + 4];   // [k][row]
    __shared__ __align__(16) float sK[64][D + 4];    // [k][col]
    const int bh = blockIdx.x, r0 = blockIdx.y * 64;
    const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
    const float* zb = z + (size_t)bh * m * m;
    const float* kb = k3v + (size_t)bh * m * D;
    float acc[4][CW];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < CW; ++j) acc[i][j] = 0.f;
    // the next 64-wide slice of Z and k3V is loaded into registers while the current one is used
    float za[16];   // scalar loads: m need not be a multiple of 4 on the float32 path
    float4 ka[D / 16];
    auto load_slice = [&](int k0) {
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            const int idx = tid + e * 256, r = idx >> 6, c = idx & 63;
            za[e] = (r0 + r < m && k0 + c < m) ? __ldg(zb + (size_t)(r0 + r) * m + k0 + c) : 0.f;
        }
#pragma unroll
        for (int e = 0; e < D / 16; ++e) {
            const int idx = tid + e * 256, r = idx / (D / 4), c4 = idx % (D / 4);
            ka[e] = (k0 + r < m) ? __ldg(reinterpret_cast<const float4*>(kb + (size_t)(k0 + r) * D) + c4)
                                 : make_float4(0.f, 0.f, 0.f, 0.f);
        }
    };
    load_slice(0);
    for (int k0 = 0; k0 < m; k0 += 64) {
        __syncthreads();   // the previous slice has been read from shared memory
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            const int idx = tid + e * 256, r = idx >> 6, c = idx & 63;
            sZ[c][r] = za[e];
        }
#pragma unroll
        for (int e = 0; e < D / 16; ++e) {
            const int idx = tid + e * 256, r = idx / (D / 4), c4 = idx % (D / 4);
            *reinterpret_cast<float4*>(&sK[r][4 * c4]) = ka[e];
        }
        __syncthreads();
        if (k0 + 64 < m) load_slice(k0 + 64);
#pragma unroll 8
        for (int kk = 0; kk < 64; ++kk) {
            const float4 a4 = *reinterpret_cast<const float4*>(&sZ[kk][ty * 4]);
            const float a[4] = {a4.x, a4.y, a4.z, a4.w};
            float bv[CW];
            if constexpr (CW == 4) {
                const float4 b4 = *reinterpret_cast<const float4*>(&sK[kk][4 * tx]);
                bv[0] = b4.x; bv[1] = b4.y; bv[2] = b4.z; bv[3] = b4.w;
            } else {
#pragma unroll
                for (int j = 0; j < CW; ++j) bv[j] = sK[kk][tx * CW + j];
            }
#pragma unroll
            for (int j = 0; j < CW; ++j)
#pragma unroll
                for (int i = 0; i < 4; ++i) acc[i][j] = fmaf(a[i], bv[j], acc[i][j]);
        }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int r = r0 + ty * 4 + i;
        if (r >= m) continue;
#pragma unroll
        for (int j = 0; j < CW; ++j) w[((size_t)bh * m + r) * D + tx * CW + j] = acc[i][j];
    }
    if (wt16 != nullptr && r0 + ty * 4 + 3 < m) {
#pragma unroll
        for (int j = 0; j < CW; ++j) {
            const int c = tx * CW + j;
            __nv_bfloat162 lo = __floats2bfloat162_rn(acc[0][j], acc[1][j]);
            __nv_bfloat162 hi = __floats2bfloat162_rn(acc[2][j], acc[3][j]);
            uint2 pk;
            pk.x = *reinterpret_cast<uint32_t*>(&lo);
            pk.y = *reinterpret_cast<uint32_t*>(&hi);
            *reinterpret_cast<uint2*>(wt16 + ((size_t)bh * D + c) * m + r0 + ty * 4) = pk;
        }
    }
}

// W = Z (k3 V) for the bf16 path (m a multiple of 32): one CTA of 128 threads per 32-row
// tile of one head, so that the 256 tiles of the headline shape spread over every SM. The
// tile's 32 Z rows (contiguous in memory) and the head's whole k3 V are staged in shared
// memory with 16-byte asynchronous copies, all in flight at once; then each thread
// accumulates a 4 x 4 block over all m in float32, reading four Z values of one row and four
// k3 V values of one k as 16-byte shared loads. Writes W (float32) and W^T (bf16, [d, m] per
// head, through a shared-memory transpose so that the stores are coalesced).
template <int D>
struct WTile {
    static constexpr int kRows = 32, kThreads = 128;
    static constexpr size_t bytes(int m) {   // sZ [32][m + 4] + sK [m][D] + sW [D][36]
        return sizeof(float) * ((size_t)32 * (m + 4) + (size_t)m * D + (size_t)D * 36);
    }
};

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(smem)),
                 "l"(gmem)
                 : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
    asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}
__device__ __forceinline__ void sm100_griddep_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <int D>
__global__ void __launch_bounds__(128)
w_tile_kernel(const float* __restrict__ z, const float* __restrict__ k3v, float* __restrict__ w,
              __nv_bfloat16* __restrict__ wt16, int m) {
    constexpr int CG = D / 4;                         // column groups of 4
    constexpr int RG = 128 / CG;                      // row groups (4 rows each): 8 (D=64) or 16 (D=32)
    static_assert(RG * 4 >= WTile<D>::kRows, "tile rows");
    extern __shared__ __align__(16) float wsm[];
    const int ldz = m + 4;                                                  // padded row: 4 rows hit 4 bank groups
    float* sZ = wsm;                                                        // [32][m + 4]
    float* sK = wsm + (size_t)32 * ldz;                                     // [m][D]
    float (*sW)[36] = reinterpret_cast<float (*)[36]>(sK + (size_t)m * D);  // [D][36]: W^T tile
    const int bh = blockIdx.y, r0 = blockIdx.x * WTile<D>::kRows;
    const int tid = threadIdx.x;
    // the output pass launched after this kernel may start its set-up now; it waits for this
    // kernel's completion before it reads W^T
    sm100_griddep_launch_dependents();
    const float* zb = z + ((size_t)bh * m + r0) * m;
    const float* kb = k3v + (size_t)bh * m * D;
    const int zc = m / 4;                             // 16-byte chunks per Z row
    for (int e = tid; e < 32 * zc; e += 128)
        cp_async16(sZ + (size_t)(e / zc) * ldz + 4 * (e % zc), zb + 4 * (size_t)e);
    for (int e = tid; e < m * D / 4; e += 128) cp_async16(sK + 4 * (size_t)e, kb + 4 * (size_t)e);
    cp_async_wait_all();
    __syncthreads();
    const int cg = tid % CG, rg = tid / CG;           // columns 4 cg .. 4 cg + 3, rows 4 rg .. 4 rg + 3
    if (4 * rg < WTile<D>::kRows) {
        float acc[4][4] = {};
        const float* zr = sZ + (size_t)(4 * rg) * ldz;
#pragma unroll 2
        for (int k = 0; k < m; k += 4) {
            float4 a[4], b[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = *reinterpret_cast<const float4*>(zr + (size_t)i * ldz + k);
#pragma unroll
            for (int j = 0; j < 4; ++j) b[j] = *reinterpret_cast<const float4*>(sK + (size_t)(k + j) * D + 4 * cg);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float ai[4] = {a[i].x, a[i].y, a[i].z, a[i].w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    acc[i][0] = fmaf(ai[j], b[j].x, acc[i][0]);
                    acc[i][1] = fmaf(ai[j], b[j].y, acc[i][1]);
                    acc[i][2] = fmaf(ai[j], b[j].z, acc[i][2]);
                    acc[i][3] = fmaf(ai[j], b[j].w, acc[i][3]);
                }
            }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int r = 4 * rg + i;
            *reinterpret_cast<float4*>(w + ((size_t)bh * m + r0 + r) * D + 4 * cg) =
                make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
#pragma unroll
            for (int j = 0; j < 4; ++j) sW[4 * cg + j][r] = acc[i][j];
        }
    }
    if (wt16 == nullptr) return;
    __syncthreads();
    // W^T tile: D rows of 32 bf16 (64 bytes) each, written as 16-byte chunks
    for (int e = tid; e < D * 4; e += 128) {
        const int c = e / 4, q = e % 4;               // column c of W, rows 8 q .. 8 q + 7 of the tile
        uint32_t pk[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            __nv_bfloat162 h = __floats2bfloat162_rn(sW[c][8 * q + 2 * j], sW[c][8 * q + 2 * j + 1]);
            pk[j] = *reinterpret_cast<uint32_t*>(&h);
        }
        *reinterpret_cast<uint4*>(wt16 + ((size_t)bh * D + c) * m + r0 + 8 * q) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
    }
}

// ------------------------------------------------------------------ output pass
// Walkthrough 2.4 and 2.6: out = softmax_row(Qs K_l^T) W + dwconv65(V).
// CTA (64 query rows, bh). Scores for all m landmarks stay in shared memory,
// so the row softmax is exact (no online rescaling).
template <typename T, int D>
struct OutSmem {
    static constexpr size_t bytes(int m) {
        return sizeof(float) * ((size_t)D * 68 * 2 + (size_t)64 * (m + 1) + (size_t)128 * (D + 4) + 72);
    }
};

template <typename T, int D>
__global__ void __launch_bounds__(256)
output_simt_kernel(const T* __restrict__ q, const float* __restrict__ kl, const float* __restrict__ w,
                   const T* __restrict__ v, const float* __restrict__ conv_w, T* __restrict__ out,
                   int H, int n, int m) {
    constexpr int CW = D / 16;
    extern __shared__ float smem[];
    float (*sQ)[68] = reinterpret_cast<float (*)[68]>(smem);              // [D][68]
    float (*sB)[68] = reinterpret_cast<float (*)[68]>(smem + D * 68);     // [D][68] K_l chunk / W chunk
    float* sS = smem + 2 * D * 68;                                        // [64][m+1]
    float (*sV)[D + 4] = reinterpret_cast<float (*)[D + 4]>(sS + 64 * (m + 1));  // [128][D+4]
    float* sw = reinterpret_cast<float*>(sV + 128);                       // [65]
    const int ldS = m + 1;
    const int bh = blockIdx.x, tile = blockIdx.y, h = bh % H;
    const int i0 = tile * 64;
    const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4, lane = tid & 31, warp = tid >> 5;
    const float s = split_scale(D);
    const T* qb = q + (size_t)bh * n * D;
    for (int e = tid; e < 64 * D; e += 256) {
        int r = e / D, c = e % D;
        sQ[c][r] = (i0 + r < n) ? s * Elt<T>::to_f(qb[(size_t)(i0 + r) * D + c]) : 0.f;
    }
    const float* klb = kl + (size_t)bh * m * D;
    for (int j0 = 0; j0 < m; j0 += 64) {
        __syncthreads();
        for (int e = tid; e < 64 * D; e += 256) {
            int r = e / D, c = e % D;
            sB[c][r] = (j0 + r < m) ? klb[(size_t)(j0 + r) * D + c] : 0.f;
        }
        __syncthreads();
        float acc[4][4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
#pragma unroll 8
        for (int e = 0; e < D; ++e) {
            float4 av = *reinterpret_cast<const float4*>(&sQ[e][ty * 4]);
            float4 bv = *reinterpret_cast<const float4*>(&sB[e][tx * 4]);
            float a4[4] = {av.x, av.y, av.z, av.w};
            float b4[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a4[i], b4[j], acc[i][j]);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                int c = j0 + tx * 4 + j;
                if (c < m) sS[(ty * 4 + i) * ldS + c] = acc[i][j];
            }
    }
    __syncthreads();
    for (int r = warp; r < 64; r += 8) {
        float* row = sS + r * ldS;
        float mx = -INFINITY;
        for (int c = lane; c < m; c += 32) mx = fmaxf(mx, row[c]);
        mx = warp_max(mx);
        float sum = 0.f;
        for (int c = lane; c < m; c += 32) {
            float e = __expf(row[c] - mx);
            row[c] = e;
            sum += e;
        }
        sum = warp_sum(sum);
        const float inv = 1.f / sum;
        for (int c = lane; c < m; c += 32) row[c] *= inv;
    }
    float o[4][CW];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < CW; ++j) o[i][j] = 0.f;
    const float* wb = w + (size_t)bh * m * D;
    for (int j0 = 0; j0 < m; j0 += 64) {
        __syncthreads();
        for (int e = tid; e < 64 * D; e += 256) {
            int r = e / D, c = e % D;
            sB[0][r * D + c] = (j0 + r < m) ? wb[(size_t)(j0 + r) * D + c] : 0.f;  // [64][D] row-major
        }
        __syncthreads();
        const float* sW = &sB[0][0];
        const int jn = min(64, m - j0);
        for (int kk = 0; kk < jn; ++kk) {
            float pv[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) pv[i] = sS[(ty * 4 + i) * ldS + j0 + kk];
#pragma unroll
            for (int j = 0; j < CW; ++j) {
                float wv = sW[kk * D + tx * CW + j];
#pragma unroll
                for (int i = 0; i < 4; ++i) o[i][j] = fmaf(pv[i], wv, o[i][j]);
            }
        }
    }
    if (conv_w != nullptr) {
        const T* vb = v + (size_t)bh * n * D;
        for (int e = tid; e < 128 * D; e += 256) {
            int r = e / D, c = e % D;
            int src = i0 - kHalfTaps + r;
            sV[r][c] = (src >= 0 && src < n) ? Elt<T>::to_f(vb[(size_t)src * D + c]) : 0.f;
        }
        if (tid < kTaps) sw[tid] = conv_w[(size_t)h * kTaps + tid];
        __syncthreads();
        for (int t = 0; t < kTaps; ++t) {
            const float wt = sw[t];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < CW; ++j) o[i][j] = fmaf(wt, sV[ty * 4 + i + t][tx * CW + j], o[i][j]);
        }
    }
    T* ob = out + (size_t)bh * n * D;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        int r = i0 + ty * 4 + i;
        if (r >= n) continue;
#pragma unroll
        for (int j = 0; j < CW; ++j) ob[(size_t)r * D + tx * CW + j] = Elt<T>::from_f(o[i][j]);
    }
}

}  // namespace nys
