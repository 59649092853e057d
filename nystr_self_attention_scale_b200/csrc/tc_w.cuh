// tc_w.cuh -- W = Z (kernel_3 V) on the tensor cores (tf32), for m = 128 and m = 256.
//
// Walkthrough (blog.gitcode.com) 2.6 computes kernel_1 Z (kernel_3 V); the library takes the
// product as kernel_1 (Z (kernel_3 V)) and forms the [m, d] factor W = Z (kernel_3 V) once per
// head, which the output pass then multiplies P by. One CTA per 128 rows of W:
//   A = 128 rows of Z, K-major (TMA tiles of 32 columns, 128-byte swizzle), as in the inverse
//   B = kernel_3 V [m, d], staged by the threads in the MN-major tf32 layout (rows of 32 values
//       along d, 32-byte granules swizzled by row % 4), rounded to tf32 (nearest, ties away)
//   D = [128, d] fp32 in TMEM: m / 8 MMAs of K = 8
// The epilogue (warp w: TMEM lanes 32 (w % 4), columns 32 (w / 4) ..; one thread per row and
// 32 columns) writes W in fp32 ([m, d] per head) and W^T in bf16 ([d, m] per head, the
// output pass's operand). A and B are rounded to tf32 (10-bit
// mantissa); the output pass reads W^T in bf16 (7-bit mantissa).
//
// The output pass is launched as a programmatic dependent of this kernel: it starts its
// prologue while this grid runs and waits for its completion before reading W^T.
#pragma once

#include "sm100.cuh"

namespace nys {

template <int D>
struct WTc {
    static constexpr int kThreads = 512;   // staging: m * D / 4 float4 over all threads, 8 each at most
    static constexpr uint32_t kAtom = 128 * 128;               // 128 rows x 32 fp32 of Z: 16 KB
    static constexpr uint32_t kMnAtom = 1024;                  // 8 K rows x 32 columns of B
    static constexpr uint32_t kKGroup = (D / 32) * kMnAtom;    // 8 K rows x D columns of B
    static constexpr uint32_t kIdesc = sm100::make_idesc(128, D, sm100::kFmtTf32, sm100::kFmtTf32, 0, 1);
    __host__ __device__ static constexpr uint32_t off_b(int m) { return (uint32_t)m / 32 * kAtom; }
    __host__ __device__ static constexpr uint32_t off_bar(int m) { return off_b(m) + (uint32_t)m / 8 * kKGroup; }
    __host__ __device__ static constexpr uint32_t bytes(int m) { return off_bar(m) + 64 + 1024; }
};

template <int D>
__global__ void __launch_bounds__(WTc<D>::kThreads, 1)
w_tc_kernel(const __grid_constant__ CUtensorMap map_z, const float* __restrict__ k3v, float* __restrict__ w,
            __nv_bfloat16* __restrict__ wt16, int m) {
    using C = WTc<D>;
    using namespace sm100;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + C::off_bar(m));
    uint64_t* z_full = bars + 0;
    uint64_t* mma_done = bars + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int row0 = blockIdx.x * 128, bh = blockIdx.y;
    const int atoms = m / 32;

    if (tid == 0) {
        mbar_init(z_full, 1);
        mbar_init(mma_done, 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, D);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (tid == 0) {
        prefetch_tmap(&map_z);
        mbar_arrive_expect_tx(z_full, (uint32_t)atoms * C::kAtom);
        for (int a = 0; a < atoms; ++a) tma_load_3d(sm + a * C::kAtom, &map_z, z_full, 32 * a, row0, bh);
    }
    // B = kernel_3 V of this head: float4 i of the [m, D] matrix is row k = i / (D / 4), columns
    // 4 (i % (D / 4)) .. + 3, i.e. 16-byte chunk (i % 8) of the 32-column atom (i % (D / 4)) / 8
    // (up to 8 loads in flight per thread, one round at m * D / 4 = 4096; the tail is predicated)
    {
        constexpr int kBatch = 8;
        const float4* src = reinterpret_cast<const float4*>(k3v + (size_t)bh * m * D);
        const int total = m * (D / 4);
#pragma unroll 1
        for (int i0 = tid; i0 < total; i0 += kBatch * C::kThreads) {
            float4 x[kBatch];
#pragma unroll
            for (int u = 0; u < kBatch; ++u) {
                const int i = i0 + u * C::kThreads;
                x[u] = i < total ? __ldg(src + i) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int u = 0; u < kBatch; ++u) {
                const int i = i0 + u * C::kThreads, k = i / (D / 4), c4 = i % (D / 4);
                if (i >= total) break;
                const uint32_t off = C::off_b(m) + (uint32_t)(k >> 3) * C::kKGroup +
                                     (uint32_t)(c4 >> 3) * C::kMnAtom + mn32_chunk(k & 7, c4 & 7);
                *reinterpret_cast<float4*>(sm + off) =
                    make_float4(tf32_rna(x[u].x), tf32_rna(x[u].y), tf32_rna(x[u].z), tf32_rna(x[u].w));
            }
        }
    }
    fence_proxy_async_shared();   // the staged B feeds the MMA
    __syncthreads();

    bool ok = true;
    if (warp == 0) {
        ok = warp_all(mbar_wait(z_full, 0));
        if (ok) {
            tc_fence_after();
            const uint32_t sa = smem_u32(sm), sb = sa + C::off_b(m);
            if (elect_one()) {
                for (int a = 0; a < atoms; ++a)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const int j = 4 * a + kk;   // K step of 8 rows
                        mma_tf32_ss(tmem, smem_desc(sa + a * C::kAtom + kk * 32, 16, 1024, kLayoutSw128),
                                    smem_desc(sb + (uint32_t)j * C::kKGroup, C::kMnAtom, 512, kLayoutSw128B32),
                                    C::kIdesc, j > 0 ? 1u : 0u);
                    }
                mma_commit(mma_done);
            }
            __syncwarp();
        }
    }
    griddep_launch_dependents();
    ok = __syncthreads_and(ok) != 0;
    if (ok) ok = mbar_wait(mma_done, 0);
    if (ok && warp < 4 * (D / 32)) {
        tc_fence_after();
        const int q = warp & 3, j = warp >> 2;      // TMEM lane quadrant, 32-column block
        const int r = row0 + 32 * q + lane;         // this thread's row of W (TMEM lane)
        float* wr = w + ((size_t)bh * m + r) * D;
        __nv_bfloat16* wtc = wt16 + (size_t)bh * D * m + r;
        {
            uint32_t v[32];
            tmem_ld32(tmem + ((uint32_t)(32 * q) << 16) + 32 * j, v);
            tmem_ld_wait();
#pragma unroll
            for (int c = 0; c < 8; ++c)
                *reinterpret_cast<float4*>(wr + 32 * j + 4 * c) =
                    make_float4(__uint_as_float(v[4 * c]), __uint_as_float(v[4 * c + 1]),
                                __uint_as_float(v[4 * c + 2]), __uint_as_float(v[4 * c + 3]));
#pragma unroll
            for (int c = 0; c < 32; ++c) wtc[(size_t)(32 * j + c) * m] = __float2bfloat16_rn(__uint_as_float(v[c]));
        }
    }
    if (!ok && tid == 0) {
        // a wait ran out: give the copies and the MMA in flight a second bounded wait before the
        // shared memory and the TMEM are released
        mbar_wait(z_full, 0);
        mbar_wait(mma_done, 0);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, D);
    }
}

}  // namespace nys
