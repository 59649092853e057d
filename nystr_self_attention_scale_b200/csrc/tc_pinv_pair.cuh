// tc_pinv_pair.cuh -- the iterative Moore-Penrose inverse for m = 256 on a CTA pair.
//
// Walkthrough (blog.gitcode.com) 2.5: Z_0 = c k2^T, then n_iter times
//   X = k2 Z;  T1 = 7I - X;  T3 = 15I - X T1;  T5 = 13I - X T3;  Z = Z T5 / 4.
//
// One head per cluster of two CTAs, and every product is one 2-CTA tcgen05 MMA
// (cta_group::2, M = N = 256, tf32): CTA r supplies rows 128r .. 128r+127 of
// the left factor A and receives the same rows of the product D in its TMEM,
// and it holds half of the right factor B in its shared memory: columns
// 128r .. 128r+127, as 128 K-major lines of 256 tf32 values (128 KB).
//
// The right factor of every product is produced by the epilogue of the
// previous one (T1, T3, T5, and Z for the next X = k2 Z), so it never leaves
// the chip: each thread owns one row of D, applies the affine step (scale and
// identity shift), rounds to tf32 and stores the row, column by column, into
// the B lines of whichever CTA owns that column -- its own shared memory or the
// peer's through distributed shared memory. X = k2 Z stays in TMEM and is the
// A operand of the next two products. The A operands that are not products of
// this iteration -- rows of k2 (for X = k2 Z) and rows of Z (for Z T5) -- are
// streamed in 32-column chunks by TMA through a 3-stage ring; the new rows of
// Z go back to L2-resident scratch with TMA stores during the same epilogue.
//
// Iteration 0 never forms Z_0 = c k2^T: its B operand is loaded as rows of k2,
// its A rows come from k2^T, and c is applied in the epilogues (X = c k2 k2^T
// is kept unscaled in TMEM, so T3 and T5 take the factor c too).
//
// Roles (320 threads): warps 0-7 epilogue (warp w reads TMEM lanes 32 (w % 4)
// and columns of half w / 4), warp 8 lane 0 TMA producer (both CTAs), warp 9
// TMEM allocation (both CTAs) and, in CTA 0 only, the MMA issuer.
#pragma once

#include "sm100.cuh"
#include "tc_pinv.cuh"

namespace nys {
namespace pair2 {

__device__ __forceinline__ uint32_t mapa(uint32_t saddr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
    return r;
}
__device__ __forceinline__ void st_local(uint32_t addr, float v) {
    asm volatile("st.shared.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}
__device__ __forceinline__ void st_remote(uint32_t addr, float v) {
    asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}
// Generic-proxy writes to this CTA's or the peer's shared memory become visible to the async proxy.
__device__ __forceinline__ void fence_proxy_async_cluster() {
    asm volatile("fence.proxy.async.shared::cluster;" ::: "memory");
}
__device__ __forceinline__ void arrive_cluster(uint32_t bar_cluster_addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster_addr) : "memory");
}
__device__ __forceinline__ bool try_wait_acq_cluster(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(sm100::smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
// Bounded wait with cluster-scope acquire (arrivals come from both CTAs).
__device__ __forceinline__ bool wait_acq_cluster(uint64_t* bar, uint32_t parity) {
    if (try_wait_acq_cluster(bar, parity)) return true;
    const uint64_t t0 = sm100::globaltimer();
    while (true) {
#pragma unroll 1
        for (int i = 0; i < 32; ++i)
            if (try_wait_acq_cluster(bar, parity)) return true;
        if (sm100::globaltimer() - t0 > sm100::kWaitLimitNs) {
            record_status(NYS_ERR_TIMEOUT);
            return false;
        }
    }
}
__device__ __forceinline__ void tmem_alloc2(uint32_t* dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(sm100::smem_u32(dst)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish2() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc2(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void mma2_ss(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::tf32 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d), "l"(a), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}
__device__ __forceinline__ void mma2_ts(uint32_t d, uint32_t a_tmem, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::tf32 [%0], [%1], %2, %3, p;\n\t}"
        ::"r"(d), "r"(a_tmem), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}
// Arrive on the barrier at the same shared-memory offset in every CTA of `mask`
// once all tcgen05 operations issued so far by this thread have completed.
__device__ __forceinline__ void commit2(uint64_t* bar, uint16_t mask) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;"
        ::"r"(sm100::smem_u32(bar)), "h"(mask)
        : "memory");
}
// TMA tile load into this CTA's shared memory whose completion is counted on the
// barrier at `bar_cluster_addr` (the pair's first CTA).
__device__ __forceinline__ void tma_load_3d_pair(void* dst, const CUtensorMap* m, uint32_t bar_cluster_addr,
                                                 int c0, int c1, int c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];"
        ::"r"(sm100::smem_u32(dst)), "l"(m), "r"(bar_cluster_addr), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}

}  // namespace pair2

struct PinvPairMaps {
    CUtensorMap a_k2;    // k2  [BH][256][256] fp32, box 32 x 128, 128-byte swizzle: A chunks
    CUtensorMap a_k2t;   // k2^T, same box: A chunks of Z_0 = c k2^T
    CUtensorMap a_z;     // Z scratch, same box: A chunks of Z and the TMA stores of new Z rows
    CUtensorMap z_out;   // the result, same box (stores)
    CUtensorMap b_k2;    // k2, box 32 x 32, 128-byte swizzle: the first right factor Z_0 (rows of k2)
};

struct PinvPairParams {
    const float* colsum_part;  // [BH][8][256] column sums of k2 per 32-row block
    const float* rowsum;       // [BH][256]
    const float* k2t;          // [BH][256][256] (n_iter = 0 only)
    float* z_out;              // [BH][256][256] (n_iter = 0 only)
    int n_iter;
};

struct PinvPair {
    static constexpr int M = 256;
    static constexpr int kStages = 3;
    static constexpr uint32_t kAtomBytes = 128 * 128;             // 128 lines x 32 tf32
    static constexpr uint32_t kBBytes = 8 * kAtomBytes;           // 8 K-atoms
    static constexpr uint32_t kAChunk = 128 * 128;                // 128 rows x 32 tf32
    static constexpr uint32_t kOffRing = kBBytes;
    static constexpr uint32_t kOffStage = kOffRing + kStages * kAChunk;   // two 16 KB store-staging tiles
    static constexpr uint32_t kOffBar = kOffStage + 2 * kAChunk;
    // barriers: full[3], empty[3], mma_done, b_ready, b_init, z_ready, drain
    static constexpr uint32_t kOffMisc = kOffBar + 16 * 8;
    static constexpr uint32_t kSmemBytes = kOffMisc + 64 + 1024;
    static constexpr int kThreads = 320;
    static constexpr uint32_t kIdesc = sm100::make_idesc(256, 256, sm100::kFmtTf32, sm100::kFmtTf32, 0, 0);
};
static_assert(PinvPair::kSmemBytes <= 227 * 1024, "pair inverse: shared memory");

__global__ void __launch_bounds__(PinvPair::kThreads, 1)
pinv_pair_kernel(const __grid_constant__ PinvPairMaps maps, const PinvPairParams prm) {
    using C = PinvPair;
    using namespace sm100;
    using namespace pair2;
    constexpr int M = C::M;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* bbuf = sm;
    uint8_t* ring = sm + C::kOffRing;
    uint8_t* stage = sm + C::kOffStage;
    uint64_t* full = reinterpret_cast<uint64_t*>(sm + C::kOffBar);
    uint64_t* empty = full + C::kStages;
    uint64_t* mma_done = empty + C::kStages;
    uint64_t* b_ready = mma_done + 1;
    uint64_t* b_init = b_ready + 1;
    uint64_t* z_ready = b_init + 1;
    uint64_t* drain = z_ready + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + C::kOffMisc);
    float* red = reinterpret_cast<float*>(sm + C::kOffMisc + 16);   // [8]

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t rank = cluster_rank();
    const bool leader = rank == 0;
    const int bh = blockIdx.x >> 1;
    const int r0 = (int)rank * 128;

    if (tid == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(mma_done, 1);
        mbar_init(b_ready, 16);    // one arrival per epilogue warp of either CTA
        mbar_init(b_init, 1);
        mbar_init(z_ready, 2);
        mbar_init(drain, 1);
        fence_mbar_init();
    }
    if (warp == 9) {
        tmem_alloc2(tmem_slot, 512);
        tmem_relinquish2();
    }
    // c = 1 / (max column sum * max row sum) of this head's kernel_2
    if (tid < 128) {
        float mc = -INFINITY, mr = -INFINITY;
        for (int c = tid; c < M; c += 128) {
            float s = 0.f;
#pragma unroll
            for (int b = 0; b < M / 32; ++b) s += prm.colsum_part[((size_t)bh * (M / 32) + b) * M + c];
            mc = fmaxf(mc, s);
            mr = fmaxf(mr, prm.rowsum[(size_t)bh * M + c]);
        }
        mc = warp_max(mc);
        mr = warp_max(mr);
        if (lane == 0) {
            red[warp] = mc;
            red[4 + warp] = mr;
        }
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();   // both CTAs' barriers initialised before any remote arrive or multicast commit
    tc_fence_after();
    const float coeff = 1.f / (fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3])) *
                               fmaxf(fmaxf(red[4], red[5]), fmaxf(red[6], red[7])));
    const uint32_t tmem = *tmem_slot;
    const uint32_t tA = tmem, tB = tmem + 256;   // X (A operand of two products) / product accumulators
    const int n_iter = prm.n_iter;

    if (n_iter == 0) {
        // Z = c k2^T
        for (int e = tid; e < 128 * (M / 4); e += C::kThreads) {
            const int r = r0 + e / (M / 4), c = (e % (M / 4)) * 4;
            const size_t o = ((size_t)bh * M + r) * M + c;
            float4 v = *reinterpret_cast<const float4*>(prm.k2t + o);
            v.x *= coeff; v.y *= coeff; v.z *= coeff; v.w *= coeff;
            *reinterpret_cast<float4*>(prm.z_out + o) = v;
        }
    } else if (warp == 8) {
        // ------------------------------------------------ TMA producer (both CTAs)
        if (lane == 0) {
            prefetch_tmap(&maps.a_k2);
            prefetch_tmap(&maps.a_k2t);
            prefetch_tmap(&maps.a_z);
            prefetch_tmap(&maps.b_k2);
            const uint32_t full0 = mapa(smem_u32(full), 0);
            // B line n of this CTA is column 128 rank + n of Z_0, i.e. row 128 rank + n of k2
            mbar_arrive_expect_tx(b_init, C::kBBytes);
            for (int a = 0; a < 8; ++a)
                for (int j = 0; j < 4; ++j)
                    tma_load_3d(bbuf + a * C::kAtomBytes + j * 4096, &maps.b_k2, b_init, 32 * a, r0 + 32 * j, bh);
            bool ok = true;
            uint32_t g = 0;
            for (int it = 0; it < n_iter && ok; ++it) {
                for (int part = 0; part < 2 && ok; ++part) {
                    const CUtensorMap* mp = part == 0 ? &maps.a_k2 : (it == 0 ? &maps.a_k2t : &maps.a_z);
                    if (part == 1 && it > 0) {
                        ok = mbar_wait(z_ready, (uint32_t)(it - 1) & 1u);   // this CTA's new Z rows are stored
                        fence_proxy_async_global();
                    }
                    for (int kc = 0; kc < 8 && ok; ++kc, ++g) {
                        const uint32_t st = g % C::kStages;
                        ok = mbar_wait(&empty[st], ((g / C::kStages) & 1u) ^ 1u);
                        if (!ok) break;
                        if (leader) mbar_arrive_expect_tx(&full[st], 2 * C::kAChunk);
                        tma_load_3d_pair(ring + st * C::kAChunk, mp, full0 + 8 * st, 32 * kc, r0, bh);
                    }
                }
            }
        }
        __syncwarp();
    } else if (warp == 9) {
        // ------------------------------------------------ MMA issuer (first CTA of the pair)
        if (leader && lane == 0) {
            const uint32_t bs = smem_u32(bbuf), rs = smem_u32(ring);
            bool ok = true;
            uint32_t g = 0, nb = 0;
            for (int it = 0; it < n_iter && ok; ++it) {
                for (int p = 0; p < 4 && ok; ++p) {
                    ok = wait_acq_cluster(b_ready, nb & 1u);   // B of this product in place, last D read
                    ++nb;
                    if (!ok) break;
                    tc_fence_after();
                    const bool from_ring = p == 0 || p == 3;
                    const uint32_t d = p == 0 ? tA : tB;
                    for (int kc = 0; kc < 8; ++kc) {
                        uint32_t sa = 0, st = 0;
                        if (from_ring) {
                            st = g % C::kStages;
                            ok = mbar_wait(&full[st], (g / C::kStages) & 1u);
                            if (!ok) break;
                            tc_fence_after();
                            sa = rs + st * C::kAChunk;
                        }
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk) {
                            const uint64_t bdesc =
                                smem_desc(bs + kc * C::kAtomBytes + kk * 32, 16, 1024, kLayoutSw128);
                            const uint32_t acc = (kc | kk) != 0 ? 1u : 0u;
                            if (from_ring)
                                mma2_ss(d, smem_desc(sa + kk * 32, 16, 1024, kLayoutSw128), bdesc, C::kIdesc, acc);
                            else
                                mma2_ts(d, tA + kc * 32 + kk * 8, bdesc, C::kIdesc, acc);
                        }
                        if (from_ring) {
                            commit2(&empty[st], 3);
                            ++g;
                        }
                    }
                    if (ok) commit2(mma_done, 3);
                }
            }
            // every MMA issued here has completed before the pair tears down
            commit2(drain, 1);
            mbar_wait(drain, 0);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------ epilogue (warps 0-7, both CTAs)
        const int q = warp & 3, h = warp >> 2;      // TMEM lane quadrant, column half
        const int lt = tid & 127;                   // thread index within the half
        const int row = r0 + 32 * q + lane;         // this thread's row of every product
        const uint32_t lane_base = (uint32_t)(32 * q) << 16;
        const uint32_t b_ready0 = mapa(smem_u32(b_ready), 0);
        // columns 128 h .. 128 h + 127 of every product belong to the B half of CTA h
        const bool to_local = (uint32_t)h == rank;
        const uint32_t b_dst = to_local ? smem_u32(bbuf) : mapa(smem_u32(bbuf), rank ^ 1u);
        // byte offset of (this row's K position) inside a B line of column i, for i % 8 = 0..7
        const uint32_t k_off = (uint32_t)(4 * (int)rank + q) * C::kAtomBytes + (uint32_t)(lane & 3) * 4u;
        const uint32_t xl = (uint32_t)(lane >> 2);
        uint8_t* stg = stage + h * C::kAChunk;
        const int bar_stage = 1 + h;                 // named barrier of this half's 128 threads

        bool failed = !mbar_wait(b_init, 0);
        failed = group_any(failed, 3, 256);
        if (!failed) {
            __syncwarp();
            if (lane == 0) arrive_cluster(b_ready0);
        }
        uint32_t nprod = 0;
        for (int it = 0; it < n_iter && !failed; ++it) {
            const float s_it = it == 0 ? coeff : 1.f;
            for (int p = 0; p < 4 && !failed; ++p) {
                const bool ok = mbar_wait(mma_done, nprod & 1u);
                ++nprod;
                failed = group_any(!ok, 3, 256);
                if (failed) break;
                tc_fence_after();
                const bool last = it + 1 == n_iter && p == 3;
                const uint32_t d = p == 0 ? tA : tB;
                const float alpha = p == 3 ? 0.25f * s_it : -s_it;
                const float diag = p == 0 ? 7.f : (p == 1 ? 15.f : (p == 2 ? 13.f : 0.f));
                const CUtensorMap* zmap = last ? &maps.z_out : &maps.a_z;
#pragma unroll 1
                for (int jj = 0; jj < 4; ++jj) {
                    const int a = 4 * h + jj;             // 32-column atom of D
                    uint32_t v[32];
                    tmem_ld32(d + lane_base + a * 32, v);
                    tmem_ld_wait();
                    float e[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i) e[i] = alpha * __uint_as_float(v[i]);
                    if (a == (row >> 5)) {
#pragma unroll
                        for (int i = 0; i < 32; ++i) e[i] += i == lane ? diag : 0.f;
                    }
                    if (!last) {
#pragma unroll
                        for (int i = 0; i < 32; ++i) e[i] = tf32_rna(e[i]);
                        // column 32 a + i is line 32 (a % 4) + i of CTA h's B half
                        const uint32_t base = b_dst + k_off + (uint32_t)(a & 3) * 4096u;
                        if (to_local) {
#pragma unroll
                            for (int i = 0; i < 32; ++i)
                                st_local(base + i * 128 + ((xl ^ (uint32_t)(i & 7)) << 4), e[i]);
                        } else {
#pragma unroll
                            for (int i = 0; i < 32; ++i)
                                st_remote(base + i * 128 + ((xl ^ (uint32_t)(i & 7)) << 4), e[i]);
                        }
                    }
                    if (p == 3) {
                        // this half's staging tile -> TMA store of rows r0.., columns 32 a ..
                        if (jj > 0) {
                            if (lt == 0) tma_store_wait_read<0>();
                            named_barrier(bar_stage, 128);
                        }
                        const int srow = 32 * q + lane;
#pragma unroll
                        for (int c = 0; c < 8; ++c)
                            *reinterpret_cast<float4*>(stg + swz<128>(srow, c)) =
                                make_float4(e[4 * c], e[4 * c + 1], e[4 * c + 2], e[4 * c + 3]);
                        fence_proxy_async_shared();
                        named_barrier(bar_stage, 128);
                        if (lt == 0) {
                            tma_store_3d(zmap, stg, 32 * a, r0, bh);
                            tma_store_commit();
                        }
                    }
                }
                if (p == 0 && it > 0 && lt == 0) {
                    // the Z rows stored at the end of the previous iteration are in L2 before the
                    // producer streams them back as the A operand of Z T5
                    tma_store_wait_all<0>();
                    fence_proxy_async_global();
                    mbar_arrive(z_ready);
                }
                if (!last) {
                    fence_proxy_async_cluster();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) arrive_cluster(b_ready0);
                }
            }
        }
        if (lt == 0) tma_store_wait_all<0>();
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync_all();   // no remote store, arrive or MMA of either CTA is still pending
    if (warp == 9) {
        tc_fence_after();
        tmem_dealloc2(tmem, 512);
    }
    cluster_sync_all();
}

}  // namespace nys
