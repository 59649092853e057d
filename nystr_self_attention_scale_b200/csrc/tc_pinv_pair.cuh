// tc_pinv_pair.cuh -- the iterative Moore-Penrose inverse for m = 256 on a CTA pair.
//
// Walkthrough (blog.gitcode.com) 2.5: Z_0 = c k2^T, then n_iter times
//   X = k2 Z;  T1 = 7I - X;  T3 = 15I - X T1;  T5 = 13I - X T3;  Z = Z T5 / 4.
//
// Two exact identities shape the kernel. (1) T1, T3 and T5 are polynomials in
// X, so they commute with X. (2) Transposing the update gives W = Z^T with
// W_0 = c k2, X^T = W k2^T and W <- T5(X^T) W / 4, where T5(X^T) is the same
// polynomial taken in X^T. The kernel iterates in X^T (called X below)
//   P1: X = W k2^T    P2: -U = T1 (-X)    P3: -V = T3 (-X)    P4: W = T5 W / 4
// (equal to the page's sequence in real arithmetic) and takes every left
// factor from TMEM: W is the raw accumulator of the previous P4; T1 = 7I - X
// is written back over P1's accumulator by its epilogue (tf32-rounded); since
// P2 and P3 multiply by -X, their accumulators -U and -V differ from
// T3 = 15I - U and T5 = 13I - V only on the diagonal, which is all their
// epilogues change (the other entries reach the MMA as fp32 bits). The right
// factors live in shared memory as K-major lines: -X, written once per
// iteration by the P1 epilogue column by column into the B half of the CTA
// that owns the column (its own or, through distributed shared memory, the
// peer's) -- X is symmetric only in exact arithmetic, and using its rows as
// its columns loses accuracy on ill-conditioned k2 -- and, streamed from L2 one
// 32-wide K atom at a time behind the previous product's MMAs, the columns of W
// (for P4; the P4 epilogue writes W^T row-major to scratch; the first P4 reads
// W_0 = c k2 by rows instead, as an MN-major operand, so that no transpose of k2
// is written) and the last three K atoms of k2's rows (for P1; its first five K
// atoms stay in shared memory for the whole kernel).
//
// One head per cluster of two CTAs, one 2-CTA tcgen05 MMA per K step
// (cta_group::2, kind::tf32, M = N = 256): CTA r holds rows 128r .. 128r+127 of
// A and D in its TMEM and lines (columns) 128r .. 128r+127 of B in its shared
// memory. TMEM: R0 = columns 0..255, R1 = 256..511; per iteration
//   P1: A = R0 (W), D -> R1;  P2: A = R1 (T1), D -> R0;
//   P3: A = R0 (T3), D -> R1; P4: A = R1 (T5), D -> R0 (the next W).
// Scale factors are folded into the epilogues: the stored W is the raw P4
// accumulator (sigma = c for W_0 = c k2 loaded unscaled, c/4 after the first
// P4, 1/4 afterwards).
//
// Roles (320 threads): warps 0-7 epilogue (warp w: TMEM lanes 32 (w % 4),
// columns 128 (w / 4) ..), warp 8 lane 0 TMA producer (both CTAs), warp 9 TMEM
// allocation (both CTAs) and, in CTA 0, the MMA issuer.
#pragma once

#include "sm100.cuh"

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
// barrier at `bar_cluster_addr` (the pair's first CTA), with an L2 cache-policy hint.
__device__ __forceinline__ void tma_load_3d_pair(void* dst, const CUtensorMap* m, uint32_t bar_cluster_addr,
                                                 int c0, int c1, int c2, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%3, %4, %5}], [%2], %6;"
        ::"r"(sm100::smem_u32(dst)), "l"(m), "r"(bar_cluster_addr), "r"(c0), "r"(c1), "r"(c2), "l"(policy)
        : "memory");
}

}  // namespace pair2

struct PinvPairMaps {
    CUtensorMap ql;    // Q_l  [BH][256][d] fp32, box 32 x 128, 128-byte swizzle: A of the kernel_2 product
    CUtensorMap kl;    // K_l, same box: B lines of the kernel_2 product
    CUtensorMap k2;    // k2   [BH][256][256] fp32, box 32 x 128: B atoms of the later P1s (and its TMA store)
    CUtensorMap k2mn;  // k2 again, box 32 x 32, 32-byte-granule 128-byte swizzle: the first P4's B atoms,
                       // MN-major (W_0 = c k2 read by rows: K row k = row k of k2)
    CUtensorMap wt;    // W^T scratch, same box: B atoms of the later P4s
};

struct PinvPairParams {
    float* k2;         // [BH][256][256] k2 (tf32), written here, read back by TMA
    float* wt;         // [BH][256][256] W^T scratch (row g = column g of W)
    float* z_out;      // [BH][256][256]
    int d, n_iter;
    int inv_init;      // NYS_INV_INIT_DEFAULT or NYS_INV_INIT_EXACT
};

struct PinvPair {
    static constexpr int M = 256;
    static constexpr uint32_t kAtomBytes = 128 * 128;          // 128 lines x 32 tf32
    static constexpr uint32_t kBBytes = 8 * kAtomBytes;        // 8 K atoms = 128 KB
    // kernel_2 operands in the B buffer: Q_l hi / lo, K_l hi / lo (d / 32 atoms each)
    static constexpr uint32_t kOffAhi = 0, kOffAlo = 2 * kAtomBytes, kOffBhi = 4 * kAtomBytes,
                              kOffBlo = 6 * kAtomBytes;
    static constexpr uint32_t kOffRed = kBBytes;                // row / column reductions
    // [2][128] row max / sum halves, [256] own column sums, [256] the peer's, [8] warp maxima,
    // [2] own and peer max row sum
    static constexpr uint32_t kOffBar = kOffRed + (2 * 128 + 2 * 128 + 256 + 256 + 8 + 8) * 4;
    // barriers: bfull[8], bfree[8], mma_done, mma4_done, e_ready, wl_ready, drain, pro_full, cs_ready,
    // e_step[2]
    static constexpr uint32_t kOffMisc = kOffBar + 26 * 8;
    // K atoms 0 .. kK2Resident - 1 of k2 (this CTA's B lines) stay in shared memory for every
    // P1; the later P1s stream only the other atoms through the B buffer
    static constexpr int kK2Resident = 5;
    static constexpr uint32_t kOffK2r = (kOffMisc + 64 + 1023) / 1024 * 1024;
    static constexpr uint32_t kSmemNeed = kOffK2r + kK2Resident * kAtomBytes + 1024;
    // more than half of the SM's shared memory: no other CTA (and no other TMEM user) shares the SM
    static constexpr uint32_t kSmemBytes = kSmemNeed < 200 * 1024 ? 200 * 1024 : kSmemNeed;
    static constexpr int kThreads = 320;
    static constexpr uint32_t kIdesc = sm100::make_idesc(256, 256, sm100::kFmtTf32, sm100::kFmtTf32, 0, 0);
    // the first P4: B MN-major (K atom kc = rows 32 kc .. + 31 of k2, this CTA's 128 columns as four
    // 4 KB column blocks of 32 rows x 128 bytes; an MMA K step is 8 rows = 1 KB into each block)
    static constexpr uint32_t kIdescBmn = sm100::make_idesc(256, 256, sm100::kFmtTf32, sm100::kFmtTf32, 0, 1);
    static constexpr uint32_t kMnBlock = 32 * 128;
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
    float* rx = reinterpret_cast<float*>(sm + C::kOffRed);   // [2][128] row max, later row sum of k2, per half
    float* sx = rx + 256;                                     // [2][128] row sums of each half
    float* cs_own = sx + 256;                                 // [256] column sums over this CTA's rows
    float* cs_peer = cs_own + 256;                            // [256] the same from the peer CTA
    float* wmax = cs_peer + 256;                              // [8]
    float* rmax = wmax + 8;                                   // [0] own, [1] peer max row sum
    uint64_t* bfull = reinterpret_cast<uint64_t*>(sm + C::kOffBar);   // [8], used in CTA 0
    uint64_t* bfree = bfull + 8;                                       // [8], both CTAs (after P3, P4)
    uint64_t* mma_done = bfree + 8;      // kernel_2 and P1..P3 accumulators complete (both CTAs)
    uint64_t* mma4_done = mma_done + 1;  // P4 accumulator complete (both CTAs)
    uint64_t* e_ready = mma4_done + 1;   // epilogue output in place for the next product (CTA 0)
    uint64_t* wl_ready = e_ready + 1;    // k2 / W^T scratch written by both CTAs (each CTA)
    uint64_t* drain = wl_ready + 1;
    uint64_t* pro_full = drain + 1;      // Q_l / K_l tiles landed (each CTA)
    uint64_t* cs_ready = pro_full + 1;   // the peer's column sums are in cs_peer (each CTA)
    uint64_t* e_step = cs_ready + 1;     // [2] CTA 0: epilogue steps 2 h, 2 h + 1 of P2 / P3 done in both CTAs
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + C::kOffMisc);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t rank = cluster_rank();
    const bool leader = rank == 0;
    const int bh = blockIdx.x >> 1;
    const int r0 = (int)rank * 128;
    const int nka = prm.d / 32;          // K atoms of the kernel_2 product
    const int n_iter = prm.n_iter;

    if (tid == 0) {
        for (int s = 0; s < 8; ++s) {
            mbar_init(&bfull[s], 1);
            mbar_init(&bfree[s], 1);
        }
        mbar_init(mma_done, 1);
        mbar_init(mma4_done, 1);
        mbar_init(e_ready, 16);    // one arrival per epilogue warp of either CTA
        mbar_init(wl_ready, 16);
        mbar_init(drain, 32);     // one commit per lane of the MMA warp
        mbar_init(pro_full, 1);
        mbar_init(cs_ready, 8);    // one arrival per epilogue warp of the peer
        for (int j = 0; j < 2; ++j) mbar_init(&e_step[j], 16);   // one arrival per epilogue warp
        fence_mbar_init();
    }
    if (warp == 9) {
        tmem_alloc2(tmem_slot, 512);
        tmem_relinquish2();
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();   // both CTAs' barriers initialised before any remote arrive or multicast commit
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t R0 = tmem, R1 = tmem + 256;

    if (warp == 8) {
        // ------------------------------------------------ TMA producer (both CTAs)
        if (lane == 0) {
            prefetch_tmap(&maps.ql);
            prefetch_tmap(&maps.kl);
            prefetch_tmap(&maps.k2);
            prefetch_tmap(&maps.k2mn);
            prefetch_tmap(&maps.wt);
            // kernel_2 operands: this CTA's rows of Q_l (A) and of K_l (its B lines)
            mbar_arrive_expect_tx(pro_full, 2u * nka * C::kAtomBytes);
            for (int a = 0; a < nka; ++a) {
                tma_load_3d(bbuf + C::kOffAhi + a * C::kAtomBytes, &maps.ql, pro_full, 32 * a, r0, bh);
                tma_load_3d(bbuf + C::kOffBhi + a * C::kAtomBytes, &maps.kl, pro_full, 32 * a, r0, bh);
            }
            const uint32_t bfull0 = mapa(smem_u32(bfull), 0);
            // k2 and W^T are streamed in again every iteration: keep them in L2
            const uint64_t keep_policy = l2_policy_evict_last();
            bool ok = true;
            for (int it = 0; it < n_iter && ok; ++it) {
                for (int part = 0; part < 2 && ok; ++part) {
                    const int p = part == 0 ? 0 : 3;
                    if (p == 0 && it == 0) continue;   // the first P1 reads k2 staged by the prologue
                    const CUtensorMap* mp = p == 0 ? &maps.k2 : &maps.wt;
                    if (p == 3) {
                        // k2 (prologue) or W^T (previous P4) of both CTAs is in global memory
                        ok = wait_acq_cluster(wl_ready, (uint32_t)it & 1u);
                        fence_proxy_async_global();
                    }
                    for (int i = 0; i < 8 && ok; ++i) {
                        // K atom kc is free once the previous product (P3 before P4, P4 before the
                        // next P1) has read it; the atoms are taken in the order those products
                        // free them. bfree[kc] completes twice per iteration, after P3 and after
                        // P4, and never runs ahead of these waits by more than one phase, so its
                        // parity is exact: every completion is waited for, also for the resident
                        // k2 atoms that the P1s do not stream.
                        const int kc = (i & 1) ? 4 + (i >> 1) : (i >> 1);
                        ok = mbar_wait(&bfree[kc], p == 3 ? 0u : 1u);
                        if (!ok) break;
                        if (p == 0 && kc < C::kK2Resident) continue;
                        if (leader) mbar_arrive_expect_tx(&bfull[kc], 2 * C::kAtomBytes);
                        if (p == 3 && it == 0) {
                            // rows 32 kc .. + 31 of k2, this CTA's columns r0 .. r0 + 127
                            for (int t = 0; t < 4; ++t)
                                tma_load_3d_pair(bbuf + kc * C::kAtomBytes + t * C::kMnBlock, &maps.k2mn, bfull0 + 8 * kc,
                                                 r0 + 32 * t, 32 * kc, bh, keep_policy);
                        } else {
                            tma_load_3d_pair(bbuf + kc * C::kAtomBytes, mp, bfull0 + 8 * kc, 32 * kc, r0, bh, keep_policy);
                        }
                    }
                }
            }
        }
        __syncwarp();
    } else if (warp == 9) {
        // ------------------------------------------------ MMA issuer (first CTA of the pair): the
        // whole warp runs the loop and the waits; one elected lane issues each MMA group and commit
        if (leader) {
            const uint32_t bs = smem_u32(bbuf);
            bool ok = true;
            uint32_t ne = 0;        // e_ready phases waited
            uint32_t fph = 0;       // bit kc: the parity of the next bfull[kc] phase to wait for
            // kernel_2: S2 = Q_l K_l^T from split tf32 operands, hi.hi + hi.lo + lo.hi
            ok = warp_all(wait_acq_cluster(e_ready, ne & 1u));
            ++ne;
            if (ok) {
                tc_fence_after();
                if (elect_one()) {
                    const uint32_t aoff[3] = {C::kOffAhi, C::kOffAhi, C::kOffAlo};
                    const uint32_t boff[3] = {C::kOffBhi, C::kOffBlo, C::kOffBhi};
                    uint32_t acc = 0;
                    for (int t = 0; t < 3; ++t)
                        for (int a = 0; a < nka; ++a)
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk) {
                                const uint32_t ka = a * C::kAtomBytes + kk * 32;
                                mma2_ss(R1, smem_desc(bs + aoff[t] + ka, 16, 1024, kLayoutSw128),
                                        smem_desc(bs + boff[t] + ka, 16, 1024, kLayoutSw128), C::kIdesc, acc);
                                acc = 1;
                            }
                }
                if (elect_one()) commit2(mma_done, 3);
            }
            uint32_t ns = 0;   // e_step phases waited
            for (int it = 0; it < n_iter && ok; ++it) {
                for (int p = 0; p < 4 && ok; ++p) {
                    const uint32_t a_col = (p == 0 || p == 2) ? R0 : R1;
                    const uint32_t d_col = (p == 0 || p == 2) ? R1 : R0;
                    const bool streamed = p == 3 || (p == 0 && it > 0);
                    // P3 and P4 start on the first half of their left factor while the epilogue of
                    // the previous product still writes the rest (its steps 0, 1 write atoms 0, 1,
                    // 4, 5 in both CTAs, steps 2, 3 the others); the other products wait for all
                    const bool stepped = p >= 2;
                    if (!stepped && (p != 0 || it == 0)) {
                        ok = warp_all(wait_acq_cluster(e_ready, ne & 1u));   // left factor (and X, or k2) in place
                        ++ne;
                        if (!ok) break;
                    }
                    tc_fence_after();
                    for (int i = 0; i < 8; ++i) {
                        // atoms 0, 4, 1, 5, ... (the later P1s: 0 .. 7, the resident ones first)
                        const bool resident_p1 = p == 0 && it > 0;
                        const int kc = resident_p1 ? i : ((i & 1) ? 4 + (i >> 1) : (i >> 1));
                        const bool resident = resident_p1 && kc < C::kK2Resident;
                        if (stepped && (i & 3) == 0) {
                            ok = warp_all(wait_acq_cluster(&e_step[i >> 2], ns & 1u));
                            if (!ok) break;
                            tc_fence_after();
                        }
                        if (streamed && !resident) {
                            ok = warp_all(mbar_wait(&bfull[kc], (fph >> kc) & 1u));
                            fph ^= 1u << kc;
                            if (!ok) break;
                            tc_fence_after();
                        }
                        if (elect_one()) {
                            if (p == 3 && it == 0) {
#pragma unroll
                                for (int kk = 0; kk < 4; ++kk)
                                    mma2_ts(d_col, a_col + kc * 32 + kk * 8,
                                            smem_desc(bs + kc * C::kAtomBytes + kk * 1024, C::kMnBlock, 512, kLayoutSw128B32),
                                            C::kIdescBmn, (i | kk) != 0 ? 1u : 0u);
                            } else {
#pragma unroll
                                for (int kk = 0; kk < 4; ++kk)
                                    mma2_ts(d_col, a_col + kc * 32 + kk * 8,
                                            smem_desc((resident ? bs + C::kOffK2r : bs) + kc * C::kAtomBytes + kk * 32, 16,
                                                      1024, kLayoutSw128),
                                            C::kIdesc, (i | kk) != 0 ? 1u : 0u);
                            }
                            if (p >= 2) commit2(&bfree[kc], 3);   // the producer refills this atom next
                        }
                    }
                    if (stepped) ++ns;
                    if (ok && elect_one()) commit2(p == 3 ? mma4_done : mma_done, 3);
                }
            }
            // every MMA issued here has completed before the pair tears down: one commit per
            // lane (drain counts 32 arrivals), so the drain covers whichever lane issued
            commit2(drain, 1);
            mbar_wait(drain, 0);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------ epilogue (warps 0-7, both CTAs)
        const int q = warp & 3, h = warp >> 2;      // TMEM lane quadrant, column half
        const int lrow = 32 * q + lane;             // TMEM lane = this CTA's row = its B line
        const int row = r0 + lrow;                  // global row of every product
        const int et = tid;                          // 0 .. 255
        const uint32_t lane_base = (uint32_t)(32 * q) << 16;
        const uint32_t e_ready0 = mapa(smem_u32(e_ready), 0);
        const uint32_t wl_loc = mapa(smem_u32(wl_ready), rank), wl_rem = mapa(smem_u32(wl_ready), rank ^ 1u);
        // X lines: columns 128 h .. 128 h + 127 belong to CTA h's B half
        const bool x_local = (uint32_t)h == rank;
        const uint32_t x_dst = x_local ? smem_u32(bbuf) : mapa(smem_u32(bbuf), rank ^ 1u);
        const uint32_t k_off = (uint32_t)(4 * (int)rank + q) * C::kAtomBytes + (uint32_t)(lane & 3) * 4u;
        const uint32_t xl = (uint32_t)(lane >> 2);
        const bool diag_half = (uint32_t)h == rank;  // this half's columns hold the diagonal element
        const int diag_atom = 4 * h + q;             // (only when diag_half)
        auto arrive_e = [&]() {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) arrive_cluster(e_ready0);
        };
        const uint32_t e_step0 = mapa(smem_u32(e_step), 0);
        auto arrive_step = [&](int half) {   // steps 2 half, 2 half + 1 of T written (this warp's part)
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) arrive_cluster(e_step0 + 8u * (uint32_t)half);
        };
        auto arrive_wl = [&]() {
            fence_proxy_async_global();   // read next by TMA
            __syncwarp();
            if (lane == 0) {
                arrive_cluster(wl_rem);
                arrive_cluster(wl_loc);
            }
        };
        // byte offset of (this row, column 32 a + 4 c) in a K-major B / staging atom
        auto stage_off = [&](int a, int c) {
            return (uint32_t)a * C::kAtomBytes + (uint32_t)lrow * 128u + (((uint32_t)c ^ (uint32_t)(lrow & 7)) << 4);
        };

        // ---- kernel_2 prologue (walkthrough 2.4: k2 = softmax_row(Q_l K_l^T); 2.5: c)
        bool failed = !mbar_wait(pro_full, 0);
        failed = group_any(failed, 3, 256);
        float coeff = 0.f;
        if (!failed) {
            // split Q_l and K_l into tf32 hi + lo in place (fp32 accuracy from three tf32 products)
            // four independent chunks per step (2 * chunks is a multiple of 1024)
            const int chunks = nka * (int)(C::kAtomBytes / 16);   // 16-byte chunks per tile
#pragma unroll 1
            for (int e0 = et; e0 < 2 * chunks; e0 += 4 * 256) {
                uint32_t off[4];
                float4 x[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int e = e0 + 256 * u;
                    off[u] = (e < chunks ? C::kOffAhi : C::kOffBhi) + (uint32_t)(e % chunks) * 16u;
                    x[u] = *reinterpret_cast<const float4*>(bbuf + off[u]);
                }
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const float4 xh = make_float4(tf32_rna(x[u].x), tf32_rna(x[u].y), tf32_rna(x[u].z), tf32_rna(x[u].w));
                    *reinterpret_cast<float4*>(bbuf + off[u]) = xh;
                    *reinterpret_cast<float4*>(bbuf + off[u] + (C::kOffAlo - C::kOffAhi)) =
                        make_float4(x[u].x - xh.x, x[u].y - xh.y, x[u].z - xh.z, x[u].w - xh.w);
                }
            }
            fence_proxy_async_shared();
            arrive_e();
            const bool ok = mbar_wait(mma_done, 0);
            failed = group_any(!ok, 3, 256);
        }
        if (!failed) {
            tc_fence_after();
            // row max: this thread's 128 columns, then the other half's through shared memory
            // (the prologue's passes over the 128 columns take two atoms per TMEM wait)
            float mq[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll 1
            for (int jp = 0; jp < 2; ++jp) {
                uint32_t v[2][32];
                tmem_ld32(R1 + lane_base + 32 * (4 * h + 2 * jp), v[0]);
                tmem_ld32(R1 + lane_base + 32 * (4 * h + 2 * jp + 1), v[1]);
                tmem_ld_wait();
#pragma unroll
                for (int e = 0; e < 2; ++e)
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        mq[i & 3] = max3(mq[i & 3], __uint_as_float(v[e][2 * i]), __uint_as_float(v[e][2 * i + 1]));
            }
            rx[h * 128 + lrow] = fmaxf(fmaxf(mq[0], mq[1]), fmaxf(mq[2], mq[3]));
            named_barrier(3, 256);
            const float mx = fmaxf(rx[lrow], rx[128 + lrow]);
            // exponentials, kept in place in TMEM; their row sum
            float ssum = 0.f;
#pragma unroll 1
            for (int jp = 0; jp < 2; ++jp) {
                uint32_t v[2][32];
                const uint32_t addr = R1 + lane_base + 32 * (4 * h + 2 * jp);
                tmem_ld32(addr, v[0]);
                tmem_ld32(addr + 32, v[1]);
                tmem_ld_wait();
#pragma unroll
                for (int e2 = 0; e2 < 2; ++e2) {
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const float e = __expf(__uint_as_float(v[e2][i]) - mx);
                        ssum += e;
                        v[e2][i] = __float_as_uint(e);
                    }
                    tmem_st32(addr + 32 * e2, v[e2]);
                }
            }
            tmem_st_wait();
            sx[h * 128 + lrow] = ssum;
            named_barrier(3, 256);
            const float inv = 1.f / (sx[lrow] + sx[128 + lrow]);
            // k2 = e / sum: into TMEM as W_0 (R0) and into the B buffer as the first P1's right
            // factor (this CTA's rows are its own B lines)
            float rsum = 0.f;
#pragma unroll 1
            for (int jp = 0; jp < 2; ++jp) {
                uint32_t vv[2][32];
                tmem_ld32(R1 + lane_base + 32 * (4 * h + 2 * jp), vv[0]);
                tmem_ld32(R1 + lane_base + 32 * (4 * h + 2 * jp + 1), vv[1]);
                tmem_ld_wait();
#pragma unroll
                for (int e2 = 0; e2 < 2; ++e2) {
                    const int a = 4 * h + 2 * jp + e2;
                    uint32_t* v = vv[e2];
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const float pv = __uint_as_float(v[i]) * inv;
                        rsum += pv;
                        const float pr = tf32_rna(pv);
                        v[i] = __float_as_uint(pr);
                    }
                    tmem_st32(R0 + lane_base + 32 * a, vv[e2]);
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        const uint4 w4 = make_uint4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
                        *reinterpret_cast<uint4*>(bbuf + stage_off(a, c)) = w4;
                        // the resident copy of k2's first K atoms (this CTA's B lines), for the later P1s
                        if (a < C::kK2Resident) *reinterpret_cast<uint4*>(sm + C::kOffK2r + stage_off(a, c)) = w4;
                    }
                }
            }
            rx[h * 128 + lrow] = rsum;   // rx is free: every thread read its row max before the last barrier
            fence_proxy_async_shared();   // the staged k2 rows feed the MMA and a TMA store
            named_barrier(3, 256);
            if (n_iter > 0) {
                // W_0 in TMEM and k2's lines in the B buffer are all that the first P1 reads (the
                // coefficient only scales its epilogue): it runs beside the column sums below
                tmem_st_wait();
                arrive_e();
                // the rows of k2 go to global memory for the later P1s. The copy has read the B
                // buffer before this CTA arrives on the peer's cs_ready and before the barrier that
                // follows this CTA's own cs_ready wait, so before either CTA's P1 epilogue writes -X
                // lines into it.
                if (et == 0) {
                    for (int a = 0; a < 8; ++a) tma_store_3d(&maps.k2, bbuf + a * C::kAtomBytes, 32 * a, r0, bh);
                    tma_store_commit();
                }
            }
            // column sums over this CTA's rows, max row sum of this CTA. Warp w sums K atom w:
            // lane (c, rq) = (lane % 8, lane / 8) adds the 16-byte chunk of columns 32 w + 4 c .. + 3
            // over rows rq, rq + 4, ... (a warp load covers four whole rows), then the four row
            // quarters are added across lanes
            {
                const int c = lane & 7, rq = lane >> 3;
                float4 s0 = make_float4(0.f, 0.f, 0.f, 0.f), s1 = s0;   // two independent chains
#pragma unroll 8
                for (int i = 0; i < 32; i += 2) {
                    const int l0 = rq + 4 * i, l1 = l0 + 4;
                    const float4 x0 = *reinterpret_cast<const float4*>(
                        bbuf + (uint32_t)warp * C::kAtomBytes + (uint32_t)l0 * 128u + (((uint32_t)c ^ (uint32_t)(l0 & 7)) << 4));
                    const float4 x1 = *reinterpret_cast<const float4*>(
                        bbuf + (uint32_t)warp * C::kAtomBytes + (uint32_t)l1 * 128u + (((uint32_t)c ^ (uint32_t)(l1 & 7)) << 4));
                    s0.x += x0.x; s0.y += x0.y; s0.z += x0.z; s0.w += x0.w;
                    s1.x += x1.x; s1.y += x1.y; s1.z += x1.z; s1.w += x1.w;
                }
                float4 cs = make_float4(s0.x + s1.x, s0.y + s1.y, s0.z + s1.z, s0.w + s1.w);
#pragma unroll
                for (int o = 8; o <= 16; o <<= 1) {
                    cs.x += __shfl_xor_sync(0xffffffffu, cs.x, o);
                    cs.y += __shfl_xor_sync(0xffffffffu, cs.y, o);
                    cs.z += __shfl_xor_sync(0xffffffffu, cs.z, o);
                    cs.w += __shfl_xor_sync(0xffffffffu, cs.w, o);
                }
                if (rq == 0) {
                    const int col = 32 * warp + 4 * c;
                    *reinterpret_cast<float4*>(cs_own + col) = cs;
                    const uint32_t pa = mapa(smem_u32(cs_peer + col), rank ^ 1u);
                    st_remote(pa, cs.x);
                    st_remote(pa + 4, cs.y);
                    st_remote(pa + 8, cs.z);
                    st_remote(pa + 12, cs.w);
                }
                const float rs = warp_max(et < 128 ? rx[et] + rx[128 + et] : 0.f);
                if (lane == 0) wmax[warp] = rs;
            }
            named_barrier(3, 256);
            if (et == 0) {
                const float rm = fmaxf(fmaxf(wmax[0], wmax[1]), fmaxf(wmax[2], wmax[3]));
                rmax[0] = rm;
                st_remote(mapa(smem_u32(rmax + 1), rank ^ 1u), rm);
            }
            if (et == 0 && n_iter > 0) tma_store_wait_read<0>();   // k2's copy has read the B buffer
            __syncwarp();
            if (lane == 0) arrive_cluster(mapa(smem_u32(cs_ready), rank ^ 1u));
            const bool ok = wait_acq_cluster(cs_ready, 0);
            failed = group_any(!ok, 3, 256);
            if (!failed) {
                const float tot = warp_max(cs_own[et] + cs_peer[et]);
                if (lane == 0) wmax[warp] = tot;
                named_barrier(3, 256);
                float mc = wmax[0];
#pragma unroll
                for (int w = 1; w < 8; ++w) mc = fmaxf(mc, wmax[w]);
                // the exact-coefficient option drops the row factor (softmax rows sum to 1)
                coeff = 1.f / (mc * (prm.inv_init == NYS_INV_INIT_EXACT ? 1.f : fmaxf(rmax[0], rmax[1])));
            }
            if (n_iter == 0 && !failed) {
                // Z = c k2^T, from the staged rows
                float* zc = prm.z_out + (size_t)bh * M * M + row;
#pragma unroll 1
                for (int jj = 0; jj < 4; ++jj) {
                    const int a = 4 * h + jj;
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        const float4 f4 = *reinterpret_cast<const float4*>(bbuf + stage_off(a, c));
                        zc[(size_t)(32 * a + 4 * c) * M] = coeff * f4.x;
                        zc[(size_t)(32 * a + 4 * c + 1) * M] = coeff * f4.y;
                        zc[(size_t)(32 * a + 4 * c + 2) * M] = coeff * f4.z;
                        zc[(size_t)(32 * a + 4 * c + 3) * M] = coeff * f4.w;
                    }
                }
            }
        }

        // ---- the iteration
        uint32_t nd = 1, n4 = 0;   // mma_done / mma4_done phases waited
        for (int it = 0; it < n_iter && !failed; ++it) {
            const float sigma = it == 0 ? coeff : (it == 1 ? 0.25f * coeff : 0.25f);
            const float lambda = it == 0 ? 0.25f * coeff : 0.25f;
            const bool last_it = it + 1 == n_iter;
            for (int p = 0; p < 4 && !failed; ++p) {
                const bool ok = p == 3 ? mbar_wait(mma4_done, (n4++) & 1u) : mbar_wait(mma_done, (nd++) & 1u);
                failed = group_any(!ok, 3, 256);
                if (failed) break;
                tc_fence_after();
                const uint32_t d_col = (p == 0 || p == 2) ? R1 : R0;
                if (p == 1 || p == 2) {
                    // the accumulator holds -U (-V): T3 = 15I - U (T5 = 13I - V) differs from it on
                    // the diagonal only, which lies in atom diag_atom of this CTA's own column half
                    if (diag_half) {
                        uint32_t v[32];
                        const uint32_t addr = d_col + lane_base + 32 * diag_atom;
                        tmem_ld32(addr, v);
                        tmem_ld_wait();
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            if (i == lane) v[i] = __float_as_uint(__uint_as_float(v[i]) + (p == 1 ? 15.f : 13.f));
                        tmem_st32(addr, v);
                    }
                    arrive_step(0);   // P3 / P4 may start on every atom
                    arrive_step(1);
                    continue;
                }
#pragma unroll 1
                for (int jj = 0; jj < 4; ++jj) {
                    const int a = 4 * h + jj;   // 32-column atom
                    uint32_t v[32];
                    tmem_ld32(d_col + lane_base + 32 * a, v);
                    tmem_ld_wait();
                    if (p == 3) {
                        // W_next = lambda D: its transpose, row-major (row g = column g of W), is both
                        // the next P4's right factor and, transposed back, the result Z = W^T
                        float* dst = last_it ? prm.z_out : prm.wt;
                        float* col = dst + (size_t)bh * M * M + (size_t)(32 * a) * M + row;
#pragma unroll
                        for (int i = 0; i < 32; ++i) {
                            const float w = lambda * __uint_as_float(v[i]);
                            col[(size_t)i * M] = last_it ? w : tf32_rna(w);
                        }
                        continue;
                    }
                    // p == 0: -X = -sigma D is the right factor of P2 and P3 as K-major lines:
                    // column g = 32 a + i of X is line 32 (a % 4) + i of CTA a / 4 (= h), and this
                    // thread's row is K position `row` of every line
                    float e[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i) e[i] = tf32_rna(-sigma * __uint_as_float(v[i]));
                    const uint32_t base = x_dst + k_off + (uint32_t)(a & 3) * 4096u;
                    if (x_local) {
#pragma unroll
                        for (int i = 0; i < 32; ++i) st_local(base + i * 128 + ((xl ^ (uint32_t)(i & 7)) << 4), e[i]);
                    } else {
#pragma unroll
                        for (int i = 0; i < 32; ++i) st_remote(base + i * 128 + ((xl ^ (uint32_t)(i & 7)) << 4), e[i]);
                    }
                    // T1 = 7I - X, back into TMEM as P2's left factor
                    if (diag_half && a == diag_atom) {
#pragma unroll
                        for (int i = 0; i < 32; ++i) e[i] += i == lane ? 7.f : 0.f;
                    }
#pragma unroll
                    for (int i = 0; i < 32; ++i) v[i] = __float_as_uint(tf32_rna(e[i]));
                    tmem_st32(d_col + lane_base + 32 * a, v);
                }
                if (p == 3) {
                    if (!last_it) arrive_wl();
                } else if (p == 0) {
                    tmem_st_wait();
                    fence_proxy_async_cluster();   // X lines (here and in the peer) feed the MMA
                    arrive_e();
                    if (it == 0) {
                        // k2's rows, the first P4's right factor (by rows, MN-major), are in global
                        // memory: the producer may stream them once P3 frees the B buffer
                        if (et == 0) tma_store_wait_all<0>();
                        arrive_wl();
                    }
                }
            }
        }
        // k2's bulk copy (waited for above unless a wait ran out) has completed before the shared
        // memory is released
        if (et == 0) tma_store_wait_all<0>();
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync_all();   // no arrive, remote store or MMA of either CTA is still pending
    if (warp == 9) {
        tc_fence_after();
        tmem_dealloc2(tmem, 512);
    }
    cluster_sync_all();
}

}  // namespace nys
