// tc_output.cuh -- bf16 output pass on the 5th-generation tensor cores.
//
// Walkthrough (blog.gitcode.com) 2.4 and 2.6:
//   out = softmax_row(Qs K_l^T) W + dwconv65(V),   W = Z (kernel_3 V)
// per 128-query tile of one (batch, head):
//   S      = Q_tile . K_l^T          tcgen05 bf16 MMA, fp32 accumulator in TMEM
//   P      = exp(s (S - rowmax))     thread-per-row softmax read from TMEM, bf16 P
//                                    written back into the S columns of TMEM
//   O_att  = P . W                   MMA with A = P straight from TMEM
//   O_conv = T . V_halo              the 65-tap conv as a 128 x 192 banded Toeplitz
//                                    matrix T times the 192 V rows around the tile
//                                    (zero outside [0, n), supplied by the TMA
//                                    out-of-bounds fill). T's three 64-column blocks
//                                    are windows of one 256 x 64 strip R,
//                                    R[u][j] = w[j - u + 128], built once per head:
//                                    block b is rows 128 - 64 b .. 255 - 64 b of R
//   out    = O_att / rowsum(P) + O_conv, bf16, TMA store
//
// Warp roles (480 threads, one persistent CTA per SM over a contiguous range of
// tiles): warp 0 TMA producer of Q and the per-head constants, and TMEM
// allocator, warp 1 MMA issuer, warps 2-5 and 6-9 two softmax warpgroups,
// warps 10-13 epilogue (and the Toeplitz build), warp 14 TMA producer of the
// V halos. A warp w reaches TMEM lanes 32 (w % 4) .. +31, so each group of four
// warps covers all 128 rows. Two TMEM slots alternate between consecutive
// tiles. Both softmax groups work on every tile, group g on the landmark
// columns [g M/2, (g+1) M/2) of each row, and exchange the row max through
// shared memory: a tile's softmax takes half as long on the chain that
// reuses its slot (S MMA, softmax, O MMAs, epilogue read), and each SM
// sub-partition runs one warp of each group on it. Each group writes its P,
// packed, over the first half of its own columns, where the P.W MMA reads its
// A operand. Every wait is bounded.
#pragma once

#include "sm100.cuh"

namespace nys {

template <int D, int M>
struct OutTc {
    static constexpr int kRows = 128;
    static constexpr int kHalo = 192;                 // 32 + 128 + 32 V rows per tile
    static constexpr int kSpan = D * 2;               // row pitch of Q/V/out tiles (bytes)
    static constexpr uint32_t kLayout = D == 64 ? sm100::kLayoutSw128 : sm100::kLayoutSw64;
    static constexpr uint32_t kSbo = 8 * kSpan;       // 8-row group stride
    static constexpr int kStages = 2;
    static constexpr uint32_t kQBytes = kRows * kSpan;
    static constexpr uint32_t kVBytes = kHalo * kSpan;
    static constexpr uint32_t kKlBytes = M * kSpan;
    static constexpr uint32_t kWtBlock = D * 128;     // [D][64] bf16 K-block of W^T
    static constexpr uint32_t kWtBytes = (M / 64) * kWtBlock;
    static constexpr uint32_t kWtLoadBytes = kWtBytes;
    static constexpr uint32_t kTBytes = 256 * 128;    // the [256][64] bf16 strip R
    static constexpr uint32_t kOutBytes = kRows * kSpan;
    // TMEM slot (256 columns): S in [0, M). Softmax group g reads S's columns [g M/2, (g+1) M/2)
    // and writes its P (bf16 pairs) over the first half of that range, columns it has already
    // read. For M = 256 the O accumulators take the second halves of the two ranges (read by
    // then); for M <= 128 they sit after S.
    static constexpr int kSlot = 256;
    static constexpr int kTmemCols = 2 * kSlot;
    static constexpr int kHalfCols = M / 2;           // S columns per softmax group
    static constexpr int kColOatt = M == 256 ? 64 : M;
    static constexpr int kColOconv = M == 256 ? 192 : M + D;
    static_assert(kColOconv + D <= kSlot && (M != 256 || kColOatt + D <= 128), "TMEM slot layout");
    // TMEM column of the packed P pair holding landmark `c` (even)
    __host__ __device__ static constexpr int p_col(int c) {
        return c < kHalfCols ? c / 2 : kHalfCols + (c - kHalfCols) / 2;
    }
    static constexpr uint32_t kOffQ = 0;
    static constexpr uint32_t kOffV = kOffQ + kStages * kQBytes;
    static constexpr uint32_t kOffKl = kOffV + kStages * kVBytes;
    static constexpr uint32_t kOffWt = kOffKl + kKlBytes;
    static constexpr uint32_t kOffT = kOffWt + kWtBytes;
    static constexpr uint32_t kOffOut = kOffT + kTBytes;
    static constexpr uint32_t kOffPsum = kOffOut + kOutBytes;   // [2 slots][2 groups][128] partial row sums
    static constexpr uint32_t kOffXch = kOffPsum + 2 * 2 * 128 * 4;   // [2 slots][2 groups][128] partial row maxima
    static constexpr uint32_t kOffBar = kOffXch + 2 * 2 * 128 * 4;
    static constexpr int kNumBars = 22;
    static constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;  // tmem base, abort flag
    static constexpr uint32_t kSmemBytes = kOffMisc + 16 + 1024;  // + alignment slack
    static_assert(kSmemBytes <= 232448, "shared memory budget");
    static_assert(kTmemCols <= 512, "TMEM budget");
    static constexpr uint32_t kIdS = sm100::make_idesc(128, M, sm100::kFmtBf16, sm100::kFmtBf16, 0, 0);
    static constexpr uint32_t kIdPW = sm100::make_idesc(128, D, sm100::kFmtBf16, sm100::kFmtBf16, 0, 0);
    static constexpr uint32_t kIdConv = sm100::make_idesc(128, D, sm100::kFmtBf16, sm100::kFmtBf16, 0, 1);
};

constexpr int kOutMaxCtas = 160;

struct OutTcParams {
    const float* conv_w;   // [H, 65] or null
    int H, n, tiles_per_head, total_tiles;
    // CTA b takes tiles tile_start[b] .. tile_start[b + 1] - 1 (contiguous, in order)
    int tile_start[kOutMaxCtas + 1];
};

template <int D, int M>
__global__ void __launch_bounds__(480, 1)
output_tc_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_v,
                 const __grid_constant__ CUtensorMap map_out, const __grid_constant__ CUtensorMap map_kl,
                 const __grid_constant__ CUtensorMap map_wt, const OutTcParams prm) {
    using C = OutTc<D, M>;
    using namespace sm100;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(sm);
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + C::kOffBar);
    uint64_t* q_full = bars + 0;     // [2] Q tile landed
    uint64_t* q_empty = bars + 2;    // [2] Q stage reusable (its S MMA completed)
    uint64_t* s_full = bars + 4;     // [2] S in TMEM
    uint64_t* p_full = bars + 6;     // [2] P in TMEM, S fully read (256 arrivals)
    uint64_t* o_full = bars + 8;     // [2] O_att, O_conv ready
    uint64_t* slot_free = bars + 10; // [2] epilogue done with the slot (128 arrivals)
    uint64_t* const_full = bars + 12;
    uint64_t* const_empty = bars + 13;
    uint64_t* mma_done = bars + 14;
    uint64_t* t_full = bars + 15;    // Toeplitz matrix built (128 arrivals)
    uint64_t* v_full = bars + 16;    // [2] V halo landed
    uint64_t* v_empty = bars + 18;   // [2] V stage reusable (its conv MMA completed)
    // [2] the second softmax group has loaded the last S columns that O_conv overlaps (m = 256)
    uint64_t* conv_free = bars + 20;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + C::kOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + C::kOffMisc + 4);
    float* psum = reinterpret_cast<float*>(sm + C::kOffPsum);
    float* pmax = reinterpret_cast<float*>(sm + C::kOffXch);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // contiguous tile range of this CTA
    const int t0 = prm.tile_start[blockIdx.x];
    const int count = prm.tile_start[blockIdx.x + 1] - t0;
    const int tph = prm.tiles_per_head;
    auto head_start = [&](int i) { return i == 0 || ((t0 + i) % tph) == 0; };

    if (threadIdx.x == 0) {
        for (int b = 0; b < 2; ++b) {
            mbar_init(&q_full[b], 1);
            mbar_init(&q_empty[b], 1);
            mbar_init(&s_full[b], 1);
            mbar_init(&p_full[b], 256);
            mbar_init(&o_full[b], 1);
            mbar_init(&slot_free[b], 128);
            mbar_init(&v_full[b], 1);
            mbar_init(&v_empty[b], 1);
            mbar_init(&conv_free[b], 128);
        }
        mbar_init(const_full, 1);
        mbar_init(t_full, 128);
        mbar_init(const_empty, 1);
        mbar_init(mma_done, 32);   // one commit per lane of the MMA warp
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&map_q);
        prefetch_tmap(&map_v);
        prefetch_tmap(&map_out);
        prefetch_tmap(&map_kl);
        prefetch_tmap(&map_wt);
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer: Q tiles and the per-head
        // constants; each Q tile is requested as soon as its stage's S MMA is done.
        if (lane == 0) {
            uint32_t ce_phase = 0;
            int last_use[2] = {-1, -1};
            int const_loads = 0;
            for (int i = 0; i < count && !*abort_flag; ++i) {
                const int t = t0 + i, bh = t / tph, row0 = (t % tph) * C::kRows;
                if (head_start(i)) {
                    if (i > 0) {
                        if (!mbar_wait(const_empty, ce_phase)) { *abort_flag = 1; break; }
                        ce_phase ^= 1;
                    } else {
                        // W^T comes from the kernel launched just before this one, and this kernel
                        // may start before that one ends (programmatic dependent launch): the set-up,
                        // the Toeplitz build and the V loads go ahead, the constants wait here
                        griddep_wait();
                    }
                    mbar_arrive_expect_tx(const_full, C::kKlBytes + C::kWtLoadBytes);
                    tma_load_3d(sm + C::kOffKl, &map_kl, const_full, 0, 0, bh);
                    for (int kb = 0; kb < M / 64; ++kb)
                        tma_load_3d(sm + C::kOffWt + kb * C::kWtBlock, &map_wt, const_full, kb * 64, 0, bh);
                    ++const_loads;
                }
                const int st = i % C::kStages, use = i / C::kStages;
                if (!mbar_wait(&q_empty[st], (use & 1) ^ 1)) { *abort_flag = 1; break; }
                mbar_arrive_expect_tx(&q_full[st], C::kQBytes);
                tma_load_3d(sm + C::kOffQ + st * C::kQBytes, &map_q, &q_full[st], 0, row0, bh);
                last_use[st] = use;
            }
            if (*abort_flag) {
                // let every copy already issued land before the CTA exits
                for (int st = 0; st < 2; ++st)
                    if (last_use[st] >= 0) mbar_wait(&q_full[st], last_use[st] & 1);
                if (const_loads > 0) mbar_wait(const_full, (const_loads - 1) & 1);
            }
        }
    } else if (warp == 14) {
        // ------------------------------------------------ TMA producer of the V halos (its own warp,
        // so that its loads are never held back behind the Q producer's waits)
        if (lane == 0 && prm.conv_w != nullptr) {
            int last_use[2] = {-1, -1};
            for (int i = 0; i < count && !*abort_flag; ++i) {
                const int t = t0 + i, bh = t / tph, row0 = (t % tph) * C::kRows;
                const int st = i % C::kStages, use = i / C::kStages;
                if (!mbar_wait(&v_empty[st], (use & 1) ^ 1)) { *abort_flag = 1; break; }
                mbar_arrive_expect_tx(&v_full[st], C::kVBytes);
                tma_load_3d(sm + C::kOffV + st * C::kVBytes, &map_v, &v_full[st], 0, row0 - 32, bh);
                last_use[st] = use;
            }
            if (*abort_flag)
                for (int st = 0; st < 2; ++st)
                    if (last_use[st] >= 0) mbar_wait(&v_full[st], last_use[st] & 1);
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer: the whole warp runs the loop and
        // the waits; one elected lane issues each MMA group and each commit
        uint32_t cf_phase = 0;
        bool ok = true;
        // operand descriptors: each buffer's is built once, and a K step or a stage advances its
        // start-address field (this warp's instructions are on every tile's critical path)
        const uint64_t dQ = smem_desc(sbase + C::kOffQ, 16, C::kSbo, C::kLayout);
        const uint64_t dKl = smem_desc(sbase + C::kOffKl, 16, C::kSbo, C::kLayout);
        const uint64_t dWt = smem_desc(sbase + C::kOffWt, 16, 1024, kLayoutSw128);
        const uint64_t dT = smem_desc(sbase + C::kOffT, 16, 1024, kLayoutSw128);
        const uint64_t dV = smem_desc(sbase + C::kOffV, C::kVBytes, C::kSbo, C::kLayout);
        auto descQ = [&](int st, int k) { return desc_advance(dQ, st * C::kQBytes + k * 32); };
        auto descKl = [&](int k) { return desc_advance(dKl, k * 32); };
        auto descWt = [&](int k) { return desc_advance(dWt, (k >> 2) * C::kWtBlock + (k & 3) * 32); };
        auto descT = [&](int k) {   // K step k of T: block k / 4 is the strip window from row 128 - 64 (k / 4)
            return desc_advance(dT, (128 - 64 * (k >> 2)) * 128 + (k & 3) * 32);
        };
        auto descV = [&](int st, int k) { return desc_advance(dV, st * C::kVBytes + k * 16 * C::kSpan); };
        auto wait = [&](uint64_t* bar, uint32_t parity) { return warp_all(mbar_wait(bar, parity)); };
        auto issue_S = [&](int j) -> bool {
            const int s = j & 1, st = j % C::kStages;
            if (!wait(&slot_free[s], ((j >> 1) & 1) ^ 1)) return false;
            if (!wait(&q_full[st], (j / C::kStages) & 1)) return false;
            tc_fence_after();
            const uint32_t slot = tmem + s * C::kSlot;
            if (elect_one()) {
#pragma unroll
                for (int k = 0; k < D / 16; ++k) mma_bf16_ss(slot, descQ(st, k), descKl(k), C::kIdS, k > 0);
            }
            if (elect_one()) {
                mma_commit(&s_full[s]);
                mma_commit(&q_empty[st]);
            }
            return true;
        };
        auto issue_O = [&](int j) -> bool {
            const int s = j & 1, st = j % C::kStages;
            const uint32_t slot = tmem + s * C::kSlot;
            // the conv product first: it does not need P, so it runs while the softmax finishes.
            // At m = 256 O_conv shares TMEM columns with the last 64 S columns of the second
            // softmax group, which that group has loaded by the time it arrives on conv_free
            if (prm.conv_w != nullptr) {
                if (M == 256 && !wait(&conv_free[s], (j >> 1) & 1)) return false;
                if (!wait(&v_full[st], (j / C::kStages) & 1)) return false;
                tc_fence_after();
                if (elect_one()) {
#pragma unroll
                    for (int k = 0; k < 12; ++k)
                        mma_bf16_ss(slot + C::kColOconv, descT(k), descV(st, k), C::kIdConv, k > 0);
                }
                if (elect_one()) mma_commit(&v_empty[st]);
            }
            if (!wait(&p_full[s], (j >> 1) & 1)) return false;
            tc_fence_after();
            if (elect_one()) {
#pragma unroll
                for (int k = 0; k < M / 16; ++k)   // landmarks 16k .. 16k+15: 8 packed P columns
                    mma_bf16_ts(slot + C::kColOatt, slot + C::p_col(16 * k), descWt(k), C::kIdPW, k > 0);
            }
            if (elect_one()) mma_commit(&o_full[s]);
            return true;
        };
        if (count > 0) {
            ok = wait(const_full, cf_phase) && wait(t_full, cf_phase);
            cf_phase ^= 1;
            tc_fence_after();
            if (ok) ok = issue_S(0);
        }
        for (int i = 0; i < count && ok && !warp_any(*abort_flag != 0); ++i) {
            const bool has_next = i + 1 < count;
            const bool next_new_head = has_next && head_start(i + 1);
            if (has_next && !next_new_head) ok = issue_S(i + 1);
            if (ok) ok = issue_O(i);
            if (ok && next_new_head) {
                if (elect_one()) mma_commit(const_empty);
                ok = wait(const_full, cf_phase) && wait(t_full, cf_phase);
                cf_phase ^= 1;
                tc_fence_after();
                if (ok) ok = issue_S(i + 1);
            }
        }
        if (!ok) *abort_flag = 1;
        // every MMA issued has completed before TMEM can be released: one commit per lane
        // (mma_done counts 32 arrivals), so the drain covers whichever lane issued
        mma_commit(mma_done);
        mbar_wait(mma_done, 0);
    } else if (warp >= 2 && warp < 10) {
        // ------------------------------------------------ softmax: both groups take every tile, group g
        // the landmark columns [g M/2, (g+1) M/2) of each row (one row per thread); the row max is
        // exchanged through shared memory
        const int g = (warp - 2) >> 2;
        const int q4 = warp & 3;
        const int r = 32 * q4 + lane;
        const uint32_t lane_base = (uint32_t)(32 * q4) << 16;
        const float sc = split_scale(D) * kLog2e;  // S holds Q . K_l^T with K_l already scaled
        constexpr int kB = C::kHalfCols < 64 ? C::kHalfCols : 64;   // S columns per TMEM wait
        const int cbase = g * C::kHalfCols;
        // one named barrier per tile (the max exchange): a group can only reach tile i + 2's
        // exchange, which reuses tile i's maxima slots, after both groups left tile i + 1's
        for (int i = 0; i < count; ++i) {
            const int s = i & 1;
            const bool ok = warp_all(mbar_wait(&s_full[s], (i >> 1) & 1));
            tc_fence_after();
            const uint32_t slot = tmem + s * C::kSlot + lane_base;
            // pass 1: this half-row's max, kB columns per wait
            float mq[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};   // four short max chains
            if (ok) {
#pragma unroll 1
                for (int c0 = cbase; c0 < cbase + C::kHalfCols; c0 += kB) {
                    uint32_t v[kB / 32][32];
#pragma unroll
                    for (int bq = 0; bq < kB / 32; ++bq) tmem_ld32(slot + c0 + bq * 32, v[bq]);
                    tmem_ld_wait();
#pragma unroll
                    for (int bq = 0; bq < kB / 32; ++bq)
#pragma unroll
                        for (int j = 0; j < 16; ++j)
                            mq[j & 3] = max3(mq[j & 3], __uint_as_float(v[bq][2 * j]), __uint_as_float(v[bq][2 * j + 1]));
                }
            }
            pmax[(s * 2 + g) * 128 + r] = fmaxf(fmaxf(mq[0], mq[1]), fmaxf(mq[2], mq[3]));
            // also publishes the maxima; a wait that ran out in either group, or an abort by another
            // role, stops both groups together
            if (group_any(!ok || *abort_flag != 0, 3, 256)) { *abort_flag = 1; break; }
            const float mo = fmaxf(pmax[(s * 2) * 128 + r], pmax[(s * 2 + 1) * 128 + r]) * sc;
            // pass 2: P over the first half of this group's columns, in increasing column order, so
            // it only overwrites scores this thread has already read.
            // exponentials on packed fp32 pairs: the MUFU unit takes 10 of every 16 pairs, the FMA
            // pipe the other 6 (polynomial 2^x), so neither pipe alone bounds the loop. P is rounded
            // to bf16 (nearest even); the row sum adds the fp32 values.
            // 32 columns per TMEM load, two register buffers: the load of the next 32 scores is in
            // flight while the current 32 are exponentiated (tcgen05.wait::ld then waits for it alone)
            const uint64_t sc2 = f2(sc, sc), nmo2 = f2(-mo, -mo);
            uint64_t acc[2] = {f2(0.f, 0.f), f2(0.f, 0.f)};
            constexpr int kChunks = C::kHalfCols / 32;
            uint32_t vb[2][32];
            tmem_ld32(slot + cbase, vb[0]);
            tmem_ld_wait();
#pragma unroll
            for (int cc = 0; cc < kChunks; ++cc) {
                if (cc + 1 < kChunks) tmem_ld32(slot + cbase + 32 * (cc + 1), vb[(cc + 1) & 1]);
                const uint32_t* v = vb[cc & 1];
                uint32_t pk[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const uint64_t x2 = f2_fma(f2(__uint_as_float(v[2 * j]), __uint_as_float(v[2 * j + 1])), sc2, nmo2);
                    float e0, e1;
                    if ((j & 7) == 2 || (j & 7) == 5 || (j & 7) == 7) {
                        exp2_poly_pair(x2, e0, e1);
                    } else {
                        float x0, x1;
                        f2_split(x2, x0, x1);
                        e0 = ex2(x0);
                        e1 = ex2(x1);
                    }
                    pk[j] = pack_bf16_rn(e0, e1);
                    acc[j & 1] = f2_add(acc[j & 1], f2(e0, e1));
                }
                // P of these 32 columns lands on scores this thread has already read (and waited for)
                tmem_st16(slot + C::p_col(cbase + 32 * cc), pk);
                if (cc + 1 < kChunks) tmem_ld_wait();
                if (M == 256 && g == 1 && cc == kChunks - 2) {
                    // every S column of this group is in registers: O_conv may overwrite the last 64
                    tc_fence_before();
                    mbar_arrive(&conv_free[s]);
                }
            }
            tmem_st_wait();
            {
                float a0, a1, b0, b1;
                f2_split(acc[0], a0, a1);
                f2_split(acc[1], b0, b1);
                psum[(s * 2 + g) * 128 + r] = (a0 + a1) + (b0 + b1);
            }
            tc_fence_before();
            mbar_arrive(&p_full[s]);
        }
    } else if (warp >= 10) {
        // ------------------------------------------------ epilogue warpgroup (+ Toeplitz build)
        const int q4 = warp & 3;
        const int r = 32 * q4 + lane;
        const uint32_t lane_base = (uint32_t)(32 * q4) << 16;
        const bool conv = prm.conv_w != nullptr;
        const bool leader = (warp == 10 && lane == 0);
        uint32_t ce_phase = 0;
        for (int i = 0; i < count; ++i) {
            if (group_any(*abort_flag != 0, 2, 128)) break;
            const int t = t0 + i, bh = t / tph, row0 = (t % tph) * C::kRows;
            if (head_start(i)) {
                if (i > 0) {
                    const bool ok = mbar_wait(const_empty, ce_phase);
                    if (group_any(!ok, 2, 128)) { *abort_flag = 1; break; }
                    ce_phase ^= 1;
                }
                if (conv) {
                    // R[u][j] = w[j - u + 128] for 0 <= j - u + 128 < 65: rows r and r + 128
                    const float* wh = prm.conv_w + (size_t)(bh % prm.H) * kTaps;
#pragma unroll 1
                    for (int hh = 0; hh < 2; ++hh) {
                        const int u = r + 128 * hh;
#pragma unroll 1
                        for (int ch = 0; ch < 8; ++ch) {
                            uint32_t pk[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const int d0 = ch * 8 + 2 * e - u + 128, d1 = d0 + 1;
                                const float w0 = (d0 >= 0 && d0 < kTaps) ? __ldg(wh + d0) : 0.f;
                                const float w1 = (d1 >= 0 && d1 < kTaps) ? __ldg(wh + d1) : 0.f;
                                pk[e] = pack_bf16(w0, w1);
                            }
                            *reinterpret_cast<uint4*>(sm + C::kOffT + swz<128>(u, ch)) =
                                make_uint4(pk[0], pk[1], pk[2], pk[3]);
                        }
                    }
                    fence_proxy_async_shared();
                }
                mbar_arrive(t_full);
            }
            const int s = i & 1;
            const bool ok = mbar_wait(&p_full[s], (i >> 1) & 1) && mbar_wait(&o_full[s], (i >> 1) & 1);
            if (group_any(!ok, 2, 128)) {
                *abort_flag = 1;
                break;
            }
            tc_fence_after();
            const float li = 1.f / (psum[(s * 2) * 128 + r] + psum[(s * 2 + 1) * 128 + r]);
            const uint32_t slot = tmem + s * C::kSlot + lane_base;
            uint32_t outp[D / 2];
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t a[32], b[32];
                tmem_ld32(slot + C::kColOatt + c * 32, a);
                if (conv) tmem_ld32(slot + C::kColOconv + c * 32, b);
                tmem_ld_wait();
                if (c + 1 == D / 32) {
                    // every TMEM column of this tile has been read: the slot is released before the
                    // last 32 columns are combined
                    tc_fence_before();
                    mbar_arrive(&slot_free[s]);
                }
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const float x0 = __uint_as_float(a[2 * j]), x1 = __uint_as_float(a[2 * j + 1]);
                    const float o0 = conv ? fmaf(x0, li, __uint_as_float(b[2 * j])) : x0 * li;
                    const float o1 = conv ? fmaf(x1, li, __uint_as_float(b[2 * j + 1])) : x1 * li;
                    outp[c * 16 + j] = pack_bf16(o0, o1);
                }
            }
            if (leader) tma_store_wait_read<0>();
            named_barrier(1, 128);
            uint8_t* stage = sm + C::kOffOut;
#pragma unroll
            for (int ch = 0; ch < D / 8; ++ch)
                *reinterpret_cast<uint4*>(stage + swz<C::kSpan>(r, ch)) =
                    make_uint4(outp[4 * ch], outp[4 * ch + 1], outp[4 * ch + 2], outp[4 * ch + 3]);
            fence_proxy_async_shared();
            named_barrier(1, 128);
            if (leader) {
                tma_store_3d(&map_out, stage, 0, row0, bh);
                tma_store_commit();
            }
        }
        if (leader) tma_store_wait_all<0>();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

}  // namespace nys
