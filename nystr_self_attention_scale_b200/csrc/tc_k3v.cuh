// tc_k3v.cuh -- bf16 kernel_3 V pass on the 5th-generation tensor cores.
//
// Walkthrough (blog.gitcode.com) 2.4: k3 = softmax_row(Q_l Ks^T + mask), new_value = k3 V.
// A work item is (batch*head, 128-landmark block, key split). For each
// 128-key chunk of the split:
//   S = Q_l_block . K_chunk^T          tcgen05 bf16 MMA into TMEM (K unscaled;
//                                      the d^-1/4 of K is applied in the exponent)
//   online softmax per landmark row    one thread per row reads S from TMEM,
//                                      masks padded keys, writes bf16 P back
//                                      (exponentials split between the MUFU unit
//                                      and a polynomial on the FMA pipe)
//   O += P . V_chunk                   MMA with A = P from TMEM, V as an MN-major
//                                      operand (keys x d straight from the TMA tile),
//                                      accumulating in TMEM across the chunks
// The exponentials use a per-row reference max that only moves when a chunk's
// max exceeds it by more than 2^8 (log2 units); then O and the running sum are
// rescaled once. Every exponential of a row uses the same reference, so the
// result is the exact softmax; P stays below 256, well inside bf16 range.
// Each item writes the unnormalised partial (O, reference max, running sum) of
// its split; a deterministic combine over splits follows.
//
// Warp roles (640 threads): warp 0 TMA producer and TMEM allocator, warp 1 MMA
// issuer, warps 4-19 four softmax warpgroups that split every chunk's 128 keys
// (32 each), exchanging the chunk max through shared memory; four warps per
// SM sub-partition hide the TMEM and MUFU latencies. Each group writes its P
// into the first half of its own 32 S columns (the P.V MMA takes its A
// operand from the four ranges). S is double buffered in TMEM; K/V chunks use
// a 3-stage shared-memory ring.
#pragma once

#include "sm100.cuh"

namespace nys {

template <int D>
struct K3vTc {
    static constexpr int kRows = 128, kChunk = 128;
    static constexpr int kSpan = D * 2;
    static constexpr uint32_t kLayout = D == 64 ? sm100::kLayoutSw128 : sm100::kLayoutSw64;
    static constexpr uint32_t kSbo = 8 * kSpan;
    static constexpr int kStages = 3;
    static constexpr uint32_t kTileBytes = 128 * kSpan;
    static constexpr uint32_t kOffQl = 0;
    static constexpr uint32_t kOffK = kOffQl + kTileBytes;
    static constexpr uint32_t kOffV = kOffK + kStages * kTileBytes;
    static constexpr uint32_t kOffBar = kOffV + kStages * kTileBytes;
    static constexpr int kNumBars = 2 + 2 * kStages + 7 + 1;
    static constexpr int kGroups = 4;                                     // softmax warpgroups
    static constexpr int kSoftmaxThreads = kGroups * 128;
    static constexpr int kThreads = 128 + kSoftmaxThreads;               // warps 0-3 + the groups
    static constexpr uint32_t kOffXch = kOffBar + kNumBars * 8;          // [2][4][128] chunk maxima
    static constexpr uint32_t kOffLx = kOffXch + 2 * kGroups * 128 * 4;  // [4][128] partial sums
    static constexpr uint32_t kOffMisc = kOffLx + kGroups * 128 * 4;
    // at least 116 KB so that only one CTA (and one 512-column TMEM allocation) fits per SM
    static constexpr uint32_t kSmemNeed = kOffMisc + 16 + 1024;
    static constexpr uint32_t kSmemBytes = kSmemNeed > 118784 ? kSmemNeed : 118784;
    static constexpr int kTmemCols = 512;
    static constexpr int kColS = 0, kColO = 256;   // S[b] at 128 b; P halves at 128 b + {0, 64}
    static constexpr uint32_t kIdS = sm100::make_idesc(128, kChunk, sm100::kFmtBf16, sm100::kFmtBf16, 0, 0);
    static constexpr uint32_t kIdPV = sm100::make_idesc(128, D, sm100::kFmtBf16, sm100::kFmtBf16, 0, 1);
};

struct K3vTcParams {
    const uint32_t* mask_bits;  // [B, n / 32] key-validity bits, or null for no mask
    float* part_o;         // [BH, splits, m, d]
    float* part_m;         // [BH, splits, m]  running max (natural-log units)
    float* part_l;         // [BH, splits, m]  running sum
    int H, n, m, halves, splits, chunks_per_split, total_items;
};

template <int D>
__global__ void __launch_bounds__(640, 1)
k3v_tc_kernel(const __grid_constant__ CUtensorMap map_ql, const __grid_constant__ CUtensorMap map_k,
              const __grid_constant__ CUtensorMap map_v, const K3vTcParams prm) {
    using C = K3vTc<D>;
    using namespace sm100;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(sm);
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + C::kOffBar);
    uint64_t* ql_full = bars + 0;
    uint64_t* ql_empty = bars + 1;
    uint64_t* kv_full = bars + 2;                  // [kStages]
    uint64_t* kv_empty = bars + 2 + C::kStages;    // [kStages]
    uint64_t* s_full = bars + 2 + 2 * C::kStages;  // [2] S(j) in TMEM
    uint64_t* p_full = s_full + 2;                 // [2] P(j) in TMEM (128 arrivals)
    uint64_t* pv_done = s_full + 4;                // [2] P(j) V(j) accumulated into O
    uint64_t* o_free = s_full + 6;                 // the item's O has been read (128 arrivals)
    uint64_t* mma_done = s_full + 7;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + C::kOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + C::kOffMisc + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int per_bh = prm.halves * prm.splits;
    const int nchunk_total = prm.n / C::kChunk;
    auto item_chunks = [&](int item, int* first) {
        const int split = item % prm.splits;
        const int c0 = split * prm.chunks_per_split;
        *first = c0;
        return min(prm.chunks_per_split, nchunk_total - c0);
    };

    if (threadIdx.x == 0) {
        mbar_init(ql_full, 1);
        mbar_init(ql_empty, 1);
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(&kv_full[s], 1);
            mbar_init(&kv_empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&s_full[b], 1);
            mbar_init(&p_full[b], C::kSoftmaxThreads);
            mbar_init(&pv_done[b], 1);
        }
        mbar_init(o_free, C::kSoftmaxThreads);
        mbar_init(mma_done, 32);   // one commit per lane of the MMA warp
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&map_ql);
        prefetch_tmap(&map_k);
        prefetch_tmap(&map_v);
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
        if (lane == 0) {
            int g = 0, it = 0;
            int last_stage_use[C::kStages];
            for (int s = 0; s < C::kStages; ++s) last_stage_use[s] = -1;
            int ql_issued = -1;
            for (int item = blockIdx.x; item < prm.total_items && !*abort_flag; item += gridDim.x, ++it) {
                const int bh = item / per_bh, half = (item / prm.splits) % prm.halves;
                int c0;
                const int nch = item_chunks(item, &c0);
                if (!mbar_wait(ql_empty, (it & 1) ^ 1)) { *abort_flag = 1; break; }
                mbar_arrive_expect_tx(ql_full, C::kTileBytes);
                tma_load_3d(sm + C::kOffQl, &map_ql, ql_full, 0, half * C::kRows, bh);
                ql_issued = it;
                for (int c = 0; c < nch; ++c, ++g) {
                    const int st = g % C::kStages;
                    if (!mbar_wait(&kv_empty[st], ((g / C::kStages) & 1) ^ 1)) { *abort_flag = 1; break; }
                    mbar_arrive_expect_tx(&kv_full[st], 2 * C::kTileBytes);
                    const int key0 = (c0 + c) * C::kChunk;
                    tma_load_3d(sm + C::kOffK + st * C::kTileBytes, &map_k, &kv_full[st], 0, key0, bh);
                    tma_load_3d(sm + C::kOffV + st * C::kTileBytes, &map_v, &kv_full[st], 0, key0, bh);
                    last_stage_use[st] = g / C::kStages;
                }
            }
            if (*abort_flag) {
                for (int s = 0; s < C::kStages; ++s)
                    if (last_stage_use[s] >= 0) mbar_wait(&kv_full[s], last_stage_use[s] & 1);
                if (ql_issued >= 0) mbar_wait(ql_full, ql_issued & 1);
            }
        }
    } else if (warp == 1) {
        // MMA issuer: the whole warp runs the loop and the waits; one elected lane issues each
        // MMA group and each commit
        bool ok = true;
        int g = 0, it = 0;
        auto descQl = [&](int k) { return smem_desc(sbase + C::kOffQl + k * 32, 16, C::kSbo, C::kLayout); };
        auto descK = [&](int st, int k) {
            return smem_desc(sbase + C::kOffK + st * C::kTileBytes + k * 32, 16, C::kSbo, C::kLayout);
        };
        auto descV = [&](int st, int k) {
            return smem_desc(sbase + C::kOffV + st * C::kTileBytes + k * 16 * C::kSpan, C::kTileBytes, C::kSbo,
                             C::kLayout);
        };
        auto wait = [&](uint64_t* bar, uint32_t parity) { return warp_all(mbar_wait(bar, parity)); };
        auto issue_S = [&](int j) -> bool {
            const int b = j & 1, st = j % C::kStages;
            // S buffer b last held S(j - 2); P(j - 2) V was accumulated once PV(j - 2) completed
            if (j >= 2 && !wait(&pv_done[b], ((j - 2) >> 1) & 1)) return false;
            if (!wait(&kv_full[st], (j / C::kStages) & 1)) return false;
            tc_fence_after();
            if (elect_one()) {
#pragma unroll
                for (int k = 0; k < D / 16; ++k)
                    mma_bf16_ss(tmem + C::kColS + b * 128, descQl(k), descK(st, k), C::kIdS, k > 0);
            }
            if (elect_one()) mma_commit(&s_full[b]);
            return true;
        };
        auto issue_PV = [&](int j, bool first, int item_it) -> bool {
            const int b = j & 1, st = j % C::kStages;
            if (!wait(&p_full[b], (j >> 1) & 1)) return false;
            // the previous item's O must have been read before it is overwritten
            if (first && !wait(o_free, (item_it & 1) ^ 1)) return false;
            tc_fence_after();
            if (elect_one()) {
#pragma unroll
                for (int k = 0; k < C::kChunk / 16; ++k) {
                    // keys 16k .. 16k+15: P of group k / 2, at the start of its 32 S columns
                    const uint32_t pa = tmem + C::kColS + b * 128 + 32 * (k >> 1) + 8 * (k & 1);
                    mma_bf16_ts(tmem + C::kColO, pa, descV(st, k), C::kIdPV, (first && k == 0) ? 0u : 1u);
                }
            }
            if (elect_one()) {
                mma_commit(&pv_done[b]);
                mma_commit(&kv_empty[st]);
            }
            return true;
        };
        for (int item = blockIdx.x; item < prm.total_items && ok && !warp_any(*abort_flag != 0);
             item += gridDim.x, ++it) {
            int c0;
            const int nch = item_chunks(item, &c0);
            ok = wait(ql_full, it & 1);
            if (!ok) break;
            tc_fence_after();
            ok = issue_S(g);
            for (int c = 0; c < nch && ok; ++c) {
                const int j = g + c;
                if (c + 1 < nch) ok = issue_S(j + 1);
                else if (elect_one()) mma_commit(ql_empty);   // every S MMA of this item is issued
                if (ok) ok = issue_PV(j, c == 0, it);
            }
            g += nch;
        }
        if (!ok) *abort_flag = 1;
        // one commit per lane (mma_done counts 32 arrivals): the drain covers whichever lane issued
        mma_commit(mma_done);
        mbar_wait(mma_done, 0);
    } else if (warp >= 4) {
        const int grp = (warp - 4) >> 2;          // softmax group: keys [32 grp, 32 grp + 32) of a chunk
        const int q4 = warp & 3;
        const int r = 32 * q4 + lane;
        const uint32_t lane_base = (uint32_t)(32 * q4) << 16;
        const float sc = split_scale(D) * kLog2e;   // exponent scale of the raw S = Q_l . K^T
        constexpr float kSlack = 8.f;               // log2 units: P stays below 2^8
        constexpr int kT = C::kSoftmaxThreads;
        float* xch = reinterpret_cast<float*>(sm + C::kOffXch);   // [2 buffers][4 groups][128]
        float* lx = reinterpret_cast<float*>(sm + C::kOffLx);     // [4 groups][128]
        int g = 0, it = 0;
        for (int item = blockIdx.x; item < prm.total_items; item += gridDim.x, ++it) {
            if (group_any(*abort_flag != 0, 1, kT)) break;
            const int bh = item / per_bh, half = (item / prm.splits) % prm.halves;
            const int split = item % prm.splits;
            const int b_idx = bh / prm.H;
            int c0;
            const int nch = item_chunks(item, &c0);
            float m_ref = -INFINITY, l_run = 0.f;   // reference max (log2 units) and this group's sum
            bool ok = true;
            for (int c = 0; c < nch; ++c) {
                const int j = g + c, b = j & 1;
                const int key0 = (c0 + c) * C::kChunk;
                // key-validity bits of this group's 32 keys (bit k = key key0 + 32 grp + k)
                const uint32_t mb = prm.mask_bits != nullptr
                                        ? __ldg(prm.mask_bits + (size_t)b_idx * (prm.n / 32) + key0 / 32 + grp)
                                        : ~0u;
                const bool full = mb == ~0u;
                // a wait that runs out leaves S unread: the group still passes the chunk's one
                // barrier below (which also ORs the failure across the groups) and then stops
                ok = warp_all(mbar_wait(&s_full[b], (j >> 1) & 1));
                tc_fence_after();
                const uint32_t sbuf = tmem + lane_base + C::kColS + b * 128;
                uint32_t v[32];
                if (ok) {
                    tmem_ld32(sbuf + 32 * grp, v);
                    tmem_ld_wait();
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e) v[e] = 0u;
                }
                if (!full) {
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        if (!((mb >> e) & 1u)) v[e] = __float_as_uint(-INFINITY);
                }
                float mq[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};   // four short max chains
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    mq[e & 3] = max3(mq[e & 3], __uint_as_float(v[2 * e]), __uint_as_float(v[2 * e + 1]));
                xch[(b * 4 + grp) * 128 + r] = fmaxf(fmaxf(mq[0], mq[1]), fmaxf(mq[2], mq[3]));
                if (group_any(!ok, 1, kT)) { ok = false; break; }   // also publishes xch
                const float* xr = xch + b * 4 * 128 + r;
                const float cmax = fmaxf(fmaxf(xr[0], xr[128]), fmaxf(xr[256], xr[384]));
                const float cm = cmax * sc;
                // move the reference only when this chunk's max exceeds it by more than the slack
                // (every group takes the same decision: same maxima, same history)
                const bool move = cm > m_ref + kSlack;
                const float m_new = move ? cm : m_ref;
                const float alpha = move ? ex2(m_ref - m_new) : 1.f;   // m_ref = -inf gives 0
                if (grp < D / 32 && c > 0 && warp_any(move && m_ref != -INFINITY)) {
                    // rescale this warp's rows of O (group g: columns 32 g .. 32 g + 31) once
                    // P(j - 1) V has been accumulated
                    ok = warp_all(mbar_wait(&pv_done[(j - 1) & 1], ((j - 1) >> 1) & 1));
                    if (ok) {
                        tc_fence_after();
                        uint32_t o[32];
                        tmem_ld32(tmem + lane_base + C::kColO + grp * 32, o);
                        tmem_ld_wait();
#pragma unroll
                        for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                        tmem_st32(tmem + lane_base + C::kColO + grp * 32, o);
                    }
                }
                const float mo = m_new == -INFINITY ? 0.f : m_new;   // rows with every key padded so far: P = 0
                // exponentials on packed fp32 pairs: in chunks without padded keys the FMA pipe takes
                // 6 of every 16 pairs (polynomial 2^x) and the MUFU unit the rest; chunks with padded
                // keys use the MUFU unit only, so that padded keys get exactly 0. P is rounded to
                // bf16 (nearest even); the running sum adds the fp32 values.
                const uint64_t sc2 = f2(sc, sc), nmo2 = f2(-mo, -mo);
                uint64_t acc[2] = {f2(0.f, 0.f), f2(0.f, 0.f)};
                uint32_t pk[16];
                if (full) {
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const uint64_t x2 =
                            f2_fma(f2(__uint_as_float(v[2 * e]), __uint_as_float(v[2 * e + 1])), sc2, nmo2);
                        float e0, e1;
                        if ((e & 7) == 2 || (e & 7) == 5 || (e & 7) == 7) {
                            exp2_poly_pair(x2, e0, e1);
                        } else {
                            float x0, x1;
                            f2_split(x2, x0, x1);
                            e0 = ex2(x0);
                            e1 = ex2(x1);
                        }
                        pk[e] = pack_bf16_rn(e0, e1);
                        acc[e & 1] = f2_add(acc[e & 1], f2(e0, e1));
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const uint64_t x2 =
                            f2_fma(f2(__uint_as_float(v[2 * e]), __uint_as_float(v[2 * e + 1])), sc2, nmo2);
                        float x0, x1;
                        f2_split(x2, x0, x1);
                        const float e0 = ex2(x0), e1 = ex2(x1);
                        pk[e] = pack_bf16_rn(e0, e1);
                        acc[e & 1] = f2_add(acc[e & 1], f2(e0, e1));
                    }
                }
                // this group's P: 16 columns at the start of its own (already read) 32 S columns
                tmem_st16(sbuf + 32 * grp, pk);
                float sum;
                {
                    float a0, a1, b0, b1;
                    f2_split(acc[0], a0, a1);
                    f2_split(acc[1], b0, b1);
                    sum = (a0 + a1) + (b0 + b1);
                }
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(&p_full[b]);
                l_run = fmaf(l_run, alpha, sum);
                m_ref = m_new;
            }
            // the item's O is complete once its last P V has been accumulated; groups 0 .. D/32 - 1
            // each stream out 32 columns, group 0 adds the four partial sums
            const int row = half * C::kRows + r;
            const size_t prow = ((size_t)bh * prm.splits + split) * prm.m + row;
            if (ok && nch > 0 && grp < D / 32) {
                const int jl = g + nch - 1;
                ok = warp_all(mbar_wait(&pv_done[jl & 1], (jl >> 1) & 1));
                if (ok) {
                    tc_fence_after();
                    uint32_t t[32];
                    tmem_ld32(tmem + lane_base + C::kColO + grp * 32, t);
                    tmem_ld_wait();
                    if (row < prm.m) {
                        float4* dst = reinterpret_cast<float4*>(prm.part_o + prow * D + grp * 32);
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            dst[e] = make_float4(__uint_as_float(t[4 * e]), __uint_as_float(t[4 * e + 1]),
                                                 __uint_as_float(t[4 * e + 2]), __uint_as_float(t[4 * e + 3]));
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(o_free);
            lx[grp * 128 + r] = l_run;
            if (group_any(!ok, 1, kT)) { *abort_flag = 1; break; }   // also publishes lx
            g += nch;
            if (grp == 0 && row < prm.m) {
                prm.part_m[prow] = m_ref == -INFINITY ? -INFINITY : m_ref * kLn2;
                prm.part_l[prow] = (lx[r] + lx[128 + r]) + (lx[256 + r] + lx[384 + r]);
            }
            named_barrier(1, kT);   // lx is read before the next item overwrites it
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

}  // namespace nys
