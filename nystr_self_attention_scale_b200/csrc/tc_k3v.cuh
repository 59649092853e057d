// tc_k3v.cuh -- bf16 kernel_3 V pass on the 5th-generation tensor cores.
//
// Walkthrough (blog.gitcode.com) 2.4: k3 = softmax_row(Q_l Ks^T + mask), new_value = k3 V.
// A work item is (batch*head, 128-landmark block, key split). For each
// 128-key chunk of the split:
//   S = Q_l_block . K_chunk^T          tcgen05 bf16 MMA into TMEM (K unscaled;
//                                      the d^-1/4 of K is applied in the exponent)
//   online softmax per landmark row    one thread per row reads S from TMEM,
//                                      masks padded keys, writes bf16 P back
//   O_chunk = P . V_chunk              MMA with A = P from TMEM, V as an MN-major
//                                      operand (keys x d straight from the TMA tile)
//   O += alpha O + O_chunk             fp32 running sum in registers (one chunk behind,
//                                      so the P.V MMA latency is hidden)
// and writes the unnormalised partial (O, running max, running sum) of the
// split; a deterministic combine over splits follows.
//
// Warp roles (256 threads): warp 0 TMA producer, warp 1 MMA issuer, warp 2
// TMEM allocator, warps 4-7 softmax + accumulation. S and O are double
// buffered in TMEM; K/V chunks use a 3-stage shared-memory ring.
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
    static constexpr int kNumBars = 2 + 2 * kStages + 8 + 1;
    static constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;
    // at least 116 KB so that only one CTA (and one 512-column TMEM allocation) fits per SM
    static constexpr uint32_t kSmemNeed = kOffMisc + 16 + 1024;
    static constexpr uint32_t kSmemBytes = kSmemNeed > 118784 ? kSmemNeed : 118784;
    static constexpr int kTmemCols = 512;
    static constexpr int kColS = 0, kColO = 256;
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
__global__ void __launch_bounds__(256, 1)
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
    uint64_t* s_full = bars + 2 + 2 * C::kStages;  // [2]
    uint64_t* p_full = s_full + 2;                 // [2] (128 arrivals)
    uint64_t* o_full = s_full + 4;                 // [2]
    uint64_t* o_free = s_full + 6;                 // [2] (128 arrivals)
    uint64_t* mma_done = s_full + 8;
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
            mbar_init(&p_full[b], 128);
            mbar_init(&o_full[b], 1);
            mbar_init(&o_free[b], 128);
        }
        mbar_init(mma_done, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&map_ql);
        prefetch_tmap(&map_k);
        prefetch_tmap(&map_v);
    }
    if (warp == 2) {
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
        if (lane == 0) {
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
            auto issue_S = [&](int j) -> bool {
                const int b = j & 1, st = j % C::kStages;
                if (j >= 2 && !mbar_wait(&o_full[b], ((j - 2) >> 1) & 1)) return false;  // P(j-2) consumed
                if (!mbar_wait(&kv_full[st], (j / C::kStages) & 1)) return false;
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < D / 16; ++k)
                    mma_bf16_ss(tmem + C::kColS + b * 128, descQl(k), descK(st, k), C::kIdS, k > 0);
                mma_commit(&s_full[b]);
                return true;
            };
            auto issue_PV = [&](int j) -> bool {
                const int b = j & 1, st = j % C::kStages;
                if (!mbar_wait(&p_full[b], (j >> 1) & 1)) return false;
                if (!mbar_wait(&o_free[b], ((j >> 1) & 1) ^ 1)) return false;
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < C::kChunk / 16; ++k)
                    mma_bf16_ts(tmem + C::kColO + b * D, tmem + C::kColS + b * 128 + k * 8, descV(st, k), C::kIdPV,
                                k > 0);
                mma_commit(&o_full[b]);
                mma_commit(&kv_empty[st]);
                return true;
            };
            for (int item = blockIdx.x; item < prm.total_items && ok && !*abort_flag; item += gridDim.x, ++it) {
                int c0;
                const int nch = item_chunks(item, &c0);
                ok = mbar_wait(ql_full, it & 1);
                if (!ok) break;
                tc_fence_after();
                ok = issue_S(g);
                for (int c = 0; c < nch && ok; ++c) {
                    const int j = g + c;
                    if (c + 1 < nch) ok = issue_S(j + 1);
                    else mma_commit(ql_empty);   // every S MMA of this item is issued
                    if (ok) ok = issue_PV(j);
                }
                g += nch;
            }
            if (!ok) *abort_flag = 1;
            mma_commit(mma_done);
            mbar_wait(mma_done, 0);
        }
    } else if (warp >= 4) {
        const int q4 = warp & 3;
        const int r = 32 * q4 + lane;
        const uint32_t lane_base = (uint32_t)(32 * q4) << 16;
        const float s_d = split_scale(D);
        const float sc = s_d * kLog2e;
        int g = 0;
        for (int item = blockIdx.x; item < prm.total_items && !warp_any(*abort_flag != 0); item += gridDim.x) {
            const int bh = item / per_bh, half = (item / prm.splits) % prm.halves;
            const int split = item % prm.splits;
            const int b_idx = bh / prm.H;
            int c0;
            const int nch = item_chunks(item, &c0);
            float o[D];
#pragma unroll
            for (int e = 0; e < D; ++e) o[e] = 0.f;
            float m_run = -INFINITY, l_run = 0.f, alpha_prev = 1.f;
            bool ok = true;
            auto accumulate = [&](int j, float alpha) -> bool {
                const int b = j & 1;
                if (!warp_all(mbar_wait(&o_full[b], (j >> 1) & 1))) return false;
                tc_fence_after();
                uint32_t v[32];
#pragma unroll
                for (int h = 0; h < D / 32; ++h) {
                    tmem_ld32(tmem + lane_base + C::kColO + b * D + h * 32, v);
                    tmem_ld_wait();
#pragma unroll
                    for (int e = 0; e < 32; ++e) o[h * 32 + e] = fmaf(o[h * 32 + e], alpha, __uint_as_float(v[e]));
                }
                tc_fence_before();
                mbar_arrive(&o_free[b]);
                return true;
            };
            for (int c = 0; c < nch && ok; ++c) {
                const int j = g + c, b = j & 1;
                const int key0 = (c0 + c) * C::kChunk;
                // key-validity bits of this chunk (bit k = key key0 + k is valid)
                uint32_t mb[4] = {~0u, ~0u, ~0u, ~0u};
                if (prm.mask_bits != nullptr) {
                    const uint4 u = __ldg(reinterpret_cast<const uint4*>(prm.mask_bits + (size_t)b_idx * (prm.n / 32) + key0 / 32));
                    mb[0] = u.x; mb[1] = u.y; mb[2] = u.z; mb[3] = u.w;
                }
                const bool full = (mb[0] & mb[1] & mb[2] & mb[3]) == ~0u;
                if (!warp_all(mbar_wait(&s_full[b], (j >> 1) & 1))) { ok = false; break; }
                tc_fence_after();
                const uint32_t sbuf = tmem + lane_base + C::kColS + b * 128;
                uint32_t v[32];
                float cmax = -INFINITY;
#pragma unroll 1
                for (int h = 0; h < 4; ++h) {
                    tmem_ld32(sbuf + h * 32, v);
                    tmem_ld_wait();
                    if (full) {
#pragma unroll
                        for (int e = 0; e < 32; ++e) cmax = fmaxf(cmax, __uint_as_float(v[e]));
                    } else {
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            if ((mb[h] >> e) & 1u) cmax = fmaxf(cmax, __uint_as_float(v[e]));
                    }
                }
                const float m_new = fmaxf(m_run, cmax);
                // a row whose keys so far are all padded keeps P = 0 (no branch around the
                // warp-collective TMEM accesses below)
                const bool live = m_new != -INFINITY;
                const float mo = live ? m_new * sc : 0.f;
                const float alpha = live ? ex2(fmaf(m_run, sc, -mo)) : 1.f;   // m_run = -inf gives 0
                float sum = 0.f;
#pragma unroll 1
                for (int h = 0; h < 4; ++h) {
                    tmem_ld32(sbuf + h * 32, v);
                    tmem_ld_wait();
                    uint32_t pk[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        float p0 = ex2(fmaf(__uint_as_float(v[2 * e]), sc, -mo));
                        float p1 = ex2(fmaf(__uint_as_float(v[2 * e + 1]), sc, -mo));
                        const bool k0 = live && (full || ((mb[h] >> (2 * e)) & 1u));
                        const bool k1 = live && (full || ((mb[h] >> (2 * e + 1)) & 1u));
                        p0 = k0 ? p0 : 0.f;
                        p1 = k1 ? p1 : 0.f;
                        sum += p0 + p1;
                        pk[e] = pack_bf16(p0, p1);
                    }
                    tmem_st16(sbuf + h * 16, pk);
                }
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(&p_full[b]);
                l_run = fmaf(l_run, alpha, sum);
                m_run = m_new;
                if (c > 0 && !accumulate(j - 1, alpha_prev)) { ok = false; break; }
                alpha_prev = alpha;
            }
            if (ok && nch > 0) ok = accumulate(g + nch - 1, alpha_prev);
            if (!ok) { *abort_flag = 1; break; }
            g += nch;
            const int row = half * C::kRows + r;
            if (row < prm.m) {
                const size_t prow = ((size_t)bh * prm.splits + split) * prm.m + row;
                float4* dst = reinterpret_cast<float4*>(prm.part_o + prow * D);
#pragma unroll
                for (int e = 0; e < D / 4; ++e) dst[e] = make_float4(o[4 * e], o[4 * e + 1], o[4 * e + 2], o[4 * e + 3]);
                prm.part_m[prow] = m_run == -INFINITY ? -INFINITY : m_run * s_d;
                prm.part_l[prow] = l_run;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 2) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

}  // namespace nys
