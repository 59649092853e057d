// tc_k3v.cuh -- bf16 kernel_3 V pass on the 5th-generation tensor cores.
//
// Walkthrough (blog.gitcode.com) 2.4: k3 = softmax_row(Q_l Ks^T + mask), new_value = k3 V.
// The same kernel runs the exact branch (walkthrough 2.1, path A) with the raw queries
// as its rows: softmax_row(Qs Ks^T + mask) V over all n query rows.
// A work item is (batch*head, 128-row block, key split). For each
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
// An item's chunks run as two independent streams: chunk c goes to stream
// c % 2, which has its own O accumulator, reference max and running sum in
// TMEM / registers. The S products go to a ring of three 128-column TMEM
// buffers shared by the two streams (chunk g of the CTA's sequence to buffer
// g % 3); each softmax group writes its P (bf16 pairs) over the first half of
// its own 64 score columns, which it has read, and the P V product takes P from
// there. A buffer is reused once that P V is done, so a stream's next S product
// waits for the P V of the chunk three places back (the other stream's previous
// chunk), not for this stream's softmax, and is mostly in place by the time the
// softmax needs it. At the end of an item
// the threads of stream 0 merge the two streams' (O, reference max, running
// sum) row by row and write the unnormalised partial of the split; a
// deterministic combine over splits follows. The stream of a chunk depends
// only on its place in its split, so a head's result does not depend on the
// rest of the batch.
//
// Warp roles (608 threads): warp 0 TMA producer and TMEM allocator, warps 1
// and 18 the MMA issuers of streams 0 and 1 (each issues in its own stream's
// order, so neither waits in program order behind the other's), warps 2-17 the softmax: stream t owns warps 2 + 8 t .. 9 + 8 t, two
// warpgroups that split each of its chunks' 128 keys (64 each), exchanging the
// chunk max through shared memory. Each SM sub-partition runs four softmax
// warps, two per stream.
// K/V chunks use a 6-stage shared-memory ring (three chunks of lookahead per stream).
#pragma once

#include "sm100.cuh"

namespace nys {

template <int D>
struct K3vTc {
    static constexpr int kRows = 128, kChunk = 128;
    static constexpr int kSpan = D * 2;
    static constexpr uint32_t kLayout = D == 64 ? sm100::kLayoutSw128 : sm100::kLayoutSw64;
    static constexpr uint32_t kSbo = 8 * kSpan;
    static constexpr int kStages = 6;
    static constexpr uint32_t kTileBytes = 128 * kSpan;
    static constexpr uint32_t kOffQl = 0;
    static constexpr uint32_t kOffK = kOffQl + kTileBytes;
    static constexpr uint32_t kOffV = kOffK + kStages * kTileBytes;
    static constexpr uint32_t kOffBar = kOffV + kStages * kTileBytes;
    static constexpr int kNumBars = 2 + 2 * kStages + 12 + 1;
    static constexpr int kStreams = 2;                                    // softmax streams
    static constexpr int kTeamThreads = 256;                              // two warpgroups per stream
    static constexpr int kThreads = 96 + kStreams * kTeamThreads;        // warps 0, 1, 18 + the streams
    static constexpr uint32_t kOffXch = kOffBar + kNumBars * 8;          // [2 streams][2 groups][128] maxima
    static constexpr uint32_t kOffLx = kOffXch + 2 * 2 * 128 * 4;        // [2 streams][2 groups][128] sums
    static constexpr uint32_t kOffMx = kOffLx + 2 * 2 * 128 * 4;         // [2 streams][128] reference maxima
    static constexpr uint32_t kOffMisc = kOffMx + 2 * 128 * 4;
    // at least 116 KB so that only one CTA (and one 512-column TMEM allocation) fits per SM
    static constexpr uint32_t kSmemNeed = kOffMisc + 16 + 1024;
    static constexpr uint32_t kSmemBytes = kSmemNeed > 118784 ? kSmemNeed : 118784;
    static constexpr int kTmemCols = 512;
    // TMEM columns: S ring buffer b at 128 b (b = 0, 1, 2; P over the first half of each
    // group's 64 columns), O of stream t at 384 + D t
    static constexpr int kColS = 0, kColO = 384;
    static constexpr uint32_t kIdS = sm100::make_idesc(128, kChunk, sm100::kFmtBf16, sm100::kFmtBf16, 0, 0);
    static constexpr uint32_t kIdPV = sm100::make_idesc(128, D, sm100::kFmtBf16, sm100::kFmtBf16, 0, 1);
};

struct K3vTcParams {
    const uint32_t* mask_bits;  // [B, n / 32] key-validity bits, or null for no mask
    float* part_o;         // [BH, splits, m, d]
    float* part_m;         // [BH, splits, m]  running max (natural-log units)
    float* part_l;         // [BH, splits, m]  running sum
    int H, n, m, halves, splits, chunks_per_split, total_items;
    float score_scale;     // exponent scale of the raw S (log2 units): d^-1/4 log2(e) for the
                           // landmark rows (K's share of the scaling), d^-1/2 log2(e) for raw queries
};

template <int D>
__global__ void __launch_bounds__(K3vTc<D>::kThreads, 1)
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
    // [3] S of the chunk in ring buffer b in TMEM: one barrier per buffer, so that a stream's next
    // S (in another buffer) may complete before its softmax has waited for the current one
    uint64_t* s_full = bars + 2 + 2 * C::kStages;
    uint64_t* p_full = s_full + 3;                 // [stream] P in TMEM (256 arrivals)
    uint64_t* pv_done = s_full + 5;                // [stream] P V accumulated into its O
    uint64_t* o_free = s_full + 7;                 // [stream] the item's O has been read (256 arrivals)
    uint64_t* buf_free = s_full + 9;               // [3] S ring buffer reusable: the P V reading it is done
    uint64_t* mma_done = s_full + 12;
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
        mbar_init(ql_empty, 2);   // one commit per MMA issuer
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(&kv_full[s], 1);
            mbar_init(&kv_empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&p_full[b], C::kTeamThreads);
            mbar_init(&pv_done[b], 1);
            mbar_init(&o_free[b], C::kTeamThreads);
        }
        for (int b = 0; b < 3; ++b) {
            mbar_init(&s_full[b], 1);
            mbar_init(&buf_free[b], 1);
        }
        mbar_init(mma_done, 64);   // one commit per lane of the two MMA warps
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
            const uint64_t stream_policy = l2_policy_evict_first();
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
                    // K and V stream through once: evict them first, so that they do not push
                    // the inverse's operands (re-read every iteration, on other SMs) out of L2
                    tma_load_3d_hint(sm + C::kOffK + st * C::kTileBytes, &map_k, &kv_full[st], 0, key0, bh, stream_policy);
                    tma_load_3d_hint(sm + C::kOffV + st * C::kTileBytes, &map_v, &kv_full[st], 0, key0, bh, stream_policy);
                    last_stage_use[st] = g / C::kStages;
                }
            }
            if (*abort_flag) {
                for (int s = 0; s < C::kStages; ++s)
                    if (last_stage_use[s] >= 0) mbar_wait(&kv_full[s], last_stage_use[s] & 1);
                if (ql_issued >= 0) mbar_wait(ql_full, ql_issued & 1);
            }
        }
    } else if (warp == 1 || warp == 18) {
        // MMA issuer of stream t (chunks c of an item with c % 2 == t): the whole warp runs the
        // loop and the waits; one elected lane issues each MMA group and each commit
        const int t = warp == 1 ? 0 : 1;
        bool ok = true;
        int g = 0, it = 0, u = 0;   // chunks before this item, items, chunks of this stream
        // operand descriptors: each buffer's is built once, and a K step or a ring stage advances
        // its start-address field (fewer instructions for this warp, which shares its issue slots
        // with four softmax warps)
        const uint64_t dQl = smem_desc(sbase + C::kOffQl, 16, C::kSbo, C::kLayout);
        const uint64_t dK = smem_desc(sbase + C::kOffK, 16, C::kSbo, C::kLayout);
        const uint64_t dV = smem_desc(sbase + C::kOffV, C::kTileBytes, C::kSbo, C::kLayout);
        auto descQl = [&](int k) { return desc_advance(dQl, k * 32); };
        auto descK = [&](int st, int k) { return desc_advance(dK, st * C::kTileBytes + k * 32); };
        auto descV = [&](int st, int k) { return desc_advance(dV, st * C::kTileBytes + k * 16 * C::kSpan); };
        auto wait = [&](uint64_t* bar, uint32_t parity) { return warp_all(mbar_wait(bar, parity)); };
        for (int item = blockIdx.x; item < prm.total_items && ok && !warp_any(*abort_flag != 0);
             item += gridDim.x, ++it) {
            int c0;
            const int nch = item_chunks(item, &c0);
            ok = wait(ql_full, it & 1);
            if (!ok) break;
            tc_fence_after();
            // S of chunk c into ring buffer (g + c) % 3, once the P V of the chunk three places
            // back (which read its P from that buffer) is done
            auto issue_S = [&](int c) -> bool {
                const int gc = g + c, st = gc % C::kStages, b = gc % 3;
                if (gc >= 3 && !wait(&buf_free[b], (gc / 3 - 1) & 1)) return false;
                if (!wait(&kv_full[st], (gc / C::kStages) & 1)) return false;
                tc_fence_after();
                if (elect_one()) {
#pragma unroll
                    for (int k = 0; k < D / 16; ++k)
                        mma_bf16_ss(tmem + C::kColS + b * 128, descQl(k), descK(st, k), C::kIdS, k > 0);
                }
                if (elect_one()) mma_commit(&s_full[b]);
                return true;
            };
            if (t < nch) ok = issue_S(t);
            for (int c = t; c < nch && ok; c += 2, ++u) {
                const int gc = g + c, st = gc % C::kStages, b = gc % 3;
                // the next S of the stream goes first, so that it runs during this chunk's softmax
                if (c + 2 < nch) {
                    if (!(ok = issue_S(c + 2))) break;
                } else if (elect_one()) {
                    mma_commit(ql_empty);   // this stream's last S of the item is issued
                }
                // P V into the stream's O, once its softmax has written P; the first of the item
                // also waits until the stream's previous O has been read
                const bool first = c < 2;
                if (!(ok = wait(&p_full[t], u & 1))) break;
                if (first && !(ok = wait(&o_free[t], (it & 1) ^ 1))) break;
                tc_fence_after();
                if (elect_one()) {
#pragma unroll
                    for (int k = 0; k < C::kChunk / 16; ++k) {
                        // keys 16k .. 16k+15: P of group k / 4, over the first half of its 64
                        // score columns in the chunk's ring buffer
                        const uint32_t pa = tmem + C::kColS + b * 128 + 64 * (k >> 2) + 8 * (k & 3);
                        mma_bf16_ts(tmem + C::kColO + t * D, pa, descV(st, k), C::kIdPV,
                                    (first && k == 0) ? 0u : 1u);
                    }
                }
                if (elect_one()) {
                    mma_commit(&pv_done[t]);
                    mma_commit(&kv_empty[st]);
                    mma_commit(&buf_free[b]);
                }
            }
            // a stream with no chunk in this item still releases Q_l once
            if (ok && t >= nch && elect_one()) mma_commit(ql_empty);
            g += nch;
        }
        if (!ok) *abort_flag = 1;
        // one commit per lane (mma_done counts both warps' 64 arrivals): the drain covers
        // whichever lane issued
        mma_commit(mma_done);
        mbar_wait(mma_done, 0);
    } else if (warp >= 2 && warp < 18) {
        const int sw = warp - 2;
        const int t = sw >> 3;                      // stream: chunks c with c % 2 == t
        const int grp = (sw >> 2) & 1;              // keys [64 grp, 64 grp + 64) of each chunk
        const int q4 = warp & 3;
        const int r = 32 * q4 + lane;
        const uint32_t lane_base = (uint32_t)(32 * q4) << 16;
        const float sc = prm.score_scale;           // exponent scale of the raw S = Q_rows . K^T
        constexpr float kSlack = 8.f;               // log2 units: P stays below 2^8
        constexpr int kT = C::kTeamThreads;
        const int bar_id = 1 + t;                   // this stream's named barrier
        float* xch = reinterpret_cast<float*>(sm + C::kOffXch) + t * 256;   // [2 groups][128]
        float* lx_all = reinterpret_cast<float*>(sm + C::kOffLx);   // [2 streams][2 groups][128]
        float* mx_all = reinterpret_cast<float*>(sm + C::kOffMx);   // [2 streams][128]
        constexpr int kCta = 2 * C::kTeamThreads;   // both streams: named barrier 3
        const uint32_t obuf = tmem + lane_base + C::kColO + t * D + 32 * grp;
        int u = 0, it = 0;   // chunks this stream has taken, items
        int g = 0;           // chunks of the CTA's earlier items (the S ring position)
        for (int item = blockIdx.x; item < prm.total_items; item += gridDim.x, ++it) {
            // both streams take every item-level decision together (barrier 3), so that neither
            // waits at that barrier for a stream that has left
            if (group_any(*abort_flag != 0, 3, kCta)) break;
            const int bh = item / per_bh, half = (item / prm.splits) % prm.halves;
            const int split = item % prm.splits;
            const int b_idx = bh / prm.H;
            int c0;
            const int nch = item_chunks(item, &c0);
            float m_ref = -INFINITY, l_run = 0.f;   // reference max (log2 units) and this group's sum
            bool ok = true;
            int mine = 0;                           // chunks of this item taken by the stream
            for (int c = t; c < nch; c += 2, ++u, ++mine) {
                const int key0 = (c0 + c) * C::kChunk + 64 * grp;
                // this group's 64 score columns in the chunk's ring buffer; its P goes over their
                // first half once they are read
                const uint32_t sbuf = tmem + lane_base + C::kColS + ((g + c) % 3) * 128 + 64 * grp;
                const uint32_t pbuf = sbuf;
                // key-validity bits of this group's 64 keys (bit k of word h = key key0 + 32 h + k)
                uint32_t mb[2] = {~0u, ~0u};
                if (prm.mask_bits != nullptr) {
                    const uint32_t* w = prm.mask_bits + (size_t)b_idx * (prm.n / 32) + key0 / 32;
                    mb[0] = __ldg(w);
                    mb[1] = __ldg(w + 1);
                }
                const bool full = (mb[0] & mb[1]) == ~0u;
                // a wait that runs out leaves S unread: the group still passes the chunk's one
                // barrier below (which also ORs the failure across the two groups) and then stops
                ok = warp_all(mbar_wait(&s_full[(g + c) % 3], ((g + c) / 3) & 1));
                tc_fence_after();
                // pass 1: the max of this group's 64 scores (the scores are loaded again for the
                // exponentials, which keeps the register footprint small)
                float mq[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};   // four short max chains
                if (ok) {
                    uint32_t v[2][32];   // keys 32 h + e of this group's 64
                    tmem_ld32(sbuf, v[0]);
                    tmem_ld32(sbuf + 32, v[1]);
                    tmem_ld_wait();
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        if (!full) {
#pragma unroll
                            for (int e = 0; e < 32; ++e)
                                if (!((mb[h] >> e) & 1u)) v[h][e] = __float_as_uint(-INFINITY);
                        }
#pragma unroll
                        for (int e = 0; e < 16; ++e)
                            mq[(2 * h + e) & 3] = max3(mq[(2 * h + e) & 3], __uint_as_float(v[h][2 * e]),
                                                       __uint_as_float(v[h][2 * e + 1]));
                    }
                }
                xch[grp * 128 + r] = fmaxf(fmaxf(mq[0], mq[1]), fmaxf(mq[2], mq[3]));
                if (group_any(!ok, bar_id, kT)) { ok = false; break; }   // also publishes xch
                const float cm = fmaxf(xch[r], xch[128 + r]) * sc;
                // move the reference only when this chunk's max exceeds it by more than the slack
                // (both groups take the same decision: same maxima, same history)
                const bool move = cm > m_ref + kSlack;
                const float m_new = move ? cm : m_ref;
                const float alpha = move ? ex2(m_ref - m_new) : 1.f;   // m_ref = -inf gives 0
                if (grp < D / 32 && mine > 0 && warp_any(move && m_ref != -INFINITY)) {
                    // rescale this warp's rows of O (group g: columns 32 g .. 32 g + 31) once the
                    // stream's previous P V has been accumulated
                    ok = warp_all(mbar_wait(&pv_done[t], (u - 1) & 1));
                    if (ok) {
                        tc_fence_after();
                        uint32_t o[32];
                        tmem_ld32(obuf, o);
                        tmem_ld_wait();
#pragma unroll
                        for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                        tmem_st32(obuf, o);
                    }
                }
                const float mo = m_new == -INFINITY ? 0.f : m_new;   // rows with every key padded so far: P = 0
                // exponentials on packed fp32 pairs: in chunks without padded keys the FMA pipe takes
                // 6 of every 16 pairs (polynomial 2^x) and the MUFU unit the rest; chunks with padded
                // keys use the MUFU unit only, so that padded keys get exactly 0. P is rounded to
                // bf16 (nearest even); the running sum adds the fp32 values.
                const uint64_t sc2 = f2(sc, sc), nmo2 = f2(-mo, -mo);
                uint64_t acc[2] = {f2(0.f, 0.f), f2(0.f, 0.f)};
                // pass 2: this group's 64 scores again, with one wait; then the S buffer is released
                // to the stream's next S MMA
                uint32_t vv[2][32];
                tmem_ld32(sbuf, vv[0]);
                tmem_ld32(sbuf + 32, vv[1]);
                tmem_ld_wait();
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    uint32_t* v = vv[h];
                    if (!full) {
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            if (!((mb[h] >> e) & 1u)) v[e] = __float_as_uint(-INFINITY);
                    }
                    uint32_t pk[16];
                    if (full) {
#pragma unroll
                        for (int e = 0; e < 16; ++e) {
                            const uint64_t x2 = f2_fma(
                                f2(__uint_as_float(v[2 * e]), __uint_as_float(v[2 * e + 1])), sc2,
                                nmo2);
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
                            const uint64_t x2 = f2_fma(
                                f2(__uint_as_float(v[2 * e]), __uint_as_float(v[2 * e + 1])), sc2,
                                nmo2);
                            float x0, x1;
                            f2_split(x2, x0, x1);
                            const float e0 = ex2(x0), e1 = ex2(x1);
                            pk[e] = pack_bf16_rn(e0, e1);
                            acc[e & 1] = f2_add(acc[e & 1], f2(e0, e1));
                        }
                    }
                    // this group's P (keys 32 h ..) over scores it has read (all 64 are in registers)
                    tmem_st16(pbuf + 16 * h, pk);
                }
                float sum;
                {
                    float a0, a1, b0, b1;
                    f2_split(acc[0], a0, a1);
                    f2_split(acc[1], b0, b1);
                    sum = (a0 + a1) + (b0 + b1);
                }
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(&p_full[t]);
                l_run = fmaf(l_run, alpha, sum);
                m_ref = m_new;
            }
            // the split's partial: each stream publishes its row statistics and waits for its last
            // P V; then the threads of stream 0 merge the two streams' O (group g: columns
            // 32 g .. 32 g + 31) and group 0 of stream 0 writes the merged maximum and sum. A
            // stream that took no chunk of the item contributes nothing (its TMEM is not read).
            lx_all[(t * 2 + grp) * 128 + r] = l_run;
            if (grp == 0) mx_all[t * 128 + r] = m_ref;
            if (ok && mine > 0) ok = warp_all(mbar_wait(&pv_done[t], (u - 1) & 1));
            if (group_any(!ok, 3, kCta)) { *abort_flag = 1; break; }   // also publishes lx, mx
            tc_fence_after();
            if (t == 0) {
                const int row = half * C::kRows + r;
                const size_t prow = ((size_t)bh * prm.splits + split) * prm.m + row;
                const bool has1 = nch > 1;                       // stream 1 took chunk 1, 3, ...
                const float m0 = mx_all[r], m1 = has1 ? mx_all[128 + r] : -INFINITY;
                const float mm = fmaxf(m0, m1);
                const float a0 = m0 == -INFINITY ? 0.f : ex2(m0 - mm);
                const float a1 = m1 == -INFINITY ? 0.f : ex2(m1 - mm);
                if (grp < D / 32) {
                    float4* dst = reinterpret_cast<float4*>(prm.part_o + prow * D + grp * 32);
#pragma unroll 1
                    for (int h = 0; h < 2; ++h) {   // 16 columns per TMEM load
                        uint32_t o0[16], o1[16];
                        tmem_ld16(obuf + 16 * h, o0);   // stream 0 always has chunk 0
                        if (has1) {
                            tmem_ld16(obuf + D + 16 * h, o1);
                        } else {
#pragma unroll
                            for (int e = 0; e < 16; ++e) o1[e] = 0u;   // a1 = 0 as well
                        }
                        tmem_ld_wait();
                        if (row < prm.m) {
#pragma unroll
                            for (int e = 0; e < 4; ++e)
                                dst[4 * h + e] = make_float4(
                                    a0 * __uint_as_float(o0[4 * e]) + a1 * __uint_as_float(o1[4 * e]),
                                    a0 * __uint_as_float(o0[4 * e + 1]) + a1 * __uint_as_float(o1[4 * e + 1]),
                                    a0 * __uint_as_float(o0[4 * e + 2]) + a1 * __uint_as_float(o1[4 * e + 2]),
                                    a0 * __uint_as_float(o0[4 * e + 3]) + a1 * __uint_as_float(o1[4 * e + 3]));
                        }
                    }
                }
                if (grp == 0 && row < prm.m) {
                    const float l0 = lx_all[r] + lx_all[128 + r];
                    const float l1 = has1 ? lx_all[256 + r] + lx_all[384 + r] : 0.f;
                    prm.part_m[prow] = mm == -INFINITY ? -INFINITY : mm * kLn2;
                    prm.part_l[prow] = a0 * l0 + a1 * l1;
                }
                // both O accumulators have been read: the next item's first P V of either stream
                // may overwrite them
                tc_fence_before();
                mbar_arrive(&o_free[0]);
                mbar_arrive(&o_free[1]);
            }
            named_barrier(3, kCta);   // the statistics are read before the next item overwrites them
            g += nch;
        }
    }

    // the split merge may launch now (it waits for this grid's completion before reading)
    griddep_launch_dependents();
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

}  // namespace nys
