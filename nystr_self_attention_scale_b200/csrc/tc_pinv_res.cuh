// tc_pinv_res.cuh -- kernel_2 and the iterative Moore-Penrose inverse for m = 128 and
// m = 64, one CTA per 128 rows, every operand on chip.
//
// Walkthrough (blog.gitcode.com) 2.4: k2 = softmax_row(Q_l K_l^T); 2.5: Z_0 = c k2^T, then
// n_iter times X = k2 Z; T1 = 7I - X; T3 = 15I - X T1; T5 = 13I - X T3; Z = Z T5 / 4.
//
// The CTA solves one 128 x 128 problem: one head at m = 128, or two heads at m = 64 held
// block-diagonally (rows and columns 0..63 the first head, 64..127 the second). Every
// product of block-diagonal matrices is block-diagonal and every T is a polynomial in X, so
// the two heads never mix; only the per-head scalars (c, and the scales derived from it)
// are taken per block.
//
// The iteration runs on W = Z^T, as in the CTA-pair kernel for m = 256 (the page's sequence
// transposed; equal in real arithmetic):
//   P1: X = W k2^T          A = W (R0: the raw previous P4 accumulator), B = k2 as K-major
//                           lines, D -> R1
//   P2: T3 = 15I + T1 (-X)  A = T1 (R1, written over P1's accumulator by its epilogue),
//                           B = -X, MN-major; D -> R2, which holds 15 I beforehand
//   P3: T5 = 13I + T3 (-X)  A = R2, B = -X; D -> R3, which holds 13 I beforehand
//   P4: W' = T5 W / 4       A = R3, B = W's rows, MN-major; D -> R0
// so only P1 has an epilogue on the chain: P2 -> P3 -> P4 wait only for the previous
// product to complete. The P1 epilogue also sets R2 and R3 to 15 I and 13 I; the P4
// epilogue, which runs beside the next P1, writes W's rows.
// k2 stays in shared memory for all P1s; -X is written by the P1 epilogue, W's rows by the
// P4 epilogue of the iteration before (or by the prologue: k2's rows, W_0 = c k2 with c folded
// into the scales). Nothing is streamed through L2. Scales are folded into the epilogues as
// in the pair kernel: X = sigma D with sigma = c, c / 4, then 1 / 4; W' = lambda D with
// lambda = c / 4, then 1 / 4.
//
// Roles (320 threads): warps 0-7 epilogue (warp w: TMEM lanes 32 (w % 4), columns 64 (w / 4)
// .. + 63), warp 8 lane 0 TMA producer of the landmarks, warp 9 TMEM allocation and MMA issue.
#pragma once

#include "sm100.cuh"

namespace nys {

struct PinvResMaps {
    CUtensorMap ql;   // Q_l [BH][m][d] fp32, box 32 x m, 128-byte swizzle
    CUtensorMap kl;   // K_l, same box
};

struct PinvResParams {
    float* z_out;     // [BH][m][m]
    int BH, d, n_iter, inv_init;
};

template <int MH>
struct PinvRes {
    static_assert(MH == 64 || MH == 128, "rows per head");
    static constexpr int M = 128;                     // rows and columns of the CTA's problem
    static constexpr int kHeads = M / MH;             // heads per CTA
    static constexpr uint32_t kAtom = 128 * 128;      // 128 lines (rows) x 32 tf32: 16 KB
    static constexpr uint32_t kMat = 4 * kAtom;       // a 128 x 128 fp32 operand: 64 KB
    static constexpr uint32_t kOffK2 = 0;             // k2 as K-major lines (P1), resident
    static constexpr uint32_t kOffX = kMat;           // -X, MN-major (P2, P3)
    static constexpr uint32_t kOffW = 2 * kMat;       // W's rows, MN-major (P4)
    // prologue: Q_l hi / lo in the X buffer, K_l hi / lo in the W buffer (d / 32 atoms each)
    static constexpr uint32_t kOffQhi = kOffX, kOffQlo = kOffX + 2 * kAtom;
    static constexpr uint32_t kOffKhi = kOffW, kOffKlo = kOffW + 2 * kAtom;
    // MN-major operand (32-byte-granule 128-byte swizzle, the layout tf32 needs):
    // [K group of 8 rows][32-column atom][two 4-row atoms of 512 B]
    static constexpr uint32_t kMnAtom = 1024, kMnGroup = 4096, kMnRow4 = 512;
    static constexpr uint32_t kOffRed = 3 * kMat;     // [2][128] row max / sums, [128] column sums, [16]
    static constexpr uint32_t kOffBar = kOffRed + (2 * 128 + 2 * 128 + 128 + 16) * 4;
    static constexpr uint32_t kOffMisc = kOffBar + 8 * 8;
    static constexpr uint32_t kSmemBytes = kOffMisc + 64 + 1024;
    static constexpr int kThreads = 320;
    static constexpr uint32_t kIdK = sm100::make_idesc(128, 128, sm100::kFmtTf32, sm100::kFmtTf32, 0, 0);
    static constexpr uint32_t kIdMN = sm100::make_idesc(128, 128, sm100::kFmtTf32, sm100::kFmtTf32, 0, 1);
};

template <int MH>
__global__ void __launch_bounds__(PinvRes<MH>::kThreads, 1)
pinv_res_kernel(const __grid_constant__ PinvResMaps maps, const PinvResParams prm) {
    using C = PinvRes<MH>;
    using namespace sm100;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float* rx = reinterpret_cast<float*>(sm + C::kOffRed);   // [2][128] row max, then row sums of the halves
    float* sx = rx + 256;                                     // [2][128] exponential sums of the halves
    float* cs = sx + 256;                                     // [128] column sums
    float* red = cs + 128;                                    // [16] per-warp maxima, [8..] per-head scalars
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + C::kOffBar);
    uint64_t* pro_full = bars + 0;    // landmarks landed
    uint64_t* e_ready = bars + 1;     // epilogue done with its part (8 warps)
    uint64_t* mma_done = bars + 2;    // kernel_2, P1..P3 accumulators complete
    uint64_t* mma4_done = bars + 3;   // P4 accumulator complete
    uint64_t* drain = bars + 4;       // every MMA issued has completed (32 lanes)
    uint64_t* chain_done = bars + 5;  // P2 / P3 complete (waited by the MMA warp)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + C::kOffMisc);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int head0 = blockIdx.x * C::kHeads;     // first head of this CTA
    const int nka = prm.d / 32;                   // K atoms of the kernel_2 product
    const int n_iter = prm.n_iter;

    if (tid == 0) {
        mbar_init(pro_full, 1);
        mbar_init(e_ready, 8);
        mbar_init(mma_done, 1);
        mbar_init(mma4_done, 1);
        mbar_init(drain, 32);
        mbar_init(chain_done, 1);
        fence_mbar_init();
    }
    if (warp == 9) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t R0 = tmem, R1 = tmem + 128, R2 = tmem + 256, R3 = tmem + 384;

    if (warp == 8) {
        // ------------------------------------------------ TMA producer: this CTA's landmarks
        if (lane == 0) {
            prefetch_tmap(&maps.ql);
            prefetch_tmap(&maps.kl);
            mbar_arrive_expect_tx(pro_full, 2u * nka * C::kAtom);
            for (int a = 0; a < nka; ++a)
                for (int hd = 0; hd < C::kHeads; ++hd) {
                    // a head past the batch reads as zeros (out-of-bounds fill) and is never written
                    const uint32_t rows = (uint32_t)hd * MH * 128u;
                    tma_load_3d(sm + C::kOffQhi + a * C::kAtom + rows, &maps.ql, pro_full, 32 * a, 0, head0 + hd);
                    tma_load_3d(sm + C::kOffKhi + a * C::kAtom + rows, &maps.kl, pro_full, 32 * a, 0, head0 + hd);
                }
        }
        __syncwarp();
    } else if (warp == 9) {
        // ------------------------------------------------ MMA issuer: the whole warp runs the loop
        // and the waits; one elected lane issues each MMA group and commit
        const uint32_t bs = smem_u32(sm);
        uint32_t ne = 0;
        bool ok = warp_all(mbar_wait(e_ready, ne & 1u));   // landmarks split into tf32 hi / lo
        ++ne;
        if (ok) {
            tc_fence_after();
            // kernel_2: S2 = Q_l K_l^T from split tf32 operands, hi.hi + hi.lo + lo.hi, into R1
            if (elect_one()) {
                const uint32_t aoff[3] = {C::kOffQhi, C::kOffQhi, C::kOffQlo};
                const uint32_t boff[3] = {C::kOffKhi, C::kOffKlo, C::kOffKhi};
                uint32_t acc = 0;
                for (int t = 0; t < 3; ++t)
                    for (int a = 0; a < nka; ++a)
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk) {
                            const uint32_t ka = a * C::kAtom + kk * 32;
                            mma_tf32_ss(R1, smem_desc(bs + aoff[t] + ka, 16, 1024, kLayoutSw128),
                                        smem_desc(bs + boff[t] + ka, 16, 1024, kLayoutSw128), C::kIdK, acc);
                            acc = 1;
                        }
            }
            if (elect_one()) mma_commit(mma_done);
        }
        uint32_t nc = 0;   // chain_done phases waited
        for (int it = 0; it < n_iter && ok; ++it) {
            for (int p = 0; p < 4 && ok; ++p) {
                // the first P1 waits for the prologue, P2 for the P1 epilogue (T1, -X, and R2 / R3
                // preset); P3 and P4 for the product before them
                if ((p == 0 && it == 0) || p == 1) {
                    ok = warp_all(mbar_wait(e_ready, ne & 1u));
                    ++ne;
                } else if (p >= 2) {
                    ok = warp_all(mbar_wait(chain_done, nc & 1u));
                    ++nc;
                }
                if (!ok) break;
                tc_fence_after();
                const uint32_t a_col = p == 0 ? R0 : (p == 1 ? R1 : (p == 2 ? R2 : R3));
                const uint32_t d_col = p == 0 ? R1 : (p == 1 ? R2 : (p == 2 ? R3 : R0));
                const bool preset = p == 1 || p == 2;   // accumulate onto 15 I / 13 I
                if (elect_one()) {
#pragma unroll 1
                    for (int ka = 0; ka < 4; ++ka)
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk) {
                            const uint32_t acc = (preset || (ka | kk) != 0) ? 1u : 0u;
                            if (p == 0) {
                                mma_tf32_ts(d_col, a_col + ka * 32 + kk * 8,
                                            smem_desc(bs + C::kOffK2 + ka * C::kAtom + kk * 32, 16, 1024, kLayoutSw128),
                                            C::kIdK, acc);
                            } else {
                                const uint32_t base = p == 3 ? C::kOffW : C::kOffX;
                                mma_tf32_ts(d_col, a_col + ka * 32 + kk * 8,
                                            smem_desc(bs + base + (4 * ka + kk) * C::kMnGroup, C::kMnAtom,
                                                      C::kMnRow4, kLayoutSw128B32),
                                            C::kIdMN, acc);
                            }
                        }
                }
                if (elect_one()) mma_commit(p == 0 ? mma_done : (p == 3 ? mma4_done : chain_done));
            }
        }
        // every MMA issued here has completed before the TMEM is released: one commit per lane
        mma_commit(drain);
        mbar_wait(drain, 0);
    } else {
        // ------------------------------------------------ epilogue (warps 0-7)
        const int q = warp & 3, h = warp >> 2;        // TMEM lane quadrant, column half
        const int lrow = 32 * q + lane;               // this thread's row of every product
        const int hd = lrow / MH;                     // its head within the CTA
        const int et = tid;                           // 0 .. 255
        const uint32_t lane_base = (uint32_t)(32 * q) << 16;
        // the columns of this half that belong to the row's own head (the others are zero)
        const bool own_half = MH == 128 || h == hd;
        // the diagonal element (lrow, lrow) lies in this half, in 32-column atom diag_jj of it
        const bool diag_half = (lrow >> 6) == h;
        const int diag_jj = (lrow >> 5) & 1;
        // v I into this thread's row of TMEM region `base` (its 64 columns): the accumulator
        // preset of P2 (15 I) and P3 (13 I)
        auto preset_diag = [&](uint32_t base, float val) {
#pragma unroll 1
            for (int jj = 0; jj < 2; ++jj) {
                uint32_t v[32];
                const bool here = diag_half && jj == diag_jj;
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] = (here && i == lane) ? __float_as_uint(val) : 0u;
                tmem_st32(base + lane_base + 64 * h + 32 * jj, v);
            }
        };
        auto arrive_e = [&]() {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(e_ready);
        };
        // offset of (row, 16-byte chunk c of column atom j) in an MN-major operand
        const uint32_t mn_row = (uint32_t)(lrow >> 3) * C::kMnGroup;
        auto mn_off = [&](int j, int c) { return mn_row + (uint32_t)j * C::kMnAtom + mn32_chunk(lrow, c); };
        // offset of (line = row, 16-byte chunk c of K atom a) in a K-major operand
        auto k_off = [&](int a, int c) {
            return (uint32_t)a * C::kAtom + (uint32_t)lrow * 128u + (((uint32_t)c ^ (uint32_t)(lrow & 7)) << 4);
        };

        // ---- kernel_2 prologue (walkthrough 2.4: k2 = softmax_row(Q_l K_l^T); 2.5: c)
        bool failed = !mbar_wait(pro_full, 0);
        failed = group_any(failed, 3, 256);
        float coeff = 0.f;
        if (!failed) {
            // split Q_l and K_l into tf32 hi + lo in place (fp32 accuracy from three tf32 products)
            // four independent chunks per step (2 * chunks is a multiple of 1024)
            const int chunks = nka * (int)(C::kAtom / 16);
            static_assert(C::kOffQlo - C::kOffQhi == C::kOffKlo - C::kOffKhi, "hi / lo distance");
#pragma unroll 1
            for (int e0 = et; e0 < 2 * chunks; e0 += 4 * 256) {
                uint32_t off[4];
                float4 x[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int e = e0 + 256 * u;
                    off[u] = (e < chunks ? C::kOffQhi : C::kOffKhi) + (uint32_t)(e % chunks) * 16u;
                    x[u] = *reinterpret_cast<const float4*>(sm + off[u]);
                }
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const float4 xh = make_float4(tf32_rna(x[u].x), tf32_rna(x[u].y), tf32_rna(x[u].z), tf32_rna(x[u].w));
                    *reinterpret_cast<float4*>(sm + off[u]) = xh;
                    *reinterpret_cast<float4*>(sm + off[u] + (C::kOffQlo - C::kOffQhi)) =
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
            // row max over the row's own head's columns (the other head's are masked)
            float mx = -INFINITY;
            if (own_half) {
#pragma unroll 1
                for (int jj = 0; jj < 2; ++jj) {
                    uint32_t v[32];
                    tmem_ld32(R1 + lane_base + 64 * h + 32 * jj, v);
                    tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 32; ++i) mx = fmaxf(mx, __uint_as_float(v[i]));
                }
            }
            // every warp reaches every TMEM load above only through warp-uniform branches
            rx[h * 128 + lrow] = mx;
            named_barrier(3, 256);
            mx = fmaxf(rx[lrow], rx[128 + lrow]);
            float ssum = 0.f;
            if (own_half) {
#pragma unroll 1
                for (int jj = 0; jj < 2; ++jj) {
                    uint32_t v[32];
                    const uint32_t addr = R1 + lane_base + 64 * h + 32 * jj;
                    tmem_ld32(addr, v);
                    tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const float e = __expf(__uint_as_float(v[i]) - mx);
                        ssum += e;
                        v[i] = __float_as_uint(e);
                    }
                    tmem_st32(addr, v);
                }
                tmem_st_wait();
            }
            sx[h * 128 + lrow] = ssum;
            named_barrier(3, 256);   // every thread has read rx; the sums are published
            const float inv = 1.f / (sx[lrow] + sx[128 + lrow]);
            // k2 = e / sum (tf32): into TMEM as W_0 / c (R0), into shared memory as K-major lines
            // (P1's right factor) and as MN-major rows (the first P4's right factor, W_0 / c)
            float rsum = 0.f;
#pragma unroll 1
            for (int jj = 0; jj < 2; ++jj) {
                uint32_t v[32];
                if (own_half) {
                    tmem_ld32(R1 + lane_base + 64 * h + 32 * jj, v);
                    tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const float pr = tf32_rna(__uint_as_float(v[i]) * inv);
                        rsum += pr;
                        v[i] = __float_as_uint(pr);
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) v[i] = 0u;
                }
                tmem_st32(R0 + lane_base + 64 * h + 32 * jj, v);
                const int a = 2 * h + jj;   // 32-column atom of the 128 columns
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const uint4 w4 = make_uint4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
                    *reinterpret_cast<uint4*>(sm + C::kOffK2 + k_off(a, c)) = w4;
                    *reinterpret_cast<uint4*>(sm + C::kOffW + mn_off(a, c)) = w4;
                }
            }
            tmem_st_wait();
            rx[h * 128 + lrow] = rsum;   // rx is free: every thread read its row max before the last barrier
            fence_proxy_async_shared();  // the staged k2 feeds the MMAs
            named_barrier(3, 256);
            // column sums (thread et < 128: column et; block-diagonal zeros add nothing) and row sums;
            // per head: the largest of each
            if (et < 128) {
                const int a = et >> 5, j = et & 31;
                float c4[4] = {0.f, 0.f, 0.f, 0.f};   // four independent chains
#pragma unroll 8
                for (int l = 0; l < 128; ++l)
                    c4[l & 3] += *reinterpret_cast<const float*>(sm + C::kOffK2 + (uint32_t)a * C::kAtom +
                                                                (uint32_t)l * 128u +
                                                                ((((uint32_t)j >> 2) ^ (uint32_t)(l & 7)) << 4) +
                                                                (uint32_t)(j & 3) * 4u);
                const float s = (c4[0] + c4[1]) + (c4[2] + c4[3]);
                const float rs = rx[et] + rx[128 + et];
                // warps 0-3 hold columns / rows 32 w .. 32 w + 31
                const float wc = warp_max(s), wr = warp_max(rs);
                if (lane == 0) {
                    red[warp] = wc;
                    red[4 + warp] = wr;
                }
            }
            named_barrier(3, 256);
            {
                const int w0 = hd * (MH / 32);   // warps of this row's head: w0 .. w0 + MH / 32 - 1
                float mc = red[w0], mr = red[4 + w0];
                for (int w = 1; w < MH / 32; ++w) {
                    mc = fmaxf(mc, red[w0 + w]);
                    mr = fmaxf(mr, red[4 + w0 + w]);
                }
                coeff = 1.f / (mc * (prm.inv_init == NYS_INV_INIT_EXACT ? 1.f : mr));
            }
            if (n_iter == 0) {
                // Z = c k2^T: column lrow of Z's head block is row lrow of k2 (this thread's half)
                const int head = head0 + hd;
                if (own_half && head < prm.BH) {
                    float* zc = prm.z_out + (size_t)head * MH * MH + (lrow % MH);
#pragma unroll 1
                    for (int jj = 0; jj < 2; ++jj) {
                        const int a = 2 * h + jj;
#pragma unroll
                        for (int c = 0; c < 8; ++c) {
                            const float4 f4 = *reinterpret_cast<const float4*>(sm + C::kOffK2 + k_off(a, c));
                            const int col = (32 * a + 4 * c) % MH;   // column within the head block
                            zc[(size_t)(col + 0) * MH] = coeff * f4.x;
                            zc[(size_t)(col + 1) * MH] = coeff * f4.y;
                            zc[(size_t)(col + 2) * MH] = coeff * f4.z;
                            zc[(size_t)(col + 3) * MH] = coeff * f4.w;
                        }
                    }
                }
            } else {
                arrive_e();   // W_0 / c in TMEM, k2 lines and rows in shared memory
            }
        }

        // ---- the iteration
        uint32_t nd = 1, n4 = 0;   // mma_done / mma4_done phases waited
        for (int it = 0; it < n_iter && !failed; ++it) {
            const float sigma = it == 0 ? coeff : (it == 1 ? 0.25f * coeff : 0.25f);
            const float lambda = it == 0 ? 0.25f * coeff : 0.25f;
            const bool last_it = it + 1 == n_iter;
            for (int p = 0; p < 4 && !failed; p += 3) {   // the P1 and P4 epilogues
                const bool ok = p == 3 ? mbar_wait(mma4_done, (n4++) & 1u) : mbar_wait(mma_done, (nd++) & 1u);
                failed = group_any(!ok, 3, 256);
                if (failed) break;
                tc_fence_after();
                const uint32_t d_col = p == 0 ? R1 : R0;
                if (p == 3) {
                    // W' = lambda D: the next P4's right factor (this thread's row, MN-major) or, at
                    // the end, Z = W'^T (column lrow of Z's head block)
                    const int head = head0 + hd;
#pragma unroll 1
                    for (int jj = 0; jj < 2; ++jj) {
                        uint32_t v[32];
                        tmem_ld32(d_col + lane_base + 64 * h + 32 * jj, v);
                        tmem_ld_wait();
                        const int a = 2 * h + jj;
                        if (last_it) {
                            if (own_half && head < prm.BH) {
                                float* zc = prm.z_out + (size_t)head * MH * MH + (lrow % MH);
#pragma unroll
                                for (int i = 0; i < 32; ++i)
                                    zc[(size_t)((32 * a + i) % MH) * MH] = lambda * __uint_as_float(v[i]);
                            }
                        } else {
#pragma unroll
                            for (int c = 0; c < 8; ++c)
                                *reinterpret_cast<float4*>(sm + C::kOffW + mn_off(a, c)) =
                                    make_float4(tf32_rna(lambda * __uint_as_float(v[4 * c])),
                                                tf32_rna(lambda * __uint_as_float(v[4 * c + 1])),
                                                tf32_rna(lambda * __uint_as_float(v[4 * c + 2])),
                                                tf32_rna(lambda * __uint_as_float(v[4 * c + 3])));
                        }
                    }
                    continue;   // the writes reach the MMA with the next fence below (P1's epilogue)
                }
                // p == 0: -X = -sigma D into the X buffer (MN-major), T1 = 7I - X back into TMEM
#pragma unroll 1
                for (int jj = 0; jj < 2; ++jj) {
                    uint32_t v[32];
                    const uint32_t addr = d_col + lane_base + 64 * h + 32 * jj;
                    tmem_ld32(addr, v);
                    tmem_ld_wait();
                    const int a = 2 * h + jj;
                    float e[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i) e[i] = -sigma * __uint_as_float(v[i]);
#pragma unroll
                    for (int c = 0; c < 8; ++c)
                        *reinterpret_cast<float4*>(sm + C::kOffX + mn_off(a, c)) =
                            make_float4(tf32_rna(e[4 * c]), tf32_rna(e[4 * c + 1]), tf32_rna(e[4 * c + 2]),
                                        tf32_rna(e[4 * c + 3]));
                    if (diag_half && jj == diag_jj) {
#pragma unroll
                        for (int i = 0; i < 32; ++i) e[i] += i == lane ? 7.f : 0.f;
                    }
#pragma unroll
                    for (int i = 0; i < 32; ++i) v[i] = __float_as_uint(tf32_rna(e[i]));
                    tmem_st32(addr, v);
                }
                // R2 / R3 back to 15 I / 13 I: their last readers, the previous P3 and P4, completed
                // before this P1 (the tensor pipe runs in issue order). Written here, while the
                // tensor pipe is idle: stores that overlap an MMA run several times slower
                preset_diag(R2, 15.f);
                preset_diag(R3, 13.f);
                tmem_st_wait();
                fence_proxy_async_shared();   // -X (and the previous P4 epilogue's W rows) feed the MMA
                arrive_e();
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 9) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace nys
