// tc_pinv.cuh -- kernel_2 and the iterative Moore-Penrose inverse on tensor cores (tf32).
//
// Walkthrough (blog.gitcode.com) 2.4 (kernel_2 = softmax(Q_l K_l^T)) and 2.5:
//   Z_0 = c k2^T,  c = 1 / (max column sum * max row sum)
//   n_iter times:  X = k2 Z;  T1 = 7I - X;  T3 = 15I - X T1;  T5 = 13I - X T3;  Z = Z T5 / 4
//
// Matrices live in L2-resident global scratch in a "blocked swizzled" layout:
// the m x m fp32 matrix is cut into m/32 column atoms of 32 floats (one
// 128-byte line per row), atom-major, and inside every 1024-byte group the
// 16-byte chunks are XOR-swizzled with the row index -- exactly the 128-byte
// swizzled shared-memory layout the tcgen05 descriptors read. A K-major A
// operand chunk (128 rows x 32 columns) is then one contiguous 16 KB run, and
// a K-major B operand chunk (all m rows of B^T x 32 columns) is one contiguous
// run too, so plain bulk copies (cp.async.bulk) reproduce the swizzled layout
// in shared memory without tensor maps. Both operands are K-major (tf32 with an
// MN-major B is not used): every matrix that serves as a right-hand factor is
// written transposed by the epilogue that produces it.
//
// kernel2_kernel (CUDA cores): rows of S2 = Q_l K_l^T, row softmax, writes k2
// and k2^T (blocked, tf32-rounded to nearest) plus the column-sum partials and
// row sums that give c.
// pinv_tc_kernel: one CTA owns 128 rows of every product (m = 256: a cluster of
// two CTAs per head). Per product, thread 0 streams the operand chunks through a
// 3-stage ring and issues the tf32 MMAs; X = k2 Z stays in TMEM and feeds the
// next two products as the A operand straight from TMEM. The 128 threads then
// read their row of the accumulator, apply the scale / identity shift, round
// to tf32 and write it back to global scratch (transposed for T1, T3, T5 and
// Z^T, by rows for Z); a cluster barrier makes it visible to the other CTA
// before the next product. Iteration 0 never forms Z_0 = c k2^T: it reads k2
// (for Z_0^T) and k2^T (for the rows of Z_0) and applies c in the epilogues.
#pragma once

#include "sm100.cuh"

namespace nys {

// byte offset of element (r, c) of an m x m matrix in the blocked swizzled layout
__host__ __device__ __forceinline__ uint32_t bsw_offset(int r, int c, int m) {
    const uint32_t line = (uint32_t)((c >> 5) * m + r);
    const uint32_t chunk = (uint32_t)((c & 31) >> 2) ^ (uint32_t)(r & 7);
    return line * 128u + (chunk << 4) + (uint32_t)(c & 3) * 4u;
}

__device__ __forceinline__ float tf32_rna(float x) {
    uint32_t y;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(y) : "f"(x));
    return __uint_as_float(y);
}

// ------------------------------------------------------------------ kernel_2 rows
// grid (BH, m / 32), 256 threads. Dynamic shared memory: (32 + m) * (D + 1) floats.
// kPlain: k2 and k2^T are written row-major (for tensor-map loads); otherwise in
// the blocked swizzled layout above (for plain bulk copies).
template <int D, bool kPlain>
__global__ void __launch_bounds__(256)
kernel2_kernel(const float* __restrict__ ql, const float* __restrict__ kl, void* __restrict__ k2out,
               void* __restrict__ k2tout, float* __restrict__ colsum_part, float* __restrict__ rowsum,
               int m) {
    extern __shared__ float sm2[];
    constexpr int d = D, ld = D + 1;
    const int bh = blockIdx.x, blk = blockIdx.y, r0 = blk * 32;
    float* sq = sm2;                 // [32][d+1]
    float* sk = sm2 + 32 * ld;       // [m][d+1]
    float* ss = sk;                  // scores [32][m+1] reuse after the products (see below)
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const float4* qb = reinterpret_cast<const float4*>(ql + ((size_t)bh * m + r0) * d);
    const float4* kb = reinterpret_cast<const float4*>(kl + (size_t)bh * m * d);
    // stage Q_l rows and all of K_l; every thread issues its loads before its stores
    {
        constexpr int kQv = 32 * D / 4 / 256;   // float4 per thread for the 32 Q_l rows
        float4 qv[kQv];
#pragma unroll
        for (int e = 0; e < kQv; ++e) qv[e] = __ldg(qb + tid + e * 256);
#pragma unroll
        for (int e = 0; e < kQv; ++e) {
            const int idx = (tid + e * 256) * 4, r = idx / D, c = idx % D;
            sq[r * ld + c] = qv[e].x; sq[r * ld + c + 1] = qv[e].y;
            sq[r * ld + c + 2] = qv[e].z; sq[r * ld + c + 3] = qv[e].w;
        }
        const int nkv = m * D / 4;
        for (int base = 0; base < nkv; base += 256 * 8) {
            float4 kv[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const int idx = base + tid + e * 256;
                kv[e] = idx < nkv ? __ldg(kb + idx) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const int idx = base + tid + e * 256;
                if (idx < nkv) {
                    const int r = (idx * 4) / D, c = (idx * 4) % D;
                    sk[r * ld + c] = kv[e].x; sk[r * ld + c + 1] = kv[e].y;
                    sk[r * ld + c + 2] = kv[e].z; sk[r * ld + c + 3] = kv[e].w;
                }
            }
        }
    }
    __syncthreads();
    // each thread: rows (warp*4 .. +4), columns lane, lane+32, ...
    constexpr int kMaxCols = 8;   // m <= 256
    float acc[4][kMaxCols];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < kMaxCols; ++j) acc[i][j] = 0.f;
    for (int e = 0; e < d; ++e) {
        float a[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) a[i] = sq[(warp * 4 + i) * ld + e];
#pragma unroll
        for (int j = 0; j < kMaxCols; ++j) {
            const int c = lane + 32 * j;
            if (c < m) {
                const float b = sk[c * ld + e];
#pragma unroll
                for (int i = 0; i < 4; ++i) acc[i][j] = fmaf(a[i], b, acc[i][j]);
            }
        }
    }
    __syncthreads();   // sk is overwritten with the scores below
    const int lds = m + 1;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float mx = -INFINITY;
#pragma unroll
        for (int j = 0; j < kMaxCols; ++j)
            if (lane + 32 * j < m) mx = fmaxf(mx, acc[i][j]);
        mx = warp_max(mx);
        float s = 0.f;
#pragma unroll
        for (int j = 0; j < kMaxCols; ++j)
            if (lane + 32 * j < m) {
                acc[i][j] = __expf(acc[i][j] - mx);
                s += acc[i][j];
            }
        s = warp_sum(s);
        const float inv = 1.f / s;
        const int r = warp * 4 + i;
        float rs = 0.f;
#pragma unroll
        for (int j = 0; j < kMaxCols; ++j) {
            const int c = lane + 32 * j;
            if (c < m) {
                const float p = acc[i][j] * inv;
                ss[r * lds + c] = p;
                rs += p;
            }
        }
        rs = warp_sum(rs);
        if (lane == 0) rowsum[(size_t)bh * m + r0 + r] = rs;
    }
    __syncthreads();
    if constexpr (kPlain) {
        float* k2h = reinterpret_cast<float*>(k2out) + (size_t)bh * m * m;
        float* k2th = reinterpret_cast<float*>(k2tout) + (size_t)bh * m * m;
        // k2 rows r0 .. r0+31, 16 bytes per thread and step
        for (int e = tid; e < 32 * (m / 4); e += 256) {
            const int r = e / (m / 4), c = (e % (m / 4)) * 4;
            *reinterpret_cast<float4*>(k2h + (size_t)(r0 + r) * m + c) =
                make_float4(tf32_rna(ss[r * lds + c]), tf32_rna(ss[r * lds + c + 1]),
                            tf32_rna(ss[r * lds + c + 2]), tf32_rna(ss[r * lds + c + 3]));
        }
        // k2^T rows c, columns r0 .. r0+31: eight threads write one 128-byte segment
        for (int e = tid; e < m * 8; e += 256) {
            const int c = e >> 3, q = e & 7;
            *reinterpret_cast<float4*>(k2th + (size_t)c * m + r0 + 4 * q) =
                make_float4(tf32_rna(ss[(4 * q) * lds + c]), tf32_rna(ss[(4 * q + 1) * lds + c]),
                            tf32_rna(ss[(4 * q + 2) * lds + c]), tf32_rna(ss[(4 * q + 3) * lds + c]));
        }
        for (int c = tid; c < m; c += 256) {
            float cs = 0.f;
#pragma unroll 8
            for (int rr = 0; rr < 32; ++rr) cs += ss[rr * lds + c];
            colsum_part[((size_t)bh * (m / 32) + blk) * m + c] = cs;
        }
    } else {
        const size_t mat = (size_t)m * m * 4;
        uint8_t* k2h = reinterpret_cast<uint8_t*>(k2out) + (size_t)bh * mat;
        uint8_t* k2th = reinterpret_cast<uint8_t*>(k2tout) + (size_t)bh * mat;
        // k2 rows r0..r0+31: 16-byte chunks
        for (int e = tid; e < 32 * (m / 4); e += 256) {
            const int r = e / (m / 4), c = (e % (m / 4)) * 4;
            float4 v = make_float4(tf32_rna(ss[r * lds + c]), tf32_rna(ss[r * lds + c + 1]),
                                   tf32_rna(ss[r * lds + c + 2]), tf32_rna(ss[r * lds + c + 3]));
            *reinterpret_cast<float4*>(k2h + bsw_offset(r0 + r, c, m)) = v;
        }
        // k2^T: column c of this block is row c of k2^T, atom blk (32 floats = one line)
        for (int c = tid; c < m; c += 256) {
            float cs = 0.f;
#pragma unroll 4
            for (int q = 0; q < 8; ++q) {
                float4 v;
                v.x = ss[(4 * q + 0) * lds + c];
                v.y = ss[(4 * q + 1) * lds + c];
                v.z = ss[(4 * q + 2) * lds + c];
                v.w = ss[(4 * q + 3) * lds + c];
                cs += (v.x + v.y) + (v.z + v.w);
                v = make_float4(tf32_rna(v.x), tf32_rna(v.y), tf32_rna(v.z), tf32_rna(v.w));
                *reinterpret_cast<float4*>(k2th + bsw_offset(c, r0 + 4 * q, m)) = v;
            }
            colsum_part[((size_t)bh * (m / 32) + blk) * m + c] = cs;
        }
    }
}

// ------------------------------------------------------------------ the iteration
template <int M>
struct PinvTc {
    static constexpr int kStages = 3;
    static constexpr int kAtoms = M / 32;
    static constexpr uint32_t kAChunk = 128 * 128;          // 128 rows x 32 floats
    static constexpr uint32_t kBChunk = M * 128;             // M rows of B^T x 32 floats
    static constexpr uint32_t kStage = kAChunk + kBChunk;
    static constexpr uint32_t kOffBar = kStages * kStage;
    static constexpr uint32_t kOffMisc = kOffBar + (2 * kStages + 2) * 8;
    static constexpr uint32_t kSmemNeed = kOffMisc + 64 + 1024;
    // M = 256 takes all 512 TMEM columns: keep other TMEM users off the SM
    // at least 116 KB: one TMEM-using CTA per SM, so TMEM allocations never wait on each other
    static constexpr uint32_t kSmemBytes = kSmemNeed < 118784 ? 118784 : kSmemNeed;
    static constexpr int kTmemCols = 2 * M < 32 ? 32 : 2 * M;
    static constexpr int kClusterSize = M > 128 ? 2 : 1;
    static constexpr uint32_t kIdesc = sm100::make_idesc(128, M, sm100::kFmtTf32, sm100::kFmtTf32, 0, 0);
};

struct PinvTcParams {
    const uint8_t* k2b;        // [BH] blocked k2
    const uint8_t* k2tb;       // [BH] blocked k2^T
    uint8_t* zb;               // [BH] blocked Z (rows)
    uint8_t* ztb;              // [BH] blocked Z^T
    uint8_t* ta;               // [BH] blocked T buffers (ping-pong)
    uint8_t* tb;
    const float* colsum_part;  // [BH][m/32][m]
    const float* rowsum;       // [BH][m]
    float* z_out;              // [BH][m][m] row-major
    int n_iter;
    int inv_init;              // NYS_INV_INIT_DEFAULT or NYS_INV_INIT_EXACT
};

__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(sm100::smem_u32(dst)), "l"(src), "r"(bytes), "r"(sm100::smem_u32(bar))
        : "memory");
}
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

template <int M>
__global__ void __launch_bounds__(128, 1) pinv_tc_kernel(const PinvTcParams prm) {
    using C = PinvTc<M>;
    using namespace sm100;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(sm);
    uint64_t* full = reinterpret_cast<uint64_t*>(sm + C::kOffBar);
    uint64_t* empty = full + C::kStages;
    uint64_t* mma_done = empty + C::kStages;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + C::kOffMisc);
    float* red = reinterpret_cast<float*>(sm + C::kOffMisc + 16);   // [8]
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + C::kOffMisc + 48);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int rank = C::kClusterSize > 1 ? (int)cluster_rank() : 0;
    const int bh = blockIdx.x / C::kClusterSize;
    const int r0 = rank * 128;                      // first row this CTA owns
    const int row = r0 + tid;                       // this thread's row (TMEM lane tid)
    const bool row_ok = row < M;
    const int rows_valid = min(128, M - r0);
    const size_t mat = (size_t)M * M * 4;
    const uint8_t* k2 = prm.k2b + bh * mat;
    const uint8_t* k2t = prm.k2tb + bh * mat;
    uint8_t* zb = prm.zb + bh * mat;
    uint8_t* ztb = prm.ztb + bh * mat;
    uint8_t* ta = prm.ta + bh * mat;
    uint8_t* tb = prm.tb + bh * mat;

    if (tid == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(mma_done, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, C::kTmemCols);
        tmem_relinquish();
    }
    // c = 1 / (max column sum * max row sum) of this head's kernel_2 (default), or
    // 1 / max column sum (the exact-coefficient option)
    float mc = -INFINITY, mr = -INFINITY;
    for (int c = tid; c < M; c += 128) {
        float s = 0.f;
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
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // the exact-coefficient option drops the row factor (the row sums of a softmax are 1)
    const float coeff = 1.f / (fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3])) *
                               (prm.inv_init == NYS_INV_INIT_EXACT
                                    ? 1.f
                                    : fmaxf(fmaxf(red[4], red[5]), fmaxf(red[6], red[7]))));
    const uint32_t tmem = *tmem_slot;
    const uint32_t tX = tmem, tOut = tmem + M;      // accumulator regions (columns)
    const uint32_t lane_base = (uint32_t)(32 * warp) << 16;

    if (prm.n_iter == 0) {
        // Z = c k2^T, straight from the blocked k2^T
        if (row_ok)
            for (int c = 0; c < M; ++c)
                prm.z_out[((size_t)bh * M + row) * M + c] =
                    coeff * *reinterpret_cast<const float*>(k2t + bsw_offset(row, c, M));
    } else {
        // Failure handling: no thread ever leaves the sequence of barriers early.
        // A bounded wait that runs out marks the CTA as failed (CTA-uniform via
        // __syncthreads_or); later products then skip their copies and MMAs but
        // every barrier (CTA and cluster) is still passed the same number of times.
        int gchunk = 0;        // chunks issued so far (ring phase bookkeeping)
        int consumed = 0;      // chunks whose copies were waited for
        int ndone = 0;         // completed mma_done phases
        bool failed = false;   // CTA-uniform
        auto product = [&](const uint8_t* a_src, int a_tmem, const uint8_t* b_src, uint32_t d_col) {
            constexpr int nch = M / 32;
            bool ok0 = true;
            if (!failed) {
                if (tid == 0) {
                    auto issue = [&](int c) {
                        const int st = (gchunk + c) % C::kStages;
                        uint8_t* sa = sm + st * C::kStage;
                        uint8_t* sb = sa + C::kAChunk;
                        const uint32_t abytes = a_src ? (uint32_t)rows_valid * 128u : 0u;
                        mbar_arrive_expect_tx(&full[st], abytes + C::kBChunk);
                        if (a_src) bulk_g2s(sa, a_src + ((size_t)c * M + r0) * 128, abytes, &full[st]);
                        bulk_g2s(sb, b_src + (size_t)c * M * 128, C::kBChunk, &full[st]);
                    };
                    int issued = 0;
                    // prime the ring; a stage is free once the MMAs of its previous use completed
                    for (int c = 0; c < nch && c < C::kStages && ok0; ++c) {
                        const int g = gchunk + c, st = g % C::kStages;
                        ok0 = mbar_wait(&empty[st], ((g / C::kStages) & 1) ^ 1);
                        if (ok0) { issue(c); ++issued; }
                    }
                    for (int c = 0; c < nch && ok0; ++c) {
                        const int g = gchunk + c, st = g % C::kStages;
                        ok0 = mbar_wait(&full[st], (g / C::kStages) & 1);
                        if (!ok0) break;
                        ++consumed;
                        tc_fence_after();
                        const uint32_t sa = sbase + st * C::kStage, sb = sa + C::kAChunk;
                        // one operand form per group of four MMAs: a run-time choice between
                        // forms inside the group serialises the MMAs
                        if (a_src) {
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk)
                                mma_tf32_ss(d_col, smem_desc(sa + kk * 32, 16, 1024, kLayoutSw128),
                                            smem_desc(sb + kk * 32, 16, 1024, kLayoutSw128), C::kIdesc,
                                            (c > 0 || kk > 0) ? 1u : 0u);
                        } else {
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk)
                                mma_tf32_ts(d_col, (uint32_t)a_tmem + c * 32 + kk * 8,
                                            smem_desc(sb + kk * 32, 16, 1024, kLayoutSw128), C::kIdesc,
                                            (c > 0 || kk > 0) ? 1u : 0u);
                        }
                        mma_commit(&empty[st]);
                        // refill the stage of the previous chunk with chunk c - 1 + kStages
                        if (c >= 1 && c - 1 + C::kStages < nch) {
                            const int gp = g - 1, sp = gp % C::kStages;
                            ok0 = mbar_wait(&empty[sp], (gp / C::kStages) & 1);
                            if (ok0) { issue(c - 1 + C::kStages); ++issued; }
                        }
                    }
                    if (!ok0) {
                        // let the copies already issued land before anything else happens
                        for (int g = consumed; g < gchunk + issued; ++g)
                            mbar_wait(&full[g % C::kStages], (g / C::kStages) & 1);
                    }
                    mma_commit(mma_done);
                    gchunk += nch;
                    consumed = gchunk;
                }
                const bool done = mbar_wait(mma_done, ndone & 1);
                ++ndone;
                failed = __syncthreads_or((!done) || (tid == 0 && !ok0)) != 0;
                tc_fence_after();
            }
        };
        // epilogue: E[row][c] = alpha * D[row][c] + (c == row ? diag : 0), rounded to tf32 and
        // written to dst (blocked, by rows) and/or dst_t (blocked, transposed: E[row][c] goes to
        // row c, column row -- a warp's 32 rows fill one 128-byte line), or plain row-major fp32
        // for the final Z. Always ends with a CTA / cluster barrier.
        auto epilogue = [&](uint32_t d_col, float alpha, float diag, uint8_t* dst, uint8_t* dst_t, float* plain) {
            if (!failed) {
#pragma unroll 1
                for (int a = 0; a < C::kAtoms; ++a) {
                    uint32_t v[32];
                    tmem_ld32(d_col + lane_base + a * 32, v);
                    tmem_ld_wait();
                    if (row_ok) {
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            float f[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const int c = a * 32 + 4 * q + e;
                                f[e] = fmaf(alpha, __uint_as_float(v[4 * q + e]), c == row ? diag : 0.f);
                            }
                            if (plain) {
                                *reinterpret_cast<float4*>(plain + ((size_t)bh * M + row) * M + a * 32 + 4 * q) =
                                    make_float4(f[0], f[1], f[2], f[3]);
                                continue;
                            }
#pragma unroll
                            for (int e = 0; e < 4; ++e) f[e] = tf32_rna(f[e]);
                            if (dst)
                                *reinterpret_cast<float4*>(dst + bsw_offset(row, a * 32 + 4 * q, M)) =
                                    make_float4(f[0], f[1], f[2], f[3]);
                            if (dst_t) {
#pragma unroll
                                for (int e = 0; e < 4; ++e)
                                    *reinterpret_cast<float*>(dst_t + bsw_offset(a * 32 + 4 * q + e, row, M)) = f[e];
                            }
                        }
                    }
                }
                fence_proxy_async_global();
            }
            tc_fence_before();
            if (C::kClusterSize > 1) cluster_sync_all(); else __syncthreads();
            tc_fence_after();
        };
        for (int it = 0; it < prm.n_iter; ++it) {
            const float s_it = it == 0 ? coeff : 1.f;
            const uint8_t* zt_src = it == 0 ? k2 : ztb;     // Z^T (Z_0^T = c k2)
            const uint8_t* z_src = it == 0 ? k2t : zb;      // rows of Z (Z_0 = c k2^T)
            const bool last = it + 1 == prm.n_iter;
            product(k2, -1, zt_src, tX);                        // X = k2 Z
            epilogue(tX, -s_it, 7.f, nullptr, ta, nullptr);     // T1 = 7I - X      (stored transposed)
            product(nullptr, (int)tX, ta, tOut);               // U = X T1
            epilogue(tOut, -s_it, 15.f, nullptr, tb, nullptr);  // T3 = 15I - U     (transposed)
            product(nullptr, (int)tX, tb, tOut);               // T = X T3
            epilogue(tOut, -s_it, 13.f, nullptr, ta, nullptr);  // T5 = 13I - T     (transposed)
            product(z_src, -1, ta, tOut);                       // Z' = Z T5 / 4 (A = this CTA's rows of Z)
            if (last)
                epilogue(tOut, 0.25f * s_it, 0.f, nullptr, nullptr, prm.z_out);
            else
                epilogue(tOut, 0.25f * s_it, 0.f, zb, ztb, nullptr);
        }
        if (failed && tid == 0) *abort_flag = 1;
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
    if (C::kClusterSize > 1) cluster_sync_all();   // keep the pair resident until both are done
}

}  // namespace nys
