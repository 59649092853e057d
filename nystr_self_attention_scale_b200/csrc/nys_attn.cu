// nys_attn.cu -- C ABI and launch sequence of the Nystromformer attention forward.
//
// Per call (walkthrough, blog.gitcode.com, section 2):
//   1. landmarks: fused d^-1/4 scale + segment means of Q and K      (2.2, 2.3)
//   2. kernel_2 + iterative inverse -> Z, on a forked stream           (2.4, 2.5)
//   3. kernel_3 V: online softmax over key splits + combine            (2.4)
//   4. W = Z (kernel_3 V)                                              (2.4)
//   5. output: softmax(Qs K_l^T) W + dwconv65(V)                       (2.4, 2.6)
// Steps 2 and 3 are independent and overlap; 4 joins them.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdio>
#include <cstring>
#include <atomic>
#include <mutex>
#include <type_traits>
#include <vector>

#include "common.cuh"
#include "exact.cuh"
#include "landmarks.cuh"
#include "probs.cuh"
#include "simt.cuh"
#include "tc_k3v.cuh"
#include "tc_output.cuh"
#include "tc_pinv_pair.cuh"
#include "tc_pinv_res.cuh"
#include "tc_w.cuh"

namespace nys {
namespace {

constexpr int kMaxDevices = 64;
constexpr int kHostChunks = 8;   // pipeline depth of the host entry (copies overlap compute)

struct DeviceState {
    bool ready = false;
    int sm_count = 0;
    cudaStream_t aux = nullptr;       // forked stream for kernel_3 V (bf16) or the inverse (float32)
    cudaEvent_t fork = nullptr, join = nullptr;
    cudaEvent_t started = nullptr;    // every CTA of the CTA-pair inverse has begun
    std::mutex launch_mu;             // serialises the fork/join event use of one device
    // host entry: copy streams and the events of its chunk pipeline
    cudaStream_t copy_in = nullptr, copy_out = nullptr;
    cudaEvent_t alloc_ev = nullptr, in_ev[kHostChunks] = {}, done_ev[kHostChunks] = {}, out_ev = nullptr;
    std::mutex host_mu;               // one host-entry call per device at a time
};

std::mutex g_mu;
DeviceState g_dev[kMaxDevices];

int device_state(DeviceState** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return NYS_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    DeviceState& st = g_dev[dev];
    if (!st.ready) {
        if (cudaDeviceGetAttribute(&st.sm_count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return NYS_ERR_CUDA;
        if (cudaStreamCreateWithFlags(&st.aux, cudaStreamNonBlocking) != cudaSuccess) return NYS_ERR_CUDA;
        if (cudaEventCreateWithFlags(&st.fork, cudaEventDisableTiming) != cudaSuccess) return NYS_ERR_CUDA;
        if (cudaEventCreateWithFlags(&st.join, cudaEventDisableTiming) != cudaSuccess) return NYS_ERR_CUDA;
        if (cudaEventCreateWithFlags(&st.started, cudaEventDisableTiming) != cudaSuccess) return NYS_ERR_CUDA;
        if (cudaStreamCreateWithFlags(&st.copy_in, cudaStreamNonBlocking) != cudaSuccess) return NYS_ERR_CUDA;
        if (cudaStreamCreateWithFlags(&st.copy_out, cudaStreamNonBlocking) != cudaSuccess) return NYS_ERR_CUDA;
        if (cudaEventCreateWithFlags(&st.alloc_ev, cudaEventDisableTiming) != cudaSuccess) return NYS_ERR_CUDA;
        if (cudaEventCreateWithFlags(&st.out_ev, cudaEventDisableTiming) != cudaSuccess) return NYS_ERR_CUDA;
        for (int c = 0; c < kHostChunks; ++c)
            if (cudaEventCreateWithFlags(&st.in_ev[c], cudaEventDisableTiming) != cudaSuccess ||
                cudaEventCreateWithFlags(&st.done_ev[c], cudaEventDisableTiming) != cudaSuccess)
                return NYS_ERR_CUDA;
        // Keep freed async allocations in the pool so per-call workspace is cheap.
        cudaMemPool_t pool;
        if (cudaDeviceGetDefaultMemPool(&pool, dev) == cudaSuccess) {
            uint64_t keep = UINT64_MAX;
            cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep);
        }
        const size_t big = 200 * 1024;
        cudaFuncSetAttribute(k3v_partial_simt_kernel<float, 32>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)big);
        cudaFuncSetAttribute(k3v_partial_simt_kernel<float, 64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)big);
        cudaFuncSetAttribute(output_simt_kernel<float, 32>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)big);
        cudaFuncSetAttribute(output_simt_kernel<float, 64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)big);
        cudaFuncSetAttribute(pinv_simt_smem_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kPinvSmemBytes);
        if (cudaGetLastError() != cudaSuccess) return NYS_ERR_CUDA;
        st.ready = true;
    }
    *out = &st;
    return NYS_OK;
}

size_t align_up(size_t x) { return (x + 255) & ~size_t(255); }

// ---------------------------------------------------------------- workspace guard mode
// With the guard mode on (nys_attn_set_workspace_guard), every workspace buffer sits between
// guard zones, the whole workspace is filled with 0xFF bytes before the first launch (a NaN
// in fp32 and bf16, so a read of an element no kernel wrote poisons the result), and after
// the last launch one CTA per zone checks that every guard byte is still 0xFF; a changed
// byte records NYS_ERR_GUARD in the device status word.
constexpr size_t kGuardBytes = 4096;
constexpr int kMaxGuards = 17;   // make_plan takes at most 16 buffers, + a trailing zone
std::atomic<int> g_guard_mode{0};

struct GuardList {
    unsigned long long off[kMaxGuards];
    int n;
};

__global__ void guard_check_kernel(const uint32_t* __restrict__ ws, const GuardList zones) {
    const uint32_t* z = ws + zones.off[blockIdx.x] / 4;
    bool bad = false;
    for (int i = threadIdx.x; i < (int)(kGuardBytes / 4); i += blockDim.x) bad |= z[i] != 0xFFFFFFFFu;
    if (__syncthreads_or(bad) && threadIdx.x == 0) record_status(NYS_ERR_GUARD);
}

// [B, n] uint8 key mask -> [B, n / 32] validity bits (bit i of word w = key 32 w + i).
__global__ void mask_bits_kernel(const uint8_t* __restrict__ mask, uint32_t* __restrict__ bits, int B, int n) {
    const int words = n / 32;
    const int w = blockIdx.x * blockDim.x + threadIdx.x;
    if (w >= B * words) return;
    const int b = w / words, wi = w % words;
    const uint4* src = reinterpret_cast<const uint4*>(mask + (size_t)b * n + (size_t)wi * 32);
    uint32_t v = 0;
#pragma unroll
    for (int q = 0; q < 2; ++q) {
        const uint4 u = src[q];
        const uint32_t x[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int e = 0; e < 16; ++e)
            v |= (((x[e >> 2] >> ((e & 3) * 8)) & 0xFFu) != 0u ? 1u : 0u) << (q * 16 + e);
    }
    bits[w] = v;
}

// ---------------------------------------------------------------- TMA tensor maps
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
        cudaGetLastError();
    });
    return fn;
}

// 3-D tensor map over a row-major [d2][d1][d0] array of `elt`-byte elements,
// box b0 x b1 x 1, out-of-bounds elements read as zero.
bool map_3d(CUtensorMap* m, CUtensorMapDataType dt, uint32_t elt, const void* base, uint64_t d0, uint64_t d1,
            uint64_t d2, uint32_t b0, uint32_t b1, CUtensorMapSwizzle sw) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {d0, d1, d2};
    const cuuint64_t strides[2] = {d0 * elt, d0 * d1 * elt};
    const cuuint32_t box[3] = {b0, b1, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, dt, 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool map_bf16_3d(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint32_t b0,
                 uint32_t b1, CUtensorMapSwizzle sw) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {d0, d1, d2};
    const cuuint64_t strides[2] = {d0 * 2, d0 * d1 * 2};
    const cuuint32_t box[3] = {b0, b1, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ---------------------------------------------------------------- per-kernel timing
// When enabled, every launch is bracketed by two CUDA events on the stream it
// runs on; nys_attn_profile_read() sums their elapsed times per kernel.
enum KernelId { K_LANDMARKS = 0, K_PINV, K_K3V, K_COMBINE, K_W, K_OUTPUT, K_MASKBITS, K_PROBS,
                K_COUNT };
const char* const kKernelNames[K_COUNT] = {"landmarks", "pinv", "k3v_partial", "k3v_combine",
                                           "w_product", "output", "mask_bits", "attn_probs"};

struct ProfRecord { int kid; cudaEvent_t a, b; };
std::mutex g_prof_mu;
bool g_prof_on = false;
unsigned int g_prof_mask = ~0u;   // kernels whose launches are timed
std::vector<ProfRecord> g_prof;
int g_prof_launches[K_COUNT];
double g_prof_ms[K_COUNT];

struct ProfScope {
    int kid;
    cudaStream_t s;
    cudaEvent_t a = nullptr, b = nullptr;
    ProfScope(int kid_, cudaStream_t s_) : kid(kid_), s(s_) {
        if (!g_prof_on || !((g_prof_mask >> kid) & 1u)) return;
        cudaEventCreate(&a);
        cudaEventCreate(&b);
        cudaEventRecord(a, s);
    }
    ~ProfScope() {
        if (!a) return;
        cudaEventRecord(b, s);
        std::lock_guard<std::mutex> lock(g_prof_mu);
        g_prof.push_back({kid, a, b});
    }
};

void prof_drain() {
    std::lock_guard<std::mutex> lock(g_prof_mu);
    for (auto& r : g_prof) {
        float ms = 0.f;
        if (cudaEventSynchronize(r.b) == cudaSuccess && cudaEventElapsedTime(&ms, r.a, r.b) == cudaSuccess) {
            g_prof_ms[r.kid] += ms;
            g_prof_launches[r.kid] += 1;
        }
        cudaEventDestroy(r.a);
        cudaEventDestroy(r.b);
    }
    g_prof.clear();
}

// Workspace carve-up (byte offsets, each 256-byte aligned).
struct Plan {
    int B, H, n, d, m, n_iter, dtype;
    int BH, splits, keys_per_split;
    size_t off_ql, off_kl, off_ql16, off_kl16, off_k3v, off_w, off_wt16, off_z, off_pinv;
    size_t off_po, off_pm, off_pl, off_mbits, total;
    size_t off_k2b, off_zb;   // CTA-pair inverse (m = 256): k2 and W^T scratch
    int tc_cps, tc_splits;  // tensor-core kernel_3 V: 128-key chunks per split, splits
    GuardList guards;       // guard zones (guard mode only; guards.n == 0 otherwise)
};

// Per-call options beyond the spec signature (nys_attn_forward_ex).
struct Options {
    int inv_init = NYS_INV_INIT_DEFAULT;   // Z_0 scaling of the iterative inverse
    bool exact = false;                    // path A: exact softmax attention (m, n_iter unused)
    float* attn_probs = nullptr;           // optional [B, H, n, m] (or [B, H, n, n] exact) weights
};

// Argument checks of the exact branch (walkthrough 2.1, path A): no landmarks.
int validate_exact(const void* q, const void* k, const void* v, const void* out, int B, int H, int n,
                   int d, int dtype) {
    if (!q || !k || !v || !out) return NYS_ERR_INVALID_ARG;
    if (B <= 0 || H <= 0 || n <= 0 || d <= 0) return NYS_ERR_INVALID_ARG;
    if (dtype != NYS_F32 && dtype != NYS_BF16) return NYS_ERR_UNSUPPORTED;
    if (d != 32 && d != 64) return NYS_ERR_UNSUPPORTED;
    if (dtype == NYS_BF16 && n % 128 != 0) return NYS_ERR_UNSUPPORTED;
    if ((long long)B * H > (1 << 24) || n / 64 >= 65535) return NYS_ERR_UNSUPPORTED;
    return NYS_OK;
}

int validate(const void* q, const void* k, const void* v, const void* out, int B, int H, int n,
             int d, int m, int n_iter, int dtype) {
    if (!q || !k || !v || !out) return NYS_ERR_INVALID_ARG;
    if (B <= 0 || H <= 0 || n <= 0 || d <= 0 || m <= 0 || n_iter < 0) return NYS_ERR_INVALID_ARG;
    if (n % m != 0 || m > n) return NYS_ERR_INVALID_ARG;
    if (dtype != NYS_F32 && dtype != NYS_BF16) return NYS_ERR_UNSUPPORTED;
    if (d != 32 && d != 64) return NYS_ERR_UNSUPPORTED;
    if (m > 256) return NYS_ERR_UNSUPPORTED;
    if (dtype == NYS_BF16 && ((m != 64 && m != 128 && m != 256) || n % 128 != 0))
        return NYS_ERR_UNSUPPORTED;
    if ((long long)B * H > (1 << 24) || n / 64 >= 65535) return NYS_ERR_UNSUPPORTED;
    return NYS_OK;
}

// Workspace of the exact branch: the key-split partials of softmax(Qs Ks^T + mask) V over all
// n query rows, and the packed key-mask bits. The key split depends on n only, as on the
// Nystrom path: one split up to n = 8192 (the rows already give B*H*n/128 work items).
Plan make_plan_exact(int B, int H, int n, int d, int dtype) {
    Plan p{};
    p.B = B; p.H = H; p.n = n; p.d = d; p.m = n; p.n_iter = 0; p.dtype = dtype;
    p.BH = B * H;
    int kps = std::min(((n + 63) / 64) * 64, 1024);
    int splits = (n + kps - 1) / kps;
    if (dtype == NYS_BF16) {
        const int chunks = n / 128;
        p.tc_cps = std::min(chunks, 64);
        p.tc_splits = (chunks + p.tc_cps - 1) / p.tc_cps;
        splits = p.tc_splits;
        kps = p.tc_cps * 128;
    }
    p.splits = splits;
    p.keys_per_split = kps;
    const size_t BH = p.BH;
    size_t o = 0;
    const bool guard = g_guard_mode.load() != 0;
    p.guards.n = 0;
    auto zone = [&]() {
        if (p.guards.n < kMaxGuards) p.guards.off[p.guards.n++] = o;
        o += kGuardBytes;
    };
    auto take = [&](size_t bytes) {
        if (guard) zone();
        size_t r = o;
        o = align_up(o + bytes);
        return r;
    };
    p.off_po = take(BH * splits * (size_t)n * d * 4);
    p.off_pm = take(BH * splits * (size_t)n * 4);
    p.off_pl = take(BH * splits * (size_t)n * 4);
    p.off_mbits = take((size_t)B * ((n + 31) / 32) * 4);
    if (guard) zone();
    p.total = o;
    return p;
}

Plan make_plan(int B, int H, int n, int d, int m, int n_iter, int dtype, int sm_count) {
    Plan p{};
    p.B = B; p.H = H; p.n = n; p.d = d; p.m = m; p.n_iter = n_iter; p.dtype = dtype;
    p.BH = B * H;
    // The key split depends on n only (never on B*H or the GPU), so a head's
    // result is bitwise the same alone or inside any batch.
    (void)sm_count;
    int kps = std::min(((n + 63) / 64) * 64, 1024);
    int splits = (n + kps - 1) / kps;
    if (dtype == NYS_BF16) {
        const int chunks = n / 128;
        // 26 chunks (3328 keys) per split from n = 16384 on: fewer, larger items (5 splits at
        // n = 16384) and fewer partials to merge
        p.tc_cps = std::min(chunks, n >= 16384 ? 26 : 8);
        p.tc_splits = (chunks + p.tc_cps - 1) / p.tc_cps;
        splits = p.tc_splits;
        kps = p.tc_cps * 128;
    }
    p.splits = splits;
    p.keys_per_split = kps;
    const size_t BH = p.BH, md = (size_t)m * d, mm = (size_t)m * m;
    size_t o = 0;
    const bool guard = g_guard_mode.load() != 0;
    p.guards.n = 0;
    auto zone = [&]() {
        if (p.guards.n < kMaxGuards) p.guards.off[p.guards.n++] = o;
        o += kGuardBytes;
    };
    auto take = [&](size_t bytes) {
        if (guard) zone();
        size_t r = o;
        o = align_up(o + bytes);
        return r;
    };
    p.off_ql = take(BH * md * 4);
    p.off_kl = take(BH * md * 4);
    p.off_ql16 = take(BH * md * 2);
    p.off_kl16 = take(BH * md * 2);
    p.off_k3v = take(BH * md * 4);
    p.off_w = take(BH * md * 4);
    p.off_wt16 = take(BH * md * 2);
    p.off_z = take(BH * mm * 4);
    p.off_pinv = take(dtype == NYS_F32 ? BH * 5 * mm * 4 : 0);
    p.off_po = take(BH * splits * md * 4);
    p.off_pm = take(BH * splits * (size_t)m * 4);
    p.off_pl = take(BH * splits * (size_t)m * 4);
    p.off_mbits = take((size_t)B * ((n + 31) / 32) * 4);
    if (dtype == NYS_BF16 && m == 256) {
        p.off_k2b = take(BH * mm * 4);
        p.off_zb = take(BH * mm * 4);
    }
    if (guard) zone();
    p.total = o;
    return p;
}

// Guard mode: fill the workspace before the first launch, check its guard zones after the last.
int guard_fill(const Plan& p, void* ws, cudaStream_t s) {
    if (p.guards.n == 0) return NYS_OK;
    return cudaMemsetAsync(ws, 0xFF, p.total, s) == cudaSuccess ? NYS_OK : NYS_ERR_CUDA;
}

int guard_check(const Plan& p, const void* ws, cudaStream_t s) {
    if (p.guards.n == 0) return NYS_OK;
    guard_check_kernel<<<p.guards.n, 256, 0, s>>>(static_cast<const uint32_t*>(ws), p.guards);
    return cudaGetLastError() == cudaSuccess ? NYS_OK : NYS_ERR_CUDA;
}

template <typename T, int D>
int launch_simt(const Plan& p, const DeviceState& st, const T* q, const T* k, const T* v,
               const uint8_t* mask, const float* conv_w, T* out, char* ws, int inv_init, cudaStream_t s) {
    float* ql = reinterpret_cast<float*>(ws + p.off_ql);
    float* kl = reinterpret_cast<float*>(ws + p.off_kl);
    float* k3v = reinterpret_cast<float*>(ws + p.off_k3v);
    float* w = reinterpret_cast<float*>(ws + p.off_w);
    float* z = reinterpret_cast<float*>(ws + p.off_z);
    float* pinv = reinterpret_cast<float*>(ws + p.off_pinv);
    float* po = reinterpret_cast<float*>(ws + p.off_po);
    float* pm = reinterpret_cast<float*>(ws + p.off_pm);
    float* pl = reinterpret_cast<float*>(ws + p.off_pl);
    const int BH = p.BH, n = p.n, m = p.m;

    {
        constexpr int V = Elt<T>::kVec;
        long long threads = (long long)BH * m * (D / V);
        dim3 grid((unsigned)((threads + 255) / 256), 2);
        ProfScope ps(K_LANDMARKS, s);
        landmarks_kernel<T><<<grid, 256, 0, s>>>(q, k, ql, kl, nullptr, nullptr, BH, n, D, m);
    }
    if (cudaEventRecord(st.fork, s) != cudaSuccess) return NYS_ERR_CUDA;
    if (cudaStreamWaitEvent(st.aux, st.fork, 0) != cudaSuccess) return NYS_ERR_CUDA;
    {
        ProfScope ps(K_PINV, st.aux);
        if (m <= 64)
            pinv_simt_smem_kernel<<<BH, 256, kPinvSmemBytes, st.aux>>>(ql, kl, z, m, D, p.n_iter, inv_init);
        else
            pinv_simt_kernel<<<BH, 256, 0, st.aux>>>(ql, kl, z, pinv, m, D, p.n_iter, inv_init);
    }
    if (cudaEventRecord(st.join, st.aux) != cudaSuccess) return NYS_ERR_CUDA;
    {
        dim3 grid(BH, (m + 63) / 64, p.splits);
        {
            ProfScope ps(K_K3V, s);
            k3v_partial_simt_kernel<T, D><<<grid, 256, k3v_simt_smem_bytes<D>(), s>>>(
                ql, k, v, mask, po, pm, pl, p.H, n, m, p.splits, p.keys_per_split, 1.f);
        }
        const long long threads = (long long)BH * m * (D / 4);
        ProfScope ps(K_COMBINE, s);
        k3v_combine_kernel<<<(unsigned)((threads + 255) / 256), 256, 0, s>>>(po, pm, pl, k3v, BH, m, D, p.splits);
    }
    if (cudaStreamWaitEvent(s, st.join, 0) != cudaSuccess) return NYS_ERR_CUDA;
    {
        ProfScope ps(K_W, s);
        w_kernel<D><<<dim3(BH, (m + 63) / 64), 256, 0, s>>>(z, k3v, w, nullptr, m);
    }
    {
        dim3 grid(BH, (n + 63) / 64);
        ProfScope ps(K_OUTPUT, s);
        output_simt_kernel<T, D><<<grid, 256, OutSmem<T, D>::bytes(m), s>>>(q, kl, w, v, conv_w, out,
                                                                          p.H, n, m);
    }
    return cudaGetLastError() == cudaSuccess ? NYS_OK : NYS_ERR_CUDA;
}

// Contiguous tile ranges for the output pass's persistent CTAs. A range that crosses into a new
// head pays for the change of per-head constants (the pipeline drains, the Toeplitz strip is
// rebuilt): about two tiles' time. The ranges are chosen greedily against a bound C on
// (tiles + 2 per head crossed), none longer than an even share of the tiles left, with the
// smallest C that fits `ctas` ranges (binary search); where no range crosses, this is the even
// split. Writes ctas + 1 boundaries.
void output_tile_ranges(int total, int tph, int ctas, int* start) {
    constexpr long long kCross = 2;
    // head starts strictly inside the range of `len` tiles from `first` (its first tile excluded)
    auto crossings = [&](long long first, long long len) {
        return len <= 1 ? 0LL : (first + len - 1) / tph - first / tph;
    };
    auto fill = [&](long long C, bool write) {
        long long t = 0;
        int b = 0;
        for (; b < ctas && t < total; ++b) {
            // no more tiles than an even share of what is left, so that ranges that cross no head
            // are not packed beyond the even split; then the longest range within the bound C
            // (its cost grows with its length)
            const long long cap = std::min<long long>((total - t + (ctas - b) - 1) / (ctas - b), total - t);
            long long lo = 1, hi = cap;
            while (lo < hi) {
                const long long mid = (lo + hi + 1) / 2;
                if (mid + kCross * crossings(t, mid) <= C) lo = mid;
                else hi = mid - 1;
            }
            if (write) start[b] = (int)t;
            t += lo;
        }
        if (t < total) return false;
        if (write)
            for (; b <= ctas; ++b) start[b] = total;
        return true;
    };
    // the even split costs at most (1 + kCross) per tile, so fill(hi) succeeds; fill(lo) fails
    const long long even = (total + ctas - 1) / ctas;
    long long lo = even - 1, hi = even * (1 + kCross);
    while (hi - lo > 1) {
        const long long mid = (lo + hi) / 2;
        (fill(mid, false) ? hi : lo) = mid;
    }
    fill(hi, true);
}

template <int D, int M>
int launch_output_tc(const Plan& p, const DeviceState& st, const __nv_bfloat16* q, const __nv_bfloat16* v,
                     const float* conv_w, __nv_bfloat16* out, const __nv_bfloat16* kl16,
                     const __nv_bfloat16* wt16, cudaStream_t s) {
    using C = OutTc<D, M>;
    CUtensorMap mq, mv, mo, mkl, mwt;
    const CUtensorMapSwizzle sw = D == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
    const uint64_t BH = p.BH, n = p.n;
    if (!map_bf16_3d(&mq, q, D, n, BH, D, 128, sw) || !map_bf16_3d(&mv, v, D, n, BH, D, 192, sw) ||
        !map_bf16_3d(&mo, out, D, n, BH, D, 128, sw) || !map_bf16_3d(&mkl, kl16, D, M, BH, D, M, sw) ||
        !map_bf16_3d(&mwt, wt16, M, D, BH, 64, D, CU_TENSOR_MAP_SWIZZLE_128B))
        return NYS_ERR_CUDA;
    OutTcParams prm{conv_w, p.H, p.n, p.n / 128, p.BH * (p.n / 128), {}};
    const int grid = std::min(std::min(prm.total_tiles, st.sm_count), kOutMaxCtas);
    output_tile_ranges(prm.total_tiles, prm.tiles_per_head, grid, prm.tile_start);
    static bool attr_set[kMaxDevices] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (!attr_set[dev]) {
        if (cudaFuncSetAttribute(output_tc_kernel<D, M>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)C::kSmemBytes) != cudaSuccess)
            return NYS_ERR_CUDA;
        attr_set[dev] = true;
    }
    // programmatic dependent launch: the kernel may start while W (the kernel before it on this
    // stream) finishes; it waits for W's completion before loading W^T
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(480);
    cfg.dynamicSmemBytes = C::kSmemBytes;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    ProfScope ps(K_OUTPUT, s);
    if (cudaLaunchKernelEx(&cfg, output_tc_kernel<D, M>, mq, mv, mo, mkl, mwt, prm) != cudaSuccess)
        return NYS_ERR_CUDA;
    return NYS_OK;
}

// kernel_3 V on the tensor cores; `rows` is the row operand [BH, p.m, D] bf16: the landmarks
// Q_l (scaled by d^-1/4 already, so the exponent carries K's d^-1/4) or, on the exact branch,
// the raw queries (p.m = n; the exponent carries the whole d^-1/2).
template <int D>
int launch_k3v_tc(const Plan& p, const DeviceState& st, const __nv_bfloat16* rows, const __nv_bfloat16* k,
                  const __nv_bfloat16* v, const uint32_t* mbits, float* po, float* pm, float* pl, int sms,
                  float score_scale, cudaStream_t s) {
    using C = K3vTc<D>;
    CUtensorMap mql, mk, mv;
    const CUtensorMapSwizzle sw = D == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
    const uint64_t BH = p.BH, n = p.n, m = p.m;
    if (!map_bf16_3d(&mql, rows, D, m, BH, D, 128, sw) || !map_bf16_3d(&mk, k, D, n, BH, D, 128, sw) ||
        !map_bf16_3d(&mv, v, D, n, BH, D, 128, sw))
        return NYS_ERR_CUDA;
    const int halves = (p.m + 127) / 128;
    K3vTcParams prm{mbits, po, pm, pl, p.H, p.n, p.m, halves, p.tc_splits, p.tc_cps,
                    p.BH * halves * p.tc_splits, score_scale};
    const int grid = std::min(prm.total_items, sms);
    static bool attr_set[kMaxDevices] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (!attr_set[dev]) {
        if (cudaFuncSetAttribute(k3v_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)C::kSmemBytes) != cudaSuccess)
            return NYS_ERR_CUDA;
        attr_set[dev] = true;
    }
    ProfScope ps(K_K3V, s);
    k3v_tc_kernel<D><<<grid, C::kThreads, C::kSmemBytes, s>>>(mql, mk, mv, prm);
    return NYS_OK;
}

// m = 64 and 128: kernel_2 and the iterative inverse in one CTA per 128 rows (two heads per CTA
// at m = 64), every operand on chip. `started` (or null) fires once every CTA has begun.
template <int MH>
int launch_pinv_res(const Plan& p, const float* ql, const float* kl, float* z, int inv_init, cudaStream_t s,
                    cudaEvent_t started) {
    using C = PinvRes<MH>;
    static bool attr_set[kMaxDevices] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (!attr_set[dev]) {
        if (cudaFuncSetAttribute(pinv_res_kernel<MH>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)C::kSmemBytes) != cudaSuccess)
            return NYS_ERR_CUDA;
        attr_set[dev] = true;
    }
    PinvResMaps maps;
    const uint64_t BH = p.BH;
    const auto f32 = CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
    if (!map_3d(&maps.ql, f32, 4, ql, p.d, MH, BH, 32, MH, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !map_3d(&maps.kl, f32, 4, kl, p.d, MH, BH, 32, MH, CU_TENSOR_MAP_SWIZZLE_128B))
        return NYS_ERR_CUDA;
    PinvResParams prm{z, p.BH, p.d, p.n_iter, inv_init};
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((p.BH + C::kHeads - 1) / C::kHeads);
    cfg.blockDim = dim3(C::kThreads);
    cfg.dynamicSmemBytes = C::kSmemBytes;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeLaunchCompletionEvent;
    attr[0].val.launchCompletionEvent.event = started;
    attr[0].val.launchCompletionEvent.flags = 0;
    cfg.attrs = attr;
    cfg.numAttrs = started != nullptr ? 1 : 0;
    ProfScope ps(K_PINV, s);
    if (cudaLaunchKernelEx(&cfg, pinv_res_kernel<MH>, maps, prm) != cudaSuccess) return NYS_ERR_CUDA;
    return NYS_OK;
}

// m = 256: kernel_2 and the iterative inverse in one CTA-pair kernel.
int launch_pinv_pair(const Plan& p, const DeviceState& st, const float* ql, const float* kl, float* z, char* ws,
                     int inv_init, cudaStream_t s, cudaEvent_t started) {
    using C = PinvPair;
    constexpr int M = 256;
    static bool attr_set[kMaxDevices] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (!attr_set[dev]) {
        if (cudaFuncSetAttribute(pinv_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)C::kSmemBytes) != cudaSuccess)
            return NYS_ERR_CUDA;
        attr_set[dev] = true;
    }
    float* k2 = reinterpret_cast<float*>(ws + p.off_k2b);
    float* zs = reinterpret_cast<float*>(ws + p.off_zb);
    PinvPairMaps maps;
    const uint64_t BH = p.BH;
    const auto f32 = CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
    const auto sw = CU_TENSOR_MAP_SWIZZLE_128B;
    if (!map_3d(&maps.ql, f32, 4, ql, p.d, M, BH, 32, 128, sw) ||
        !map_3d(&maps.kl, f32, 4, kl, p.d, M, BH, 32, 128, sw) ||
        !map_3d(&maps.k2, f32, 4, k2, M, M, BH, 32, 128, sw) ||
        !map_3d(&maps.k2mn, f32, 4, k2, M, M, BH, 32, 32, CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B) ||
        !map_3d(&maps.wt, f32, 4, zs, M, M, BH, 32, 128, sw))
        return NYS_ERR_CUDA;
    PinvPairParams prm{k2, zs, z, p.d, p.n_iter, inv_init};
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.BH * 2);
    cfg.blockDim = dim3(C::kThreads);
    cfg.dynamicSmemBytes = C::kSmemBytes;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    // `started` fires once every CTA pair has begun: kernel_3 V is held back until then, so
    // that its persistent grid takes the SMs the pairs leave instead of splitting SM pairs
    attr[1].id = cudaLaunchAttributeLaunchCompletionEvent;
    attr[1].val.launchCompletionEvent.event = started;
    attr[1].val.launchCompletionEvent.flags = 0;
    cfg.attrs = attr;
    cfg.numAttrs = started != nullptr ? 2 : 1;
    ProfScope ps(K_PINV, s);
    if (cudaLaunchKernelEx(&cfg, pinv_pair_kernel, maps, prm) != cudaSuccess) return NYS_ERR_CUDA;
    return NYS_OK;
}

template <int D>
int launch_bf16(const Plan& p, const DeviceState& st, const __nv_bfloat16* q, const __nv_bfloat16* k,
                const __nv_bfloat16* v, const uint8_t* mask, const float* conv_w, __nv_bfloat16* out, char* ws,
                int inv_init, cudaStream_t s) {
    using bf = __nv_bfloat16;
    float* ql = reinterpret_cast<float*>(ws + p.off_ql);
    float* kl = reinterpret_cast<float*>(ws + p.off_kl);
    bf* ql16 = reinterpret_cast<bf*>(ws + p.off_ql16);
    bf* kl16 = reinterpret_cast<bf*>(ws + p.off_kl16);
    float* k3v = reinterpret_cast<float*>(ws + p.off_k3v);
    float* w = reinterpret_cast<float*>(ws + p.off_w);
    bf* wt16 = reinterpret_cast<bf*>(ws + p.off_wt16);
    float* z = reinterpret_cast<float*>(ws + p.off_z);
    float* po = reinterpret_cast<float*>(ws + p.off_po);
    float* pm = reinterpret_cast<float*>(ws + p.off_pm);
    float* pl = reinterpret_cast<float*>(ws + p.off_pl);
    uint32_t* mbits = mask ? reinterpret_cast<uint32_t*>(ws + p.off_mbits) : nullptr;
    const int BH = p.BH, n = p.n, m = p.m;
    int rc = NYS_OK;
    {
        ProfScope ps(K_LANDMARKS, s);
        constexpr int rows_per_instr = 32 / (D / 8);
        if ((n / m) % rows_per_instr == 0) {
            // as many CTAs of eight warps per SM as fit, striding over the landmarks, and just
            // enough of them that every warp takes the same number of landmarks (no partly-filled
            // last round)
            static int per_sm[kMaxDevices] = {};
            int dev = 0;
            cudaGetDevice(&dev);
            if (per_sm[dev] == 0 &&
                (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm[dev], landmarks_warp_kernel<D>, 256, 0) !=
                     cudaSuccess ||
                 per_sm[dev] < 1)) {
                per_sm[dev] = 0;
                return NYS_ERR_CUDA;
            }
            const long long units = 2LL * BH * m, slots = 8LL * per_sm[dev] * st.sm_count;
            const long long per_warp = (units + slots - 1) / slots;
            const int ctas = (int)((units + 8 * per_warp - 1) / (8 * per_warp));
            landmarks_warp_kernel<D><<<ctas, 256, 0, s>>>(q, k, ql, kl, ql16, kl16, BH, n, m);
        } else {
            long long threads = (long long)BH * m * (D / 8);
            dim3 grid((unsigned)((threads + 255) / 256), 2);
            landmarks_kernel<bf><<<grid, 256, 0, s>>>(q, k, ql, kl, ql16, kl16, BH, n, D, m);
        }
    }
    // kernel_3 V (+ mask bits, + combine) runs on the auxiliary stream, concurrently with the
    // inverse on the caller's stream: the inverse is the longer branch at the supported sizes,
    // and a kernel that follows its predecessor on the same stream starts sooner than one
    // released by a cross-stream event. At m = 256 the auxiliary stream waits until every
    // CTA pair of the inverse has started (see launch_pinv_pair); otherwise until the
    // landmarks are done.
    // one wave of CTA pairs: kernel_3 V waits until every pair has started and takes the SMs they
    // leave; more pairs than SMs (B*H > SMs / 2): "every pair has started" would only come after a
    // whole wave of the inverse, so kernel_3 V is released with the landmarks instead and its
    // persistent grid spans every SM, taking SMs as the inverse's waves free them
    const bool one_wave = m == 256 && 2 * BH <= st.sm_count;
    if (m == 256 && one_wave) {
        rc = launch_pinv_pair(p, st, ql, kl, z, ws, inv_init, s, st.started);
        if (rc != NYS_OK) return rc;
        if (cudaStreamWaitEvent(st.aux, st.started, 0) != cudaSuccess) return NYS_ERR_CUDA;
    } else if (m == 256) {
        if (cudaEventRecord(st.fork, s) != cudaSuccess) return NYS_ERR_CUDA;
        if (cudaStreamWaitEvent(st.aux, st.fork, 0) != cudaSuccess) return NYS_ERR_CUDA;
        rc = launch_pinv_pair(p, st, ql, kl, z, ws, inv_init, s, nullptr);
        if (rc != NYS_OK) return rc;
    } else {
        // m = 64 / 128: the resident inverse is much shorter than kernel_3 V; kernel_3 V is released
        // once every inverse CTA has started (one wave) and takes every SM, those of the inverse as
        // they free up; with more inverse CTAs than SMs it is released with the landmarks
        const int res_ctas = m == 128 ? BH : (BH + 1) / 2;
        if (res_ctas <= st.sm_count) {
            rc = m == 64 ? launch_pinv_res<64>(p, ql, kl, z, inv_init, s, st.started)
               : m == 128 ? launch_pinv_res<128>(p, ql, kl, z, inv_init, s, st.started) : NYS_ERR_UNSUPPORTED;
            if (rc != NYS_OK) return rc;
            if (cudaStreamWaitEvent(st.aux, st.started, 0) != cudaSuccess) return NYS_ERR_CUDA;
        } else {
            if (cudaEventRecord(st.fork, s) != cudaSuccess) return NYS_ERR_CUDA;
            if (cudaStreamWaitEvent(st.aux, st.fork, 0) != cudaSuccess) return NYS_ERR_CUDA;
            rc = m == 64 ? launch_pinv_res<64>(p, ql, kl, z, inv_init, s, nullptr)
               : m == 128 ? launch_pinv_res<128>(p, ql, kl, z, inv_init, s, nullptr) : NYS_ERR_UNSUPPORTED;
            if (rc != NYS_OK) return rc;
        }
    }
    if (mask) {
        const int words = p.B * (n / 32);
        ProfScope ps(K_MASKBITS, st.aux);
        mask_bits_kernel<<<(words + 255) / 256, 256, 0, st.aux>>>(mask, mbits, p.B, n);
    }
    // the inverse runs concurrently on its own SMs (one CTA per SM, one per 128 landmark
    // rows of each head); the persistent kernel_3 V grid takes the rest
    const int pinv_ctas = BH * ((m + 127) / 128);
    // one wave of CTA pairs at m = 256 (as long as kernel_3 V): the SMs the pairs leave; otherwise
    // (several waves, or the short resident inverse at m <= 128) every SM
    const int k3v_sms = m == 256 && one_wave ? std::max(st.sm_count / 4, st.sm_count - pinv_ctas) : st.sm_count;
    rc = launch_k3v_tc<D>(p, st, ql16, k, v, mbits, po, pm, pl, k3v_sms, split_scale(D) * kLog2e, st.aux);
    if (rc != NYS_OK) return rc;
    {
        // a programmatic dependent of kernel_3 V: launched while its last CTAs finish
        const long long threads = (long long)BH * m * (D / 4);
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)((threads + 255) / 256));
        cfg.blockDim = dim3(256);
        cfg.stream = st.aux;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        ProfScope ps(K_COMBINE, st.aux);
        if (cudaLaunchKernelEx(&cfg, k3v_combine_kernel, (const float*)po, (const float*)pm, (const float*)pl, k3v,
                               BH, m, (int)D, p.splits) != cudaSuccess)
            return NYS_ERR_CUDA;
    }
    if (cudaEventRecord(st.join, st.aux) != cudaSuccess) return NYS_ERR_CUDA;
    if (cudaStreamWaitEvent(s, st.join, 0) != cudaSuccess) return NYS_ERR_CUDA;
    {
        static bool attr_set[kMaxDevices] = {};
        int dev = 0;
        cudaGetDevice(&dev);
        if (!attr_set[dev]) {
            if (cudaFuncSetAttribute(w_tile_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)WTile<D>::bytes(256)) != cudaSuccess ||
                cudaFuncSetAttribute(w_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)WTc<D>::bytes(256)) != cudaSuccess)
                return NYS_ERR_CUDA;
            attr_set[dev] = true;
        }
        ProfScope ps(K_W, s);
        if (m % 128 == 0) {
            // tensor cores: one CTA per 128 rows of W, Z rows by TMA
            CUtensorMap map_z;
            if (!map_3d(&map_z, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, z, m, m, BH, 32, 128, CU_TENSOR_MAP_SWIZZLE_128B))
                return NYS_ERR_CUDA;
            w_tc_kernel<D><<<dim3(m / 128, BH), WTc<D>::kThreads, WTc<D>::bytes(m), s>>>(map_z, k3v, w, wt16, m);
        } else {
            w_tile_kernel<D><<<dim3(m / WTile<D>::kRows, BH), WTile<D>::kThreads, WTile<D>::bytes(m), s>>>(
                z, k3v, w, wt16, m);
        }
    }
    switch (m) {
        case 64: rc = launch_output_tc<D, 64>(p, st, q, v, conv_w, out, kl16, wt16, s); break;
        case 128: rc = launch_output_tc<D, 128>(p, st, q, v, conv_w, out, kl16, wt16, s); break;
        case 256: rc = launch_output_tc<D, 256>(p, st, q, v, conv_w, out, kl16, wt16, s); break;
        default: return NYS_ERR_UNSUPPORTED;
    }
    if (rc != NYS_OK) return rc;
    return cudaGetLastError() == cudaSuccess ? NYS_OK : NYS_ERR_CUDA;
}

// Exact branch (walkthrough 2.1, path A): softmax(Qs Ks^T + mask) V over all n query rows on
// the kernel_3 V machinery (tensor cores for bf16, CUDA cores for float32), then the split
// merge, normalisation and conv; optionally the n x n weights.
template <typename T, int D>
int launch_exact(const Plan& p, const DeviceState& st, const T* q, const T* k, const T* v,
                 const uint8_t* mask, const float* conv_w, T* out, float* attn_probs, char* ws, cudaStream_t s) {
    float* po = reinterpret_cast<float*>(ws + p.off_po);
    float* pm = reinterpret_cast<float*>(ws + p.off_pm);
    float* pl = reinterpret_cast<float*>(ws + p.off_pl);
    const int BH = p.BH, n = p.n;
    if constexpr (std::is_same<T, __nv_bfloat16>::value) {
        uint32_t* mbits = mask ? reinterpret_cast<uint32_t*>(ws + p.off_mbits) : nullptr;
        if (mask) {
            const int words = p.B * (n / 32);
            ProfScope ps(K_MASKBITS, s);
            mask_bits_kernel<<<(words + 255) / 256, 256, 0, s>>>(mask, mbits, p.B, n);
        }
        const float sc = split_scale(D) * split_scale(D) * kLog2e;   // Q and K both raw
        const int rc = launch_k3v_tc<D>(p, st, q, k, v, mbits, po, pm, pl, st.sm_count, sc, s);
        if (rc != NYS_OK) return rc;
    } else {
        dim3 grid(BH, (n + 63) / 64, p.splits);
        ProfScope ps(K_K3V, s);
        k3v_partial_simt_kernel<T, D><<<grid, 256, k3v_simt_smem_bytes<D>(), s>>>(
            q, k, v, mask, po, pm, pl, p.H, n, n, p.splits, p.keys_per_split, split_scale(D));
    }
    {
        ProfScope ps(K_OUTPUT, s);
        exact_finish_kernel<T, D><<<dim3((n + 63) / 64, BH), 256, 0, s>>>(po, pm, pl, v, conv_w, out, p.H, n,
                                                                          p.splits);
    }
    if (attn_probs) {
        ProfScope ps(K_PROBS, s);
        exact_probs_kernel<T, D><<<dim3((n + 63) / 64, BH), 256, 0, s>>>(q, k, mask, attn_probs, p.H, n);
    }
    return cudaGetLastError() == cudaSuccess ? NYS_OK : NYS_ERR_CUDA;
}

// kernel_1 Z (walkthrough 2.7) from the call's float32 K_l and Z, after the forward.
template <typename T, int D>
int launch_nystrom_probs(const Plan& p, const T* q, float* attn_probs, char* ws, cudaStream_t s) {
    const float* kl = reinterpret_cast<const float*>(ws + p.off_kl);
    const float* z = reinterpret_cast<const float*>(ws + p.off_z);
    const size_t smem = ProbsSmem<D>::bytes(p.m);
    static bool attr_set[kMaxDevices] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (!attr_set[dev]) {
        if (cudaFuncSetAttribute(nystrom_probs_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)ProbsSmem<D>::bytes(256)) != cudaSuccess)
            return NYS_ERR_CUDA;
        attr_set[dev] = true;
    }
    ProfScope ps(K_PROBS, s);
    nystrom_probs_kernel<T, D><<<dim3((p.n + 63) / 64, p.BH), 256, smem, s>>>(q, kl, z, attn_probs, p.n, p.m);
    return cudaGetLastError() == cudaSuccess ? NYS_OK : NYS_ERR_CUDA;
}

int run_exact(const void* q, const void* k, const void* v, const uint8_t* mask, const float* conv_w,
              int B, int H, int n, int d, int dtype, void* out, float* attn_probs, cudaStream_t s) {
    int rc = validate_exact(q, k, v, out, B, H, n, d, dtype);
    if (rc != NYS_OK) return rc;
    DeviceState* st = nullptr;
    rc = device_state(&st);
    if (rc != NYS_OK) return rc;
    cudaGetLastError();   // an earlier, unrelated launch error is not this call's
    const Plan p = make_plan_exact(B, H, n, d, dtype);
    void* ws = nullptr;
    if (cudaMallocAsync(&ws, p.total, s) != cudaSuccess) {
        cudaGetLastError();
        return NYS_ERR_NOMEM;
    }
    char* w = static_cast<char*>(ws);
    std::unique_lock<std::mutex> launch_lock(st->launch_mu);
    using bf = __nv_bfloat16;
    rc = guard_fill(p, ws, s);
    if (rc != NYS_OK) {
        cudaFreeAsync(ws, s);
        return rc;
    }
    if (dtype == NYS_F32)
        rc = d == 64 ? launch_exact<float, 64>(p, *st, (const float*)q, (const float*)k, (const float*)v, mask,
                                               conv_w, (float*)out, attn_probs, w, s)
                     : launch_exact<float, 32>(p, *st, (const float*)q, (const float*)k, (const float*)v, mask,
                                               conv_w, (float*)out, attn_probs, w, s);
    else
        rc = d == 64 ? launch_exact<bf, 64>(p, *st, (const bf*)q, (const bf*)k, (const bf*)v, mask, conv_w,
                                            (bf*)out, attn_probs, w, s)
                     : launch_exact<bf, 32>(p, *st, (const bf*)q, (const bf*)k, (const bf*)v, mask, conv_w,
                                            (bf*)out, attn_probs, w, s);
    if (rc == NYS_OK) rc = guard_check(p, ws, s);
    if (cudaFreeAsync(ws, s) != cudaSuccess && rc == NYS_OK) rc = NYS_ERR_CUDA;
    return rc;
}

int run(const void* q, const void* k, const void* v, const uint8_t* mask, const float* conv_w,
        int B, int H, int n, int d, int m, int n_iter, int dtype, void* out, float* dbg_ql,
        float* dbg_kl, float* dbg_z, float* dbg_k3v, float* dbg_w, cudaStream_t s,
        const Options& opt = Options()) {
    if (opt.exact) return run_exact(q, k, v, mask, conv_w, B, H, n, d, dtype, out, opt.attn_probs, s);
    if (opt.inv_init != NYS_INV_INIT_DEFAULT && opt.inv_init != NYS_INV_INIT_EXACT) return NYS_ERR_INVALID_ARG;
    int rc = validate(q, k, v, out, B, H, n, d, m, n_iter, dtype);
    if (rc != NYS_OK) return rc;
    DeviceState* st = nullptr;
    rc = device_state(&st);
    if (rc != NYS_OK) return rc;
    cudaGetLastError();   // an earlier, unrelated launch error is not this call's
    const Plan p = make_plan(B, H, n, d, m, n_iter, dtype, st->sm_count);
    void* ws = nullptr;
    if (cudaMallocAsync(&ws, p.total, s) != cudaSuccess) {
        cudaGetLastError();
        return NYS_ERR_NOMEM;
    }
    char* w = static_cast<char*>(ws);
    std::unique_lock<std::mutex> launch_lock(st->launch_mu);
    using bf = __nv_bfloat16;
    rc = guard_fill(p, ws, s);
    if (rc != NYS_OK) {
        cudaFreeAsync(ws, s);
        return rc;
    }
    if (dtype == NYS_F32) {
        rc = d == 64 ? launch_simt<float, 64>(p, *st, (const float*)q, (const float*)k, (const float*)v,
                                              mask, conv_w, (float*)out, w, opt.inv_init, s)
                     : launch_simt<float, 32>(p, *st, (const float*)q, (const float*)k, (const float*)v,
                                              mask, conv_w, (float*)out, w, opt.inv_init, s);
    } else {
        rc = d == 64 ? launch_bf16<64>(p, *st, (const bf*)q, (const bf*)k, (const bf*)v, mask, conv_w,
                                       (bf*)out, w, opt.inv_init, s)
                     : launch_bf16<32>(p, *st, (const bf*)q, (const bf*)k, (const bf*)v, mask, conv_w,
                                       (bf*)out, w, opt.inv_init, s);
    }
    if (rc == NYS_OK && opt.attn_probs) {
        if (dtype == NYS_F32)
            rc = d == 64 ? launch_nystrom_probs<float, 64>(p, (const float*)q, opt.attn_probs, w, s)
                         : launch_nystrom_probs<float, 32>(p, (const float*)q, opt.attn_probs, w, s);
        else
            rc = d == 64 ? launch_nystrom_probs<bf, 64>(p, (const bf*)q, opt.attn_probs, w, s)
                         : launch_nystrom_probs<bf, 32>(p, (const bf*)q, opt.attn_probs, w, s);
    }
    if (rc == NYS_OK) {
        const size_t BH = p.BH, md = (size_t)m * d, mm = (size_t)m * m;
        struct { float* dst; size_t off; size_t bytes; } copies[] = {
            {dbg_ql, p.off_ql, BH * md * 4}, {dbg_kl, p.off_kl, BH * md * 4},
            {dbg_z, p.off_z, BH * mm * 4}, {dbg_k3v, p.off_k3v, BH * md * 4},
            {dbg_w, p.off_w, BH * md * 4}};
        for (auto& c : copies)
            if (c.dst && cudaMemcpyAsync(c.dst, w + c.off, c.bytes, cudaMemcpyDeviceToDevice, s) != cudaSuccess)
                rc = NYS_ERR_CUDA;
    }
    if (rc == NYS_OK) rc = guard_check(p, ws, s);
    if (cudaFreeAsync(ws, s) != cudaSuccess && rc == NYS_OK) rc = NYS_ERR_CUDA;
    return rc;
}

// ---------------------------------------------------------------- allocation-free inverse
// Scratch of nys_attn_pinv_static(): a fixed 8 MiB array in device memory.
// Each head of the iterative inverse needs 5 m x m float32 matrices; heads
// are processed in batches that fit. Every GPU that loads this library holds
// the array until the process exits. In host code the name below is only a
// host-side stand-in: its device address comes from cudaGetSymbolAddress().
constexpr size_t kStaticScratchFloats = (8u << 20) / sizeof(float);
constexpr int kStaticMaxM = 256;   // the largest m any entry point accepts
static_assert((size_t)5 * kStaticMaxM * kStaticMaxM <= kStaticScratchFloats,
              "one head of the largest supported m must fit the static scratch");
static __device__ __align__(256) float g_static_scratch[kStaticScratchFloats];

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
CtxGetCurrentFn ctx_get_current_fn() {
    static CtxGetCurrentFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<CtxGetCurrentFn>(p);
        cudaGetLastError();
    });
    return fn;
}

std::mutex g_static_mu;
// device address of g_static_scratch per device, with the context it was looked up in: a
// device reset (or any teardown of the context) reloads the module, so the address is looked
// up again when the current context is not the one recorded
struct StaticScratchAddr { CUcontext ctx = nullptr; float* ptr = nullptr; };
StaticScratchAddr g_static_addr[kMaxDevices];

// Once per device (and context), with that device current: look up the array's address.
int static_scratch(float** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return NYS_ERR_CUDA;
    CtxGetCurrentFn get_ctx = ctx_get_current_fn();
    if (!get_ctx) return NYS_ERR_CUDA;
    CUcontext ctx = nullptr;   // null before the runtime has made its context current
    if (get_ctx(&ctx) != CUDA_SUCCESS) return NYS_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_static_mu);
    StaticScratchAddr& a = g_static_addr[dev];
    if (a.ptr == nullptr || ctx == nullptr || a.ctx != ctx) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || p == nullptr) {
            cudaGetLastError();
            return NYS_ERR_CUDA;
        }
        if (get_ctx(&ctx) != CUDA_SUCCESS || ctx == nullptr) return NYS_ERR_CUDA;
        a.ctx = ctx;
        a.ptr = static_cast<float*>(p);
    }
    *out = a.ptr;
    return NYS_OK;
}

}  // namespace
}  // namespace nys

extern "C" {

int nys_attn_forward(const void* q, const void* k, const void* v, const uint8_t* key_mask,
                     const float* conv_w, int B, int H, int n, int d, int m, int n_iter, int dtype,
                     void* out, void* stream) {
    return nys::run(q, k, v, key_mask, conv_w, B, H, n, d, m, n_iter, dtype, out, nullptr, nullptr,
                    nullptr, nullptr, nullptr, static_cast<cudaStream_t>(stream));
}

int nys_attn_forward_debug(const void* q, const void* k, const void* v, const uint8_t* key_mask,
                           const float* conv_w, int B, int H, int n, int d, int m, int n_iter,
                           int dtype, void* out, float* q_l, float* k_l, float* z, float* k3v,
                           float* w, void* stream) {
    return nys::run(q, k, v, key_mask, conv_w, B, H, n, d, m, n_iter, dtype, out, q_l, k_l, z, k3v,
                    w, static_cast<cudaStream_t>(stream));
}

int nys_attn_forward_ex(const void* q, const void* k, const void* v, const uint8_t* key_mask,
                        const float* conv_w, int B, int H, int n, int d, int m, int n_iter, int dtype,
                        int inv_init, int exact, void* out, float* attn_probs, void* stream) {
    nys::Options opt;
    opt.inv_init = inv_init;
    opt.exact = exact != 0;
    opt.attn_probs = attn_probs;
    return nys::run(q, k, v, key_mask, conv_w, B, H, n, d, m, n_iter, dtype, out, nullptr, nullptr,
                    nullptr, nullptr, nullptr, static_cast<cudaStream_t>(stream), opt);
}

int nys_attn_host_plan(int B, int H, int* chunks, int max_chunks) {
    // Chunks of (batch, head) slices, contiguous in every [B, H, n, d] tensor: whole batch
    // elements when B >= kHostChunks, otherwise head ranges of one batch element, B * g <= 8.
    if (B <= 0 || H <= 0 || !chunks || max_chunks < nys::kHostChunks) return NYS_ERR_INVALID_ARG;
    int nch = 0;
    if (B >= nys::kHostChunks) {
        for (int c = 0; c < nys::kHostChunks; ++c) {
            const int b0 = (int)((long long)B * c / nys::kHostChunks);
            const int b1 = (int)((long long)B * (c + 1) / nys::kHostChunks);
            chunks[4 * nch] = b0; chunks[4 * nch + 1] = b1 - b0; chunks[4 * nch + 2] = 0; chunks[4 * nch + 3] = H;
            ++nch;
        }
    } else {
        const int g = std::max(1, std::min(H, nys::kHostChunks / B));   // head groups per batch element
        for (int bb = 0; bb < B; ++bb)
            for (int c = 0; c < g; ++c) {
                const int h0 = H * c / g, h1 = H * (c + 1) / g;
                chunks[4 * nch] = bb; chunks[4 * nch + 1] = 1; chunks[4 * nch + 2] = h0; chunks[4 * nch + 3] = h1 - h0;
                ++nch;
            }
    }
    return nch;
}

int nys_attn_forward_host(const void* q, const void* k, const void* v, const uint8_t* key_mask,
                          const float* conv_w, int B, int H, int n, int d, int m, int n_iter,
                          int dtype, void* out, void* stream) {
    int rc = nys::validate(q, k, v, out, B, H, n, d, m, n_iter, dtype);
    if (rc != NYS_OK) return rc;
    nys::DeviceState* st = nullptr;
    rc = nys::device_state(&st);
    if (rc != NYS_OK) return rc;
    std::lock_guard<std::mutex> host_lock(st->host_mu);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t elt = dtype == NYS_F32 ? 4 : 2;
    const size_t head = (size_t)n * d * elt;            // bytes of one (batch, head) slice
    const size_t tensor = (size_t)B * H * head;
    const size_t mask_bytes = key_mask ? (size_t)B * n : 0;
    const size_t w_bytes = conv_w ? (size_t)H * NYS_CONV_TAPS * sizeof(float) : 0;
    const size_t o_q = 0, o_k = nys::align_up(tensor), o_v = 2 * o_k, o_o = 3 * o_k;
    const size_t o_mask = 4 * o_k, o_w = o_mask + nys::align_up(mask_bytes);
    const size_t total = o_w + nys::align_up(w_bytes);
    void* buf = nullptr;
    if (cudaMallocAsync(&buf, total, s) != cudaSuccess) {
        cudaGetLastError();
        return NYS_ERR_NOMEM;
    }
    char* b = static_cast<char*>(buf);
    const char* hq = static_cast<const char*>(q);
    const char* hk = static_cast<const char*>(k);
    const char* hv = static_cast<const char*>(v);
    char* ho = static_cast<char*>(out);
    // Chunks of (batch, head) slices, contiguous in every tensor: whole batch elements when
    // B >= kHostChunks, otherwise head ranges of one batch element. A head's result does not
    // depend on the rest of the batch, so chunk c's forward runs while chunk c + 1's inputs
    // are copied in and chunk c - 1's output is copied out (three streams, two copy engines).
    int plan[4 * nys::kHostChunks];
    const int nch = nys_attn_host_plan(B, H, plan, nys::kHostChunks);
    if (nch <= 0) {
        cudaFreeAsync(buf, s);
        cudaStreamSynchronize(s);
        return NYS_ERR_INVALID_ARG;
    }
    struct Chunk { int b0, nb, h0, nh; };
    Chunk ch[nys::kHostChunks];
    for (int c = 0; c < nch; ++c) ch[c] = {plan[4 * c], plan[4 * c + 1], plan[4 * c + 2], plan[4 * c + 3]};
    bool ok = cudaEventRecord(st->alloc_ev, s) == cudaSuccess &&
              cudaStreamWaitEvent(st->copy_in, st->alloc_ev, 0) == cudaSuccess;
    if (ok && conv_w) ok = cudaMemcpyAsync(b + o_w, conv_w, w_bytes, cudaMemcpyHostToDevice, st->copy_in) == cudaSuccess;
    int issued = 0;
    for (int c = 0; c < nch && ok && rc == NYS_OK; ++c) {
        const Chunk& k_ = ch[c];
        const size_t off = ((size_t)k_.b0 * H + k_.h0) * head;
        const size_t bytes = (size_t)k_.nb * k_.nh * head;
        ok = cudaMemcpyAsync(b + o_q + off, hq + off, bytes, cudaMemcpyHostToDevice, st->copy_in) == cudaSuccess &&
             cudaMemcpyAsync(b + o_k + off, hk + off, bytes, cudaMemcpyHostToDevice, st->copy_in) == cudaSuccess &&
             cudaMemcpyAsync(b + o_v + off, hv + off, bytes, cudaMemcpyHostToDevice, st->copy_in) == cudaSuccess;
        if (ok && key_mask && k_.h0 == 0)   // a batch element's mask rows, with its first chunk
            ok = cudaMemcpyAsync(b + o_mask + (size_t)k_.b0 * n, key_mask + (size_t)k_.b0 * n, (size_t)k_.nb * n,
                                 cudaMemcpyHostToDevice, st->copy_in) == cudaSuccess;
        ok = ok && cudaEventRecord(st->in_ev[c], st->copy_in) == cudaSuccess &&
             cudaStreamWaitEvent(s, st->in_ev[c], 0) == cudaSuccess;
        if (!ok) break;
        rc = nys_attn_forward(b + o_q + off, b + o_k + off, b + o_v + off,
                              key_mask ? (const uint8_t*)(b + o_mask) + (size_t)k_.b0 * n : nullptr,
                              conv_w ? (const float*)(b + o_w) + (size_t)k_.h0 * NYS_CONV_TAPS : nullptr, k_.nb,
                              k_.nh, n, d, m, n_iter, dtype, b + o_o + off, s);
        if (rc != NYS_OK) break;
        ok = cudaEventRecord(st->done_ev[c], s) == cudaSuccess &&
             cudaStreamWaitEvent(st->copy_out, st->done_ev[c], 0) == cudaSuccess &&
             cudaMemcpyAsync(ho + off, b + o_o + off, bytes, cudaMemcpyDeviceToHost, st->copy_out) == cudaSuccess;
        ++issued;
    }
    if (rc == NYS_OK && (!ok || issued != nch)) rc = NYS_ERR_CUDA;
    // the buffer is released on `stream` after every copy that uses it
    cudaEventRecord(st->out_ev, st->copy_out);
    cudaStreamWaitEvent(s, st->out_ev, 0);
    cudaEventRecord(st->alloc_ev, st->copy_in);
    cudaStreamWaitEvent(s, st->alloc_ev, 0);
    cudaFreeAsync(buf, s);
    if (cudaStreamSynchronize(s) != cudaSuccess && rc == NYS_OK) rc = NYS_ERR_CUDA;
    return rc;
}

int nys_attn_device_status(void) {
    if (cudaDeviceSynchronize() != cudaSuccess) return NYS_ERR_CUDA;
    int val = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&val, nys::g_status, sizeof(int)) != cudaSuccess) return NYS_ERR_CUDA;
    if (cudaMemcpyToSymbol(nys::g_status, &zero, sizeof(int)) != cudaSuccess) return NYS_ERR_CUDA;
    return val;
}

size_t nys_attn_workspace_bytes(int B, int H, int n, int d, int m, int dtype) {
    const char dummy = 0;
    if (nys::validate(&dummy, &dummy, &dummy, &dummy, B, H, n, d, m, 0, dtype) != NYS_OK) return 0;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaGetLastError();
    return nys::make_plan(B, H, n, d, m, 0, dtype, sms).total;
}

const char* nys_strerror(int status) {
    switch (status) {
        case NYS_OK: return "ok";
        case NYS_ERR_INVALID_ARG: return "invalid argument";
        case NYS_ERR_UNSUPPORTED: return "unsupported shape or dtype";
        case NYS_ERR_CUDA: return "CUDA error";
        case NYS_ERR_NOMEM: return "device workspace allocation failed";
        case NYS_ERR_TIMEOUT: return "bounded device wait timed out";
        case NYS_ERR_SCRATCH_LIMIT: return "problem exceeds the library's fixed static scratch";
        case NYS_ERR_GUARD: return "a workspace guard zone was overwritten (guard mode)";
        default: return "unknown status";
    }
}

int nys_attn_version(void) { return 200; }   // 0.2.0: forward_ex, guard mode, self-tests

namespace nys {
__global__ void exp2_selftest_kernel(int n, float lo, float hi, unsigned int* worst) {
    float w = 0.f;
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; 2 * i + 1 < n; i += gridDim.x * blockDim.x) {
        const float x0 = lo + (hi - lo) * (float)(2 * i) / (float)(n - 1);
        const float x1 = lo + (hi - lo) * (float)(2 * i + 1) / (float)(n - 1);
        float e0, e1;
        sm100::exp2_poly_pair(sm100::f2(x0, x1), e0, e1);
        const float r0 = exp2f(x0), r1 = exp2f(x1);
        w = fmaxf(w, fmaxf(fabsf(e0 - r0) / r0, fabsf(e1 - r1) / r1));
    }
    atomicMax(worst, __float_as_uint(w));   // non-negative floats order like their bits
}
}  // namespace nys

namespace nys {
// One CTA waits on an mbarrier that nothing arrives on, with the bounded wait every kernel
// uses (limit given here instead of the kernels' one second); no copy or MMA is in flight.
__global__ void wait_timeout_selftest_kernel(uint64_t limit_ns, int* result) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        sm100::mbar_init(&bar, 1);
        sm100::fence_mbar_init();
    }
    __syncthreads();
    const bool ok = sm100::warp_all(sm100::mbar_wait_limit(&bar, 0, limit_ns));
    if (threadIdx.x == 0) *result = ok ? 1 : 0;
}
}  // namespace nys

int nys_attn_selftest_wait_timeout(unsigned long long limit_ns, int* completed) {
    if (!completed || limit_ns == 0 || limit_ns > 1000000000ull) return NYS_ERR_INVALID_ARG;
    int* d = nullptr;
    if (cudaMalloc(&d, sizeof(int)) != cudaSuccess) return NYS_ERR_CUDA;
    int h = -1, rc = NYS_OK;
    if (cudaMemset(d, 0xFF, sizeof(int)) != cudaSuccess) rc = NYS_ERR_CUDA;
    if (rc == NYS_OK) {
        nys::wait_timeout_selftest_kernel<<<1, 32>>>((uint64_t)limit_ns, d);
        if (cudaGetLastError() != cudaSuccess || cudaMemcpy(&h, d, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess)
            rc = NYS_ERR_CUDA;
    }
    cudaFree(d);
    *completed = h;
    return rc;
}

int nys_attn_set_workspace_guard(int enable) {
    if (enable != 0 && enable != 1) return NYS_ERR_INVALID_ARG;
    return nys::g_guard_mode.exchange(enable);
}

int nys_attn_selftest_guard(int corrupt, int* status) {
    if (!status || (corrupt != 0 && corrupt != 1)) return NYS_ERR_INVALID_ARG;
    nys::Plan p{};
    p.guards.n = 2;
    p.guards.off[0] = 0;
    p.guards.off[1] = 2 * nys::kGuardBytes;   // a 4 KiB "buffer" between the zones
    p.total = 3 * nys::kGuardBytes;
    void* ws = nullptr;
    if (cudaMalloc(&ws, p.total) != cudaSuccess) return NYS_ERR_CUDA;
    int rc = cudaDeviceSynchronize() == cudaSuccess ? NYS_OK : NYS_ERR_CUDA;
    int prior = 0;
    if (rc == NYS_OK && cudaMemcpyFromSymbol(&prior, nys::g_status, sizeof(int)) != cudaSuccess) rc = NYS_ERR_CUDA;
    if (rc == NYS_OK && prior != NYS_OK) rc = NYS_ERR_INVALID_ARG;   // the caller must read the word first
    if (rc == NYS_OK) rc = nys::guard_fill(p, ws, 0);
    // the buffer itself may be written freely; with corrupt = 1 one byte of the second zone changes
    if (rc == NYS_OK && cudaMemset(static_cast<char*>(ws) + nys::kGuardBytes, 0, nys::kGuardBytes) != cudaSuccess)
        rc = NYS_ERR_CUDA;
    if (rc == NYS_OK && corrupt &&
        cudaMemset(static_cast<char*>(ws) + 2 * nys::kGuardBytes + 1000, 0x7F, 1) != cudaSuccess)
        rc = NYS_ERR_CUDA;
    if (rc == NYS_OK) rc = nys::guard_check(p, ws, 0);
    if (rc == NYS_OK && cudaDeviceSynchronize() != cudaSuccess) rc = NYS_ERR_CUDA;
    cudaFree(ws);
    if (rc == NYS_OK) rc = nys_attn_device_status();
    if (rc < 0 && rc != NYS_ERR_GUARD) return rc;
    *status = rc;
    return NYS_OK;
}

int nys_attn_selftest_exp2(float* max_rel_err) {
    if (!max_rel_err) return NYS_ERR_INVALID_ARG;
    unsigned int* d = nullptr;
    if (cudaMalloc(&d, sizeof(unsigned int)) != cudaSuccess) return NYS_ERR_CUDA;
    unsigned int h = 0;
    int rc = NYS_OK;
    if (cudaMemset(d, 0, sizeof(unsigned int)) != cudaSuccess) rc = NYS_ERR_CUDA;
    if (rc == NYS_OK) {
        nys::exp2_selftest_kernel<<<256, 256>>>(1 << 20, -125.f, 8.f, d);
        if (cudaGetLastError() != cudaSuccess || cudaMemcpy(&h, d, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess)
            rc = NYS_ERR_CUDA;
    }
    cudaFree(d);
    std::memcpy(max_rel_err, &h, sizeof(float));
    return rc;
}

int nys_attn_pinv_static(const float* q_l, const float* k_l, float* z, int BH, int m, int d,
                         int n_iter, void* stream) {
    if (!q_l || !k_l || !z) return NYS_ERR_INVALID_ARG;
    if (BH <= 0 || m <= 0 || d <= 0 || n_iter < 0) return NYS_ERR_INVALID_ARG;
    if ((d != 32 && d != 64) || m > nys::kStaticMaxM) return NYS_ERR_UNSUPPORTED;
    const size_t per_head = (size_t)5 * m * m;   // k2, X, T, U and the second Z buffer
    if (per_head > nys::kStaticScratchFloats) return NYS_ERR_SCRATCH_LIMIT;   // unreachable at m <= 256
    float* scratch = nullptr;
    int rc = nys::static_scratch(&scratch);
    if (rc != NYS_OK) return rc;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaGetLastError();   // an earlier, unrelated launch error is not this call's
    const int per_launch = (int)(nys::kStaticScratchFloats / per_head);
    for (int h0 = 0; h0 < BH; h0 += per_launch) {
        const int nh = BH - h0 < per_launch ? BH - h0 : per_launch;
        const size_t md = (size_t)h0 * m * d, mm = (size_t)h0 * m * m;
        nys::pinv_simt_kernel<<<nh, 256, 0, s>>>(q_l + md, k_l + md, z + mm, scratch, m, d, n_iter,
                                                 NYS_INV_INIT_DEFAULT);
        if (cudaGetLastError() != cudaSuccess) return NYS_ERR_CUDA;   // stop at the first failed launch
    }
    return NYS_OK;
}

int nys_attn_profile_enable(int on) {
    nys::prof_drain();
    std::lock_guard<std::mutex> lock(nys::g_prof_mu);
    nys::g_prof_on = on != 0;
    for (int i = 0; i < nys::K_COUNT; ++i) {
        nys::g_prof_ms[i] = 0.0;
        nys::g_prof_launches[i] = 0;
    }
    return NYS_OK;
}

int nys_attn_profile_mask(unsigned int mask) {
    std::lock_guard<std::mutex> lock(nys::g_prof_mu);
    nys::g_prof_mask = mask;
    return NYS_OK;
}

int nys_attn_profile_read(int kernel_id, int* launches, double* total_ms) {
    if (kernel_id < 0 || kernel_id >= nys::K_COUNT || !launches || !total_ms) return NYS_ERR_INVALID_ARG;
    nys::prof_drain();
    std::lock_guard<std::mutex> lock(nys::g_prof_mu);
    *launches = nys::g_prof_launches[kernel_id];
    *total_ms = nys::g_prof_ms[kernel_id];
    return NYS_OK;
}

int nys_attn_kernel_count(void) { return nys::K_COUNT; }

const char* nys_attn_kernel_name(int kernel_id) {
    if (kernel_id < 0 || kernel_id >= nys::K_COUNT) return "";
    return nys::kKernelNames[kernel_id];
}

}  // extern "C"
