/*
 * nys_attn.h -- C ABI of the B200 (sm_100a) Nystromformer self-attention forward.
 *
 * The operation (per batch b and head h), as the Nystromformer source
 * walkthrough (blog.gitcode.com) describes it in section 2:
 *   2.2  Qs = d^-1/4 Q,  Ks = d^-1/4 K            (1/sqrt(d) split over Q and K)
 *   2.3  Q_l[j] = mean_{t < L} Qs[j L + t],  K_l likewise,  L = n / m
 *   2.4  k1 = softmax_row(Qs K_l^T)    [n x m]
 *        k2 = softmax_row(Q_l K_l^T)   [m x m]
 *        k3 = softmax_row(Q_l Ks^T + mask)   [m x n], padded keys -> probability 0
 *   2.5  Z  = iterative Moore-Penrose inverse of k2: Z_0 = c k2^T with
 *        c = 1 / (max column sum * max row sum); n_iter times
 *        Z <- 1/4 Z (13 I - X (15 I - X (7 I - X))),  X = k2 Z
 *   2.4  out = k1 Z (k3 V)            (computed as k1 (Z (k3 V)))
 *   2.6  out += depthwise conv of V along the sequence, 65 taps per head,
 *        zero padding 32 on each side, no bias (Conv2d kernel (65,1), groups = H)
 *
 * Layouts: q, k, v, out are [B, H, n, d] row-major and contiguous (the head
 * split of walkthrough 2.2). key_mask is [B, n] uint8 with 1 = valid key and
 * 0 = padded key (the model API's attention_mask convention; HF docs,
 * NystromformerModel forward). conv_w is [H, 65] float32, the depthwise
 * Conv2d weight [H, 1, 65, 1] flattened; tap t multiplies V[i + t - 32].
 *
 * Ownership: every pointer belongs to the caller; the library keeps none of
 * them after the call returns. Calls are reentrant.
 *
 * Errors: every entry point returns an nys_status_t. Argument checks happen
 * before anything is launched; NYS_ERR_CUDA wraps a CUDA error reported at
 * launch time. Device-side waits are bounded: a wait that runs out records
 * NYS_ERR_TIMEOUT in a device status word that nys_attn_device_status()
 * returns (and clears).
 *
 * Precondition (documented, not checked): every sequence has at least one
 * valid key; otherwise kernel_3 is 0/0 for that sequence.
 */
#ifndef NYS_ATTN_H
#define NYS_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Depthwise conv taps: the conv_kernel_size default of NystromformerConfig
 * (walkthrough section 3.1; HF docs NystromformerConfig). */
#define NYS_CONV_TAPS 65
/* Default iteration count of the iterative inverse (walkthrough 2.5). */
#define NYS_DEFAULT_N_ITER 6
/* Z_0 scaling of the iterative inverse (walkthrough 2.5, the two bullets; the
 * inv_coeff_init_option row of the 3.1 table): DEFAULT takes
 * c = 1 / (max column sum * max row sum) of kernel_2, EXACT (the option set
 * to True) takes c = 1 / max column sum = 1 / ||kernel_2||_1. */
#define NYS_INV_INIT_DEFAULT 0
#define NYS_INV_INIT_EXACT 1

typedef enum {
    NYS_F32 = 0,   /* float32 in, float32 out, float32 arithmetic               */
    NYS_BF16 = 1   /* bf16 in, bf16 out (round to nearest even), float32 accumulate */
} nys_dtype_t;

typedef enum {
    NYS_OK = 0,
    NYS_ERR_INVALID_ARG = -1,  /* null pointer, non-positive size, n % m != 0, m > n, n_iter < 0 */
    NYS_ERR_UNSUPPORTED = -2,  /* shape or dtype outside what the kernels implement            */
    NYS_ERR_CUDA = -3,         /* a CUDA call failed                                           */
    NYS_ERR_NOMEM = -4,        /* workspace allocation failed                                  */
    NYS_ERR_TIMEOUT = -5,      /* a bounded device-side wait ran out                           */
    NYS_ERR_SCRATCH_LIMIT = -6, /* needs more than the fixed static scratch (nys_attn_pinv_static) */
    NYS_ERR_GUARD = -7          /* a workspace guard zone was overwritten (guard mode only)    */
} nys_status_t;

/*
 * nys_attn_forward -- the whole forward of walkthrough section 2 on device memory.
 *
 *   q, k, v   device pointers, [B, H, n, d], element type `dtype`
 *   key_mask  device pointer [B, n] uint8 (1 valid, 0 padded), or NULL for no mask
 *   conv_w    device pointer [H, 65] float32, or NULL to skip the conv
 *             (the conv_kernel_size = None case of walkthrough 2.6)
 *   m         landmarks; n % m == 0 (segment length L = n / m)
 *   n_iter    iterations of the iterative inverse (the pages' default is 6)
 *   out       device pointer [B, H, n, d], element type `dtype`; must not alias inputs
 *   stream    a cudaStream_t (NULL = legacy default stream)
 *
 * Supported: d in {32, 64}. float32: 1 <= m <= 256. bf16: m in {64, 128, 256}
 * and n % 128 == 0. Anything else returns NYS_ERR_UNSUPPORTED.
 *
 * Asynchronous: work is enqueued on `stream` and the call returns without a
 * host synchronisation. Scratch memory comes from cudaMallocAsync on
 * `stream` and is released with cudaFreeAsync on the same stream.
 */
int nys_attn_forward(const void* q, const void* k, const void* v, const uint8_t* key_mask,
                     const float* conv_w, int B, int H, int n, int d, int m, int n_iter,
                     int dtype, void* out, void* stream);

/*
 * nys_attn_forward_ex -- nys_attn_forward with the layer's other options.
 *
 *   inv_init    NYS_INV_INIT_DEFAULT, or NYS_INV_INIT_EXACT for the
 *               "exact coefficient" Z_0 = k2^T / ||k2||_1 (walkthrough 2.5,
 *               second bullet; inv_coeff_init_option = True in the 3.1 table)
 *   exact       0: the Nystrom path. Nonzero: path A of walkthrough 2.1, the
 *               branch the layer takes when num_landmarks equals the segment
 *               length: out = softmax_row(Qs Ks^T + mask) V + dwconv65(V), with
 *               Qs, Ks scaled by d^-1/4 as in 2.2 and the same mask and conv
 *               conventions. m, n_iter and inv_init are then ignored (not
 *               checked); bf16 needs n % 128 == 0.
 *   attn_probs  NULL, or a device float32 buffer for the attention weights the
 *               layer returns with output_attentions (walkthrough 2.7):
 *               [B, H, n, m] = kernel_1 Z on the Nystrom path, [B, H, n, n]
 *               = softmax_row(Qs Ks^T + mask) on the exact path. Computed in
 *               float32 on CUDA cores from the inputs and the call's float32
 *               stages; it does not feed the main output.
 * Everything else (layouts, checks, asynchrony, scratch) is as for
 * nys_attn_forward; an inv_init other than the two values returns
 * NYS_ERR_INVALID_ARG.
 */
int nys_attn_forward_ex(const void* q, const void* k, const void* v, const uint8_t* key_mask,
                        const float* conv_w, int B, int H, int n, int d, int m, int n_iter,
                        int dtype, int inv_init, int exact, void* out, float* attn_probs,
                        void* stream);

/*
 * nys_attn_forward_host -- the same operation on HOST buffers (same shapes,
 * layouts and checks). Copies the inputs to the device, runs the forward on
 * `stream`, copies the result back into `out` and synchronises `stream`
 * before returning. The batch is processed in up to 8 chunks of (batch, head)
 * slices, contiguous in every tensor, so that the copy of one chunk's inputs
 * and of another's output overlap the forward of a third (two library-owned
 * copy streams); the result is bitwise the same as one forward over the whole
 * batch. One call per device at a time (calls from several host threads are
 * serialised). Host buffers should be pinned (cudaHostAlloc) for full copy
 * bandwidth and overlap; pageable memory works but is slower. Device buffers
 * are taken with cudaMallocAsync and released before return.
 */
int nys_attn_forward_host(const void* q, const void* k, const void* v, const uint8_t* key_mask,
                          const float* conv_w, int B, int H, int n, int d, int m, int n_iter,
                          int dtype, void* out, void* stream);

/*
 * nys_attn_host_plan -- the chunks nys_attn_forward_host runs the batch in (host
 * only, no GPU work): up to 8 chunks of (batch, head) slices, each contiguous in
 * every [B, H, n, d] tensor -- whole batch elements when B >= 8, otherwise head
 * ranges of one batch element -- covering every slice exactly once. Writes
 * (b0, nb, h0, nh) per chunk into `chunks` (room for max_chunks >= 8 chunks,
 * 4 ints each) and returns the count, or NYS_ERR_INVALID_ARG.
 */
int nys_attn_host_plan(int B, int H, int* chunks, int max_chunks);

/*
 * nys_attn_forward_debug -- nys_attn_forward plus copies of the intermediate
 * stages, for tests. Each stage pointer is a device float32 buffer or NULL:
 *   q_l, k_l [B, H, m, d]   landmarks of the scaled Q and K (walkthrough 2.3)
 *   z        [B, H, m, m]   iterative inverse of kernel_2 (2.5)
 *   k3v      [B, H, m, d]   kernel_3 V (2.4)
 *   w        [B, H, m, d]   Z (kernel_3 V)
 * The main output is written as in nys_attn_forward.
 */
int nys_attn_forward_debug(const void* q, const void* k, const void* v, const uint8_t* key_mask,
                           const float* conv_w, int B, int H, int n, int d, int m, int n_iter,
                           int dtype, void* out, float* q_l, float* k_l, float* z, float* k3v,
                           float* w, void* stream);

/*
 * nys_attn_pinv_static -- kernel_2 and its iterative inverse for a batch of
 * heads, using no memory allocation at all. (The pages have no counterpart
 * of this entry point; it exists for callers, not for the method.)
 *
 * Who needs it: callers that cannot call cudaMalloc / cudaMallocAsync --
 * for example a host application that reserves all device memory up front
 * and forbids any later allocation, or a latency-critical loop that cannot
 * afford an allocation's cost or its failure. nys_attn_forward takes its
 * scratch from cudaMallocAsync; this entry point takes it from a fixed 8 MiB
 * array in the library's device memory instead.
 *
 *   q_l, k_l  device float32 [BH, m, d]: landmarks of the scaled Q and K
 *             (as nys_attn_forward_debug returns them)
 *   z         device float32 [BH, m, m] output: Z = iterative inverse of
 *             kernel_2 = softmax_row(Q_l K_l^T), n_iter iterations,
 *             Z_0 = k2^T / (max column sum * max row sum)
 *   stream    a cudaStream_t (NULL = legacy default stream)
 * Supported: d in {32, 64}, 1 <= m <= 256, any BH >= 1 (heads run in
 * batches that fit the array; one head needs 5 m^2 floats, at most
 * 1.25 MiB at m = 256, so a batch holds at least 6 heads). m > 256 returns
 * NYS_ERR_UNSUPPORTED; NYS_ERR_SCRATCH_LIMIT is reserved for a head larger
 * than the array, which no supported m reaches. Bad arguments return
 * NYS_ERR_INVALID_ARG / NYS_ERR_UNSUPPORTED before any launch; a failed
 * launch returns NYS_ERR_CUDA at once, without launching the remaining
 * batches. The call allocates nothing (no cudaMalloc, cudaFree or
 * allocating library routine). The buffers are not checked beyond null:
 * q_l, k_l must hold BH*m*d floats and z BH*m*m floats.
 *
 * Set-up: the first call on a device (with that device current) looks up
 * the array's device address once; make that first call before any stream
 * capture begins. The address is looked up again if the device's context
 * changed since (after cudaDeviceReset, for example). The array is held by
 * every GPU that loads the library until the process exits.
 *
 * Sharing: every call uses the same array, which keeps the previous call's
 * contents (nothing in it needs to start at zero: each launch writes every
 * scratch element before reading it). Calls whose work overlaps on the GPU
 * -- on different streams, or from different host threads -- race on the
 * array and corrupt each other's results; order them on one stream.
 */
int nys_attn_pinv_static(const float* q_l, const float* k_l, float* z, int BH, int m, int d,
                         int n_iter, void* stream);

/* Synchronises the current device, then returns and clears the device status
 * word (NYS_OK, NYS_ERR_TIMEOUT or NYS_ERR_GUARD); NYS_ERR_CUDA if the
 * synchronisation fails. */
int nys_attn_device_status(void);

/* Bytes of device scratch nys_attn_forward takes for this shape (0 if invalid). */
size_t nys_attn_workspace_bytes(int B, int H, int n, int d, int m, int dtype);

/* Short English text for a status code; never NULL. */
const char* nys_strerror(int status);

/* Library ABI version: major * 10000 + minor * 100 + patch. */
int nys_attn_version(void);

/*
 * Self-test of the FMA-pipe 2^x approximation that the bf16 softmax passes
 * use for part of their exponentials (the pages fix no exponential; this is
 * an implementation check, with no counterpart in them). Evaluates it on
 * 2^20 evenly spaced points of [-125, 8] on the current device and writes
 * the maximum relative error against CUDA's exp2f to *max_rel_err (host
 * pointer). Synchronous. NYS_ERR_INVALID_ARG for a null pointer,
 * NYS_ERR_CUDA on a CUDA failure.
 */
int nys_attn_selftest_exp2(float* max_rel_err);

/*
 * Self-test of the bounded device-side wait (an implementation check with no
 * counterpart in the pages). Launches one CTA on the current device that
 * waits on an mbarrier nothing arrives on, with the same bounded wait every
 * kernel of the library uses but a limit of `limit_ns` nanoseconds (at most
 * one second) instead of one second; no copy or tensor-core operation is in
 * flight. The wait runs out, the kernel records NYS_ERR_TIMEOUT in the
 * device status word (read it with nys_attn_device_status) and returns, so
 * the context stays usable. Synchronous. *completed (host pointer) is set to
 * 0 when the wait ran out and 1 if it had completed (which nothing can
 * cause). NYS_ERR_INVALID_ARG for a null pointer or a limit of 0 or more than
 * one second, NYS_ERR_CUDA on a CUDA failure.
 */
int nys_attn_selftest_wait_timeout(unsigned long long limit_ns, int* completed);

/*
 * nys_attn_set_workspace_guard -- a checking mode for the workspace of
 * nys_attn_forward / _ex / _debug / _host (an implementation check with no
 * counterpart in the pages). enable = 1 turns it on for every later call in
 * the process, 0 turns it off; returns the previous setting, or
 * NYS_ERR_INVALID_ARG for any other value. While it is on, each workspace
 * buffer lies between 4 KiB guard zones, the whole workspace is set to 0xFF
 * bytes before the first kernel (a NaN in float32 and bf16, so a read of an
 * element that no kernel wrote makes the result non-finite), and after the
 * last kernel a check records NYS_ERR_GUARD in the device status word (read
 * it with nys_attn_device_status) if any guard byte changed. The calls stay
 * asynchronous; the workspace grows by at most 17 zones (68 KiB) and each
 * call adds one memset and one small kernel. nys_attn_workspace_bytes
 * reports the size for the current setting.
 */
int nys_attn_set_workspace_guard(int enable);

/*
 * Self-test of the guard check (an implementation check with no counterpart
 * in the pages). Allocates a 12 KiB buffer holding two guard zones around a
 * 4 KiB region, fills it as the guard mode does, overwrites the region in
 * the middle (which is allowed) and, with corrupt = 1, one byte of the second
 * zone from the host (cudaMemset, inside the allocation), then runs the
 * check. *status (host pointer) receives what the device status word then
 * holds: NYS_OK for corrupt = 0, NYS_ERR_GUARD for corrupt = 1. Synchronous;
 * the status word is read and cleared. NYS_ERR_INVALID_ARG for a null
 * pointer, a corrupt value other than 0 / 1, or a status word that already
 * held an error when the call began; NYS_ERR_CUDA on a CUDA failure.
 */
int nys_attn_selftest_guard(int corrupt, int* status);

/*
 * Per-kernel timing, for benchmarks. While enabled, each kernel launch of
 * the forward is bracketed by two CUDA events recorded on the stream the
 * kernel runs on. nys_attn_profile_enable() clears the counters (and turns
 * recording on or off); nys_attn_profile_read() waits for the recorded
 * events and returns, for one kernel id in [0, nys_attn_kernel_count()),
 * the number of timed launches and their summed device time in ms.
 */
int nys_attn_profile_enable(int on);
int nys_attn_profile_read(int kernel_id, int* launches, double* total_ms);
/*
 * nys_attn_profile_mask -- restricts the timing to the kernels whose bit
 * (1 << kernel_id) is set in `mask` (all of them by default). Each timed
 * launch adds two event records to its stream, which delay the next launch,
 * so a benchmark that times the whole forward brackets only the kernel it
 * reports. Takes effect for launches after the call; the counters are not
 * cleared. Returns NYS_OK.
 */
int nys_attn_profile_mask(unsigned int mask);
int nys_attn_kernel_count(void);
const char* nys_attn_kernel_name(int kernel_id);

#ifdef __cplusplus
}
#endif

#endif /* NYS_ATTN_H */
