/*
 * nys_oracle.c -- plain, slow fp64 CPU oracle of the Nystromformer
 * approximate self-attention forward.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the product path may call, link or
 * load this file; it is used by the tests, by the smoke check, and by the
 * benchmark's CPU-baseline leg. It shares no code, header, table or helper
 * with the CUDA library.
 *
 * Every step follows "Nystromformer source walkthrough" (blog.gitcode.com),
 * section 2, in the page's own order and association:
 *   2.2  Q and K are each divided by sqrt(sqrt(d))           (d^-1/4 each)
 *   2.3  landmarks = mean of n/m consecutive rows (segment means)
 *   2.4  kernel_1 = softmax(Q K_l^T), kernel_2 = softmax(Q_l K_l^T),
 *        kernel_3 = softmax(Q_l K^T + mask);
 *        attention_probs = kernel_1 * iterative_inv(kernel_2),
 *        new_value = kernel_3 * V, context = attention_probs * new_value
 *   2.5  iterative Moore-Penrose inverse, default 6 iterations:
 *        Z <- 1/4 Z (13I - X(15I - X(7I - X))), X = kernel_2 Z
 *   2.6  context += depthwise Conv2d over the sequence axis of V,
 *        kernel (65,1), padding (32,0), groups = heads, no bias
 *   2.7  output_attentions returns attention_probs = kernel_1 Z [n x m]
 *   2.1  path A (num_landmarks == segment length): exact softmax attention,
 *        softmax(Q K^T + mask) V, with the same d^-1/4 scaling and conv
 *
 * Readings where the pages are silent or ambiguous (all listed in the
 * design notes):
 *   - the segment length is the runtime n / m (n divisible by m);
 *   - the Nystrom path is taken for every m, including m == n, unless the
 *     caller asks for path A explicitly;
 *   - Z_0 = c * kernel_2^T with c = 1 / (max column sum * max row sum),
 *     both taken per (batch, head); with the exact-coefficient option
 *     c = 1 / max column sum (the row sums of a softmax are 1);
 *   - path A adds the conv of 2.6 like the Nystrom path;
 *   - a masked key gets score -inf in kernel_3 only (probability exactly 0);
 *   - Conv2d is cross-correlation: tap t multiplies V[i + t - 32], zero
 *     outside [0, n).
 *
 * All arithmetic is double; inputs arrive as float32 (bf16 inputs are
 * exactly representable in float32) and are widened without rounding.
 * Loops only; no BLAS, no blocking, no reordering beyond the page's.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define NYS_ORACLE_TAPS 65

static void scaled_copy(const float* x, int n, int d, double s, double* y);

/* Walkthrough 2.2: the 1/sqrt(d) softmax scale split evenly over Q and K. */
static double split_scale(int d) { return 1.0 / sqrt(sqrt((double)d)); }

/* Walkthrough 2.3: x is [n, d]; xl[j] = (1/L) sum_{t<L} s * x[j*L + t], L = n/m. */
void nys_oracle_landmarks(const float* x, int n, int d, int m, double* xl) {
    const int L = n / m;
    const double s = split_scale(d);
    for (int j = 0; j < m; ++j) {
        for (int c = 0; c < d; ++c) {
            double acc = 0.0;
            for (int t = 0; t < L; ++t) acc += s * (double)x[(size_t)(j * L + t) * d + c];
            xl[(size_t)j * d + c] = acc / (double)L;
        }
    }
}

/* Row softmax in place; keep[c] == 0 puts -inf at column c (walkthrough 2.4, mask add). */
void nys_oracle_softmax_rows(double* S, int rows, int cols, const uint8_t* keep) {
    for (int r = 0; r < rows; ++r) {
        double* row = S + (size_t)r * cols;
        if (keep)
            for (int c = 0; c < cols; ++c)
                if (!keep[c]) row[c] = -INFINITY;
        double mx = -INFINITY;
        for (int c = 0; c < cols; ++c) mx = row[c] > mx ? row[c] : mx;
        double sum = 0.0;
        for (int c = 0; c < cols; ++c) {
            row[c] = exp(row[c] - mx);
            sum += row[c];
        }
        for (int c = 0; c < cols; ++c) row[c] /= sum;
    }
}

/* C[r][c] = sum_k A[r][k] * B[k][c]; A is rows x inner, B is inner x cols. */
static void matmul(const double* A, const double* B, int rows, int inner, int cols, double* C) {
    for (int r = 0; r < rows; ++r)
        for (int c = 0; c < cols; ++c) {
            double acc = 0.0;
            for (int k = 0; k < inner; ++k) acc += A[(size_t)r * inner + k] * B[(size_t)k * cols + c];
            C[(size_t)r * cols + c] = acc;
        }
}

/* C[r][c] = sum_k A[r][k] * B[c][k]  (A times B transposed). */
static void matmul_bt(const double* A, const double* B, int rows, int inner, int cols, double* C) {
    for (int r = 0; r < rows; ++r)
        for (int c = 0; c < cols; ++c) {
            double acc = 0.0;
            for (int k = 0; k < inner; ++k) acc += A[(size_t)r * inner + k] * B[(size_t)c * inner + k];
            C[(size_t)r * cols + c] = acc;
        }
}

/* M <- diag_value * I - M */
static void sub_from_scaled_identity(double* M, int m, double diag_value) {
    for (int r = 0; r < m; ++r)
        for (int c = 0; c < m; ++c) {
            double e = (r == c ? diag_value : 0.0) - M[(size_t)r * m + c];
            M[(size_t)r * m + c] = e;
        }
}

/* Scalar of the default Z_0 initialisation: 1 / (max column sum * max row sum). */
double nys_oracle_init_coeff(const double* A, int m) {
    double max_col = -INFINITY, max_row = -INFINITY;
    for (int c = 0; c < m; ++c) {
        double s = 0.0;
        for (int r = 0; r < m; ++r) s += A[(size_t)r * m + c];
        max_col = s > max_col ? s : max_col;
    }
    for (int r = 0; r < m; ++r) {
        double s = 0.0;
        for (int c = 0; c < m; ++c) s += A[(size_t)r * m + c];
        max_row = s > max_row ? s : max_row;
    }
    return 1.0 / (max_col * max_row);
}

/*
 * Scalar of the "exact coefficient" Z_0 initialisation (walkthrough 2.5, second
 * bullet; the inv_coeff_init_option row of the 3.1 table): c = 1 / ||A||_1, the
 * largest column sum. Reading: the rows of kernel_2 are normalised by its softmax,
 * so ||A||_inf = 1 and the exact coefficient 1 / (||A||_1 ||A||_inf) is 1 / ||A||_1;
 * the row factor is taken as 1, not computed.
 */
double nys_oracle_init_coeff_exact(const double* A, int m) {
    double max_col = -INFINITY;
    for (int c = 0; c < m; ++c) {
        double s = 0.0;
        for (int r = 0; r < m; ++r) s += A[(size_t)r * m + c];
        max_col = s > max_col ? s : max_col;
    }
    return 1.0 / max_col;
}

/*
 * Walkthrough 2.5: iterative Moore-Penrose inverse of the m x m matrix A.
 *   Z = c A^T;  repeat n_iter times:
 *     X = A Z;  T = 7I - X;  T = X T;  T = 15I - T;  T = X T;  T = 13I - T;  Z = 1/4 Z T
 * init_option 0: c from nys_oracle_init_coeff (the default); 1: from
 * nys_oracle_init_coeff_exact (inv_coeff_init_option = True).
 */
void nys_oracle_iterative_inv_opt(const double* A, int m, int n_iter, int init_option, double* Z) {
    const size_t mm = (size_t)m * m;
    double* X = (double*)malloc(mm * sizeof(double));
    double* T = (double*)malloc(mm * sizeof(double));
    double* U = (double*)malloc(mm * sizeof(double));
    const double c = init_option ? nys_oracle_init_coeff_exact(A, m) : nys_oracle_init_coeff(A, m);
    for (int r = 0; r < m; ++r)
        for (int k = 0; k < m; ++k) Z[(size_t)r * m + k] = c * A[(size_t)k * m + r];
    for (int it = 0; it < n_iter; ++it) {
        matmul(A, Z, m, m, m, X);                 /* X = A Z          */
        memcpy(T, X, mm * sizeof(double));
        sub_from_scaled_identity(T, m, 7.0);      /* T = 7I - X       */
        matmul(X, T, m, m, m, U);                 /* U = X (7I - X)   */
        sub_from_scaled_identity(U, m, 15.0);     /* U = 15I - U      */
        matmul(X, U, m, m, m, T);                 /* T = X U          */
        sub_from_scaled_identity(T, m, 13.0);     /* T = 13I - T      */
        matmul(Z, T, m, m, m, U);                 /* U = Z T          */
        for (size_t e = 0; e < mm; ++e) Z[e] = 0.25 * U[e];
    }
    free(X);
    free(T);
    free(U);
}

void nys_oracle_iterative_inv(const double* A, int m, int n_iter, double* Z) {
    nys_oracle_iterative_inv_opt(A, m, n_iter, 0, Z);
}

/* Walkthrough 2.6: out[i][c] += sum_t w[t] * v[i + t - 32][c], zero outside [0, n). */
void nys_oracle_dwconv_add(const float* v, const float* w, int n, int d, double* out) {
    const int half = NYS_ORACLE_TAPS / 2;
    for (int i = 0; i < n; ++i)
        for (int c = 0; c < d; ++c) {
            double acc = 0.0;
            for (int t = 0; t < NYS_ORACLE_TAPS; ++t) {
                int src = i + t - half;
                if (src < 0 || src >= n) continue;
                acc += (double)w[t] * (double)v[(size_t)src * d + c];
            }
            out[(size_t)i * d + c] += acc;
        }
}

/* 2.6 for selected rows: out[r][c] += sum_t w[t] * v[rows[r] + t - 32][c] (rows == NULL: all n). */
static void conv_rows_add(const float* v, const float* w, int n, int d, const int* rows, int nr,
                          double* out) {
    if (!rows) {
        nys_oracle_dwconv_add(v, w, n, d, out);
        return;
    }
    const int half = NYS_ORACLE_TAPS / 2;
    for (int r = 0; r < nr; ++r)
        for (int c = 0; c < d; ++c) {
            double acc = 0.0;
            for (int t = 0; t < NYS_ORACLE_TAPS; ++t) {
                int src = rows[r] + t - half;
                if (src < 0 || src >= n) continue;
                acc += (double)w[t] * (double)v[(size_t)src * d + c];
            }
            out[(size_t)r * d + c] += acc;
        }
}

/*
 * Walkthrough 2.1, path A: when num_landmarks equals the segment length the layer
 * computes full softmax attention instead of the approximation. One (batch, head):
 * with Qs = d^-1/4 Q and Ks = d^-1/4 K (2.2, applied before either path),
 *   probs = softmax_row(Qs Ks^T + mask)   [n x n], padded keys -> 0
 *   out   = probs V, then the conv of 2.6 is added.
 * rows / n_rows select the query rows as in nys_oracle_head; probs_out (or NULL)
 * receives the selected rows of probs, [n_rows, n].
 */
int nys_oracle_exact_head(const float* q, const float* k, const float* v, const uint8_t* keep,
                          const float* w, int n, int d, const int* rows, int n_rows, double* out,
                          double* probs_out) {
    if (n <= 0 || d <= 0) return -1;
    const double s = split_scale(d);
    const int nr = rows ? n_rows : n;
    double* ks = (double*)malloc((size_t)n * d * sizeof(double));
    double* vd = (double*)malloc((size_t)n * d * sizeof(double));
    double* qs = (double*)malloc((size_t)nr * d * sizeof(double));
    double* p = (double*)malloc((size_t)nr * n * sizeof(double));
    scaled_copy(k, n, d, s, ks);
    scaled_copy(v, n, d, 1.0, vd);
    for (int r = 0; r < nr; ++r) {
        int i = rows ? rows[r] : r;
        for (int c = 0; c < d; ++c) qs[(size_t)r * d + c] = s * (double)q[(size_t)i * d + c];
    }
    matmul_bt(qs, ks, nr, d, n, p);
    nys_oracle_softmax_rows(p, nr, n, keep);
    matmul(p, vd, nr, n, d, out);
    if (w) conv_rows_add(v, w, n, d, rows, nr, out);
    if (probs_out) memcpy(probs_out, p, (size_t)nr * n * sizeof(double));
    free(ks); free(vd); free(qs); free(p);
    return 0;
}

/* Scaled copy of a [n, d] float32 block into double. */
static void scaled_copy(const float* x, int n, int d, double s, double* y) {
    for (size_t e = 0; e < (size_t)n * d; ++e) y[e] = s * (double)x[e];
}

/*
 * One (batch, head). q, k, v: [n, d]; keep: [n] or NULL; w: [65] or NULL.
 * rows/n_rows select the query rows whose output is returned in out
 * (rows == NULL means all n rows in order). Optional stage outputs (may be
 * NULL): ql, kl [m, d]; k2, z [m, m]; k3v [m, d].
 */
int nys_oracle_head(const float* q, const float* k, const float* v, const uint8_t* keep,
                    const float* w, int n, int d, int m, int n_iter, int init_option,
                    const int* rows, int n_rows, double* out,
                    double* ql_out, double* kl_out, double* k2_out, double* z_out,
                    double* k3v_out, double* probs_out) {
    if (n <= 0 || d <= 0 || m <= 0 || n % m != 0 || m > n || n_iter < 0) return -1;
    const double s = split_scale(d);
    const int nr = rows ? n_rows : n;
    double* ql = (double*)malloc((size_t)m * d * sizeof(double));
    double* kl = (double*)malloc((size_t)m * d * sizeof(double));
    double* k2 = (double*)malloc((size_t)m * m * sizeof(double));
    double* z = (double*)malloc((size_t)m * m * sizeof(double));
    double* ks = (double*)malloc((size_t)n * d * sizeof(double));
    double* vd = (double*)malloc((size_t)n * d * sizeof(double));
    double* k3 = (double*)malloc((size_t)m * n * sizeof(double));
    double* k3v = (double*)malloc((size_t)m * d * sizeof(double));
    double* qs = (double*)malloc((size_t)nr * d * sizeof(double));
    double* k1 = (double*)malloc((size_t)nr * m * sizeof(double));
    double* probs = (double*)malloc((size_t)nr * m * sizeof(double));

    /* 2.3 landmarks of the scaled Q and K */
    nys_oracle_landmarks(q, n, d, m, ql);
    nys_oracle_landmarks(k, n, d, m, kl);

    /* 2.4 kernel_2 = softmax(Q_l K_l^T) */
    matmul_bt(ql, kl, m, d, m, k2);
    nys_oracle_softmax_rows(k2, m, m, NULL);

    /* 2.5 Z = iterative_inv(kernel_2) */
    nys_oracle_iterative_inv_opt(k2, m, n_iter, init_option, z);

    /* 2.4 kernel_3 = softmax(Q_l Ks^T + mask); new_value = kernel_3 V */
    scaled_copy(k, n, d, s, ks);
    scaled_copy(v, n, d, 1.0, vd);
    matmul_bt(ql, ks, m, d, n, k3);
    nys_oracle_softmax_rows(k3, m, n, keep);
    matmul(k3, vd, m, n, d, k3v);

    /* 2.4 kernel_1 = softmax(Qs K_l^T) for the requested rows */
    for (int r = 0; r < nr; ++r) {
        int i = rows ? rows[r] : r;
        for (int c = 0; c < d; ++c) qs[(size_t)r * d + c] = s * (double)q[(size_t)i * d + c];
    }
    matmul_bt(qs, kl, nr, d, m, k1);
    nys_oracle_softmax_rows(k1, nr, m, NULL);

    /* 2.4 attention_probs = kernel_1 Z; context = attention_probs new_value */
    matmul(k1, z, nr, m, m, probs);
    matmul(probs, k3v, nr, m, d, out);

    /* 2.6 context += depthwise conv of V */
    if (w) conv_rows_add(v, w, n, d, rows, nr, out);
    /* 2.7 the attention weights returned for output_attentions: attention_probs = kernel_1 Z */
    if (probs_out) memcpy(probs_out, probs, (size_t)nr * m * sizeof(double));

    if (ql_out) memcpy(ql_out, ql, (size_t)m * d * sizeof(double));
    if (kl_out) memcpy(kl_out, kl, (size_t)m * d * sizeof(double));
    if (k2_out) memcpy(k2_out, k2, (size_t)m * m * sizeof(double));
    if (z_out) memcpy(z_out, z, (size_t)m * m * sizeof(double));
    if (k3v_out) memcpy(k3v_out, k3v, (size_t)m * d * sizeof(double));
    free(ql); free(kl); free(k2); free(z); free(ks); free(vd);
    free(k3); free(k3v); free(qs); free(k1); free(probs);
    return 0;
}

/*
 * Whole batch: q, k, v [B, H, n, d]; mask [B, n] or NULL; conv_w [H, 65] or NULL.
 * rows/n_rows as in nys_oracle_head (the same rows for every head); out is
 * [B, H, n_rows, d] (n_rows = n when rows == NULL). Optional per-head stage
 * outputs: ql, kl, k3v [B, H, m, d]; k2, z [B, H, m, m]; probs [B, H, n_rows, m]
 * (kernel_1 Z), or [B, H, n_rows, n] on the exact path. init_option selects the
 * Z_0 coefficient (0 default, 1 exact); exact != 0 takes path A (m, n_iter and
 * init_option unused; the stage outputs other than probs are not written).
 * threads <= 0 uses the OpenMP default. Returns 0, or -1 on an invalid shape.
 */
int nys_oracle_forward(const float* q, const float* k, const float* v, const uint8_t* mask,
                       const float* conv_w, int B, int H, int n, int d, int m, int n_iter,
                       int init_option, int exact, const int* rows, int n_rows, int threads,
                       double* out, double* ql, double* kl, double* k2, double* z, double* k3v,
                       double* probs) {
    if (B <= 0 || H <= 0 || n <= 0 || d <= 0) return -1;
    if (!exact && (m <= 0 || n % m != 0 || m > n || n_iter < 0)) return -1;
    const int nr = rows ? n_rows : n;
    int bad = 0;
#ifdef _OPENMP
    if (threads > 0) omp_set_num_threads(threads);
#else
    (void)threads;
#endif
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int bh = 0; bh < B * H; ++bh) {
        const int b = bh / H, h = bh % H;
        const size_t off = (size_t)bh * n * d;
        const size_t md = (size_t)bh * m * d, mm = (size_t)bh * m * m;
        const uint8_t* keep = mask ? mask + (size_t)b * n : NULL;
        const float* wh = conv_w ? conv_w + (size_t)h * NYS_ORACLE_TAPS : NULL;
        if (exact) {
            bad |= nys_oracle_exact_head(q + off, k + off, v + off, keep, wh, n, d, rows, nr,
                                         out + (size_t)bh * nr * d,
                                         probs ? probs + (size_t)bh * nr * n : NULL) != 0;
        } else {
            bad |= nys_oracle_head(q + off, k + off, v + off, keep, wh, n, d, m, n_iter, init_option,
                                   rows, nr, out + (size_t)bh * nr * d,
                                   ql ? ql + md : NULL, kl ? kl + md : NULL, k2 ? k2 + mm : NULL,
                                   z ? z + mm : NULL, k3v ? k3v + md : NULL,
                                   probs ? probs + (size_t)bh * nr * m : NULL) != 0;
        }
    }
    return bad ? -1 : 0;
}

int nys_oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
