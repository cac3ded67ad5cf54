/*
 * Plain FP64 CPU oracle for the strided-view GEMM   C = alpha * A * B + beta * C.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  It shares no code,
 * header, table or constant with the CUDA library it checks.
 *
 * What it follows:
 *  - Definition of the operation: every output element is
 *      C[m][n] = alpha * sum_k A[m][k] * B[k][n] + beta * C[m][n]
 *    ("DeepGEMM: a recalibration of the compute paradigm", §2.3 and the
 *    problem template of §4.1; "DeepGEMM deep dive", §1.1).
 *  - Addressing: an element of a view lives at  base + sum_d idx_d * stride_d,
 *    strides in BYTES (recalibration page, §2.3 address formula and §3.2
 *    byte-stride rule).  The matrix row index is unflattened row-major over the
 *    first row_dims dims and the column index over the remaining dims.
 *  - FP8 E4M3 with per-row (A) and per-column (B) scales applied once in the
 *    rescale step ("DeepGEMM deep dive", §2.4 precision modes; §4.2 warns about
 *    a scale applied twice).
 *
 *  - The fused epilogue: a bias vector broadcast over rows and an
 *    element-wise activation applied to the result before it is stored
 *    ("DeepGEMM is not a new model: the inner discipline of GPU matrix
 *    multiplication", §3.3, GEMM + BiasAdd + GeLU with GeLU in its tanh
 *    form; "DeepGEMM deep dive", §5.1 epilogue fusion):
 *      out[m][n] = act( alpha * sa[m] * sb[n] * sum_k A[m][k] B[k][n]
 *                       + beta * C[m][n] + bias[n] )
 *    act is the identity, ReLU, or GeLU in the tanh form
 *      gelu(z) = z/2 * (1 + tanh( sqrt(2/pi) * (z + 0.044715 z^3) )).
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *  - beta == 0: C is not read (BLAS convention), so NaN in C does not leak.
 *  - alpha == 0: the product is not formed; the result is beta * C, as the
 *    recalibration page's troubleshooting note (§4.3) requires beta to be
 *    applied even when the A-load is skipped.
 *  - scale pointers may be NULL, meaning all-ones scales.
 *  - the bias is indexed by the output column n (one value per output
 *    feature, the same for every row m) and may be NULL (no bias); the
 *    activation is the last step before the store, after beta * C.
 *  - ReLU keeps NaN (z < 0 ? 0 : z), so a NaN of the sum still reaches C.
 *  - Accumulation is FP64 in ascending k; no blocking or reordering.
 *
 * Decoders are written from the format definitions: IEEE binary16, bfloat16
 * (the top half of an IEEE binary32) and OCP FP8 E4M3 ("fn": no infinities,
 * S.1111.111 is NaN, largest finite 448).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

enum { DGO_F32 = 0, DGO_F16 = 1, DGO_BF16 = 2, DGO_E4M3 = 3 };

enum { DGO_ACT_NONE = 0, DGO_ACT_RELU = 1, DGO_ACT_GELU_TANH = 2 };

enum {
    DGO_OK = 0,
    DGO_BAD_ARG = 1,
    DGO_BAD_SHAPE = 2,
    DGO_NO_MEMORY = 3,
};

typedef struct {
    const unsigned char *base; /* address of element (0,...,0) */
    int32_t ndim;              /* 1..4 */
    int32_t row_dims;          /* 0..ndim */
    int32_t dtype;             /* DGO_* */
    int32_t pad_;
    int64_t shape[4];
    int64_t stride[4];         /* bytes */
} dgo_view;

/* ------------------------------------------------------------- decoders */

static double dec_f32(const unsigned char *p) {
    float f;
    memcpy(&f, p, 4);
    return (double)f;
}

/* IEEE binary16: 1 sign, 5 exponent (bias 15), 10 fraction bits. */
static double dec_f16(const unsigned char *p) {
    uint16_t h;
    memcpy(&h, p, 2);
    int s = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int f = h & 0x3ff;
    double v;
    if (e == 0)
        v = ldexp((double)f, -24); /* subnormal: f * 2^-14 * 2^-10 */
    else if (e == 31)
        v = (f == 0) ? INFINITY : NAN;
    else
        v = ldexp(1.0 + (double)f / 1024.0, e - 15);
    return s ? -v : v;
}

/* bfloat16: the upper 16 bits of an IEEE binary32. */
static double dec_bf16(const unsigned char *p) {
    uint16_t h;
    memcpy(&h, p, 2);
    uint32_t w = (uint32_t)h << 16;
    float f;
    memcpy(&f, &w, 4);
    return (double)f;
}

/* OCP FP8 E4M3 ("fn"): 1 sign, 4 exponent (bias 7), 3 fraction bits.
 * e == 0 is subnormal: f * 2^-9.  e == 15 with f == 7 is NaN (no infinities). */
double dgo_decode_e4m3(unsigned int code) {
    int s = (code >> 7) & 1;
    int e = (code >> 3) & 0xf;
    int f = code & 0x7;
    double v;
    if (e == 0)
        v = ldexp((double)f, -9);
    else if (e == 15 && f == 7)
        v = NAN;
    else
        v = ldexp(1.0 + (double)f / 8.0, e - 7);
    return s ? -v : v;
}

static double dec(int dtype, const unsigned char *p) {
    switch (dtype) {
    case DGO_F32: return dec_f32(p);
    case DGO_F16: return dec_f16(p);
    case DGO_BF16: return dec_bf16(p);
    case DGO_E4M3: return dgo_decode_e4m3(*p);
    default: return NAN;
    }
}

/* Element decoders exposed for the pins (format tables, round trips). */
double dgo_decode(int dtype, const void *p) { return dec(dtype, (const unsigned char *)p); }

/* ------------------------------------------------------------ addressing */

int64_t dgo_rows(const dgo_view *v) {
    int64_t r = 1;
    for (int d = 0; d < v->row_dims; ++d) r *= v->shape[d];
    return r;
}

int64_t dgo_cols(const dgo_view *v) {
    int64_t c = 1;
    for (int d = v->row_dims; d < v->ndim; ++d) c *= v->shape[d];
    return c;
}

/* Byte offset of matrix element (r, c): unflatten r over dims [0, row_dims)
 * and c over [row_dims, ndim), both row-major (last dim fastest), then
 * sum idx_d * stride_d. */
int64_t dgo_offset(const dgo_view *v, int64_t r, int64_t c) {
    int64_t off = 0;
    for (int d = v->row_dims - 1; d >= 0; --d) {
        int64_t i = r % v->shape[d];
        r /= v->shape[d];
        off += i * v->stride[d];
    }
    for (int d = v->ndim - 1; d >= v->row_dims; --d) {
        int64_t i = c % v->shape[d];
        c /= v->shape[d];
        off += i * v->stride[d];
    }
    return off;
}

static double elem(const dgo_view *v, int64_t r, int64_t c) {
    return dec(v->dtype, v->base + dgo_offset(v, r, c));
}

static int check_views(const dgo_view *A, const dgo_view *B, const dgo_view *C,
                       int64_t *M, int64_t *N, int64_t *K) {
    if (!A || !B || !C) return DGO_BAD_ARG;
    const dgo_view *vs[3] = {A, B, C};
    for (int i = 0; i < 3; ++i) {
        if (vs[i]->ndim < 1 || vs[i]->ndim > 4) return DGO_BAD_ARG;
        if (vs[i]->row_dims < 0 || vs[i]->row_dims > vs[i]->ndim) return DGO_BAD_ARG;
    }
    *M = dgo_rows(A);
    *K = dgo_cols(A);
    *N = dgo_cols(B);
    if (dgo_rows(B) != *K || dgo_rows(C) != *M || dgo_cols(C) != *N) return DGO_BAD_SHAPE;
    return DGO_OK;
}

/* ------------------------------------------------------------ activation */

/* The element-wise activation of the fused epilogue, in FP64. */
double dgo_activation(int act, double z) {
    switch (act) {
    case DGO_ACT_RELU: return z < 0.0 ? 0.0 : z;
    case DGO_ACT_GELU_TANH: {
        const double c = sqrt(2.0 / acos(-1.0)); /* sqrt(2 / pi) */
        return 0.5 * z * (1.0 + tanh(c * (z + 0.044715 * z * z * z)));
    }
    default: return z;
    }
}

/* -------------------------------------------------------------- the GEMM */

/*
 * Full oracle.  out[m*N + n] receives
 *     z = alpha * sa[m] * sb[n] * sum_k a(m,k) b(k,n)  +  beta * c(m,n)  +  bias[n]
 *     out = act(z)
 * in FP64 (c read only when beta != 0; the sum skipped when alpha == 0; the
 * bias term 0 when bias is NULL), bound[m*N + n] (if non-NULL) receives
 * |alpha * sa[m] * sb[n]| * sum_k |a b|, the scale against which rounding of
 * the sum is judged, and pre[m*N + n] (if non-NULL) receives z.
 *
 * A and B are first decoded into FP64 matrices through the view addressing
 * (B stored transposed so the k loop walks memory in order); the triple loop
 * is then the definition written out, k ascending.
 */
int dgo_gemm(const dgo_view *A, const dgo_view *B, const dgo_view *C,
             double alpha, double beta, const float *sa, const float *sb,
             const float *bias, int act,
             double *out, double *bound, double *pre, int nthreads) {
    int64_t M, N, K;
    int st = check_views(A, B, C, &M, &N, &K);
    if (st) return st;
    if (!out) return DGO_BAD_ARG;
    if (M == 0 || N == 0) return DGO_OK;

    double *a = NULL, *bt = NULL;
    if (alpha != 0.0 && K > 0) {
        a = (double *)malloc(sizeof(double) * (size_t)(M * K));
        bt = (double *)malloc(sizeof(double) * (size_t)(N * K));
        if (!a || !bt) {
            free(a);
            free(bt);
            return DGO_NO_MEMORY;
        }
    }
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
    if (a) {
#pragma omp parallel for schedule(static)
        for (int64_t m = 0; m < M; ++m)
            for (int64_t k = 0; k < K; ++k) a[m * K + k] = elem(A, m, k);
#pragma omp parallel for schedule(static)
        for (int64_t n = 0; n < N; ++n)
            for (int64_t k = 0; k < K; ++k) bt[n * K + k] = elem(B, k, n);
    }

#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t m = 0; m < M; ++m) {
        double s_m = sa ? (double)sa[m] : 1.0;
        for (int64_t n = 0; n < N; ++n) {
            double s_n = sb ? (double)sb[n] : 1.0;
            double acc = 0.0, mag = 0.0;
            if (a) {
                const double *ar = a + m * K;
                const double *br = bt + n * K;
                for (int64_t k = 0; k < K; ++k) {
                    double p = ar[k] * br[k];
                    acc += p;
                    mag += fabs(p);
                }
            }
            double s = alpha * s_m * s_n;
            double r = (a ? s * acc : 0.0);
            if (beta != 0.0) r += beta * elem(C, m, n);
            if (bias) r += (double)bias[n];
            out[m * N + n] = dgo_activation(act, r);
            if (pre) pre[m * N + n] = r;
            if (bound) bound[m * N + n] = (a ? fabs(s) * mag : 0.0);
        }
    }
    free(a);
    free(bt);
    return DGO_OK;
}

/*
 * The same definition evaluated one output at a time, straight from the
 * views (no pre-decoded copies): used to check sampled outputs of problems
 * too large for the full oracle.  out, bound and pre as in dgo_gemm, one
 * entry per point (ms[i], ns[i]).
 */
int dgo_gemm_points(const dgo_view *A, const dgo_view *B, const dgo_view *C,
                    double alpha, double beta, const float *sa, const float *sb,
                    const float *bias, int act,
                    const int64_t *ms, const int64_t *ns, int64_t npts,
                    double *out, double *bound, double *pre, int nthreads) {
    int64_t M, N, K;
    int st = check_views(A, B, C, &M, &N, &K);
    if (st) return st;
    if (!ms || !ns || !out) return DGO_BAD_ARG;
    for (int64_t i = 0; i < npts; ++i)
        if (ms[i] < 0 || ms[i] >= M || ns[i] < 0 || ns[i] >= N) return DGO_BAD_ARG;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
#pragma omp parallel for schedule(dynamic, 16)
    for (int64_t i = 0; i < npts; ++i) {
        int64_t m = ms[i], n = ns[i];
        double acc = 0.0, mag = 0.0;
        int use_ab = (alpha != 0.0);
        if (use_ab)
            for (int64_t k = 0; k < K; ++k) {
                double p = elem(A, m, k) * elem(B, k, n);
                acc += p;
                mag += fabs(p);
            }
        double s = alpha * (sa ? (double)sa[m] : 1.0) * (sb ? (double)sb[n] : 1.0);
        double r = use_ab ? s * acc : 0.0;
        if (beta != 0.0) r += beta * elem(C, m, n);
        if (bias) r += (double)bias[n];
        out[i] = dgo_activation(act, r);
        if (pre) pre[i] = r;
        if (bound) bound[i] = use_ab ? fabs(s) * mag : 0.0;
    }
    return DGO_OK;
}

int dgo_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
