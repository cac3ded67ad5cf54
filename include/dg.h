/*
 * libdg — strided-view GEMM for NVIDIA B200 (sm_100a).
 *
 * C ABI.  Every entry point computes (part of) the deep-learning GEMM
 *
 *     C[m][n] = alpha * sa[m] * sb[n] * sum_k A[m][k] * B[k][n]  +  beta * C[m][n]
 *
 * ("DeepGEMM: a recalibration of the compute paradigm", §2.3 and the problem
 * template of §4.1; "DeepGEMM deep dive", §1.1 for the operation and §2.4 for
 * the FP8 rescale), with FP32 accumulation, over operands given as strided
 * "views" that are read in place (recalibration page, §2.1-§2.2: no reshape or
 * contiguous() copy).
 *
 * Conventions shared by all entry points
 *  - Memory: the caller owns every buffer.  Data pointers are DEVICE pointers
 *    (cudaMalloc / torch CUDA tensors / managed memory) on the current device.
 *    The library keeps no pointer after a call returns.  It owns one
 *    4-byte device status word per device, allocated on the first call on
 *    that device (that first call should therefore come before any CUDA
 *    stream capture), and one Stream-K workspace per stream that runs a
 *    Stream-K plan (see DG_OPT_STREAM_K; about 19 MB for a 4096^3 product),
 *    allocated on that stream's first such call outside a capture; a call
 *    captured on a stream that has none runs without Stream-K.
 *  - Streams: `stream` is a cudaStream_t passed as void* (NULL = the legacy
 *    default stream).  Calls are asynchronous on that stream.
 *  - Errors: argument errors are returned synchronously, before anything is
 *    launched, and leave C untouched.  A device-side wait that gives up (see
 *    dg_sync_status) is reported by dg_sync_status.
 *  - Thread safety: calls may be made from several host threads and their
 *    kernels may run concurrently on different streams: split-K partial
 *    sums stay in on-chip (cluster) shared memory, and Stream-K partials go
 *    through the workspace of the call's own stream, so calls on different
 *    streams share no scratch buffers.  dg_set_option is process-global and
 *    should not race with running calls.
 */
#ifndef DG_H_
#define DG_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Element types.  A and B must have the same type (F16, BF16 or E4M3; F32
 * inputs are accepted on the CUDA-core path only).  C may be F32, F16 or BF16.
 * E4M3 is OCP FP8 E4M3 ("fn": largest finite 448, no infinities). */
typedef enum {
    DG_F32 = 0,
    DG_F16 = 1,
    DG_BF16 = 2,
    DG_E4M3 = 3
} dg_dtype;

/* Status codes.  The error table of the recalibration page (§5.1) names the
 * failure classes: stride overflow, pointers not on the device, non-finite
 * alpha/beta, unsupported combinations. */
typedef enum {
    DG_OK = 0,
    DG_ERR_NULL = 1,        /* a required pointer is NULL                        */
    DG_ERR_NDIM = 2,        /* ndim not in 1..4 or row_dims not in 0..ndim        */
    DG_ERR_SHAPE = 3,       /* negative size, or A/B/C sizes disagree (K, M, N)   */
    DG_ERR_DTYPE = 4,       /* unsupported type or A/B type mismatch              */
    DG_ERR_STRIDE = 5,      /* negative stride, byte extent overflows int64, or
                               C has two elements at one address                 */
    DG_ERR_ALIGN = 6,       /* pointer or stride not a multiple of the element    */
    DG_ERR_POINTER = 7,     /* pointer is not device-accessible                   */
    DG_ERR_VALUE = 8,       /* alpha or beta not finite                           */
    DG_ERR_UNSUPPORTED = 9, /* valid request this build does not implement        */
    DG_ERR_CUDA = 10,       /* a CUDA runtime call failed                          */
    DG_ERR_TIMEOUT = 11     /* a device-side wait gave up (see dg_sync_status)    */
} dg_status;

/*
 * A strided view ("DeepGEMM: a recalibration of the compute paradigm", §3.2).
 *  ptr       address of element (0,...,0); device memory.
 *  ndim      1..4 dims; shape[d] >= 0 elements; stride[d] >= 0 in BYTES
 *            (not elements: §3.2 fixes byte strides).
 *  row_dims  the first row_dims dims flatten row-major (last fastest) into the
 *            matrix row index, the remaining dims into the column index.  So a
 *            [M,K] row-major matrix is shape {M,K}, stride {K*es, es},
 *            row_dims 1; its transpose as a [K,M] operand is shape {K,M},
 *            stride {es, K*es}; an NCHW tensor read as [N*H*W, C] is shape
 *            {N,H,W,C}, strides {sN,sH,sW,sC}, row_dims 3.
 *  dtype     a dg_dtype value.
 * The page's `layout` tag and `align` hint are not fields: strides are
 * authoritative and alignment is derived from ptr and strides.  A zero stride
 * broadcasts (allowed for A and B, rejected for C unless the dim has size 1).
 */
typedef struct {
    void *ptr;
    int32_t ndim;
    int32_t row_dims;
    int64_t shape[4];
    int64_t stride[4];
    int32_t dtype;
    int32_t reserved; /* set to 0 */
} dg_view;

/*
 * dg_gemm — C = alpha * diag(sa) * (A B) * diag(sb) + beta * C.
 *  A [M x K], B [K x N], C [M x N]: views as above (C is read when beta != 0
 *  and written always; it must not overlap A or B).
 *  alpha, beta: finite.  beta == 0 never reads C (NaN in C does not leak);
 *  alpha == 0 never reads A or B and yields beta * C.
 *  scale_a: device float32[M] or NULL (all ones); scale_b: device float32[N]
 *  or NULL.  They are the per-row (per-token) scale of A and the per-column
 *  (per-channel) scale of B of the FP8 precision mode ("DeepGEMM deep dive",
 *  §2.4), applied exactly once in the epilogue; allowed for every input type.
 * Returns DG_OK once the work is enqueued on `stream`.
 */
dg_status dg_gemm(const dg_view *A, const dg_view *B, const dg_view *C,
                  float alpha, float beta,
                  const float *scale_a, const float *scale_b,
                  void *stream);

/* Activations of the fused epilogue. */
typedef enum {
    DG_ACT_NONE = 0,       /* identity                                              */
    DG_ACT_RELU = 1,       /* z < 0 ? 0 : z (a NaN stays NaN)                        */
    DG_ACT_GELU_TANH = 2   /* z/2 * (1 + tanh(sqrt(2/pi) * (z + 0.044715 z^3)))      */
} dg_activation;

/*
 * The fused epilogue ("DeepGEMM is not a new model: the inner discipline of
 * GPU matrix multiplication", §3.3: GEMM + BiasAdd + GeLU in one kernel, the
 * bias broadcast in registers and GeLU in its tanh form before the store;
 * "DeepGEMM deep dive", §5.1 epilogue fusion).  The GEMM result is turned
 * into
 *     C[m][n] = act( alpha * sa[m] * sb[n] * sum_k A[m][k] B[k][n]
 *                    + beta * C[m][n] + bias[n] )
 * before it is stored, so no intermediate output goes through memory.
 *  bias        device float32[N] (one value per output column n, the same for
 *              every row m), or NULL for no bias.  Read only; owned by the
 *              caller.
 *  activation  a dg_activation value; anything else is DG_ERR_VALUE.
 *  reserved    set to 0 (anything else is DG_ERR_VALUE).
 * The layout transform of the fusion (e.g. writing an NCHW output from an
 * [N*H*W, C] product) needs no field: C is a strided view, and the
 * tensor-core epilogue addresses a row of C through any number of dims.
 * Accuracy: everything before the store is FP32; GeLU's tanh is the hardware
 * approximation for F16/BF16 outputs (relative error about 2^-11, below their
 * rounding) and the accurate tanhf for FP32 outputs.
 */
typedef struct {
    const float *bias;
    int32_t activation;
    int32_t reserved;
} dg_epilogue;

/*
 * dg_gemm_ex — dg_gemm with a fused epilogue (above).  `epilogue` NULL (or
 * no bias with DG_ACT_NONE) is exactly dg_gemm.  The epilogue runs on every
 * path: the tensor-core kernels (single CTA, CTA pairs, split-K clusters,
 * gathered operands), the GEMVs, the CUDA-core kernel, and alpha == 0 or
 * K == 0, where C = act(beta * C + bias).  Errors as dg_gemm, plus
 * DG_ERR_VALUE for a bad activation or reserved field and DG_ERR_POINTER for
 * a bias that is not device memory of the current device.
 */
dg_status dg_gemm_ex(const dg_view *A, const dg_view *B, const dg_view *C,
                     float alpha, float beta,
                     const float *scale_a, const float *scale_b,
                     const dg_epilogue *epilogue, void *stream);

/*
 * dg_gemv — y = alpha * x W + beta * y for a single row (or up to 8 rows) of
 * activations: the decode-time thin GEMM of "DeepGEMM is not a new model: the
 * inner discipline of GPU matrix multiplication" (§2, [1,4096]x[4096,14336];
 * §4, [1,4096]x[4096,128]).  x is [R x K] with R <= 8 (a 1-D view of K
 * elements is one row), W is [K x N], y is [R x N].  It is dg_gemm with no
 * scales; dg_gemm itself also routes M <= 8 here when W's layout allows.
 * Returns DG_ERR_UNSUPPORTED if R > 8.
 */
dg_status dg_gemv(const dg_view *x, const dg_view *W, const dg_view *y,
                  float alpha, float beta, void *stream);

/* Human-readable name of a status code (static storage). */
const char *dg_status_string(dg_status s);

/*
 * dg_sync_status — synchronise `stream`, then return and clear the device
 * error word of the current device: DG_ERR_TIMEOUT if a kernel's bounded wait
 * gave up since the last check (its output is then undefined), DG_ERR_CUDA if
 * the synchronisation failed, DG_OK otherwise.
 */
dg_status dg_sync_status(void *stream);

/* ----------------------------------------------------------- introspection
 * Host-only helpers: they read no device memory and launch nothing, so they
 * also work on a machine without a GPU. */

/* Result of view analysis (recalibration page, §2.2: effective span,
 * contiguous segments).  Size-1 dims are dropped and neighbouring dims merged
 * when stride[i] == stride[i+1] * shape[i+1], separately for the row group and
 * the column group. */
typedef struct {
    int64_t rows, cols;
    int32_t n_row, n_col;       /* merged dims in each group (0 = extent 1)     */
    int64_t row_shape[4], row_stride[4];
    int64_t col_shape[4], col_stride[4];
    int32_t unit_dim;           /* 1: columns unit-stride (row-major), 2: rows
                                   unit-stride (column-major), 0: neither          */
    int32_t tma_ok;             /* expressible as one 2-D TMA tensor map         */
    int64_t span_bytes;         /* max byte offset touched + element size         */
    int32_t vec_bytes;          /* widest aligned contiguous run (1..16 bytes)    */
    int32_t reserved;
} dg_view_info;

dg_status dg_analyse_view(const dg_view *v, dg_view_info *out);

/* Kernel families the dispatcher chooses between. */
typedef enum {
    DG_KIND_NONE = 0,      /* nothing to do (M == 0 or N == 0)                     */
    DG_KIND_SCALE_C = 1,   /* alpha == 0 or K == 0: C = beta * C                   */
    DG_KIND_SIMT = 2,      /* CUDA-core tiled kernel, any view                      */
    DG_KIND_GEMV_N = 3,    /* M <= 8, W unit-stride along N                         */
    DG_KIND_GEMV_K = 4,    /* M <= 8, W unit-stride along K                         */
    DG_KIND_UMMA = 5       /* tcgen05 tensor-core kernel, TMEM accumulators          */
} dg_kind;

typedef struct {
    int32_t kind;          /* dg_kind                                               */
    int32_t swap_ab;       /* UMMA: computes C^T = B^T A^T (tensor-core M runs on N) */
    int32_t p_gather;      /* UMMA: the M-side operand is loaded by threads, not TMA */
    int32_t p_mn_major;    /* UMMA: operand layouts in smem (0 K-major, 1 MN-major)  */
    int32_t q_mn_major;
    int32_t block_m, block_n, block_k;  /* tile rows, columns, and k per pipeline stage */
    int32_t stages;
    int32_t split_k;
    int32_t grid;          /* CTAs launched                                          */
    int32_t vec_bytes;     /* gather / GEMV vector width                             */
    int64_t M, N, K;
    int32_t cta_pair;      /* UMMA: two CTAs of a cluster share each 256-row tile     */
    int32_t epi_tma_store; /* UMMA: the epilogue writes C in 32-row x 128-byte blocks
                              through tensor stores (beta == 0, C row-major along N)  */
    int32_t gather_cluster;/* UMMA, gathered operand: CTAs per cluster that share each
                              gathered tile, each loading 1/gather_cluster of it and
                              copying it to the others (1 = no sharing)             */
    int32_t pair_half_tiles;/* UMMA, CTA pairs: tiles of the last, partial wave that run
                              as two half-width tiles each                          */
    int32_t stream_k_tiles; /* UMMA, CTA pairs: tiles of the last, partial wave whose k
                              blocks are shared out over all pairs (Stream-K); their
                              owners add the other pairs' partials                   */
    int32_t split_reduce_add;/* UMMA, split-K with beta == 1 and FP32 C: each split adds
                              its partial straight into C (tensor reduce-add in L2)
                              instead of the cluster's fixed-order reduction, when the
                              call has no activation (see DG_OPT_DETERMINISTIC)       */
} dg_plan_info;

/* The dispatch decision dg_gemm would take for these views (pointers are only
 * used for their alignment).  `num_sms` <= 0 means the current device's count
 * (148 when no device is present). */
dg_status dg_plan(const dg_view *A, const dg_view *B, const dg_view *C,
                  float alpha, float beta, int has_scales, int num_sms,
                  dg_plan_info *out);

/*
 * dg_autotune — the call of dg_gemm_ex, after timing the kernel variants that
 * can serve it on these very operands ("DeepGEMM deep dive", §5.3: the best
 * tile and pipeline settings depend on the shape and are found by measuring;
 * "DeepGEMM: a recalibration of the compute paradigm", §6.1: the chosen
 * configuration is cached per problem).  The variants are the tensor-core
 * tile width (32..256 columns), k splits (1..8, on-chip cluster reduction),
 * CTA pairs with or without the Stream-K tail and with one or two 128-byte
 * k sub-blocks per stage, the gather-cluster size and the tensor-store
 * epilogue; for the memory-bound GEMV, its k splits.  Each
 * is run `reps` times (1..1000) after a warm-up and timed with CUDA events;
 * the fastest is kept in a process-wide table keyed by the views (shapes,
 * strides, types, pointer alignment), beta == 0, alpha == 0, the device and
 * its SM count, and every later dg_gemm / dg_gemm_ex with the same key uses
 * it.  Calls whose plan has no variants (CUDA-core kernel, K-contiguous GEMV,
 * alpha == 0) just run.
 *  On return C holds the product, as after dg_gemm_ex: the trials overwrite
 *  C, and when beta != 0 its bytes are saved first (a temporary device
 *  buffer of C's span) and put back before the final call.  The function
 *  synchronises `stream`; it is DG_ERR_UNSUPPORTED while the stream is being
 *  captured into a graph.  `out` (may be NULL) receives the number of
 *  variants timed, the time per call of the rule's plan and of the chosen
 *  one, and the chosen plan.
 */
typedef struct {
    int32_t candidates;   /* variants timed                                  */
    int32_t reserved;
    float default_us;     /* time per call of the dispatcher's own plan       */
    float best_us;        /* time per call of the chosen variant              */
    dg_plan_info plan;    /* the chosen plan                                  */
} dg_tune_result;

dg_status dg_autotune(const dg_view *A, const dg_view *B, const dg_view *C,
                      float alpha, float beta,
                      const float *scale_a, const float *scale_b,
                      const dg_epilogue *epilogue, void *stream, int reps,
                      dg_tune_result *out);

/* Forget every tuned variant (later calls plan by the rules again). */
dg_status dg_tune_clear(void);

/*
 * dg_gemm_static — dg_gemm for callers that cannot let a library allocate
 * device memory: work captured into a CUDA graph (an allocation there fails
 * or ends the capture), frameworks whose own pool owns and accounts for every
 * byte of device memory, and serving loops where an allocation's implicit
 * device synchronisation is not allowed.  The paper has no counterpart; this
 * is an interface for such callers.
 *
 * Same arguments and result as dg_gemm.  It calls no cudaMalloc, cudaFree or
 * other allocating routine: the status word and the Stream-K workspace (the
 * scratch memory of the CTA-pair kernel's Stream-K tail) live in one
 * file-scope device array of 24 MiB, which the CUDA runtime places on every
 * device that loads the library and which stays there until the process
 * exits.  The caller still passes A, B, C and the scales.
 *  - A problem whose Stream-K workspace would exceed the array (more than
 *    about 24 MiB of FP32 partial tiles; a 4096^3 product on 148 SMs needs
 *    19.4 MB) returns DG_ERR_UNSUPPORTED before anything is launched; with
 *    DG_OPT_STREAM_K set to 0 such a problem runs without scratch.
 *  - The first call on a device does a set-up: it looks up the array's
 *    device address with the device current and clears the words that must
 *    start at zero (the status word, the Stream-K sequence header and flags)
 *    with cudaMemsetAsync on `stream`.  Make that first call before any stream
 *    capture.
 *  - Every call on a device shares the array, which keeps the last call's
 *    contents (the Stream-K flags carry sequence tags, so a later call never
 *    reads an earlier call's partials).  Calls whose kernels overlap on the
 *    GPU (concurrent streams, host threads) race on it: serialise them.
 *  - A device-side wait that gives up leaves C undefined and is recorded in
 *    the array's status word, which dg_sync_status does not read.
 */
dg_status dg_gemm_static(const dg_view *A, const dg_view *B, const dg_view *C,
                         float alpha, float beta,
                         const float *scale_a, const float *scale_b,
                         void *stream);

/* Number of kernels this library has launched in this process. */
uint64_t dg_launch_count(void);

/* Process-global options (tests and benchmarks). */
typedef enum {
    DG_OPT_FORCE_KIND = 1,        /* 0 = automatic, else a dg_kind to use when it is
                                     applicable (DG_KIND_SIMT always is)              */
    DG_OPT_WAIT_TIMEOUT_MS = 2,   /* bound on every device-side wait (default 2000)   */
    DG_OPT_TEST_STALL = 3,        /* tests of the bounds: 1 the tensor-core kernel's
                                     loader issues no copies; 2 the split-K CTAs send
                                     no partial slices to their owners.  Either way
                                     waits run out and the call reports
                                     DG_ERR_TIMEOUT                                     */
    DG_OPT_MAX_SPLIT_K = 4,       /* upper bound on the tensor-core kernel's split-K
                                     (default and cluster limit 8; 1 disables)         */
    DG_OPT_CTA_PAIR = 5,          /* paired-CTA (256-row) tensor-core tiles: 0 never,
                                     1 for large problems (default), 2 whenever the
                                     operands allow                                    */
    DG_OPT_EARLY_LAUNCH = 6,      /* programmatic dependent launch: 0 off, 1 release the
                                     next kernel at the start of each kernel, 2 release
                                     it near the end of long kernels, 3 (default) for
                                     the K-contiguous GEMV (its 64 blocks leave room
                                     for the next launch) and the tensor-core kernels
                                     (released once their MMAs are issued), not for
                                     the N-contiguous GEMV (1 and 2 slowed the decode
                                     step: two W-streaming blocks fill an SM).  Every
                                     kernel waits for the previous one before it
                                     touches memory, so all modes give the same
                                     results.                                          */
    DG_OPT_TRACE = 7,             /* device address of 64 uint64 slots (0 = off): the
                                     single-CTA tensor-core kernel's CTA 0 writes
                                     its SM cycle counter (%clock64) at its phase
                                     boundaries (analysis)                             */
    DG_OPT_EPI_TMA = 8,           /* 1 (default): tensor-core epilogues store C through
                                     tensor copies where the plan allows; 0: thread
                                     stores only                                        */
    DG_OPT_GATHER_CLUSTER = 9,    /* 1 (default): CTAs that need the same gathered
                                     operand tile share the loads through distributed
                                     shared memory; 0: each gathers the whole tile      */
    DG_OPT_PAIR_TAIL = 10,        /* 1 (default): CTA pairs run the last, partial wave
                                     of tiles as half-width tiles; 0: whole tiles only  */
    DG_OPT_DETERMINISTIC = 12,    /* 0 (default): split-K with beta == 1 and FP32 C adds
                                     the splits' partials into C in the memory system
                                     (their order, and so the last bits, can vary from
                                     run to run); 1: always the cluster reduction in a
                                     fixed order (bit-identical runs)                    */
    DG_OPT_STREAM_K = 11,         /* 1: CTA pairs share the k blocks of the last,
                                     partial wave of tiles out over all pairs (Stream-K,
                                     "DeepGEMM deep dive" §5.2) when a workspace for the
                                     stream is available; 0 (default): the half-width
                                     tail above.  On 4096^3 the tail measured faster on
                                     B200 (BF16 104 against 106 us, E4M3 58 against
                                     63 us); dg_autotune times both per shape           */
    DG_OPT_PAIR_DEEP_STAGES = 13  /* 1 (default): CTA-pair stages two 128-byte k
                                     sub-blocks deep (block_k = 256 bytes of K) when an
                                     operand is MN-major and K is a whole number of such
                                     stages, so MN-major tiles arrive in half as many,
                                     twice as tall copies (4096^3 on B200: BF16 103.6 ->
                                     96.4 us, E4M3 57.7 -> 56.8 us); 0: one sub-block  */
} dg_option;

dg_status dg_set_option(int option, int64_t value);

/* Library version: major*10000 + minor*100 + patch. */
int dg_version(void);

#ifdef __cplusplus
}
#endif

#endif /* DG_H_ */
