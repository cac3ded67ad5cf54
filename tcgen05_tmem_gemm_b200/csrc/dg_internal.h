// Internal interfaces of libdg: the device-side view description, the
// per-kernel parameter blocks and the launchers each kernel file exports to
// the dispatcher.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/dg.h"

namespace dg {

constexpr int kMaxDims = 4;

// One group (rows or columns) of a view after size-1 dims are dropped and
// contiguous neighbours merged; dims are listed outermost first.  An index in
// [0, prod(size)) is unflattened row-major over the group.
struct Axis {
    int32_t n;
    int32_t pad_;
    int64_t size[kMaxDims];
    int64_t stride[kMaxDims];  // bytes
};

// A view as the kernels see it: element (r, c) lives at ptr + off(row, r) + off(col, c).
struct DevView {
    const char *ptr;
    Axis row, col;
    int32_t dtype;
    int32_t pad_;
};

__host__ __device__ inline int64_t axis_offset(const Axis &a, int64_t idx) {
    if (a.n == 1) return idx * a.stride[0];  // one merged dim: no division
    if (a.n == 0) return 0;
    int64_t off = 0;
    for (int d = a.n - 1; d >= 0; --d) {
        const int64_t s = a.size[d];
        const int64_t q = idx / s;
        off += (idx - q * s) * a.stride[d];
        idx = q;
    }
    return off;
}

// Host-side analysis of one view (see view.cpp).
struct ViewInfo {
    int64_t rows = 0, cols = 0;
    Axis row{}, col{};
    int unit_dim = 0;      // 1: col group is one unit-stride dim, 2: row group is
    bool tma_ok = false;   // one 2-D TMA map covers it
    int vec_bytes = 1;     // widest aligned run along the unit-stride dim
    int64_t span = 0;      // bytes touched from ptr
    int es = 0;            // element size
};

dg_status analyse(const dg_view *v, bool is_output, ViewInfo *info);
int elem_size(int dtype);

// ------------------------------------------------------------- kernel params

// Epilogue target: C viewed as (i, j) with byte strides, i on the tensor-core
// M side, j on the N side (swapped when the kernel computes C^T).  The
// epilogue computes  out = act(alpha * s_i * s_j * acc + beta * C + bias)
// with the bias indexed by the output column n, which is j, or i when the
// operands are swapped.
struct EpiParams {
    char *c;
    int64_t ci, cj;          // byte strides of C along i and j (ci: when ci_multi == 0)
    int32_t c_dtype;
    int32_t vec_ok;          // C contiguous along j with 16-byte aligned rows
    float alpha, beta;
    const float *scale_i;    // per-i scale or null
    const float *scale_j;    // per-j scale or null
    const float *bias_i;     // fused bias along i (swapped operands) or null
    const float *bias_j;     // fused bias along j or null
    int32_t act;             // fused activation (dg_activation)
    int32_t ci_multi;        // C's i index spans several dims (e.g. an NCHW output): row offsets from ci_axis
    Axis ci_axis;            // C's i group, outermost dim first
};

// Byte offset of C's row i.  Every loop over the axis is unrolled with
// constant indices, so the epilogue's copy of EpiParams stays in registers.
__host__ __device__ inline int64_t epi_row_offset(const EpiParams &e, int64_t i) {
    if (!e.ci_multi) return i * e.ci;
    int64_t off = 0;
#if defined(__CUDA_ARCH__)
#pragma unroll
#endif
    for (int d = kMaxDims - 1; d >= 0; --d) {
        if (d < e.ci_axis.n) {
            const int64_t s = e.ci_axis.size[d];
            const int64_t q = i / s;
            off += (i - q * s) * e.ci_axis.stride[d];
            i = q;
        }
    }
    return off;
}

struct UmmaParams {
    int32_t Mi, Nj, K;       // tensor-core problem: D[Mi x Nj] = P[Mi x K] Q[K x Nj]
    int32_t bn;              // tile width along j (64, 128 or 256)
    int32_t bk;              // tile depth (128 bytes of K)
    int32_t ksub;            // CTA pairs: k sub-blocks of bk per stage (1 or 2); a stage is ksub * bk deep
    int32_t stages;
    int32_t tiles_i, tiles_j, split_k, kb_per_split, kb_total;
    int32_t num_units;       // tiles_i * tiles_j * split_k
    int32_t p_mn_major, q_mn_major;
    uint32_t idesc;          // instruction descriptor
    int32_t tmem_cols;
    EpiParams epi;
    // thread-loaded P operand (gather variant)
    DevView pv;              // rows = i, cols = k
    int32_t gather_vec;      // elements per load
    int32_t epi_tma;         // 1: the epilogue writes C through tensor stores (third map)
    int32_t gather_cluster;  // > 1: CTAs of a cluster (same i tile) each gather 1/gather_cluster of
                             // every P stage and copy it into the others' stages
    // CTA pairs: units [0, full_units) are whole 256 x bn tiles; the tiles after
    // them (the last, partial wave) run as two 256 x bn/2 units each, with
    // instruction descriptor idesc_half
    int32_t full_units;
    uint32_t idesc_half;
    // split-K with beta = 1 and FP32 C: every split adds its scaled partial
    // straight into C with tensor reduce-adds (third map: C, 32 x 32 FP32
    // boxes), instead of the cluster exchange; red_inner_i: C is unit-stride
    // along i (the map's inner dim is i), else along j
    int32_t red_add;
    int32_t red_inner_i;
    // Stream-K (CTA pairs): the first dp_tiles tiles run whole, one pair
    // each; the last sk_tiles tiles form one run of k blocks shared out evenly
    // over all pairs.  A tile's owner (the pair holding its last k blocks)
    // adds the partials the other pairs left in the workspace, in pair order.
    int32_t sk_tiles;
    int32_t dp_tiles;
    float *sk_part;          // per (pair, CTA): 128 rows x bn FP32, column by column
    uint32_t *sk_flag;       // per (pair, CTA, epilogue warp): sequence tag of the partial rows last written
    uint32_t *sk_hdr;        // [0] sequence number of the last completed launch, [1] CTAs done
    // control
    int *err_word;
    uint64_t timeout_ns;
    int32_t stall_loader;    // test hooks: 1 loaders issue nothing, 2 split-K sends no slices
    int32_t pdl;             // 0 off, 1 release dependents at start, 2 near the end
    uint64_t *trace;         // optional phase timestamps of CTA 0 (SM cycles, %clock64)
};

struct GemvParams {
    DevView x;               // [R x K]
    const char *w;           // W base
    int64_t w_ld;            // bytes between consecutive k (GEMV_N) or n (GEMV_K)
    int32_t R, K, N;
    int32_t in_dtype;
    EpiParams epi;           // i = row of x, j = n
    int32_t kper;            // GEMV_N: rows of W per block (a multiple of the 64-row TMA stage)
    int32_t x_vec16;         // x unit-stride along k, 16-byte aligned rows, K % 8 == 0
    int64_t x_ld;            // bytes between rows of x (x_vec16 only)
    int *err_word;
    uint64_t timeout_ns;
    int32_t pdl;             // 0 off, 1 release dependents at start, 2 near the end
};

struct SimtParams {
    DevView a, b;            // a: rows m, cols k;  b: rows k, cols n
    DevView c;               // rows m, cols n
    int32_t M, N, K;
    EpiParams epi;           // i = m, j = n (c pointer unused; see c view)
    int32_t pdl;
};

// ------------------------------------------------------------------ launchers
// Each returns cudaSuccess or the launch error; `launches` is incremented by
// the number of kernels enqueued.

// tc: C's tensor map when p.epi_tma (otherwise not read)
using UmmaKernelFn = void (*)(const CUtensorMap, const CUtensorMap, const CUtensorMap, const UmmaParams);
UmmaKernelFn umma_gather_kernel(bool fp8, bool split);  // the gather instances (umma_gather.cu)
UmmaKernelFn umma_gather_kernel_split(bool fp8);        // those for split-K plans (umma_gather_split.cu)
cudaError_t launch_umma(const UmmaParams &p, const CUtensorMap *tp, const CUtensorMap *tq, const CUtensorMap *tc,
                        bool fp8, bool gather, int grid, size_t smem, cudaStream_t s);
size_t umma_smem_bytes(int bn, int stages, bool gather, bool epi_tma, int split);
int umma_max_stages(int bn, bool gather, bool epi_tma, int split);
uint32_t umma_split_out_bytes(int bn, int split);  // ring bytes a split-K partial is staged in
cudaError_t launch_umma_pair(const UmmaParams &p, const CUtensorMap *tp, const CUtensorMap *tq,
                             const CUtensorMap *tc, bool fp8, int grid, size_t smem, cudaStream_t s);
size_t umma_pair_smem_bytes(int bn, int stages, bool epi_tma, int ksub);
int umma_pair_max_stages(int bn, bool epi_tma, int ksub);

cudaError_t launch_gemv_n(const GemvParams &p, const CUtensorMap *tmap_w, cudaStream_t s, int *grid_out);
size_t gemv_n_smem_bytes(int r_inst, int kper);
cudaError_t launch_gemv_k(const GemvParams &p, cudaStream_t s, int *grid_out);
cudaError_t launch_simt(const SimtParams &p, cudaStream_t s);
cudaError_t launch_scale_c(const DevView &c, int64_t M, int64_t N, float beta, const float *bias, int act, int pdl,
                           cudaStream_t s);

}  // namespace dg
