// CUDA-core kernels that accept any view:
//  - simt_gemm: a plain shared-memory tiled GEMM (64x64 tile, 4x4 per thread)
//    reading every operand through the view addressing, FP32 accumulation.
//    It is the bisection baseline (DG_OPT_FORCE_KIND = DG_KIND_SIMT) and the
//    path for layouts the tensor-core kernel does not take.
//  - scale_c: C = beta * C (or 0 when beta == 0), then the fused bias and
//    activation, for alpha == 0 or K == 0, where the product is not formed
//    ("DeepGEMM: a recalibration of the compute paradigm", §4.3: beta must
//    still be applied when A is skipped).
#include "common.cuh"

namespace dg {

namespace {

constexpr int TM = 64, TN = 64, TK = 16, NT = 256;

__global__ void __launch_bounds__(NT) simt_gemm_kernel(const SimtParams p) {
    pdl_wait_then_release();
    __shared__ float As[TK][TM + 4];
    __shared__ float Bs[TK][TN + 4];
    __shared__ int64_t a_row_off[TM], b_col_off[TN];
    __shared__ int64_t a_col_off[TK], b_row_off[TK];

    const int tid = threadIdx.x;
    const int m0 = blockIdx.y * TM, n0 = blockIdx.x * TN;
    if (tid < TM) a_row_off[tid] = (m0 + tid < p.M) ? axis_offset(p.a.row, m0 + tid) : -1;
    else if (tid < TM + TN) {
        const int j = tid - TM;
        b_col_off[j] = (n0 + j < p.N) ? axis_offset(p.b.col, n0 + j) : -1;
    }
    const int tx = tid % 16, ty = tid / 16;  // 16 x 16 threads, 4 x 4 outputs each
    float acc[4][4] = {};

    for (int k0 = 0; k0 < p.K; k0 += TK) {
        __syncthreads();
        if (tid < TK) a_col_off[tid] = (k0 + tid < p.K) ? axis_offset(p.a.col, k0 + tid) : -1;
        else if (tid < 2 * TK) {
            const int kk = tid - TK;
            b_row_off[kk] = (k0 + kk < p.K) ? axis_offset(p.b.row, k0 + kk) : -1;
        }
        __syncthreads();
        for (int e = tid; e < TK * TM; e += NT) {
            const int kk = e / TM, mm = e % TM;
            const int64_t ro = a_row_off[mm], co = a_col_off[kk];
            As[kk][mm] = (ro >= 0 && co >= 0) ? load_elem(p.a.ptr + ro + co, p.a.dtype) : 0.f;
        }
        for (int e = tid; e < TK * TN; e += NT) {
            const int kk = e / TN, nn = e % TN;
            const int64_t ro = b_row_off[kk], co = b_col_off[nn];
            Bs[kk][nn] = (ro >= 0 && co >= 0) ? load_elem(p.b.ptr + ro + co, p.b.dtype) : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < TK; ++kk) {
            float a[4], b[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
            for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx * 4 + j];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
        }
    }

    const EpiParams &e = p.epi;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int m = m0 + ty * 4 + i;
        if (m >= p.M) continue;
        const float asi = e.alpha * (e.scale_i ? e.scale_i[m] : 1.f);
        const int64_t cro = axis_offset(p.c.row, m);
        char *cp[4];
        float cin[4], sj[4], bj[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {  // every load before the first store
            const int n = n0 + tx * 4 + j;
            cp[j] = n < p.N ? const_cast<char *>(p.c.ptr) + cro + axis_offset(p.c.col, n) : nullptr;
            cin[j] = (cp[j] && e.beta != 0.f) ? load_elem(cp[j], p.c.dtype) : 0.f;
            sj[j] = (cp[j] && e.scale_j) ? e.scale_j[n] : 1.f;
            bj[j] = (cp[j] && e.bias_j) ? e.bias_j[n] : 0.f;
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            if (!cp[j]) continue;
            float v = (asi * sj[j]) * acc[i][j];
            if (e.beta != 0.f) v = fmaf(e.beta, cin[j], v);
            if (e.bias_j != nullptr || e.act != DG_ACT_NONE) v = act_apply(e.act, v + bj[j], p.c.dtype != DG_F32);
            store_elem(cp[j], p.c.dtype, v);
        }
    }
}

// C = act(beta * C + bias[n]) (the product term is zero).
__global__ void scale_c_kernel(const DevView c, int64_t M, int64_t N, float beta, const float *bias, int act) {
    pdl_wait_then_release();
    const int64_t total = M * N;
    const bool fused = bias != nullptr || act != DG_ACT_NONE;
    for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total;
         e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t m = e / N, n = e - (e / N) * N;
        char *cp = const_cast<char *>(c.ptr) + axis_offset(c.row, m) + axis_offset(c.col, n);
        float v = beta != 0.f ? beta * load_elem(cp, c.dtype) : 0.f;
        if (fused) v = epi_fuse(v, bias, n, act, c.dtype != DG_F32);
        store_elem(cp, c.dtype, v);
    }
}

}  // namespace

cudaError_t launch_simt(const SimtParams &p, cudaStream_t s) {
    dim3 grid((p.N + TN - 1) / TN, (p.M + TM - 1) / TM);
    if (grid.y > 65535) return cudaErrorInvalidConfiguration;
    return launch_ex(simt_gemm_kernel, grid, dim3(NT), 0, s, dim3(1, 1, 1), p.pdl, p);
}

cudaError_t launch_scale_c(const DevView &c, int64_t M, int64_t N, float beta, const float *bias, int act, int pdl,
                           cudaStream_t s) {
    const int64_t total = M * N;
    int blocks = (int)std::min<int64_t>((total + 255) / 256, 148 * 16);
    if (blocks < 1) blocks = 1;
    return launch_ex(scale_c_kernel, dim3(blocks), dim3(256), 0, s, dim3(1, 1, 1), pdl, c, M, N, beta, bias, act);
}

}  // namespace dg
