// Memory-bound GEMV for up to 8 activation rows: y = alpha * x W + beta * y.
//
// The decode-time thin GEMMs of "DeepGEMM is not a new model: the inner
// discipline of GPU matrix multiplication" (§2: [1,4096]x[4096,14336]; §4:
// [1,4096]x[4096,128], the single-token Q K^T) stream W once from HBM and do
// two flops per weight, so they are judged on bytes per second.  Tensor cores
// would waste 127/128 of every instruction at M = 1; these kernels use CUDA
// cores with 16-byte coalesced loads, FP32 accumulation and a warp-shuffle
// plus shared-memory reduction (inner-discipline page §3.2, the shuffle
// exchange), and no atomics, so results are deterministic.
//
//  gemv_n:  W unit-stride along n (row-major [K, N]).  A thread owns 8
//           consecutive columns; a warp covers TX threads along n and 32/TX
//           rows along k; the block's 8 warps split k further.
//  gemv_k:  W unit-stride along k (e.g. K^T read in place from a row-major
//           [N, K] key matrix).  A warp walks one column's k range with
//           16-byte loads; four warps share one column and meet in shared
//           memory.
#include "common.cuh"

namespace dg {

namespace {

constexpr int NT = 256;       // threads per block
constexpr int KC = 1024;      // k rows of x staged in shared memory at a time

template <typename T>
__device__ __forceinline__ void unpack8(const uint4 &v, float (&f)[8]);

template <>
__device__ __forceinline__ void unpack8<__nv_bfloat16>(const uint4 &v, float (&f)[8]) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}

template <>
__device__ __forceinline__ void unpack8<__half>(const uint4 &v, float (&f)[8]) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        __half2 h = *reinterpret_cast<const __half2 *>(&w[i]);
        float2 t = __half22float2(h);
        f[2 * i] = t.x;
        f[2 * i + 1] = t.y;
    }
}

__device__ __forceinline__ uint4 ldg_stream(const void *p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

// Stage x[r][k0 .. k0+KC) as float (zero beyond K or R).
template <int R>
__device__ __forceinline__ void stage_x(float *xs, const GemvParams &p, int k0) {
    for (int e = threadIdx.x; e < R * KC; e += NT) {
        const int r = e / KC, kk = e % KC, k = k0 + kk;
        float v = 0.f;
        if (r < p.R && k < p.K)
            v = load_elem(p.x.ptr + axis_offset(p.x.row, r) + axis_offset(p.x.col, k), p.x.dtype);
        xs[r * KC + kk] = v;
    }
}

__device__ __forceinline__ void store_out(const EpiParams &e, int r, int n, float acc) {
    char *cp = e.c + (int64_t)r * e.ci + (int64_t)n * e.cj;
    const float asi = e.alpha * (e.scale_i ? e.scale_i[r] : 1.f);
    const float sj = e.scale_j ? e.scale_j[n] : 1.f;
    store_elem(cp, e.c_dtype, epi_value(acc, asi, sj, e.beta, cp, e.c_dtype));
}

template <typename T, int R, int TX>
__global__ void __launch_bounds__(NT) gemv_n_kernel(const GemvParams p) {
    constexpr int KY_W = 32 / TX;           // k rows per warp step
    constexpr int KY = KY_W * (NT / 32);    // k rows per block step
    constexpr int NB = 8 * TX;              // columns per block
    extern __shared__ float smem[];
    float *xs = smem;                       // [R][KC]
    float *red = smem + R * KC;             // [8 warps][R][NB]

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int tx = lane % TX, ky = warp * KY_W + lane / TX;
    const int n = blockIdx.x * NB + tx * 8;
    const bool col_ok = n < p.N;            // N % 8 == 0 is guaranteed by the dispatcher
    float acc[R][8];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[r][c] = 0.f;

    const char *wcol = p.w + (int64_t)n * sizeof(T);
    for (int k0 = 0; k0 < p.K; k0 += KC) {
        __syncthreads();
        stage_x<R>(xs, p, k0);
        __syncthreads();
        const int kend = min(KC, p.K - k0);
        if (col_ok) {
            int kk = ky;
            constexpr int U = 4;
            for (; kk + (U - 1) * KY < kend; kk += U * KY) {
                uint4 v[U];
#pragma unroll
                for (int u = 0; u < U; ++u) v[u] = ldg_stream(wcol + (int64_t)(k0 + kk + u * KY) * p.w_ld);
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    float f[8];
                    unpack8<T>(v[u], f);
#pragma unroll
                    for (int r = 0; r < R; ++r) {
                        const float xv = xs[r * KC + kk + u * KY];
#pragma unroll
                        for (int c = 0; c < 8; ++c) acc[r][c] = fmaf(xv, f[c], acc[r][c]);
                    }
                }
            }
            for (; kk < kend; kk += KY) {
                uint4 v = ldg_stream(wcol + (int64_t)(k0 + kk) * p.w_ld);
                float f[8];
                unpack8<T>(v, f);
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    const float xv = xs[r * KC + kk];
#pragma unroll
                    for (int c = 0; c < 8; ++c) acc[r][c] = fmaf(xv, f[c], acc[r][c]);
                }
            }
        }
    }
    // reduce the KY_W rows inside the warp (lanes tx, tx+TX, ...)
#pragma unroll
    for (int off = TX; off < 32; off <<= 1)
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int c = 0; c < 8; ++c) acc[r][c] += __shfl_xor_sync(0xffffffffu, acc[r][c], off);
    if (lane < TX) {
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int c = 0; c < 8; ++c) red[(warp * R + r) * NB + tx * 8 + c] = acc[r][c];
    }
    __syncthreads();
    // across the 8 warps, in warp order, then the epilogue
    for (int e = threadIdx.x; e < R * NB; e += NT) {
        const int r = e / NB, j = e % NB;
        const int nn = blockIdx.x * NB + j;
        if (r >= p.R || nn >= p.N) continue;
        float s = 0.f;
#pragma unroll
        for (int w = 0; w < NT / 32; ++w) s += red[(w * R + r) * NB + j];
        store_out(p.epi, r, nn, s);
    }
}

// Four warps per column; a block covers two columns.
template <typename T, int R>
__global__ void __launch_bounds__(NT) gemv_k_kernel(const GemvParams p) {
    constexpr int WPC = 4;                  // warps per column
    constexpr int CPB = (NT / 32) / WPC;    // columns per block
    extern __shared__ float smem[];
    float *xs = smem;                       // [R][KC]
    float *red = smem + R * KC;             // [8 warps][R]

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int n = blockIdx.x * CPB + warp / WPC;
    const int q = warp % WPC;
    const bool col_ok = n < p.N;
    const char *wrow = p.w + (int64_t)(col_ok ? n : 0) * p.w_ld;
    float acc[R];
#pragma unroll
    for (int r = 0; r < R; ++r) acc[r] = 0.f;

    for (int k0 = 0; k0 < p.K; k0 += KC) {
        __syncthreads();
        stage_x<R>(xs, p, k0);
        __syncthreads();
        const int kend = min(KC, p.K - k0);   // K % 8 == 0 is guaranteed
        if (col_ok) {
            // this warp's quarter of the chunk, 8 elements per lane per step
            for (int kk = (q * 32 + lane) * 8; kk < kend; kk += WPC * 32 * 8) {
                uint4 v = ldg_stream(wrow + (int64_t)(k0 + kk) * sizeof(T));
                float f[8];
                unpack8<T>(v, f);
#pragma unroll
                for (int r = 0; r < R; ++r)
#pragma unroll
                    for (int c = 0; c < 8; ++c) acc[r] = fmaf(xs[r * KC + kk + c], f[c], acc[r]);
            }
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
#pragma unroll
        for (int r = 0; r < R; ++r) acc[r] += __shfl_xor_sync(0xffffffffu, acc[r], off);
    if (lane == 0)
#pragma unroll
        for (int r = 0; r < R; ++r) red[warp * R + r] = acc[r];
    __syncthreads();
    if (threadIdx.x < CPB * R) {
        const int c = threadIdx.x / R, r = threadIdx.x % R;
        const int nn = blockIdx.x * CPB + c;
        if (r < p.R && nn < p.N) {
            float s = 0.f;
#pragma unroll
            for (int w = 0; w < WPC; ++w) s += red[((c * WPC) + w) * R + r];
            store_out(p.epi, r, nn, s);
        }
    }
}

template <typename T, int R, int TX>
cudaError_t run_n(const GemvParams &p, cudaStream_t s, int *grid_out) {
    constexpr int NB = 8 * TX;
    const int grid = (p.N + NB - 1) / NB;
    const size_t smem = sizeof(float) * (R * KC + (NT / 32) * R * NB);
    auto kern = gemv_n_kernel<T, R, TX>;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    kern<<<grid, NT, smem, s>>>(p);
    *grid_out = grid;
    return cudaGetLastError();
}

template <typename T, int R>
cudaError_t run_n_tx(const GemvParams &p, cudaStream_t s, int num_sms, int *grid_out) {
    // widest warp footprint along n that still gives every SM a block
    const int blocks32 = (p.N + 255) / 256, blocks16 = (p.N + 127) / 128, blocks8 = (p.N + 63) / 64;
    if (blocks32 >= num_sms) return run_n<T, R, 32>(p, s, grid_out);
    if (blocks16 >= num_sms) return run_n<T, R, 16>(p, s, grid_out);
    if (blocks8 >= num_sms) return run_n<T, R, 8>(p, s, grid_out);
    return run_n<T, R, 4>(p, s, grid_out);
}

template <typename T>
cudaError_t run_n_r(const GemvParams &p, cudaStream_t s, int num_sms, int *grid_out) {
    if (p.R <= 1) return run_n_tx<T, 1>(p, s, num_sms, grid_out);
    if (p.R <= 2) return run_n_tx<T, 2>(p, s, num_sms, grid_out);
    if (p.R <= 4) return run_n_tx<T, 4>(p, s, num_sms, grid_out);
    return run_n_tx<T, 8>(p, s, num_sms, grid_out);
}

template <typename T, int R>
cudaError_t run_k(const GemvParams &p, cudaStream_t s, int *grid_out) {
    constexpr int CPB = 2;
    const int grid = (p.N + CPB - 1) / CPB;
    const size_t smem = sizeof(float) * (R * KC + (NT / 32) * R);
    auto kern = gemv_k_kernel<T, R>;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    kern<<<grid, NT, smem, s>>>(p);
    *grid_out = grid;
    return cudaGetLastError();
}

template <typename T>
cudaError_t run_k_r(const GemvParams &p, cudaStream_t s, int *grid_out) {
    if (p.R <= 1) return run_k<T, 1>(p, s, grid_out);
    if (p.R <= 2) return run_k<T, 2>(p, s, grid_out);
    if (p.R <= 4) return run_k<T, 4>(p, s, grid_out);
    return run_k<T, 8>(p, s, grid_out);
}

}  // namespace

cudaError_t launch_gemv_n(const GemvParams &p, cudaStream_t s, int num_sms, int *grid_out) {
    if (p.in_dtype == DG_BF16) return run_n_r<__nv_bfloat16>(p, s, num_sms, grid_out);
    if (p.in_dtype == DG_F16) return run_n_r<__half>(p, s, num_sms, grid_out);
    return cudaErrorInvalidValue;
}

cudaError_t launch_gemv_k(const GemvParams &p, cudaStream_t s, int num_sms, int *grid_out) {
    (void)num_sms;
    if (p.in_dtype == DG_BF16) return run_k_r<__nv_bfloat16>(p, s, grid_out);
    if (p.in_dtype == DG_F16) return run_k_r<__half>(p, s, grid_out);
    return cudaErrorInvalidValue;
}

}  // namespace dg
