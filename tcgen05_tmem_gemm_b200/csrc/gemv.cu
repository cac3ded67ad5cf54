// Memory-bound GEMV for up to 8 activation rows: y = alpha * x W + beta * y.
//
// The decode-time thin GEMMs of "DeepGEMM is not a new model: the inner
// discipline of GPU matrix multiplication" (§2: [1,4096]x[4096,14336]; §4:
// [1,4096]x[4096,128], the single-token Q K^T) stream W once from HBM and do
// two flops per weight, so they are judged on bytes per second.  Tensor cores
// would waste 127/128 of every instruction at M = 1; these kernels use CUDA
// cores with FP32 accumulation, and reductions in a fixed order (warp
// shuffles and shared memory, the inner-discipline page's §3.2 exchange), so
// results are deterministic.
//
//  gemv_n:  W unit-stride along n (row-major [K, N]).  A block owns a strip of
//           256 columns and a range of k.  One producer lane streams 64 x 256
//           tiles of W into a ring of shared-memory stages with TMA (the bytes
//           in flight per SM are the ring, not registers); eight consumer
//           warps read them (a lane = 8 columns) and accumulate.  The k ranges
//           of one strip form a thread-block cluster: each block leaves its
//           256 partial sums in shared memory and, after a cluster barrier,
//           block s adds slice s of the strip across the cluster through
//           distributed shared memory, in rank order ("DeepGEMM deep dive",
//           §5.2 split-K, reduced here on chip instead of through HBM).
//  gemv_k:  W unit-stride along k (K^T read in place from a row-major [N, K]
//           key matrix).  Four warps share one column, each walking a quarter
//           of k with every 16-byte load of its range in flight at once.
#include <atomic>

#include "common.cuh"
#include "sm100.cuh"

namespace dg {

namespace {

constexpr int kNB = 256;        // columns per gemv_n block
constexpr int kRows = 64;       // rows of W per TMA stage (one 32 KB box: a TMA unit's byte rate grows with box size).
                                // A block's k range (kper) is a whole number of stages, so no stage of one
                                // k split reads rows of the next split.
constexpr int kStages = 3;      // ring depth
constexpr int kCW = 8;          // consumer warps
constexpr int kNT = 32 * (kCW + 1);
constexpr int kReleaseStages = 3;  // dependents are released this many stages before the end

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

// x[r][k0 .. k0+len) -> xs[r * pitch + kk] as float, zero beyond K or R.
// 16-byte loads when x is unit-stride along k and aligned, else element loads.
template <typename T, int R>
__device__ __forceinline__ void stage_x(float *xs, int pitch, const GemvParams &p, int k0, int len, int tid,
                                        int nthreads) {
    const bool fast = p.x_vec16 && (k0 % 8 == 0);
    if (fast) {
        const int nv = (len + 7) / 8;
        for (int e = tid; e < R * nv; e += nthreads) {
            const int r = e / nv, v8 = e - r * nv, kk = v8 * 8, k = k0 + kk;
            float f[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            if (r < p.R && k < p.K) {
                const uint4 v = *reinterpret_cast<const uint4 *>(p.x.ptr + (int64_t)r * p.x_ld + (int64_t)k * 2);
                unpack8<T>(v, f);
            }
#pragma unroll
            for (int c = 0; c < 8; ++c)
                if (kk + c < len) xs[r * pitch + kk + c] = (k + c < p.K) ? f[c] : 0.f;
        }
    } else {
        for (int e = tid; e < R * len; e += nthreads) {
            const int r = e / len, kk = e - r * len, k = k0 + kk;
            float v = 0.f;
            if (r < p.R && k < p.K)
                v = load_elem(p.x.ptr + axis_offset(p.x.row, r) + axis_offset(p.x.col, k), p.x.dtype);
            xs[r * pitch + kk] = v;
        }
    }
}

__device__ __forceinline__ void store_out(const EpiParams &e, int r, int n, float acc) {
    char *cp = e.c + (int64_t)r * e.ci + (int64_t)n * e.cj;
    const float asi = e.alpha * (e.scale_i ? e.scale_i[r] : 1.f);
    const float sj = e.scale_j ? e.scale_j[n] : 1.f;
    float v = epi_value(acc, asi, sj, e.beta, cp, e.c_dtype);
    if (e.bias_j != nullptr || e.act != DG_ACT_NONE)
        v = epi_fuse(v, e.bias_j, n, e.act, e.c_dtype != DG_F32);  // bias per column n
    store_elem(cp, e.c_dtype, v);
}

struct GemvNLayout {
    uint32_t ring, xs, part, bars, flag, total;
};

__host__ __device__ inline GemvNLayout gemv_n_layout(int R, int kper) {
    GemvNLayout L;
    L.ring = 0;
    L.xs = kStages * kRows * kNB * 2;                    // 16-bit W tiles
    L.part = L.xs + (uint32_t)(R * kper * 4);
    L.bars = L.part + (uint32_t)(R * kNB * 4);
    L.flag = L.bars + 8 * 2 * kStages;
    L.total = L.flag + 16 + 1024;                        // + alignment slack
    return L;
}

template <typename T, int R>
__global__ void __launch_bounds__(kNT) gemv_n_kernel(const __grid_constant__ CUtensorMap tmap_w,
                                                     const GemvParams p) {
    if (threadIdx.x == 0) tma_prefetch_desc(&tmap_w);  // the descriptor fetch overlaps the set-up
    pdl_wait();
    if (p.pdl == 1) pdl_release();
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const GemvNLayout L = gemv_n_layout(R, p.kper);
    float *xs = reinterpret_cast<float *>(smem + L.xs);
    float *part = reinterpret_cast<float *>(smem + L.part);
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar_full = sbase + L.bars, bar_empty = bar_full + 8 * kStages;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L.flag);
    const WaitCtl wc{abort_flag, p.err_word, p.timeout_ns};

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n0 = blockIdx.x * kNB;
    const int kb0 = blockIdx.y * p.kper;
    const int kn = min(p.K - kb0, p.kper);
    const int nst = (kn + kRows - 1) / kRows;
    const int nsplit = gridDim.y;

    // The producer lane sets up the barriers and puts the first round of W
    // stages in flight (every stage is free) before x is staged, so the two
    // trips to memory overlap; the consumers see the barriers after the
    // block-wide barrier below.
    const int first_round = min(kStages, nst);
    if (warp == kCW && lane == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(bar_full + 8 * s, 1);
            mbar_init(bar_empty + 8 * s, kCW);
        }
        *abort_flag = 0;
        fence_barrier_init();
        fence_proxy_async_smem();
        for (int it = 0; it < first_round; ++it) {
            mbar_arrive_expect_tx(bar_full + 8 * it, kRows * kNB * 2);
            tma_load_2d(sbase + L.ring + it * (kRows * kNB * 2), &tmap_w, bar_full + 8 * it, n0, kb0 + it * kRows);
        }
    }
    stage_x<T, R>(xs, p.kper, p, kb0, kn, threadIdx.x, kNT);
    __syncthreads();

    if (warp == kCW) {
        // ----------------------------------------------------- TMA producer
        if (lane == 0) {
            int it = first_round;
            const int release_at = max(0, nst - kReleaseStages);
            if (release_at < first_round && p.pdl == 2) pdl_release();
            for (; it < nst; ++it) {
                const int s = it % kStages;
                const uint32_t ph = (uint32_t)(it / kStages) & 1u;
                // a few stages before the end: let the next kernel be scheduled, so its
                // launch latency overlaps this kernel's last loads and reduction
                if (it == release_at && p.pdl == 2) pdl_release();
                if (!mbar_wait(bar_empty + 8 * s, ph ^ 1u, wc)) break;
                mbar_arrive_expect_tx(bar_full + 8 * s, kRows * kNB * 2);
                tma_load_2d(sbase + L.ring + s * (kRows * kNB * 2), &tmap_w, bar_full + 8 * s, n0, kb0 + it * kRows);
            }
            for (int d = 1; d <= kStages && it - d >= 0; ++d) {
                const int j = it - d;
                mbar_wait_drain(bar_full + 8 * (j % kStages), (uint32_t)(j / kStages) & 1u, p.timeout_ns);
            }
        }
    } else {
        // -------------------------------------------------------- consumers
        float acc[R][8];
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int c = 0; c < 8; ++c) acc[r][c] = 0.f;
        for (int it = 0; it < nst; ++it) {
            const int s = it % kStages;
            const uint32_t ph = (uint32_t)(it / kStages) & 1u;
            if (!mbar_wait(bar_full + 8 * s, ph, wc)) break;
            const uint8_t *tile = smem + L.ring + s * (kRows * kNB * 2);
            uint4 v[kRows / kCW];
#pragma unroll
            for (int j = 0; j < kRows / kCW; ++j)
                v[j] = *reinterpret_cast<const uint4 *>(tile + (warp + kCW * j) * (kNB * 2) + lane * 16);
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_empty + 8 * s);
#pragma unroll
            for (int j = 0; j < kRows / kCW; ++j) {
                const int kk = it * kRows + warp + kCW * j;
                if (kk >= kn) continue;  // rows past this block's range (TMA fills past K with zeros)
                float f[8];
                unpack8<T>(v[j], f);
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    const float xv = xs[r * p.kper + kk];
#pragma unroll
                    for (int c = 0; c < 8; ++c) acc[r][c] = fmaf(xv, f[c], acc[r][c]);
                }
            }
        }
        // the ring is free once every consumer warp is past its loop
        asm volatile("bar.sync 1, %0;" ::"n"(kCW * 32) : "memory");
        float *red = reinterpret_cast<float *>(smem + L.ring);   // [kCW][R][kNB]
#pragma unroll
        for (int r = 0; r < R; ++r) {
            float4 *dst = reinterpret_cast<float4 *>(red + (warp * R + r) * kNB + lane * 8);
            dst[0] = make_float4(acc[r][0], acc[r][1], acc[r][2], acc[r][3]);
            dst[1] = make_float4(acc[r][4], acc[r][5], acc[r][6], acc[r][7]);
        }
        asm volatile("bar.sync 1, %0;" ::"n"(kCW * 32) : "memory");
        for (int e = threadIdx.x; e < R * kNB; e += kCW * 32) {
            const int r = e / kNB, j = e - r * kNB;
            float sum = 0.f;
#pragma unroll
            for (int w = 0; w < kCW; ++w) sum += red[(w * R + r) * kNB + j];
            if (nsplit == 1) {
                if (r < p.R && n0 + j < p.N) store_out(p.epi, r, n0 + j, sum);
            } else {
                part[r * kNB + j] = sum;
            }
        }
    }
    if (nsplit == 1) return;

    // ---------------------------------------------- cluster reduction of k splits
    __syncthreads();
    cluster_sync();
    {
        const uint32_t rank = cluster_ctarank();
        const int c0 = (int)(rank * kNB / nsplit), c1 = (int)((rank + 1) * kNB / nsplit);
        const int width = c1 - c0;
        const uint32_t part_addr = sbase + L.part;
        for (int e = threadIdx.x; e < R * width; e += kNT) {
            const int r = e / width, j = c0 + (e - r * width);
            if (r >= p.R || n0 + j >= p.N) continue;
            // all remote loads issued before the sum, which runs in rank order
            float v[8];
#pragma unroll
            for (int q = 0; q < 8; ++q)
                v[q] = q < nsplit ? dsmem_ld_f32(dsmem_map(part_addr + (r * kNB + j) * 4, q)) : 0.f;
            float sum = 0.f;
#pragma unroll
            for (int q = 0; q < 8; ++q)
                if (q < nsplit) sum += v[q];
            store_out(p.epi, r, n0 + j, sum);
        }
    }
    cluster_sync();  // keep every block's partials alive until all remote reads are done
}

// Four warps per column; a block covers two columns.  A warp's loads over its
// quarter of k are all issued before any is used.
template <typename T, int R>
__global__ void __launch_bounds__(256) gemv_k_kernel(const GemvParams p) {
    constexpr int WPC = 4;
    constexpr int CPB = 8 / WPC;
    constexpr int MAXV = 8;                 // 16-byte loads per lane kept in flight
    pdl_wait_then_release();
    extern __shared__ float smem[];
    float *xs = smem;                       // [R][K]
    float *red = smem + R * p.K;            // [8 warps][R]

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int n = blockIdx.x * CPB + warp / WPC;
    const int q = warp % WPC;
    const bool col_ok = n < p.N;
    const char *wrow = p.w + (int64_t)(col_ok ? n : 0) * p.w_ld;
    // this warp's k range, a multiple of 8 elements
    const int kq = ((p.K / 8 + WPC - 1) / WPC) * 8;
    const int ka = q * kq, kb = min(p.K, ka + kq);

    // the first batch of this warp's W loads goes out before x is staged, so
    // the two round trips to memory overlap
    const int kfirst = ka + lane * 8;
    uint4 vfirst[MAXV];
#pragma unroll
    for (int u = 0; u < MAXV; ++u) {
        const int k = kfirst + u * 256;
        vfirst[u] = (col_ok && k < kb) ? ldg_stream(wrow + (int64_t)k * sizeof(T)) : make_uint4(0, 0, 0, 0);
    }
    stage_x<T, R>(xs, p.K, p, 0, p.K, threadIdx.x, 256);
    __syncthreads();
    float acc[R];
#pragma unroll
    for (int r = 0; r < R; ++r) acc[r] = 0.f;
    // one batch of MAXV 16-byte loads per lane: the first was issued above
    auto consume = [&](int k0, const uint4 (&v)[MAXV]) {
#pragma unroll
        for (int u = 0; u < MAXV; ++u) {
            const int k = k0 + u * 256;
            if (k >= kb) break;
            float f[8];
            unpack8<T>(v[u], f);
#pragma unroll
            for (int r = 0; r < R; ++r) {
                const float4 x0 = *reinterpret_cast<const float4 *>(xs + r * p.K + k);
                const float4 x1 = *reinterpret_cast<const float4 *>(xs + r * p.K + k + 4);
                acc[r] = fmaf(x0.x, f[0], acc[r]);
                acc[r] = fmaf(x0.y, f[1], acc[r]);
                acc[r] = fmaf(x0.z, f[2], acc[r]);
                acc[r] = fmaf(x0.w, f[3], acc[r]);
                acc[r] = fmaf(x1.x, f[4], acc[r]);
                acc[r] = fmaf(x1.y, f[5], acc[r]);
                acc[r] = fmaf(x1.z, f[6], acc[r]);
                acc[r] = fmaf(x1.w, f[7], acc[r]);
            }
        }
    };
    if (col_ok) {
        consume(kfirst, vfirst);
        for (int k0 = kfirst + 32 * 8 * MAXV; k0 < kb; k0 += 32 * 8 * MAXV) {
            uint4 v[MAXV];
#pragma unroll
            for (int u = 0; u < MAXV; ++u) {
                const int k = k0 + u * 256;
                v[u] = (k < kb) ? ldg_stream(wrow + (int64_t)k * sizeof(T)) : make_uint4(0, 0, 0, 0);
            }
            consume(k0, v);
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

// Raise a kernel's dynamic shared-memory limit once per device and size, not
// per call (`Tag` gives each kernel instantiation its own record).
template <typename Tag, typename K>
cudaError_t ensure_smem(K kern, size_t smem, bool prefer_max_shared = false) {
    static SmemLimit limit;
    return limit.ensure(kern, smem, prefer_max_shared);
}

template <typename T, int R, int Kind>
struct KernelTag {};

template <typename T, int R>
cudaError_t run_n(const GemvParams &p, const CUtensorMap *tmap, cudaStream_t s, int *grid_out) {
    if (p.kper <= 0 || p.kper % kRows != 0) return cudaErrorInvalidValue;  // whole stages per k split
    const int gx = (p.N + kNB - 1) / kNB;
    const int gy = (p.K + p.kper - 1) / p.kper;
    const size_t smem = gemv_n_layout(R, p.kper).total;
    auto kern = gemv_n_kernel<T, R>;
    cudaError_t e = ensure_smem<KernelTag<T, R, 0>>(kern, smem);
    if (e != cudaSuccess) return e;
    e = launch_ex(kern, dim3(gx, gy), dim3(kNT), smem, s, dim3(1, gy, 1), p.pdl, *tmap, p);
    *grid_out = gx * gy;
    return e;
}

template <typename T>
cudaError_t run_n_r(const GemvParams &p, const CUtensorMap *tmap, cudaStream_t s, int *grid_out) {
    if (p.R <= 1) return run_n<T, 1>(p, tmap, s, grid_out);
    if (p.R <= 2) return run_n<T, 2>(p, tmap, s, grid_out);
    if (p.R <= 4) return run_n<T, 4>(p, tmap, s, grid_out);
    return run_n<T, 8>(p, tmap, s, grid_out);
}

template <typename T, int R>
cudaError_t run_k(const GemvParams &p, cudaStream_t s, int *grid_out) {
    const int grid = (p.N + 1) / 2;
    const size_t smem = sizeof(float) * ((size_t)R * p.K + 8 * R);
    auto kern = gemv_k_kernel<T, R>;
    // it often runs beside the N-contiguous GEMV (decode steps): keep SMs shared-memory heavy
    cudaError_t e = ensure_smem<KernelTag<T, R, 1>>(kern, smem, true);
    if (e != cudaSuccess) return e;
    *grid_out = grid;
    return launch_ex(kern, dim3(grid), dim3(256), smem, s, dim3(1, 1, 1), p.pdl, p);
}

template <typename T>
cudaError_t run_k_r(const GemvParams &p, cudaStream_t s, int *grid_out) {
    if (p.R <= 1) return run_k<T, 1>(p, s, grid_out);
    if (p.R <= 2) return run_k<T, 2>(p, s, grid_out);
    if (p.R <= 4) return run_k<T, 4>(p, s, grid_out);
    return run_k<T, 8>(p, s, grid_out);
}

}  // namespace

size_t gemv_n_smem_bytes(int r_inst, int kper) { return gemv_n_layout(r_inst, kper).total; }

cudaError_t launch_gemv_n(const GemvParams &p, const CUtensorMap *tmap, cudaStream_t s, int *grid_out) {
    if (p.in_dtype == DG_BF16) return run_n_r<__nv_bfloat16>(p, tmap, s, grid_out);
    if (p.in_dtype == DG_F16) return run_n_r<__half>(p, tmap, s, grid_out);
    return cudaErrorInvalidValue;
}

cudaError_t launch_gemv_k(const GemvParams &p, cudaStream_t s, int *grid_out) {
    if (p.in_dtype == DG_BF16) return run_k_r<__nv_bfloat16>(p, s, grid_out);
    if (p.in_dtype == DG_F16) return run_k_r<__half>(p, s, grid_out);
    return cudaErrorInvalidValue;
}

}  // namespace dg
