// Element load/store helpers and the shared epilogue arithmetic.
#pragma once

#include <atomic>
#include <mutex>

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "dg_internal.h"

namespace dg {

// The dynamic shared-memory limit of one kernel, raised per device: the
// attribute set by cudaFuncSetAttribute belongs to the current device, so a
// record per process would skip the call on a second device.  The limit only
// ever grows (under a lock), so a launch that needs less never lowers it
// beneath a concurrent launch that needs more.
struct SmemLimit {
    static constexpr int kDevices = 64;
    std::atomic<int> bytes[kDevices] = {};
    std::atomic<int> carve[kDevices] = {};
    std::mutex mu;

    // prefer_max_shared: also ask that an SM running this kernel keep its
    // whole unified L1/shared memory as shared memory, so that blocks of a
    // shared-memory-hungry kernel on another stream (two 104 KB blocks of
    // the N-contiguous GEMV per SM) still fit beside it.  A kernel with a
    // small footprint otherwise gets an L1-heavy split, and an SM configured
    // that way takes no large blocks until it drains.
    template <typename Kern>
    cudaError_t ensure(Kern kern, size_t need, bool prefer_max_shared = false) {
        if (need <= 48 * 1024 && !prefer_max_shared) return cudaSuccess;  // the default limit
        int dev = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e != cudaSuccess) return e;
        if (dev < 0 || dev >= kDevices) return cudaErrorInvalidDevice;
        if (prefer_max_shared && carve[dev].load(std::memory_order_acquire) == 0) {
            std::lock_guard<std::mutex> lk(mu);
            if (carve[dev].load(std::memory_order_relaxed) == 0) {
                e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                                         (int)cudaSharedmemCarveoutMaxShared);
                if (e != cudaSuccess) return e;
                carve[dev].store(1, std::memory_order_release);
            }
        }
        if (need <= 48 * 1024) return cudaSuccess;
        if (bytes[dev].load(std::memory_order_acquire) >= (int)need) return cudaSuccess;
        std::lock_guard<std::mutex> lk(mu);
        if (bytes[dev].load(std::memory_order_relaxed) >= (int)need) return cudaSuccess;
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)need);
        if (e == cudaSuccess) bytes[dev].store((int)need, std::memory_order_release);
        return e;
    }
};

// Programmatic dependent launch.  Every kernel here is launched with
// programmatic stream serialisation: it may be scheduled while the previous
// kernel on the stream is still running, so its very first action is to wait
// for that kernel to complete (and its writes to be visible) before touching
// global memory.  Short kernels then release their dependents at once; long
// ones release them at their tail (after the main loop), so waiting
// dependents do not hold SM slots while the main loop runs.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_release() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait_then_release() {
    pdl_wait();
    pdl_release();
}

// cudaLaunchKernelEx with programmatic stream serialisation and an optional
// thread-block cluster shape.
template <typename Kern, typename... Args>
cudaError_t launch_ex(Kern kern, dim3 grid, dim3 block, size_t smem, cudaStream_t s, dim3 cluster, int pdl,
                      Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    int n = 0;
    if (pdl) {
        attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[n].val.programmaticStreamSerializationAllowed = 1;
        ++n;
    }
    if (cluster.x * cluster.y * cluster.z > 1) {
        attr[n].id = cudaLaunchAttributeClusterDimension;
        attr[n].val.clusterDim.x = cluster.x;
        attr[n].val.clusterDim.y = cluster.y;
        attr[n].val.clusterDim.z = cluster.z;
        ++n;
    }
    cfg.attrs = attr;
    cfg.numAttrs = n;
    // The launch's own result is the return value.  A failed launch also
    // leaves its error as the thread's last error: consume it, so that it is
    // not reported again by a later call (the library's or the caller's); an
    // error someone else left pending is not this launch's and is left alone.
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, args...);
    if (e != cudaSuccess) cudaGetLastError();
    return e;
}

__device__ __forceinline__ float load_elem(const char *p, int dtype) {
    switch (dtype) {
    case DG_F32: return *reinterpret_cast<const float *>(p);
    case DG_F16: return __half2float(*reinterpret_cast<const __half *>(p));
    case DG_BF16: return __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(p));
    case DG_E4M3: {
        __half_raw h = __nv_cvt_fp8_to_halfraw(*reinterpret_cast<const __nv_fp8_storage_t *>(p), __NV_E4M3);
        return __half2float(__half(h));
    }
    default: return 0.f;
    }
}

__device__ __forceinline__ void store_elem(char *p, int dtype, float v) {
    switch (dtype) {
    case DG_F32: *reinterpret_cast<float *>(p) = v; break;
    case DG_F16: *reinterpret_cast<__half *>(p) = __float2half_rn(v); break;
    case DG_BF16: *reinterpret_cast<__nv_bfloat16 *>(p) = __float2bfloat16_rn(v); break;
    default: break;
    }
}

__host__ __device__ __forceinline__ int elem_bytes(int dtype) {
    return dtype == DG_F32 ? 4 : dtype == DG_E4M3 ? 1 : 2;
}

// The hardware's tanh approximation (one instruction; the PTX ISA gives its
// largest relative error as about 2^-11).
__device__ __forceinline__ float tanh_approx(float x) {
    float y;
    asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// The fused activation ("DeepGEMM is not a new model: the inner discipline of
// GPU matrix multiplication", §3.3: GeLU in its tanh form after the bias add,
// with a fast tanh).  ReLU keeps NaN; GeLU is
// z/2 (1 + tanh(sqrt(2/pi) (z + 0.044715 z^3))), evaluated as h + h tanh(u)
// with h = z/2 and u = z (sqrt(2/pi) + 0.044715 sqrt(2/pi) z^2): six
// operations, one of them the tanh.  For a 16-bit output (`FAST`) the tanh is
// the hardware approximation, whose error (2^-11 of the tanh) stays below the
// output's own rounding (2^-9 for BF16, 2^-11 for FP16); an FP32 output takes
// the accurate tanhf, so it keeps FP32 accuracy.
template <bool FAST>
__device__ __forceinline__ float gelu_tanh(float z) {
    const float u = z * fmaf(0.035677408136300125f, z * z, 0.7978845608028654f);
    const float t = FAST ? tanh_approx(u) : tanhf(u);
    const float h = 0.5f * z;
    return fmaf(h, t, h);
}

// The activation chosen at compile time (the epilogues pick the instance once
// per tile, so no element pays for the choice).
template <int ACT, bool FAST>
__device__ __forceinline__ float act_fn(float z) {
    if (ACT == DG_ACT_RELU) return z < 0.f ? 0.f : z;
    if (ACT == DG_ACT_GELU_TANH) return gelu_tanh<FAST>(z);
    return z;
}

__device__ __forceinline__ float act_apply(int act, float z, bool fast = false) {
    if (act == DG_ACT_RELU) return act_fn<DG_ACT_RELU, false>(z);
    if (act == DG_ACT_GELU_TANH) return fast ? gelu_tanh<true>(z) : gelu_tanh<false>(z);
    return z;
}

// The bias add and activation of the epilogue, for an epilogue that has them.
__device__ __forceinline__ float epi_fuse(float z, const float *bias, int64_t idx, int act, bool fast) {
    if (bias != nullptr) z += bias[idx];
    return act_apply(act, z, fast);
}

// out = act(alpha * s_i * s_j * acc + beta * c_in + bias)   (c_in read only when beta != 0)
__device__ __forceinline__ float epi_value(float acc, float alpha_si, float sj, float beta, const char *c,
                                           int c_dtype) {
    float v = (alpha_si * sj) * acc;
    if (beta != 0.f) v = fmaf(beta, load_elem(c, c_dtype), v);
    return v;
}

}  // namespace dg
