// Element load/store helpers and the shared epilogue arithmetic.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "dg_internal.h"

namespace dg {

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

// out = alpha * s_i * s_j * acc + beta * c_in   (c_in read only when beta != 0)
__device__ __forceinline__ float epi_value(float acc, float alpha_si, float sj, float beta, const char *c,
                                           int c_dtype) {
    float v = (alpha_si * sj) * acc;
    if (beta != 0.f) v = fmaf(beta, load_elem(c, c_dtype), v);
    return v;
}

}  // namespace dg
