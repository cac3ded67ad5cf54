// Epilogue pieces shared by the tensor-core kernels.
#pragma once

#include "common.cuh"

namespace dg {

// Apply  out = alpha * s_i * s_j * acc + beta * C  to the 16 consecutive
// columns jb .. jb+15 of one output row (row pointer `crow`, per-row factor
// asi = alpha * s_i) and store them: 16-byte vector stores when C is
// contiguous along j and the chunk is whole, otherwise element stores for any
// strides, with every C load of the chunk issued before the first store.
__device__ __forceinline__ void epilogue_chunk16(const EpiParams &e, char *crow, float asi, int jb, int Nj,
                                                 const uint32_t (&r)[16]) {
    if (e.vec_ok && jb + 16 <= Nj) {
        float v[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) {
            const float sj = e.scale_j ? e.scale_j[jb + c] : 1.f;
            v[c] = (asi * sj) * __uint_as_float(r[c]);
        }
        if (e.c_dtype == DG_F32) {
            float4 *dst = reinterpret_cast<float4 *>(crow + (int64_t)jb * 4);
            if (e.beta != 0.f) {
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float4 o = dst[q];
                    v[4 * q + 0] = fmaf(e.beta, o.x, v[4 * q + 0]);
                    v[4 * q + 1] = fmaf(e.beta, o.y, v[4 * q + 1]);
                    v[4 * q + 2] = fmaf(e.beta, o.z, v[4 * q + 2]);
                    v[4 * q + 3] = fmaf(e.beta, o.w, v[4 * q + 3]);
                }
            }
#pragma unroll
            for (int q = 0; q < 4; ++q) dst[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
        } else {
            // 16-bit output: two 16-byte stores
            uint4 *dst = reinterpret_cast<uint4 *>(crow + (int64_t)jb * 2);
            uint32_t w[8];
            if (e.beta != 0.f) {
                const uint4 o0 = dst[0], o1 = dst[1];
                const uint32_t ow[8] = {o0.x, o0.y, o0.z, o0.w, o1.x, o1.y, o1.z, o1.w};
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    float lo, hi;
                    if (e.c_dtype == DG_BF16) {
                        lo = __uint_as_float(ow[q] << 16);
                        hi = __uint_as_float(ow[q] & 0xffff0000u);
                    } else {
                        const float2 t = __half22float2(*reinterpret_cast<const __half2 *>(&ow[q]));
                        lo = t.x;
                        hi = t.y;
                    }
                    v[2 * q] = fmaf(e.beta, lo, v[2 * q]);
                    v[2 * q + 1] = fmaf(e.beta, hi, v[2 * q + 1]);
                }
            }
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                if (e.c_dtype == DG_BF16) {
                    __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * q], v[2 * q + 1]);
                    w[q] = *reinterpret_cast<uint32_t *>(&h);
                } else {
                    __half2 h = __floats2half2_rn(v[2 * q], v[2 * q + 1]);
                    w[q] = *reinterpret_cast<uint32_t *>(&h);
                }
            }
            dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
            dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
        }
    } else {
        float cin[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) {
            const int j = jb + c;
            cin[c] = (e.beta != 0.f && j < Nj) ? load_elem(crow + (int64_t)j * e.cj, e.c_dtype) : 0.f;
        }
#pragma unroll
        for (int c = 0; c < 16; ++c) {
            const int j = jb + c;
            if (j < Nj) {
                const float sj = e.scale_j ? e.scale_j[j] : 1.f;
                float val = (asi * sj) * __uint_as_float(r[c]);
                if (e.beta != 0.f) val = fmaf(e.beta, cin[c], val);
                store_elem(crow + (int64_t)j * e.cj, e.c_dtype, val);
            }
        }
    }
}

}  // namespace dg
