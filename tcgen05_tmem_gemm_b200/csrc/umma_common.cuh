// Epilogue pieces shared by the tensor-core kernels.
#pragma once

#include "common.cuh"
#include "sm100.cuh"

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

constexpr int kStagePitch = 33;                          // floats per row of a staged 32 x 32 block
constexpr int kEpiStageBytes = 32 * kStagePitch * 4;     // per epilogue warp

// One epilogue warp's 32 accumulator rows (TMEM lanes) x bn columns, for C
// contiguous along j (16-byte aligned rows).  A row lives in one thread after
// tcgen05.ld, which would make every store instruction touch 32 rows; each
// 32 x 32 block is therefore passed through `stage` (this warp's shared
// memory) so that a store instruction writes 4 rows x 32 contiguous columns.
// All 32 lanes call it together (tcgen05.ld is warp-collective).
__device__ __forceinline__ void epilogue_rows_staged(const EpiParams &e, float *stage, uint32_t t_warp,
                                                     int i_base, int Mi, int j0, int bn, int Nj) {
    const int lane = threadIdx.x & 31;
    const int sub = lane & 7, rq = lane >> 3;   // 4 columns of one of 4 rows per step
    const int es = elem_bytes(e.c_dtype);
    for (int c0 = 0; c0 < bn; c0 += 32) {
        uint32_t r[32];
        __syncwarp();
        tmem_ld32(t_warp + c0, r);
        tmem_ld_wait();
#pragma unroll
        for (int c = 0; c < 32; ++c) stage[lane * kStagePitch + c] = __uint_as_float(r[c]);
        __syncwarp();
        const int jb = j0 + c0 + sub * 4;
        float sj[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) sj[q] = (e.scale_j && jb + q < Nj) ? e.scale_j[jb + q] : 1.f;
        // every C load of the block first (beta != 0), then the arithmetic and the stores
        float cin[8][4];
#pragma unroll
        for (int rr = 0; rr < 8; ++rr) {
            const int i = i_base + rr * 4 + rq;
#pragma unroll
            for (int q = 0; q < 4; ++q) cin[rr][q] = 0.f;
            if (e.beta != 0.f && i < Mi) {
                const char *crow = e.c + (int64_t)i * e.ci;
                if (jb + 4 <= Nj) {
                    if (es == 4) {
                        const float4 o = *reinterpret_cast<const float4 *>(crow + (int64_t)jb * 4);
                        cin[rr][0] = o.x; cin[rr][1] = o.y; cin[rr][2] = o.z; cin[rr][3] = o.w;
                    } else {
#pragma unroll
                        for (int q = 0; q < 4; ++q) cin[rr][q] = load_elem(crow + (int64_t)(jb + q) * es, e.c_dtype);
                    }
                } else {
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        if (jb + q < Nj) cin[rr][q] = load_elem(crow + (int64_t)(jb + q) * es, e.c_dtype);
                }
            }
        }
#pragma unroll
        for (int rr = 0; rr < 8; ++rr) {
            const int row = rr * 4 + rq;
            const int i = i_base + row;
            if (i >= Mi || jb >= Nj) continue;
            const float asi = e.alpha * (e.scale_i ? e.scale_i[i] : 1.f);
            float v[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                v[q] = (asi * sj[q]) * stage[row * kStagePitch + sub * 4 + q];
                if (e.beta != 0.f) v[q] = fmaf(e.beta, cin[rr][q], v[q]);
            }
            char *dst = e.c + (int64_t)i * e.ci + (int64_t)jb * es;
            if (jb + 4 <= Nj) {
                if (e.c_dtype == DG_F32) {
                    *reinterpret_cast<float4 *>(dst) = make_float4(v[0], v[1], v[2], v[3]);
                } else if (e.c_dtype == DG_BF16) {
                    __nv_bfloat162 a = __floats2bfloat162_rn(v[0], v[1]), b = __floats2bfloat162_rn(v[2], v[3]);
                    *reinterpret_cast<uint2 *>(dst) =
                        make_uint2(*reinterpret_cast<uint32_t *>(&a), *reinterpret_cast<uint32_t *>(&b));
                } else {
                    __half2 a = __floats2half2_rn(v[0], v[1]), b = __floats2half2_rn(v[2], v[3]);
                    *reinterpret_cast<uint2 *>(dst) =
                        make_uint2(*reinterpret_cast<uint32_t *>(&a), *reinterpret_cast<uint32_t *>(&b));
                }
            } else {
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    if (jb + q < Nj) store_elem(dst + q * es, e.c_dtype, v[q]);
            }
        }
    }
    __syncwarp();
}

}  // namespace dg
