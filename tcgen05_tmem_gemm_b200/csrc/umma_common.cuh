// Epilogue pieces shared by the tensor-core kernels.
#pragma once

#include "common.cuh"
#include "sm100.cuh"

namespace dg {

// Apply  out = act(alpha * s_i * s_j * acc + beta * C + bias)  to the 16
// consecutive columns jb .. jb+15 of output row i (row pointer `crow`,
// per-row factor asi = alpha * s_i) and store them: 16-byte vector stores
// when C is contiguous along j and the chunk is whole, otherwise element
// stores for any strides, with every C load of the chunk issued before the
// first store.  The bias add and activation run only when the call has them.
// The bias and activation of 16 whole columns jb.. of row i (after beta * C).
__device__ __forceinline__ void fuse16(const EpiParams &e, float (&v)[16], int i, int jb) {
#pragma unroll
    for (int c = 0; c < 16; ++c) {
        float z = v[c];
        if (e.bias_i) z += e.bias_i[i];
        if (e.bias_j) z += e.bias_j[jb + c];
        v[c] = act_apply(e.act, z, e.c_dtype != DG_F32);
    }
}

__device__ __forceinline__ void epilogue_chunk16(const EpiParams &e, char *crow, float asi, int i, int jb, int Nj,
                                                 const uint32_t (&r)[16]) {
    const bool fused = e.bias_i != nullptr || e.bias_j != nullptr || e.act != DG_ACT_NONE;
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
            if (fused) fuse16(e, v, i, jb);  // C was loaded first: the whole sum
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
            if (fused) fuse16(e, v, i, jb);  // C was loaded first: the whole sum
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
        // Every load of the chunk (C, column scales, bias) is issued before
        // the first store: the stores go through a plain pointer the compiler
        // cannot tell apart from the scale and bias arrays, so a load placed
        // after a store would wait for it, one element at a time.
        float cin[16], sjv[16], bjv[16];
        const float bi = e.bias_i ? e.bias_i[i] : 0.f;
#pragma unroll
        for (int c = 0; c < 16; ++c) {
            const int j = jb + c;
            const bool ok = j < Nj;
            cin[c] = (e.beta != 0.f && ok) ? load_elem(crow + (int64_t)j * e.cj, e.c_dtype) : 0.f;
            sjv[c] = (e.scale_j && ok) ? e.scale_j[j] : 1.f;
            bjv[c] = (e.bias_j && ok) ? e.bias_j[j] : 0.f;
        }
#pragma unroll
        for (int c = 0; c < 16; ++c) {
            const int j = jb + c;
            if (j < Nj) {
                float val = (asi * sjv[c]) * __uint_as_float(r[c]);
                if (e.beta != 0.f) val = fmaf(e.beta, cin[c], val);
                if (fused) {
                    if (e.bias_i) val += bi;
                    if (e.bias_j) val += bjv[c];
                    val = act_apply(e.act, val, e.c_dtype != DG_F32);
                }
                store_elem(crow + (int64_t)j * e.cj, e.c_dtype, val);
            }
        }
    }
}

// Shared memory of the TMA-store epilogue: two blocks of 32 rows x 128 bytes
// for each of the four epilogue warps.
constexpr uint32_t kEpiBlockBytes = 32 * 128;
constexpr uint32_t kEpiStoreBytes = 4 * 2 * kEpiBlockBytes;

// Epilogue of one warp's 32 accumulator rows (TMEM lanes) x bn columns through
// tensor stores, for beta == 0 and C unit-stride along j (with the fused bias
// and activation when the call has them).  After tcgen05.ld a
// thread holds one row, so direct stores would touch 32 rows per instruction.
// Instead the warp writes 32 rows x 128 bytes of output at a time into a
// shared-memory block in the 128-byte-swizzle layout (row r's 16-byte unit u
// sits at unit u ^ (r & 7), so the eight lanes of each store phase hit
// different banks) and one lane stores the block with a tensor copy, which
// writes whole lines and skips everything outside C.  Two blocks alternate,
// so packing one overlaps the copy of the other.  `stage` is this warp's
// 2 x kEpiBlockBytes (1024-byte aligned), `nblk` counts the blocks the warp
// has issued; the caller waits for its copies (bulk_wait_all) before exit.
// The warp stores 128-byte column blocks blk_first, blk_first + blk_step, ...
template <int ES>
__device__ __forceinline__ void epilogue_rows_tma(const EpiParams &e, const CUtensorMap *cmap, uint32_t stage,
                                                  uint32_t t_row, int i_base, int Mi, int j0, int bn, int Nj,
                                                  int lane, uint32_t &nblk, int blk_first = 0, int blk_step = 1) {
    constexpr int W = 128 / ES;  // output columns per block
    if (i_base >= Mi) return;    // the whole warp is below C (warp-uniform)
    // parameters in registers: nothing below re-reads the parameter block
    const float *const scale_j = e.scale_j;
    const float *const bias_j = e.bias_j;
    const int act = e.act;
    const bool fused = e.bias_i != nullptr || bias_j != nullptr || act != DG_ACT_NONE;
    const bool bf16_out = e.c_dtype == DG_BF16;
    const int i = i_base + lane;
    const float asi = i < Mi ? e.alpha * (e.scale_i ? e.scale_i[i] : 1.f) : 0.f;
    const bool has_bi = e.bias_i != nullptr;
    const float bi = (i < Mi && has_bi) ? e.bias_i[i] : 0.f;
    // blocks blk_first, blk_first + blk_step, ... of the row strip (warps that
    // share TMEM lanes split a strip this way)
    for (int c0 = blk_first * W; c0 < bn && j0 + c0 < Nj; c0 += blk_step * W) {
        uint32_t r[W];
#pragma unroll
        for (int q = 0; q < W / 16; ++q)
            tmem_ld16(t_row + (uint32_t)(c0 + 16 * q), *reinterpret_cast<uint32_t(*)[16]>(&r[16 * q]));
        tmem_ld_wait();
        float v[W];
        if (scale_j != nullptr) {  // per-column scales (FP8): read once per block, clamped at the edge
            const int jb = j0 + c0;
#pragma unroll
            for (int c = 0; c < W; ++c) {
                const float sj = scale_j[jb + c < Nj ? jb + c : Nj - 1];
                v[c] = (asi * sj) * __uint_as_float(r[c]);
            }
        } else {
#pragma unroll
            for (int c = 0; c < W; ++c) v[c] = asi * __uint_as_float(r[c]);
        }
        if (fused) {  // bias (per row or per column, clamped at the edge) and activation
            const int jb = j0 + c0;
#pragma unroll
            for (int c = 0; c < W; ++c) {
                float z = v[c];
                if (has_bi) z += bi;
                if (bias_j) z += bias_j[jb + c < Nj ? jb + c : Nj - 1];
                v[c] = act_apply(act, z, ES == 2);  // 16-bit output: the hardware tanh
            }
        }
        uint32_t w[32];
        if (ES == 4) {
#pragma unroll
            for (int c = 0; c < 32; ++c) w[c] = __float_as_uint(v[c]);
        } else {
#pragma unroll
            for (int c = 0; c < 32; ++c) {
                if (bf16_out) {
                    __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * c], v[2 * c + 1]);
                    w[c] = *reinterpret_cast<uint32_t *>(&h);
                } else {
                    __half2 h = __floats2half2_rn(v[2 * c], v[2 * c + 1]);
                    w[c] = *reinterpret_cast<uint32_t *>(&h);
                }
            }
        }
        const uint32_t buf = stage + (nblk & 1u) * kEpiBlockBytes;
        if (lane == 0) bulk_wait_read<1>();  // the copy that last read this block is done with it
        __syncwarp();
        const uint32_t rowa = buf + (uint32_t)lane * 128u;
#pragma unroll
        for (int u = 0; u < 8; ++u)
            st_shared_v4(rowa + ((uint32_t)(u ^ (lane & 7)) << 4), w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
            tma_store_2d(cmap, buf, j0 + c0, i_base);
            bulk_commit();
        }
        ++nblk;
    }
}

}  // namespace dg
