// Epilogue pieces shared by the tensor-core kernels.
#pragma once

#include "common.cuh"
#include "sm100.cuh"

namespace dg {

// Sixteen per-column factors arr[jb .. jb+15] (scales or bias; jb a multiple
// of 16): four 16-byte loads when the array is 16-byte aligned and the chunk
// whole, else element loads clamped to the last column (their values past Nj
// are never stored).  A null array gives `dflt`.
__device__ __forceinline__ void load_cols16(float (&b)[16], const float *arr, int jb, int Nj, float dflt) {
    if (arr == nullptr) {
#pragma unroll
        for (int c = 0; c < 16; ++c) b[c] = dflt;
    } else if ((reinterpret_cast<uintptr_t>(arr) & 15u) == 0 && jb + 16 <= Nj) {
        const float4 *q = reinterpret_cast<const float4 *>(arr + jb);
#pragma unroll
        for (int g = 0; g < 4; ++g) {
            const float4 t = q[g];
            b[4 * g] = t.x;
            b[4 * g + 1] = t.y;
            b[4 * g + 2] = t.z;
            b[4 * g + 3] = t.w;
        }
    } else {
#pragma unroll
        for (int c = 0; c < 16; ++c) b[c] = arr[jb + c < Nj ? jb + c : Nj - 1];
    }
}

// v[c] = act(v[c] + bi + bias[jb + c]) for W columns, 16 at a time (bias_i
// and bias_j are never both set, so bi + bias is one of them exactly).
template <int ACT, bool FAST, int W>
__device__ __forceinline__ void fuse_cols(float (&v)[W], float bi, const float *bias, int jb, int Nj) {
#pragma unroll
    for (int q = 0; q < W / 16; ++q) {
        float b[16];
        load_cols16(b, bias, jb + 16 * q, Nj, 0.f);
#pragma unroll
        for (int c = 0; c < 16; ++c) v[16 * q + c] = act_fn<ACT, FAST>(v[16 * q + c] + (bi + b[c]));
    }
}

// Output element access for a C dtype fixed at compile time.
template <int CD>
__device__ __forceinline__ float ld_out(const char *p) {
    if (CD == DG_F32) return *reinterpret_cast<const float *>(p);
    if (CD == DG_BF16) return __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(p));
    return __half2float(*reinterpret_cast<const __half *>(p));
}
template <int CD>
__device__ __forceinline__ void st_out(char *p, float v) {
    if (CD == DG_F32) *reinterpret_cast<float *>(p) = v;
    else if (CD == DG_BF16) *reinterpret_cast<__nv_bfloat16 *>(p) = __float2bfloat16_rn(v);
    else *reinterpret_cast<__half *>(p) = __float2half_rn(v);
}
template <bool B16>
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
    if (B16) {
        __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
        return *reinterpret_cast<uint32_t *>(&h);
    }
    __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
}

// The 16 consecutive columns jb .. jb+15 of output row i through element
// stores at any column stride (C's row pointer `crow`), in two halves of 8.
// Every load of a half (C, column scales, bias) is issued before its first
// store: the stores go through a plain pointer the compiler cannot tell apart
// from the scale and bias arrays, so a load placed after a store would wait
// for it.  (Halves keep the loads of a chunk in registers without spilling.)
template <int CD, bool FUSED, int ACT>
__device__ __forceinline__ void chunk16_elem(const EpiParams &e, char *crow, float asi, float bi, int jb, int Nj,
                                             const uint32_t (&r)[16]) {
    const int64_t cj = e.cj;
#pragma unroll
    for (int h = 0; h < 16; h += 8) {
        char *p = crow + (int64_t)(jb + h) * cj;
        float cin[8], sjv[8], bjv[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const int j = jb + h + c;
            const int jc = j < Nj ? j : Nj - 1;  // loads past Nj are clamped; their values are never stored
            cin[c] = (e.beta != 0.f && j < Nj) ? ld_out<CD>(p + c * cj) : 0.f;
            sjv[c] = e.scale_j ? e.scale_j[jc] : 1.f;
            bjv[c] = FUSED && e.bias_j ? e.bias_j[jc] : 0.f;
        }
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            float val = (asi * sjv[c]) * __uint_as_float(r[h + c]);
            if (e.beta != 0.f) val = fmaf(e.beta, cin[c], val);
            if (FUSED) val = act_fn<ACT, CD != DG_F32>(val + (bi + bjv[c]));
            if (jb + h + c < Nj) st_out<CD>(p + c * cj, val);
        }
    }
}

// The same 16 columns when C is contiguous along j and the chunk whole:
// 16-byte vector loads and stores.
template <int CD, bool FUSED, int ACT>
__device__ __forceinline__ void chunk16_vec(const EpiParams &e, char *crow, float asi, float bi, int jb, int Nj,
                                            const uint32_t (&r)[16]) {
    float sjv[16], v[16];
    load_cols16(sjv, e.scale_j, jb, Nj, 1.f);
#pragma unroll
    for (int c = 0; c < 16; ++c) v[c] = (asi * sjv[c]) * __uint_as_float(r[c]);
    if (CD == DG_F32) {
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
        if (FUSED) fuse_cols<ACT, false>(v, bi, e.bias_j, jb, Nj);  // C was loaded first: the whole sum
#pragma unroll
        for (int q = 0; q < 4; ++q) dst[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
    } else {
        uint4 *dst = reinterpret_cast<uint4 *>(crow + (int64_t)jb * 2);
        if (e.beta != 0.f) {
            const uint4 o0 = dst[0], o1 = dst[1];
            const uint32_t ow[8] = {o0.x, o0.y, o0.z, o0.w, o1.x, o1.y, o1.z, o1.w};
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                float lo, hi;
                if (CD == DG_BF16) {
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
        if (FUSED) fuse_cols<ACT, true>(v, bi, e.bias_j, jb, Nj);  // C was loaded first: the whole sum
        uint32_t w[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) w[q] = pack2<CD == DG_BF16>(v[2 * q], v[2 * q + 1]);
        dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
        dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
    }
}

template <bool FUSED, int ACT>
__device__ __forceinline__ void chunk16_any(const EpiParams &e, char *crow, float asi, float bi, int jb, int Nj,
                                            const uint32_t (&r)[16]) {
    const bool vec = e.vec_ok && jb + 16 <= Nj;
    switch (e.c_dtype) {
    case DG_F32:
        if (vec) chunk16_vec<DG_F32, FUSED, ACT>(e, crow, asi, bi, jb, Nj, r);
        else chunk16_elem<DG_F32, FUSED, ACT>(e, crow, asi, bi, jb, Nj, r);
        break;
    case DG_BF16:
        if (vec) chunk16_vec<DG_BF16, FUSED, ACT>(e, crow, asi, bi, jb, Nj, r);
        else chunk16_elem<DG_BF16, FUSED, ACT>(e, crow, asi, bi, jb, Nj, r);
        break;
    default:
        if (vec) chunk16_vec<DG_F16, FUSED, ACT>(e, crow, asi, bi, jb, Nj, r);
        else chunk16_elem<DG_F16, FUSED, ACT>(e, crow, asi, bi, jb, Nj, r);
        break;
    }
}

// Thread-store epilogue of one warp's 32 accumulator rows (TMEM lanes at
// t_row; this thread's row i): the 16-column chunks c_first, c_first +
// c_step, ... of the tile's bn columns from j0.  The activation and bias
// choice is made once for the whole strip.
template <bool FUSED, int ACT>
__device__ __forceinline__ void rows_thread_t(const EpiParams &e, uint32_t t_row, int i, int Mi, int j0, int bn,
                                              int Nj, int c_first, int c_step) {
    const bool row_ok = i < Mi;
    const float asi = row_ok ? e.alpha * (e.scale_i ? e.scale_i[i] : 1.f) : 0.f;
    const float bi = (row_ok && e.bias_i != nullptr) ? e.bias_i[i] : 0.f;
    char *crow = e.c + epi_row_offset(e, row_ok ? i : 0);
    for (int c0 = c_first; c0 < bn; c0 += c_step) {
        uint32_t r[16];
        __syncwarp();
        tmem_ld16(t_row + (uint32_t)c0, r);
        tmem_ld_wait();
        if (row_ok) chunk16_any<FUSED, ACT>(e, crow, asi, bi, j0 + c0, Nj, r);
    }
}

__device__ __forceinline__ void epilogue_rows_thread(const EpiParams &e, uint32_t t_row, int i, int Mi, int j0,
                                                     int bn, int Nj, int c_first = 0, int c_step = 16) {
    if (e.act == DG_ACT_GELU_TANH)
        rows_thread_t<true, DG_ACT_GELU_TANH>(e, t_row, i, Mi, j0, bn, Nj, c_first, c_step);
    else if (e.act == DG_ACT_RELU)
        rows_thread_t<true, DG_ACT_RELU>(e, t_row, i, Mi, j0, bn, Nj, c_first, c_step);
    else if (e.bias_i != nullptr || e.bias_j != nullptr)
        rows_thread_t<true, DG_ACT_NONE>(e, t_row, i, Mi, j0, bn, Nj, c_first, c_step);
    else
        rows_thread_t<false, DG_ACT_NONE>(e, t_row, i, Mi, j0, bn, Nj, c_first, c_step);
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
// has issued; before exit the caller waits until its copies have read shared
// memory (bulk_wait_read<0>); their writes land before the grid completes.
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
    const float bi = (i < Mi && e.bias_i != nullptr) ? e.bias_i[i] : 0.f;
    // blocks blk_first, blk_first + blk_step, ... of the row strip (warps that
    // share TMEM lanes split a strip this way)
    for (int c0 = blk_first * W; c0 < bn && j0 + c0 < Nj; c0 += blk_step * W) {
        uint32_t r[W];
#pragma unroll
        for (int q = 0; q < W / 16; ++q)
            tmem_ld16(t_row + (uint32_t)(c0 + 16 * q), *reinterpret_cast<uint32_t(*)[16]>(&r[16 * q]));
        tmem_ld_wait();
        float v[W];
        {
            const int jb = j0 + c0;
            if (scale_j != nullptr) {
#pragma unroll
                for (int q = 0; q < W / 16; ++q) {  // per-column scales (FP8), 16 at a time
                    float sj[16];
                    load_cols16(sj, scale_j, jb + 16 * q, Nj, 1.f);
#pragma unroll
                    for (int c = 0; c < 16; ++c) v[16 * q + c] = (asi * sj[c]) * __uint_as_float(r[16 * q + c]);
                }
            } else {
#pragma unroll
                for (int c = 0; c < W; ++c) v[c] = asi * __uint_as_float(r[c]);
            }
            if (fused) {  // bias and activation, the activation picked once per block
                if (act == DG_ACT_GELU_TANH) fuse_cols<DG_ACT_GELU_TANH, ES == 2>(v, bi, bias_j, jb, Nj);
                else if (act == DG_ACT_RELU) fuse_cols<DG_ACT_RELU, ES == 2>(v, bi, bias_j, jb, Nj);
                else fuse_cols<DG_ACT_NONE, ES == 2>(v, bi, bias_j, jb, Nj);
            }
        }
        uint32_t w[32];
        if (ES == 4) {
#pragma unroll
            for (int c = 0; c < 32; ++c) w[c] = __float_as_uint(v[c]);
        } else if (bf16_out) {
#pragma unroll
            for (int c = 0; c < 32; ++c) w[c] = pack2<true>(v[2 * c], v[2 * c + 1]);
        } else {
#pragma unroll
            for (int c = 0; c < 32; ++c) w[c] = pack2<false>(v[2 * c], v[2 * c + 1]);
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
