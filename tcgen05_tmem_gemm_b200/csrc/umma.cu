// Tensor-core GEMM for sm_100a: tcgen05.mma with TMEM accumulators.
//
// Computes D[i][j] = sum_k P[i][k] Q[k][j] tile by tile and applies the
// epilogue  out = alpha * s_i * s_j * D + beta * C_in  on the way out.  P is A
// (i = m) and Q is B (j = n), or, when the dispatcher swaps the operands to
// put a long N on the tensor core's 128-row side, P = B^T and Q = A^T.
//
// Structure ("DeepGEMM deep dive" §2.1-§2.3 describe the blocking, register
// accumulation and the load/compute overlap this re-designs for Blackwell;
// §3.4 the shared-memory swizzle):
//  - one CTA per SM, persistent over tiles (i-tile, j-tile, k-split);
//  - warp 0, one lane: TMA loads of the P and Q tiles into a ring of
//    `stages` shared-memory buffers in the 128-byte swizzled layout the
//    tensor core reads, each stage guarded by a full/empty mbarrier pair;
//  - warp 1: allocates TMEM (two accumulators of bn FP32 columns each), and one
//    lane issues tcgen05.mma (128 x bn x 16 for 16-bit inputs, x32 for E4M3)
//    and tcgen05.commit, which frees a stage once its MMAs have read it and
//    signals a finished accumulator;
//  - warps 2-5: the epilogue, each owning 32 TMEM lanes (rows): tcgen05.ld,
//    scale, optional beta * C, convert and store, while the MMA warp already
//    fills the other accumulator;
//  - warps 6-9 (gather variant): thread loads of a P operand that TMA cannot
//    describe (e.g. an NCHW feature map read as [N*H*W, C] with a 392-byte
//    channel stride), written into the same swizzled layout
//    ("DeepGEMM: a recalibration of the compute paradigm", §2.2: scatter-gather
//    loads for the non-contiguous segments of a view).
//  - split-K: partial tiles go to a workspace; per 32-row quarter the last
//    arriving split adds the partials in split order (deterministic) and runs
//    the epilogue ("DeepGEMM deep dive", §5.2).
// Every wait is bounded (WaitCtl); on expiry the CTA records DG_ERR_TIMEOUT,
// drains what it has in flight, frees TMEM and exits.
#include <atomic>

#include "common.cuh"
#include "sm100.cuh"
#include "umma_common.cuh"

namespace dg {

namespace {

constexpr int kBM = 128;             // tensor-core tile rows (TMEM lanes)
constexpr int kTileBytesK = 128;     // one swizzle row: 64 x 16-bit or 128 x 8-bit
constexpr int kGatherWarps = 4;

struct SmemLayout {
    uint32_t stage_bytes, p_bytes, q_bytes;
    uint32_t bar_off;                // after the stages
    uint32_t aux_off;                // tmem address, abort flag, gather tables
    uint32_t total;
};

__host__ __device__ inline SmemLayout smem_layout(int bn, int stages, bool gather) {
    SmemLayout L;
    L.p_bytes = kBM * kTileBytesK;
    L.q_bytes = (uint32_t)bn * kTileBytesK;
    L.stage_bytes = L.p_bytes + L.q_bytes;
    L.bar_off = L.stage_bytes * stages;
    // full[S], empty[S], tfull[2], tempty[2], drain
    L.aux_off = L.bar_off + 8 * (2 * stages + 5);
    uint32_t aux = 16;  // tmem base + abort flag
    if (gather) aux += 8 * kBM;  // row offsets of the tile
    L.total = L.aux_off + aux + 1024;  // + slack to align the base to 1024
    return L;
}

struct TileCoord {
    int ti, tj, split;
};

__device__ __forceinline__ TileCoord unit_coord(int u, const UmmaParams &p) {
    TileCoord c;
    c.split = u % p.split_k;
    const int t = u / p.split_k;
    c.ti = t % p.tiles_i;
    c.tj = t / p.tiles_i;
    return c;
}

// Byte offset inside a 128-byte-swizzled tile of an element at (mn, k) for
// the two layouts the tensor core reads.  `bytek` = k * element size.
__device__ __forceinline__ uint32_t sw128_kmajor(int mn, int bytek) {
    return (uint32_t)((mn >> 3) * 1024 + (mn & 7) * 128 + ((((bytek >> 4) ^ (mn & 7)) << 4) | (bytek & 15)));
}
__device__ __forceinline__ uint32_t sw128_mnmajor(int bytemn, int k, int chunk_bytes) {
    const int c = bytemn >> 7, w = bytemn & 127;
    return (uint32_t)(c * chunk_bytes + (k >> 3) * 1024 + (k & 7) * 128 + ((((w >> 4) ^ (k & 7)) << 4) | (w & 15)));
}

template <int BYTES> struct VecOf;
template <> struct VecOf<16> { using T = uint4; };
template <> struct VecOf<8> { using T = uint2; };
template <> struct VecOf<4> { using T = uint32_t; };
template <> struct VecOf<2> { using T = unsigned short; };
template <> struct VecOf<1> { using T = unsigned char; };

template <int BYTES>
__device__ __forceinline__ typename VecOf<BYTES>::T gather_load_one(const char *src, bool valid) {
    using V = typename VecOf<BYTES>::T;
    if (!valid) return V{};
    return __ldg(reinterpret_cast<const V *>(src));
}

template <int BYTES>
__device__ __forceinline__ void st_shared_vec(uint32_t dst, const typename VecOf<BYTES>::T &v) {
    if constexpr (BYTES == 16) {
        asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w));
    } else if constexpr (BYTES == 8) {
        asm volatile("st.shared.v2.u32 [%0], {%1, %2};" ::"r"(dst), "r"(v.x), "r"(v.y));
    } else if constexpr (BYTES == 4) {
        asm volatile("st.shared.u32 [%0], %1;" ::"r"(dst), "r"(v));
    } else if constexpr (BYTES == 2) {
        asm volatile("st.shared.u16 [%0], %1;" ::"r"(dst), "h"(v));
    } else {
        asm volatile("st.shared.u8 [%0], %1;" ::"r"(dst), "r"((uint32_t)v));
    }
}

// Phase timestamps of CTA 0 for performance analysis (DG_OPT_TRACE): slot 0
// entry, 1 set-up done, 2+kb first-unit loads issued (k block kb < 16),
// 18+kb MMAs of k block kb issued, 34 first accumulator complete (seen by the
// epilogue), 35 first epilogue done, 36 teardown, 37..52 gather k block kb
// written (first unit); split-K: 53 accumulator complete, 54 first cluster
// barrier passed, 55 partials pushed and second barrier passed, 56 reduced.
__device__ __forceinline__ void trace_at(const UmmaParams &p, int slot) {
    if (p.trace != nullptr && blockIdx.x == 0) p.trace[slot] = globaltimer_ns();
}

// OR of `pred` over the gather warps (named barrier 1), returned to all of them.
__device__ __forceinline__ bool named_bar_or(bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, 1, %2, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)pred), "n"(kGatherWarps * 32)
        : "memory");
    return r != 0;
}

// Thread loads of one stage of the P tile (kBM rows of i, bk of k), split in
// two halves so that a stage's loads can be in flight while the previous
// stage is stored: gather_load fills registers (at most kGatherUnroll copies
// per thread), gather_store writes them in the 128-byte-swizzled layout.
// Copy u of a stage covers `vec` consecutive elements along the unit-stride
// dimension; consecutive threads take consecutive copies.
constexpr int kGatherUnroll = 16;

struct GatherGeom {
    bool mn;
    int vec, runs, total, chunk_bytes, es;
};

__device__ __forceinline__ GatherGeom gather_geom(const UmmaParams &p, int VB, int bk, int es) {
    GatherGeom g;
    g.mn = p.p_mn_major != 0;
    g.vec = VB / es;
    g.runs = g.mn ? kBM / g.vec : bk / g.vec;
    g.total = g.mn ? g.runs * bk : kBM * g.runs;
    g.chunk_bytes = bk * 128;
    g.es = es;
    return g;
}

// Copies first, first + 128, first + 256, ... of a stage: along the unit-
// stride dim their position is fixed and the other index advances by
// 128 / runs per copy (runs is a power of two dividing 128), so no index is
// divided inside the loops.
template <int VB>
__device__ __forceinline__ void gather_load(const UmmaParams &p, const GatherGeom &g, const int64_t *row_off,
                                            int kbase, int first, typename VecOf<VB>::T (&v)[kGatherUnroll]) {
    const int nthreads = kGatherWarps * 32;
    const int step = nthreads / g.runs;
    if (g.mn) {
        // fixed i (a run of vec rows), k advancing by `step`
        const int i = (first % g.runs) * g.vec;
        const int64_t ro = row_off[i];
        const int k0 = first / g.runs;
#pragma unroll
        for (int r = 0; r < kGatherUnroll; ++r) {
            const int u = first + r * nthreads;
            const int kg = kbase + k0 + r * step;
            const bool ok = u < g.total && ro >= 0 && kg < p.K;
            v[r] = gather_load_one<VB>(p.pv.ptr + (ok ? ro + axis_offset(p.pv.col, kg) : 0), ok);
        }
    } else {
        // fixed k (a run of vec columns), i advancing by `step`
        const int kg = kbase + (first % g.runs) * g.vec;
        const int64_t co = kg < p.K ? axis_offset(p.pv.col, kg) : -1;
        const int i0 = first / g.runs;
#pragma unroll
        for (int r = 0; r < kGatherUnroll; ++r) {
            const int u = first + r * nthreads;
            const int i = i0 + r * step;
            const int64_t ro = (u < g.total) ? row_off[i] : -1;
            const bool ok = ro >= 0 && co >= 0;
            v[r] = gather_load_one<VB>(p.pv.ptr + (ok ? ro + co : 0), ok);
        }
    }
}

template <int VB>
__device__ __forceinline__ void gather_store(const GatherGeom &g, uint32_t p_smem, int first,
                                             const typename VecOf<VB>::T (&v)[kGatherUnroll]) {
    const int nthreads = kGatherWarps * 32;
    const int step = nthreads / g.runs;
    const int fixed = (first % g.runs) * g.vec, moving0 = first / g.runs;
#pragma unroll
    for (int r = 0; r < kGatherUnroll; ++r) {
        const int u = first + r * nthreads;
        if (u >= g.total) continue;
        const int moving = moving0 + r * step;
        st_shared_vec<VB>(p_smem + (g.mn ? sw128_mnmajor(fixed * g.es, moving, g.chunk_bytes)
                                         : sw128_kmajor(moving, fixed * g.es)),
                          v[r]);
    }
}

// cp.async version of a batch: the same copies as gather_load/gather_store,
// issued as asynchronous global -> shared copies (no register staging).
template <int VB>
__device__ __forceinline__ void gather_issue_async(const UmmaParams &p, const GatherGeom &g, const int64_t *row_off,
                                                   int kbase, int first, uint32_t p_smem) {
    const int nthreads = kGatherWarps * 32;
    const int step = nthreads / g.runs;
    const int fixed = (first % g.runs) * g.vec, moving0 = first / g.runs;
    if (g.mn) {
        const int64_t ro = row_off[fixed];
#pragma unroll
        for (int r = 0; r < kGatherUnroll; ++r) {
            const int u = first + r * nthreads;
            if (u >= g.total) break;
            const int k = moving0 + r * step, kg = kbase + k;
            const bool ok = ro >= 0 && kg < p.K;
            cp_async_zfill<VB>(p_smem + sw128_mnmajor(fixed * g.es, k, g.chunk_bytes),
                               p.pv.ptr + (ok ? ro + axis_offset(p.pv.col, kg) : 0), ok);
        }
    } else {
        const int kg = kbase + fixed;
        const int64_t co = kg < p.K ? axis_offset(p.pv.col, kg) : -1;
#pragma unroll
        for (int r = 0; r < kGatherUnroll; ++r) {
            const int u = first + r * nthreads;
            if (u >= g.total) break;
            const int i = moving0 + r * step;
            const int64_t ro = row_off[i];
            const bool ok = ro >= 0 && co >= 0;
            cp_async_zfill<VB>(p_smem + sw128_kmajor(i, fixed * g.es), p.pv.ptr + (ok ? ro + co : 0), ok);
        }
    }
}

// The gather role for one vector width.  Per tile: row offsets once.  When
// a stage is at most one batch per thread (kGatherUnroll copies), the next
// k block's loads are issued before this block is stored, so two stages of
// loads are in flight; wider stages are loaded and stored batch by batch.
// Every exit decision is voted on across the gather warps (bar.red), so no
// warp is left waiting at their named barrier.
template <int VB>
__device__ __forceinline__ void gather_role(const UmmaParams &p, const SmemLayout &L, uint32_t sbase,
                                            uint32_t bar_full, uint32_t bar_empty, int64_t *g_row_off,
                                            volatile int *abort_flag, const WaitCtl &wc, int bk, int es, int gtid,
                                            int lane) {
    using V = typename VecOf<VB>::T;
    const GatherGeom g = gather_geom(p, VB, bk, es);
    const int nthreads = kGatherWarps * 32;
    const bool one_batch = VB < 4 && g.total <= nthreads * kGatherUnroll;  // register path look-ahead
    int it = 0;
    for (int u = blockIdx.x; u < p.num_units; u += gridDim.x) {
        if (named_bar_or(*abort_flag != 0)) break;
        const TileCoord tc = unit_coord(u, p);
        const int kb0 = tc.split * p.kb_per_split;
        const int kb1 = min(p.kb_total, kb0 + p.kb_per_split);
        for (int r = gtid; r < kBM; r += nthreads) {
            const int i = tc.ti * kBM + r;
            g_row_off[r] = i < p.Mi ? axis_offset(p.pv.row, i) : -1;
        }
        asm volatile("bar.sync 1, %0;" ::"n"(kGatherWarps * 32) : "memory");
        bool ok = true;
        V cur[kGatherUnroll], nxt[kGatherUnroll];
        if (one_batch && kb0 < kb1) gather_load<VB>(p, g, g_row_off, kb0 * bk, gtid, cur);
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
            const int s = it % p.stages;
            const uint32_t ph = (uint32_t)(it / p.stages) & 1u;
            if (one_batch && kb + 1 < kb1) gather_load<VB>(p, g, g_row_off, (kb + 1) * bk, gtid, nxt);
            ok = mbar_wait(bar_empty + 8 * s, ph ^ 1u, wc);
            if (named_bar_or(!ok)) { ok = false; break; }
            if (!p.stall_loader && VB >= 4) {
                // asynchronous copies: the stage completes on the full barrier
                // when they land, and this warp moves on at once
                const uint32_t ps = sbase + s * L.stage_bytes;
                for (int f = gtid; f < g.total; f += nthreads * kGatherUnroll)
                    gather_issue_async<(VB >= 4 ? VB : 4)>(p, g, g_row_off, kb * bk, f, ps);
                cp_async_arrive_noinc(bar_full + 8 * s);
                if (it < 16 && gtid == 0) trace_at(p, 37 + it);
            } else if (!p.stall_loader) {
                const uint32_t ps = sbase + s * L.stage_bytes;
                if (one_batch) {
                    gather_store<VB>(g, ps, gtid, cur);
                } else {
                    for (int f = gtid; f < g.total; f += nthreads * kGatherUnroll) {
                        gather_load<VB>(p, g, g_row_off, kb * bk, f, cur);
                        gather_store<VB>(g, ps, f, cur);
                    }
                }
                fence_proxy_async_smem();  // make the stores visible to the tensor core
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_full + 8 * s);
                if (it < 16 && gtid == 0) trace_at(p, 37 + it);
            }
            if (one_batch) {
#pragma unroll
                for (int r = 0; r < kGatherUnroll; ++r) cur[r] = nxt[r];
            }
        }
        // row offsets of this tile stay in use until every gather warp is past it
        asm volatile("bar.sync 1, %0;" ::"n"(kGatherWarps * 32) : "memory");
        if (!ok) break;
    }
    // nothing this thread copied may land after the CTA has gone
    asm volatile("cp.async.wait_all;" ::: "memory");
}

template <bool FP8, bool GATHER>
__global__ void __launch_bounds__(GATHER ? 320 : 192, 1)
    umma_gemm_kernel(const __grid_constant__ CUtensorMap tmap_p, const __grid_constant__ CUtensorMap tmap_q,
                     const UmmaParams p) {
    if (threadIdx.x == 0) trace_at(p, 0);
    pdl_wait();
    if (p.pdl == 1) pdl_release();
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1024-byte alignment for the 128-byte swizzle atoms
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const SmemLayout L = smem_layout(p.bn, p.stages, GATHER);
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar_full = sbase + L.bar_off;
    const uint32_t bar_empty = bar_full + 8 * p.stages;
    const uint32_t bar_tfull = bar_empty + 8 * p.stages;
    const uint32_t bar_tempty = bar_tfull + 16;
    const uint32_t bar_drain = bar_tempty + 16;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L.aux_off);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L.aux_off + 4);
    int64_t *g_row_off = reinterpret_cast<int64_t *>(smem + L.aux_off + 16);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr int kEpiWarp0 = 2;
    const WaitCtl wc{abort_flag, p.err_word, p.timeout_ns};

    if (threadIdx.x == 0) {
        for (int s = 0; s < p.stages; ++s) {
            // gather stages: one arrival per gather thread when its cp.async
            // copies land (4..16-byte copies), else one per gather warp
            mbar_init(bar_full + 8 * s, GATHER ? 1 + (p.gather_vec * (FP8 ? 1 : 2) >= 4 ? kGatherWarps * 32 : kGatherWarps) : 1);
            mbar_init(bar_empty + 8 * s, 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar_tfull + 8 * b, 1);
            mbar_init(bar_tempty + 8 * b, 4);
        }
        mbar_init(bar_drain, 1);
        *abort_flag = 0;
        fence_barrier_init();
        fence_proxy_async_smem();
        tma_prefetch_desc(&tmap_q);
        if (!GATHER) tma_prefetch_desc(&tmap_p);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), (uint32_t)p.tmem_cols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    if (threadIdx.x == 0) trace_at(p, 1);

    const int es = FP8 ? 1 : 2;
    const int bk = p.bk;
    constexpr int kUmmaK = FP8 ? 32 : 16;           // K per instruction
    const uint32_t q_box_bytes = (uint32_t)(p.q_mn_major ? bk * 128 : p.bn * 128);

    if (warp == 0) {
        // ------------------------------------------------------ TMA producer
        if (lane == 0) {
            int it = 0;  // global k-block counter across tiles
            const uint32_t tx = (GATHER ? 0u : L.p_bytes) + L.q_bytes;
            for (int u = blockIdx.x; u < p.num_units && !*abort_flag; u += gridDim.x) {
                const TileCoord tc = unit_coord(u, p);
                const int kb0 = tc.split * p.kb_per_split;
                const int kb1 = min(p.kb_total, kb0 + p.kb_per_split);
                for (int kb = kb0; kb < kb1; ++kb, ++it) {
                    const int s = it % p.stages;
                    const uint32_t ph = (uint32_t)(it / p.stages) & 1u;
                    if (!mbar_wait(bar_empty + 8 * s, ph ^ 1u, wc)) break;
                    if (p.stall_loader) continue;  // test hook: nothing arrives, consumers time out
                    const uint32_t full = bar_full + 8 * s;
                    mbar_arrive_expect_tx(full, tx);
                    const uint32_t ps = sbase + s * L.stage_bytes;
                    const uint32_t qs = ps + L.p_bytes;
                    const int k0 = kb * bk;
                    if (!GATHER) {
                        if (p.p_mn_major) {
                            const int per = 128 / es;  // i per box
                            for (int c = 0; c < kBM / per; ++c)
                                tma_load_2d(ps + c * bk * 128, &tmap_p, full, tc.ti * kBM + c * per, k0);
                        } else {
                            tma_load_2d(ps, &tmap_p, full, k0, tc.ti * kBM);
                        }
                    }
                    if (p.q_mn_major) {
                        const int per = 128 / es;
                        for (int c = 0; c < p.bn / per; ++c)
                            tma_load_2d(qs + c * q_box_bytes, &tmap_q, full, tc.tj * p.bn + c * per, k0);
                    } else {
                        tma_load_2d(qs, &tmap_q, full, k0, tc.tj * p.bn);
                    }
                    if (it < 16) trace_at(p, 2 + it);
                }
            }
            // let the copies already issued land before the CTA can exit
            const int last = it;
            for (int d = 1; d <= p.stages && last - d >= 0; ++d) {
                const int j = last - d;
                if (p.stall_loader) break;
                mbar_wait_drain(bar_full + 8 * (j % p.stages), (uint32_t)(j / p.stages) & 1u, p.timeout_ns);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------- MMA issuer
        if (lane == 0) {
            int it = 0, local = 0;
            const uint32_t idesc = p.idesc;
            // descriptor strides: K-major tiles step 1024 B per 8 rows; MN-major
            // tiles step 1024 B per 8 k and one 128-byte MN chunk per bk*128 B.
            const uint32_t p_lbo = p.p_mn_major ? (uint32_t)(bk * 128) : 16u;
            const uint32_t q_lbo = p.q_mn_major ? (uint32_t)(bk * 128) : 16u;
            const uint32_t p_kstep = p.p_mn_major ? kUmmaK * 128 : kUmmaK * es;
            const uint32_t q_kstep = p.q_mn_major ? kUmmaK * 128 : kUmmaK * es;
            bool ok = true;
            for (int u = blockIdx.x; u < p.num_units && ok; u += gridDim.x, ++local) {
                const TileCoord tc = unit_coord(u, p);
                const int kb0 = tc.split * p.kb_per_split;
                const int kb1 = min(p.kb_total, kb0 + p.kb_per_split);
                const int b = local & 1;
                const uint32_t tph = (uint32_t)(local >> 1) & 1u;
                if (!mbar_wait(bar_tempty + 8 * b, tph ^ 1u, wc)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(b * p.bn);
                for (int kb = kb0; kb < kb1; ++kb, ++it) {
                    const int s = it % p.stages;
                    const uint32_t ph = (uint32_t)(it / p.stages) & 1u;
                    if (!mbar_wait(bar_full + 8 * s, ph, wc)) { ok = false; break; }
                    tc_fence_after();
                    if (GATHER) fence_proxy_async_smem();  // thread-written P stage -> tensor-core reads
                    const uint32_t ps = sbase + s * L.stage_bytes;
                    const uint32_t qs = ps + L.p_bytes;
#pragma unroll
                    for (int kk = 0; kk < kTileBytesK / (kUmmaK * es); ++kk) {
                        const uint64_t da = make_sw128_desc(ps + kk * p_kstep, p_lbo, 1024);
                        const uint64_t db = make_sw128_desc(qs + kk * q_kstep, q_lbo, 1024);
                        const uint32_t acc = (kb > kb0 || kk > 0) ? 1u : 0u;
                        if (FP8) umma_f8(d_tmem, da, db, idesc, acc);
                        else umma_f16(d_tmem, da, db, idesc, acc);
                    }
                    tc_commit(bar_empty + 8 * s);  // stage is free once these MMAs have read it
                    if (it < 16) trace_at(p, 18 + it);
                }
                if (!ok) break;
                tc_commit(bar_tfull + 8 * b);      // accumulator b is complete
            }
            pdl_release();  // every MMA is issued: the next kernel may be scheduled during the epilogue
            // wait for every MMA this thread issued before TMEM can be freed
            tc_commit(bar_drain);
            mbar_wait_drain(bar_drain, 0, p.timeout_ns);
        }
    } else if (warp < kEpiWarp0 + 4) {
        // ---------------------------------------------------------- epilogue
        const int quarter = warp & 3;               // TMEM lanes 32*quarter .. +31
        const int row = quarter * 32 + lane;         // row inside the tile
        const EpiParams &e = p.epi;
        int local = 0;
        for (int u = blockIdx.x; u < p.num_units; u += gridDim.x, ++local) {
            const TileCoord tc = unit_coord(u, p);
            const int b = local & 1;
            const uint32_t tph = (uint32_t)(local >> 1) & 1u;
            if (!mbar_wait(bar_tfull + 8 * b, tph, wc)) break;
            tc_fence_after();
            if (local == 0 && threadIdx.x == kEpiWarp0 * 32) trace_at(p, 34);
            const int i = tc.ti * kBM + row;
            const uint32_t t_row = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(b * p.bn);
            const int j0 = tc.tj * p.bn;

            if (p.split_k > 1) {
                // one unit per CTA: the partial stays in TMEM until the cluster
                // has finished its main loops (see the reduction below)
                tc_fence_before();
                if (threadIdx.x == kEpiWarp0 * 32) trace_at(p, 53);
                continue;
            }

            const bool row_ok = i < p.Mi;
            const float asi = row_ok ? e.alpha * (e.scale_i ? e.scale_i[i] : 1.f) : 0.f;
            char *crow = e.c + (int64_t)(row_ok ? i : 0) * e.ci;
            for (int c0 = 0; c0 < p.bn; c0 += 16) {
                uint32_t r[16];
                __syncwarp();
                tmem_ld16(t_row + c0, r);
                tmem_ld_wait();
                if (!row_ok) continue;
                epilogue_chunk16(e, crow, asi, j0 + c0, p.Nj, r);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_tempty + 8 * b);
            if (local == 0 && threadIdx.x == kEpiWarp0 * 32) trace_at(p, 35);
        }
    } else if (GATHER) {
        // ------------------------------------------------ gather producers
        const int gtid = threadIdx.x - (kEpiWarp0 + 4) * 32;
        switch (p.gather_vec * es) {
        case 16: gather_role<16>(p, L, sbase, bar_full, bar_empty, g_row_off, abort_flag, wc, bk, es, gtid, lane); break;
        case 8: gather_role<8>(p, L, sbase, bar_full, bar_empty, g_row_off, abort_flag, wc, bk, es, gtid, lane); break;
        case 4: gather_role<4>(p, L, sbase, bar_full, bar_empty, g_row_off, abort_flag, wc, bk, es, gtid, lane); break;
        case 2: gather_role<2>(p, L, sbase, bar_full, bar_empty, g_row_off, abort_flag, wc, bk, es, gtid, lane); break;
        default: gather_role<1>(p, L, sbase, bar_full, bar_empty, g_row_off, abort_flag, wc, bk, es, gtid, lane); break;
        }
    }

    if (p.split_k > 1) {
        // ------------------------------------------ cluster reduction of k splits
        // CTA s of the cluster owns rows [128 s / S, 128 (s+1) / S) of the tile.
        // After every CTA's main loop (barrier 1: all operand rings are idle),
        // each CTA pushes every row of its partial from TMEM into the owner's
        // ring with remote shared-memory stores (which do not wait), as
        // recv[source][column][row - first owned row]; after barrier 2 each
        // owner adds its S slices in rank order from its own shared memory
        // and runs the epilogue.
        const int S = p.split_k;
        const int rs_max = (kBM + S - 1) / S;
        const uint32_t rank = cluster_ctarank();
        tc_fence_before();
        __syncthreads();
        cluster_sync();
        if (threadIdx.x == kEpiWarp0 * 32) trace_at(p, 54);
        if (warp >= kEpiWarp0 && warp < kEpiWarp0 + 4) {
            tc_fence_after();
            const int quarter = warp & 3;
            const int row = quarter * 32 + lane;
            int d = 0;
            while (d + 1 < S && (d + 1) * kBM / S <= row) ++d;
            const int rl = row - d * kBM / S;
            const uint32_t dst = dsmem_map(sbase, (uint32_t)d);
            const uint32_t t_row = tmem_base + ((uint32_t)(quarter * 32) << 16);
            for (int c0 = 0; c0 < p.bn; c0 += 16) {
                uint32_t r[16];
                __syncwarp();
                tmem_ld16(t_row + c0, r);
                tmem_ld_wait();
#pragma unroll
                for (int c = 0; c < 16; ++c)
                    dsmem_st_f32(dst + (uint32_t)((((int)rank * p.bn + c0 + c) * rs_max + rl) * 4), __uint_as_float(r[c]));
            }
        }
        __syncthreads();
        cluster_sync();
        if (threadIdx.x == kEpiWarp0 * 32) trace_at(p, 55);
        if (warp >= kEpiWarp0 && warp < kEpiWarp0 + 4) {
            const EpiParams &e = p.epi;
            const TileCoord tc = unit_coord(blockIdx.x, p);
            const int r0 = (int)(rank * kBM / S), r1 = (int)((rank + 1) * kBM / S), rs = r1 - r0;
            const int t = threadIdx.x - kEpiWarp0 * 32;
            const bool along_i = (e.ci == (int64_t)elem_bytes(e.c_dtype));  // C contiguous along i
            const float *recv = reinterpret_cast<const float *>(smem);
            // element e of the owned rs x bn slice: r = e % rs, c = e / rs when C
            // is contiguous along i (consecutive threads, consecutive addresses),
            // else c = e % bn, r = e / bn; indices advance without division
            const int total = rs * p.bn;
            int r = along_i ? t % rs : t / p.bn, c = along_i ? t / rs : t % p.bn;
            const int dr = along_i ? 128 % rs : 128 / p.bn, dc = along_i ? 128 / rs : 128 % p.bn;
            constexpr int kB = 8;  // outputs per thread per batch: their C loads are in flight together
            for (int base = t; base < total; base += 128 * kB) {
                int ii[kB], jj[kB];
                float acc[kB], cin[kB];
#pragma unroll
                for (int b = 0; b < kB; ++b) {
                    const int i = tc.ti * kBM + r0 + r, j = tc.tj * p.bn + c;
                    const bool ok = base + b * 128 < total && i < p.Mi && j < p.Nj;
                    ii[b] = ok ? i : -1;
                    jj[b] = j;
                    float a = 0.f;
                    if (ok)
                        for (int q = 0; q < S; ++q) a += recv[(q * p.bn + c) * rs_max + r];
                    acc[b] = a;
                    cin[b] = (ok && e.beta != 0.f) ? load_elem(e.c + (int64_t)i * e.ci + (int64_t)j * e.cj, e.c_dtype)
                                                   : 0.f;
                    // advance by 128 elements
                    if (along_i) {
                        r += dr;
                        c += dc;
                        if (r >= rs) { r -= rs; ++c; }
                    } else {
                        c += dc;
                        r += dr;
                        if (c >= p.bn) { c -= p.bn; ++r; }
                    }
                }
#pragma unroll
                for (int b = 0; b < kB; ++b) {
                    if (ii[b] < 0) continue;
                    const int i = ii[b], j = jj[b];
                    const float asi = e.alpha * (e.scale_i ? e.scale_i[i] : 1.f);
                    const float sj = e.scale_j ? e.scale_j[j] : 1.f;
                    float val = (asi * sj) * acc[b];
                    if (e.beta != 0.f) val = fmaf(e.beta, cin[b], val);
                    store_elem(e.c + (int64_t)i * e.ci + (int64_t)j * e.cj, e.c_dtype, val);
                }
            }
        }
        if (threadIdx.x == kEpiWarp0 * 32) trace_at(p, 56);
        // no CTA touches another's shared memory after the second barrier
    }

    // --------------------------------------------------------------- teardown
    if (threadIdx.x == 0) trace_at(p, 36);
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem_base, (uint32_t)p.tmem_cols);
    }
}

}  // namespace

size_t umma_smem_bytes(int bn, int bk_bytes, int stages, bool gather) {
    (void)bk_bytes;
    return smem_layout(bn, stages, gather).total;
}

int umma_max_stages(int bn, bool gather) {
    int s = 2;
    while (s < 12 && smem_layout(bn, s + 1, gather).total <= 227 * 1024) ++s;
    return s;
}

cudaError_t launch_umma(const UmmaParams &p, const CUtensorMap *tp, const CUtensorMap *tq, bool fp8, bool gather,
                        int grid, size_t smem, cudaStream_t s) {
    void (*kern)(const CUtensorMap, const CUtensorMap, const UmmaParams);
    if (fp8) kern = gather ? umma_gemm_kernel<true, true> : umma_gemm_kernel<true, false>;
    else kern = gather ? umma_gemm_kernel<false, true> : umma_gemm_kernel<false, false>;
    // raise the kernel's dynamic shared-memory limit once per size, not per call
    static std::atomic<int> s_limit[4];
    std::atomic<int> &lim = s_limit[(fp8 ? 2 : 0) + (gather ? 1 : 0)];
    cudaError_t e = cudaSuccess;
    if ((int)smem > lim.load()) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        lim.store((int)smem);
    }
    return launch_ex(kern, dim3(grid), dim3(gather ? 320 : 192), smem, s, dim3(p.split_k, 1, 1), p.pdl, *tp, *tq, p);
}

}  // namespace dg
