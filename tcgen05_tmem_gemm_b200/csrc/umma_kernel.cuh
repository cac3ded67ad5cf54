// Tensor-core GEMM for sm_100a: tcgen05.mma with TMEM accumulators.
// (The kernel template; umma.cu, umma_gather.cu and umma_gather_split.cu each instantiate part of it.)
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
//    signals a finished accumulator; with a gather cluster a second lane
//    forwards this CTA's gathered parts to the other CTAs;
//  - warps 2-5: the epilogue, each owning 32 TMEM lanes (rows): tcgen05.ld,
//    scale, optional beta * C, convert, and tensor stores of 32-row x 128-byte
//    blocks (or thread stores), while the MMA warp already fills the other
//    accumulator;
//  - warps 6-13 (gather variant): cp.async loads of a P operand that TMA
//    cannot describe (e.g. an NCHW feature map read as [N*H*W, C] with a
//    392-byte channel stride), written into the same swizzled layout
//    ("DeepGEMM: a recalibration of the compute paradigm", §2.2: scatter-gather
//    loads for the non-contiguous segments of a view).  The CTAs that need the
//    same rows of P form a cluster and each gathers one k-slice of every stage,
//    copied to the others through distributed shared memory.  With one tile
//    per CTA these warps then take part of the epilogue;
//  - split-K ("DeepGEMM deep dive", §5.2), no global workspace either way:
//    with beta = 1 and FP32 C (and no activation) each split adds its scaled
//    partial into C with tensor reduce-adds, with no cluster; otherwise the
//    splits of a tile form a cluster, each CTA sends the rows other CTAs own
//    from its partial into their shared memory, and each owner adds the
//    slices in split order (deterministic) and runs the epilogue.
// The template's SPLIT parameter leaves the split-K paths out of instances
// that only run unsplit plans.  Every wait is bounded (WaitCtl); on expiry the
// CTA records DG_ERR_TIMEOUT, drains what it has in flight, frees TMEM and
// exits.
#pragma once

#include <atomic>
#include <type_traits>

#include "common.cuh"
#include "sm100.cuh"
#include "umma_common.cuh"

namespace dg {

namespace {

constexpr int kBM = 128;             // tensor-core tile rows (TMEM lanes)
constexpr int kMaxSplit = 8;         // k splits of a tile: one portable cluster
constexpr int kTileBytesK = 128;     // one swizzle row: 64 x 16-bit or 128 x 8-bit
constexpr int kGatherWarps = 8;     // gather warps: cp.async latency-bound, so more warps keep more copies in flight

// Split-K reduction: a CTA's partial is staged in its own operand ring (idle
// once its main loop is done) as S slices of `slice` bytes from offset 0,
// slice d holding the rows CTA d of the cluster owns (column-major); the
// slices the other CTAs send it land in a region of its own (S slots, by
// source rank), so they can arrive while its main loop still runs.
__host__ __device__ inline uint32_t split_slice_bytes(int bn, int S) {
    return (uint32_t)(bn * ((kBM + S - 1) / S) * 4);
}
__host__ __device__ inline uint32_t split_out_bytes(int bn, int S) { return S * split_slice_bytes(bn, S); }
__host__ __device__ inline uint32_t split_in_bytes(int bn, int S) {
    return S > 1 ? (S * split_slice_bytes(bn, S) + 1023u) & ~1023u : 0u;
}

struct SmemLayout {
    uint32_t stage_bytes, p_bytes, q_bytes;
    uint32_t epi_off;                // TMA-store epilogue blocks (epi_tma), after the stages
    uint32_t recv_off;               // split-K slices received from the other CTAs
    uint32_t bar_off;
    uint32_t aux_off;                // tmem address, abort flag, gather tables
    uint32_t total;
};

__host__ __device__ inline SmemLayout smem_layout(int bn, int stages, bool gather, bool epi_tma, int split) {
    SmemLayout L;
    L.p_bytes = kBM * kTileBytesK;
    L.q_bytes = (uint32_t)bn * kTileBytesK;
    L.stage_bytes = L.p_bytes + L.q_bytes;  // a multiple of 1024: bn is a multiple of 8
    L.epi_off = L.stage_bytes * stages;
    L.recv_off = L.epi_off + (epi_tma ? kEpiStoreBytes : 0u);
    L.bar_off = L.recv_off + split_in_bytes(bn, split);
    // full[S], empty[S], part[S] (gather cluster), tfull[2], tempty[2], drain,
    // recv (split-K slices)
    L.aux_off = L.bar_off + 8 * (3 * stages + 6);
    uint32_t aux = 16;  // tmem base + abort flag
    if (gather) aux += 8 * kBM;  // row offsets of the tile
    L.total = L.aux_off + aux + 1024;  // + slack to align the base to 1024
    return L;
}

struct TileCoord {
    int ti, tj, split;
};

// Unit u of the persistent schedule.  With split-K, the splits of a tile are
// consecutive (one cluster).  With a gather cluster of G CTAs, u = g * G + r:
// the G CTAs of a cluster take tiles (ti, jg * G + r) of group g, the same
// rows of P.
__device__ __forceinline__ TileCoord unit_coord(int u, const UmmaParams &p) {
    TileCoord c;
    if (p.gather_cluster > 1) {
        const int G = p.gather_cluster, g = u / G;
        c.split = 0;
        c.ti = g % p.tiles_i;
        c.tj = (g / p.tiles_i) * G + u % G;
        return c;
    }
    c.split = u % p.split_k;
    const int t = u / p.split_k;
    c.ti = t % p.tiles_i;
    c.tj = t / p.tiles_i;
    return c;
}

// Byte offset inside a 128-byte-swizzled K-major tile of the element at
// (mn, k); `bytek` = k * element size.
__device__ __forceinline__ uint32_t sw128_kmajor(int mn, int bytek) {
    return (uint32_t)((mn >> 3) * 1024 + (mn & 7) * 128 + ((((bytek >> 4) ^ (mn & 7)) << 4) | (bytek & 15)));
}
// Gathered MN-major tiles are laid out k-slice by k-slice: the 2^ks_log2 rows
// of k that one MMA instruction consumes (every 128-byte MN chunk of them)
// are kGatherSliceBytes contiguous bytes, so the k range one CTA of a gather
// cluster loads is a single block of shared memory.  Within a slice, chunk c
// starts at c * 2^ks_log2 * 128 bytes; 8-row swizzle atoms of 1024 bytes.
constexpr int kGatherSliceBytes = 4096;  // 128 rows x 16 (16-bit) or 32 (8-bit) k
__device__ __forceinline__ uint32_t sw128_mnmajor_ks(int bytemn, int k, int ks_log2) {
    const int c = bytemn >> 7, w = bytemn & 127;
    const int kk = k & ((1 << ks_log2) - 1);
    return (uint32_t)((k >> ks_log2) * kGatherSliceBytes + (c << ks_log2) * 128 + (kk >> 3) * 1024 + (k & 7) * 128 +
                      ((((w >> 4) ^ (k & 7)) << 4) | (w & 15)));
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

// Phase timestamps of CTA 0 for performance analysis (DG_OPT_TRACE), in SM
// cycles (the cycle counter costs a few cycles to read): slot 0
// entry, 1 set-up done, 2+kb first-unit loads issued (k block kb < 16),
// 18+kb MMAs of k block kb issued, 34 first accumulator complete (seen by the
// epilogue), 35 first epilogue done, 36 teardown, 37..52 gather k block kb
// written (first unit); split-K: 53 accumulator complete, 54 first cluster
// barrier passed, 55 partials pushed and second barrier passed, 56 reduced.
__device__ __forceinline__ void trace_at(const UmmaParams &p, int slot) {
    if (p.trace != nullptr && blockIdx.x == 0) p.trace[slot] = (uint64_t)clock64();
}

// The tensor copies of k block k0.. of tile (ti, tj) into the stage at `ps`
// (P, unless it is gathered) and `qs` (Q), completing on barrier `full`.
// MN-major operands come as boxes of 128 bytes along i or j.
template <bool GATHER>
__device__ __forceinline__ void load_kblock(const CUtensorMap *tp, const CUtensorMap *tq, uint32_t full, uint32_t ps,
                                            uint32_t qs, int ti, int tj, int k0, int bn, int bk, int es, bool p_mn,
                                            bool q_mn, uint32_t q_box_bytes) {
    if (!GATHER) {
        if (p_mn) {
            const int per = 128 / es;  // i per box
            for (int c = 0; c < kBM / per; ++c) tma_load_2d(ps + c * bk * 128, tp, full, ti * kBM + c * per, k0);
        } else {
            tma_load_2d(ps, tp, full, k0, ti * kBM);
        }
    }
    if (q_mn) {
        const int per = 128 / es;
        for (int c = 0; c < bn / per; ++c) tma_load_2d(qs + c * q_box_bytes, tq, full, tj * bn + c * per, k0);
    } else {
        tma_load_2d(qs, tq, full, k0, tj * bn);
    }
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
    int vec, runs, total, es;
    int runs_log2;  // runs is a power of two: indices split with shifts and masks
    int ks_log2;    // MN-major: log2 of the k rows per slice (one MMA instruction's K)
};

// The gathered operand's base and k axis, read from the parameter block once:
// the copy loops then keep them in registers instead of re-reading them after
// every asynchronous copy.
struct GatherSrc {
    const char *ptr;
    int64_t kstride;     // byte stride of k when k is one merged dim (k1)
    const Axis *kaxis;   // otherwise the whole axis
    int K;
    bool k1;
    __device__ __forceinline__ int64_t koff(int kg) const {
        return k1 ? (int64_t)kg * kstride : axis_offset(*kaxis, kg);
    }
};

__device__ __forceinline__ GatherSrc gather_src(const UmmaParams &p) {
    GatherSrc s;
    s.ptr = p.pv.ptr;
    s.k1 = p.pv.col.n == 1;
    s.kstride = p.pv.col.stride[0];
    s.kaxis = &p.pv.col;
    s.K = p.K;
    return s;
}

__device__ __forceinline__ GatherGeom gather_geom(const UmmaParams &p, int VB, int bk, int es) {
    GatherGeom g;
    g.mn = p.p_mn_major != 0;
    g.vec = VB / es;
    g.runs = g.mn ? kBM / g.vec : bk / g.vec;
    g.total = g.mn ? g.runs * bk : kBM * g.runs;
    g.runs_log2 = __ffs(g.runs) - 1;
    g.ks_log2 = es == 1 ? 5 : 4;  // 32 E4M3 or 16 F16/BF16 k per MMA instruction
    g.es = es;
    return g;
}

// Copies first, first + 128, first + 256, ... of a stage: along the unit-
// stride dim their position is fixed and the other index advances by
// 128 / runs per copy (runs is a power of two dividing 128), so no index is
// divided inside the loops.
template <int VB>
__device__ __forceinline__ void gather_load(const GatherSrc &src, const GatherGeom &g, const int64_t *row_off,
                                            int kbase, int first, typename VecOf<VB>::T (&v)[kGatherUnroll]) {
    const int nthreads = kGatherWarps * 32;
    const int step = nthreads >> g.runs_log2;
    if (g.mn) {
        // fixed i (a run of vec rows), k advancing by `step`
        const int i = (first & (g.runs - 1)) * g.vec;
        const int64_t ro = row_off[i];
        const int k0 = first >> g.runs_log2;
#pragma unroll
        for (int r = 0; r < kGatherUnroll; ++r) {
            const int u = first + r * nthreads;
            const int kg = kbase + k0 + r * step;
            const bool ok = u < g.total && ro >= 0 && kg < src.K;
            v[r] = gather_load_one<VB>(src.ptr + (ok ? ro + src.koff(kg) : 0), ok);
        }
    } else {
        // fixed k (a run of vec columns), i advancing by `step`
        const int kg = kbase + (first & (g.runs - 1)) * g.vec;
        const int64_t co = kg < src.K ? src.koff(kg) : -1;
        const int i0 = first >> g.runs_log2;
#pragma unroll
        for (int r = 0; r < kGatherUnroll; ++r) {
            const int u = first + r * nthreads;
            const int i = i0 + r * step;
            const int64_t ro = (u < g.total) ? row_off[i] : -1;
            const bool ok = ro >= 0 && co >= 0;
            v[r] = gather_load_one<VB>(src.ptr + (ok ? ro + co : 0), ok);
        }
    }
}

template <int VB>
__device__ __forceinline__ void gather_store(const GatherGeom &g, uint32_t p_smem, int first,
                                             const typename VecOf<VB>::T (&v)[kGatherUnroll]) {
    const int nthreads = kGatherWarps * 32;
    const int step = nthreads >> g.runs_log2;
    const int fixed = (first & (g.runs - 1)) * g.vec, moving0 = first >> g.runs_log2;
#pragma unroll
    for (int r = 0; r < kGatherUnroll; ++r) {
        const int u = first + r * nthreads;
        if (u >= g.total) continue;
        const int moving = moving0 + r * step;
        st_shared_vec<VB>(p_smem + (g.mn ? sw128_mnmajor_ks(fixed * g.es, moving, g.ks_log2)
                                         : sw128_kmajor(moving, fixed * g.es)),
                          v[r]);
    }
}

// cp.async version of a batch: the same copies as gather_load/gather_store,
// issued as asynchronous global -> shared copies (no register staging).
template <int VB>
__device__ __forceinline__ void gather_issue_async(const GatherSrc &src, const GatherGeom &g,
                                                   const int64_t *row_off, int kbase, int first, int uend,
                                                   uint32_t p_smem) {
    const int nthreads = kGatherWarps * 32;
    const int step = nthreads >> g.runs_log2;
    const int fixed = (first & (g.runs - 1)) * g.vec, moving0 = first >> g.runs_log2;
    if (g.mn) {
        const int64_t ro = row_off[fixed];
#pragma unroll
        for (int r = 0; r < kGatherUnroll; ++r) {
            const int u = first + r * nthreads;
            if (u >= uend) break;
            const int k = moving0 + r * step, kg = kbase + k;
            const bool ok = ro >= 0 && kg < src.K;
            cp_async_zfill<VB>(p_smem + sw128_mnmajor_ks(fixed * g.es, k, g.ks_log2),
                               src.ptr + (ok ? ro + src.koff(kg) : 0), ok);
        }
    } else {
        const int kg = kbase + fixed;
        const int64_t co = kg < src.K ? src.koff(kg) : -1;
#pragma unroll
        for (int r = 0; r < kGatherUnroll; ++r) {
            const int u = first + r * nthreads;
            if (u >= uend) break;
            const int i = moving0 + r * step;
            const int64_t ro = row_off[i];
            const bool ok = ro >= 0 && co >= 0;
            cp_async_zfill<VB>(p_smem + sw128_kmajor(i, fixed * g.es), src.ptr + (ok ? ro + co : 0), ok);
        }
    }
}

// The gather role for one vector width.  Per tile: row offsets once.  When
// a stage is at most one batch per thread (kGatherUnroll copies), the next
// k block's loads are issued before this block is stored, so two stages of
// loads are in flight; wider stages are loaded and stored batch by batch.
// Every exit decision is voted on across the gather warps (bar.red) at tile
// boundaries, so no warp is left waiting at their named barrier.
template <int VB>
__device__ __forceinline__ void gather_role(const UmmaParams &p, const SmemLayout &L, uint32_t sbase,
                                            uint32_t bar_full, uint32_t bar_empty, uint32_t bar_part,
                                            int64_t *g_row_off,
                                            volatile int *abort_flag, const WaitCtl &wc, int bk, int es, int gtid,
                                            int lane) {
    using V = typename VecOf<VB>::T;
    const GatherGeom g = gather_geom(p, VB, bk, es);
    const GatherSrc src = gather_src(p);
    const int stages = p.stages;
    const bool stall = p.stall_loader == 1;
    const int nthreads = kGatherWarps * 32;
    const bool one_batch = VB < 4 && g.total <= nthreads * kGatherUnroll;  // register path look-ahead
    // a gather cluster splits every stage's copies among its CTAs (cp.async
    // path only); this CTA's copies complete on its part barrier
    const int G = p.gather_cluster > 1 ? p.gather_cluster : 1;
    const int grank = G > 1 ? (int)cluster_ctarank() : 0;
    const int ubeg = grank * (g.total / G), uend = (grank + 1) * (g.total / G);
    const uint32_t bar_done = G > 1 ? bar_part : bar_full;
    int it = 0, gs = 0;
    uint32_t gph = 0;
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
        pdl_wait();  // before the first copy (returns at once after the first unit)
        bool ok = true;
        V cur[kGatherUnroll], nxt[kGatherUnroll];
        if (one_batch && kb0 < kb1) gather_load<VB>(src, g, g_row_off, kb0 * bk, gtid, cur);
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
            const int s = gs;
            const uint32_t ph = gph;
            if (++gs == stages) {  // stage and phase of the next k block, without division
                gs = 0;
                gph ^= 1u;
            }
            if (one_batch && kb + 1 < kb1) gather_load<VB>(src, g, g_row_off, (kb + 1) * bk, gtid, nxt);
            ok = mbar_wait(bar_empty + 8 * s, ph ^ 1u, wc);
            if (!ok) break;  // the other warps see the abort flag; the vote below makes the exit uniform
            if (!stall && VB >= 4) {
                // asynchronous copies: the stage completes on the full barrier
                // when they land, and this warp moves on at once
                const uint32_t ps = sbase + s * L.stage_bytes;
                for (int f = ubeg + gtid; f < uend; f += nthreads * kGatherUnroll)
                    gather_issue_async<(VB >= 4 ? VB : 4)>(src, g, g_row_off, kb * bk, f, uend, ps);
                cp_async_arrive_noinc(bar_done + 8 * s);
                if (it < 16 && gtid == 0) trace_at(p, 37 + it);
            } else if (!stall) {
                const uint32_t ps = sbase + s * L.stage_bytes;
                if (one_batch) {
                    gather_store<VB>(g, ps, gtid, cur);
                } else {
                    for (int f = gtid; f < g.total; f += nthreads * kGatherUnroll) {
                        gather_load<VB>(src, g, g_row_off, kb * bk, f, cur);
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
        // row offsets of this tile stay in use until every gather warp is past
        // it; the vote is that barrier, and every warp leaves together
        if (named_bar_or(!ok)) break;
    }
    // nothing this thread copied may land after the CTA has gone
    asm volatile("cp.async.wait_all;" ::: "memory");
}

template <bool FP8, bool GATHER, bool SPLIT>
__global__ void __launch_bounds__(GATHER ? 448 : 192, 1)
    umma_gemm_kernel(const __grid_constant__ CUtensorMap tmap_p, const __grid_constant__ CUtensorMap tmap_q,
                     const __grid_constant__ CUtensorMap tmap_c, const UmmaParams p) {
    // instances for unsplit plans carry no split-K paths (a smaller
    // instruction footprint: every phase of a one-tile CTA is a first pass
    // through its code)
    constexpr bool kSplit = SPLIT;
    if (threadIdx.x == 0) trace_at(p, 0);
    if (threadIdx.x == 64) {
        // descriptor fetches start at once, while thread 0 sets up the barriers
        tma_prefetch_desc(&tmap_q);
        if (!GATHER) tma_prefetch_desc(&tmap_p);
        if (p.epi_tma || p.red_add) tma_prefetch_desc(&tmap_c);
    }
    if (p.pdl == 1) pdl_release();
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1024-byte alignment for the 128-byte swizzle atoms
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    // split-K partials added into C (red_add) need no receive region
    const SmemLayout L = smem_layout(p.bn, p.stages, GATHER, p.epi_tma != 0, p.red_add ? 1 : p.split_k);
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar_full = sbase + L.bar_off;
    const uint32_t bar_empty = bar_full + 8 * p.stages;
    const uint32_t bar_part = bar_empty + 8 * p.stages;
    const uint32_t bar_tfull = bar_part + 8 * p.stages;
    const uint32_t bar_tempty = bar_tfull + 16;
    const uint32_t bar_drain = bar_tempty + 16;
    const uint32_t bar_recv = bar_drain + 8;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L.aux_off);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L.aux_off + 4);
    int64_t *g_row_off = reinterpret_cast<int64_t *>(smem + L.aux_off + 16);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr int kEpiWarp0 = 2;
    const WaitCtl wc{abort_flag, p.err_word, p.timeout_ns};

    const int G = GATHER && p.gather_cluster > 1 ? p.gather_cluster : 1;  // gather cluster size
    // gather warps help the epilogue when every CTA has exactly one tile (their
    // tensor-store blocks then live in the idle operand ring; thread stores
    // need no staging)
    const bool helpers = GATHER && p.split_k == 1 && p.num_units == (int)gridDim.x &&
                         (!p.epi_tma ||
                          L.stage_bytes * (uint32_t)p.stages >= (uint32_t)kGatherWarps * 2u * kEpiBlockBytes);
    int pre_issued = 0;  // k blocks of the first unit copied during the set-up (thread 0)
    if (threadIdx.x == 0) {
        for (int s = 0; s < p.stages; ++s) {
            // gather stages: one arrival per gather thread when its cp.async
            // copies land (4..16-byte copies), else one per gather warp; with
            // a gather cluster those land on the part barrier and the
            // forwarding thread arrives once on the stage's full barrier
            const int gather_arrivals = p.gather_vec * (FP8 ? 1 : 2) >= 4 ? kGatherWarps * 32 : kGatherWarps;
            mbar_init(bar_full + 8 * s, GATHER ? 1 + (G > 1 ? 1 : gather_arrivals) : 1);
            // a stage is free once every CTA of a gather cluster has consumed it
            mbar_init(bar_empty + 8 * s, (uint32_t)G);
            mbar_init(bar_part + 8 * s, (uint32_t)gather_arrivals);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar_tfull + 8 * b, 1);
            mbar_init(bar_tempty + 8 * b, 4);
        }
        mbar_init(bar_drain, 1);
        mbar_init(bar_recv, 1);
        // split-K: the slices of this CTA's rows from the other CTAs of the cluster
        if (kSplit && p.split_k > 1 && !p.red_add)
            mbar_arrive_expect_tx(bar_recv, (uint32_t)(p.split_k - 1) * split_slice_bytes(p.bn, p.split_k));
        *abort_flag = 0;
        fence_barrier_init();
        fence_proxy_async_smem();
        // Every stage is free: for a unit that streams more k blocks than the
        // ring holds, this thread, the producer lane, puts the first round of
        // copies in flight now, while the other warps finish the set-up
        // (their first global access waits for the previous kernel, and so
        // does this one).  Not in a cluster (a gather cluster, or split-K
        // reduced on chip), whose start would wait for these copies; and not
        // for short units, whose set-up measured faster without it.
        const bool no_cluster = !GATHER && !(kSplit && p.split_k > 1 && !p.red_add);
        if (no_cluster && p.stall_loader != 1 && (int)blockIdx.x < p.num_units) {
            const TileCoord tc = unit_coord(blockIdx.x, p);
            const int kb0 = tc.split * p.kb_per_split;
            const int nkb = min(p.kb_total, kb0 + p.kb_per_split) - kb0;
            pre_issued = nkb > p.stages ? p.stages : 0;
            const uint32_t tx0 = (GATHER ? (uint32_t)(G - 1) * (L.p_bytes / G) : L.p_bytes) + L.q_bytes;
            const uint32_t qbb = (uint32_t)(p.q_mn_major ? p.bk * 128 : p.bn * 128);
            if (pre_issued > 0) pdl_wait();
            for (int q = 0; q < pre_issued; ++q) {
                const uint32_t full = bar_full + 8 * q;
                const uint32_t ps = sbase + q * L.stage_bytes;
                mbar_arrive_expect_tx(full, tx0);
                load_kblock<GATHER>(&tmap_p, &tmap_q, full, ps, ps + L.p_bytes, tc.ti, tc.tj, (kb0 + q) * p.bk, p.bn,
                                    p.bk, FP8 ? 1 : 2, p.p_mn_major != 0, p.q_mn_major != 0, qbb);
            }
        }
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), (uint32_t)p.tmem_cols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    // CTAs of a cluster write into each other's shared memory and barriers
    // (split-K slices, gather-cluster parts and stage releases).  Every thread
    // arrives on the cluster barrier once this CTA's barriers are initialised;
    // a thread waits for it before its first access to another CTA, and at the
    // latest before the next cluster barrier, so the start is not delayed.
    // Cluster barrier operations are always issued by whole, converged warps.
    // split-K CTAs that add into C (red_add) exchange nothing: no cluster
    const bool clustered = (kSplit && p.split_k > 1 && !p.red_add) || G > 1;
    bool cluster_ready = !clustered;  // warp-uniform
    if (clustered) {
        __syncwarp();
        cluster_arrive();
    }
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    // The set-up above touches only this CTA's shared memory and TMEM, so it
    // runs while the previous kernel finishes (programmatic dependent launch).
    // Each role waits for that kernel right before its first global access,
    // after the work it can do from the parameters alone (the gather's row
    // offsets, the producer's unit coordinates); the MMA issuer and the
    // gather-cluster forwarder touch no global memory and do not wait.
    if (threadIdx.x == 0) trace_at(p, 1);

    const int es = FP8 ? 1 : 2;
    const int bk = p.bk;
    constexpr int kUmmaK = FP8 ? 32 : 16;           // K per instruction
    const uint32_t q_box_bytes = (uint32_t)(p.q_mn_major ? bk * 128 : p.bn * 128);

    if (warp == 0) {
        // ------------------------------------------------------ TMA producer
        if (lane == 0) {
            // everything the loop needs in registers (the copies' memory
            // clobbers would otherwise make it re-read the parameters); stage
            // and phase advance without division
            const int stages = p.stages, num_units = p.num_units, kb_total = p.kb_total;
            const int kb_per_split = p.kb_per_split, bn = p.bn;
            const bool stall = p.stall_loader == 1, p_mn = p.p_mn_major != 0, q_mn = p.q_mn_major != 0;
            const uint32_t stage_bytes = L.stage_bytes, p_bytes = L.p_bytes;
            // the set-up issued stages 0 .. pre_issued-1 of the first unit
            int it = pre_issued, s = pre_issued == stages ? 0 : pre_issued;  // k-block counter, its stage
            uint32_t ph = pre_issued == stages ? 1u : 0u;
            int skip = pre_issued;
            // gathered P: the parts of the other CTAs of a gather cluster arrive as bytes
            const uint32_t tx = (GATHER ? (uint32_t)(G - 1) * (p_bytes / G) : p_bytes) + L.q_bytes;
            pdl_wait();
            for (int u = blockIdx.x; u < num_units && !*abort_flag; u += gridDim.x) {
                const TileCoord tc = unit_coord(u, p);
                const int kb0 = tc.split * kb_per_split;
                const int kb1 = min(kb_total, kb0 + kb_per_split);
                bool ok = true;
                for (int kb = kb0 + skip; kb < kb1; ++kb, ++it) {
                    if (!mbar_wait(bar_empty + 8 * s, ph ^ 1u, wc)) { ok = false; break; }
                    if (!stall) {  // test hook: with stall nothing arrives, consumers time out
                        const uint32_t full = bar_full + 8 * s;
                        mbar_arrive_expect_tx(full, tx);
                        const uint32_t ps = sbase + s * stage_bytes;
                        load_kblock<GATHER>(&tmap_p, &tmap_q, full, ps, ps + p_bytes, tc.ti, tc.tj, kb * bk, bn, bk,
                                            es, p_mn, q_mn, q_box_bytes);
                        if (it < 16) trace_at(p, 2 + it);
                    }
                    if (++s == stages) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                skip = 0;
                if (!ok) break;
            }
            // let the copies already issued land before the CTA can exit
            const int last = it;
            for (int d = 1; d <= p.stages && last - d >= 0; ++d) {
                const int j = last - d;
                if (p.stall_loader == 1) break;
                mbar_wait_drain(bar_full + 8 * (j % p.stages), (uint32_t)(j / p.stages) & 1u, p.timeout_ns);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------- MMA issuer
        if (G > 1) {
            // the whole warp, converged: its stage releases and the forwarder's
            // copies reach the other CTAs, whose barriers must be initialised
            __syncwarp();
            cluster_wait();
            cluster_ready = true;
        }
        if (lane == 0) {
            const int stages = p.stages, num_units = p.num_units, kb_total = p.kb_total;
            const int kb_per_split = p.kb_per_split, bn = p.bn;
            const uint32_t idesc = p.idesc, stage_bytes = L.stage_bytes;
            // descriptor strides: K-major tiles step 1024 B per 8 rows; MN-major
            // tiles step 1024 B per 8 k and one 128-byte MN chunk per bk*128 B.
            // gathered MN-major P is laid out k-slice by k-slice (one slice per
            // MMA step, its MN chunks kUmmaK * 128 bytes apart)
            const bool p_ks = GATHER && p.p_mn_major;
            const uint32_t p_lbo = p_ks ? (uint32_t)(kUmmaK * 128) : p.p_mn_major ? (uint32_t)(bk * 128) : 16u;
            const uint32_t q_lbo = p.q_mn_major ? (uint32_t)(bk * 128) : 16u;
            const uint32_t p_kstep = p_ks ? (uint32_t)kGatherSliceBytes : p.p_mn_major ? kUmmaK * 128 : kUmmaK * es;
            const uint32_t q_kstep = p.q_mn_major ? kUmmaK * 128 : kUmmaK * es;
            // descriptors of stage 0; a stage's differ only in the start address
            // field (address >> 4, below 2^14 for any shared-memory address)
            const uint64_t da0 = make_sw128_desc(sbase, p_lbo, 1024);
            const uint64_t db0 = make_sw128_desc(sbase + L.p_bytes, q_lbo, 1024);
            const uint16_t cl_mask = (uint16_t)((1u << G) - 1u);
            int it = 0, local = 0, s = 0;
            uint32_t ph = 0;
            bool ok = true;
            for (int u = blockIdx.x; u < num_units && ok; u += gridDim.x, ++local) {
                const TileCoord tc = unit_coord(u, p);
                const int kb0 = tc.split * kb_per_split;
                const int kb1 = min(kb_total, kb0 + kb_per_split);
                const int b = local & 1;
                const uint32_t tph = (uint32_t)(local >> 1) & 1u;
                if (!mbar_wait(bar_tempty + 8 * b, tph ^ 1u, wc)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(b * bn);
                for (int kb = kb0; kb < kb1; ++kb, ++it) {
                    if (!mbar_wait(bar_full + 8 * s, ph, wc)) { ok = false; break; }
                    tc_fence_after();
                    if (GATHER) fence_proxy_async_smem();  // thread-written P stage -> tensor-core reads
                    const uint64_t soff = (uint64_t)((s * stage_bytes) >> 4);
#pragma unroll
                    for (int kk = 0; kk < kTileBytesK / (kUmmaK * es); ++kk) {
                        const uint64_t da = da0 + soff + (uint64_t)((kk * p_kstep) >> 4);
                        const uint64_t db = db0 + soff + (uint64_t)((kk * q_kstep) >> 4);
                        const uint32_t acc = (kb > kb0 || kk > 0) ? 1u : 0u;
                        if (FP8) umma_f8(d_tmem, da, db, idesc, acc);
                        else umma_f16(d_tmem, da, db, idesc, acc);
                    }
                    // the stage is free once these MMAs have read it (in every
                    // CTA of a gather cluster: they all write into it)
                    if (G > 1) tc_commit_mc(bar_empty + 8 * s, cl_mask);
                    else tc_commit(bar_empty + 8 * s);
                    if (it < 16) trace_at(p, 18 + it);
                    if (++s == stages) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                if (!ok) break;
                tc_commit(bar_tfull + 8 * b);      // accumulator b is complete
            }
            pdl_release();  // every MMA is issued: the next kernel may be scheduled during the epilogue
            // wait for every MMA this thread issued before TMEM can be freed
            tc_commit(bar_drain);
            mbar_wait_drain(bar_drain, 0, p.timeout_ns);
        } else if (GATHER && G > 1 && lane == 1) {
            // ---------------------------------------- gather-cluster forwarder
            // Once this CTA's part of a stage has landed, copy it into the same
            // stage of every other CTA of the cluster (their full barriers count
            // the bytes), then count the part as arrived here.  The part is one
            // contiguous block: whole k-slices (MN-major) or a row range.
            const uint32_t grank = cluster_ctarank();
            const uint32_t part = L.p_bytes / (uint32_t)G;
            const uint32_t first_off = grank * part;
            const int stages = p.stages;
            int fs = 0;  // stage and phase, advanced without division
            uint32_t fph = 0;
            bool ok = true;
            for (int u = blockIdx.x; u < p.num_units && ok; u += gridDim.x) {
                const TileCoord tc = unit_coord(u, p);
                const int kb0 = tc.split * p.kb_per_split;
                const int kb1 = min(p.kb_total, kb0 + p.kb_per_split);
                for (int kb = kb0; kb < kb1; ++kb) {
                    const int s = fs;
                    const uint32_t ph = fph;
                    if (++fs == stages) {
                        fs = 0;
                        fph ^= 1u;
                    }
                    if (!mbar_wait(bar_part + 8 * s, ph, wc)) { ok = false; break; }
                    fence_proxy_async_smem();  // cp.async writes -> bulk-copy reads
                    const uint32_t ps = sbase + s * L.stage_bytes;
                    for (int q = 1; q < G; ++q) {
                        uint32_t d = grank + (uint32_t)q;  // the other CTAs, without division
                        if (d >= (uint32_t)G) d -= (uint32_t)G;
                        bulk_copy_to_cluster(dsmem_map(ps + first_off, d), ps + first_off, part,
                                             dsmem_map(bar_full + 8 * s, d));
                    }
                    mbar_arrive(bar_full + 8 * s);
                }
            }
        }
    } else if (warp < kEpiWarp0 + 4) {
        // ---------------------------------------------------------- epilogue
        pdl_wait();
        const int quarter = warp & 3;               // TMEM lanes 32*quarter .. +31
        const int row = quarter * 32 + lane;         // row inside the tile
        const EpiParams e = p.epi;  // a local copy: its fields stay in registers
        int local = 0;
        uint32_t nblk = 0;  // tensor-store blocks this warp has issued
        if (kSplit && p.split_k > 1 && e.beta != 0.f && !e.ci_multi && blockIdx.x < p.num_units) {
            // the rows this CTA will reduce (cluster reduction), or a 1/split
            // share of the tile it adds into (reduce-add): pull their C lines
            // into L2 while the main loops run, so that the epilogue's reads
            // or adds find them there
            const TileCoord tc = unit_coord(blockIdx.x, p);
            const int S = p.split_k, rank = p.red_add ? tc.split : (int)cluster_ctarank();
            const int r0 = rank * kBM / S, rs = (rank + 1) * kBM / S - r0;
            const int ces = elem_bytes(e.c_dtype);
            const int t = threadIdx.x - kEpiWarp0 * 32;
            const int i0 = tc.ti * kBM + r0, jt = tc.tj * p.bn;
            const int ni = min(rs, p.Mi - i0), nj = min(p.bn, p.Nj - jt);
            if (ni > 0 && nj > 0) {
                // every 128-byte line a run touches: offsets 0, 128, ... clamped
                // to the run's last byte (never past the run)
                if (e.ci == ces) {  // a run of ni elements per column
                    const int len = ni * ces, per = (len + 127) / 128 + 1;
                    for (int q = t; q < nj * per; q += 128) {
                        const int c = q / per, l = q % per;
                        prefetch_l2(e.c + (int64_t)i0 * e.ci + (int64_t)(jt + c) * e.cj + min(l * 128, len - 1));
                    }
                } else if (e.cj == ces) {  // a run of nj elements per row
                    const int len = nj * ces, per = (len + 127) / 128 + 1;
                    for (int q = t; q < ni * per; q += 128) {
                        const int r = q / per, l = q % per;
                        prefetch_l2(e.c + (int64_t)(i0 + r) * e.ci + (int64_t)jt * e.cj + min(l * 128, len - 1));
                    }
                }
            }
        }
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

            if (kSplit && p.split_k > 1) {
                // one unit per CTA: the partial stays in TMEM until the cluster
                // has finished its main loops (see the reduction below)
                tc_fence_before();
                if (threadIdx.x == kEpiWarp0 * 32) trace_at(p, 53);
                continue;
            }

            if (p.epi_tma) {
                const uint32_t blocks = sbase + L.epi_off + (uint32_t)quarter * 2u * kEpiBlockBytes;
                const int i_base = tc.ti * kBM + quarter * 32;
                // one tile per CTA with a gather: the gather warps share the strip
                const int step = helpers ? 3 : 1;
                __syncwarp();
                if (e.c_dtype == DG_F32)
                    epilogue_rows_tma<4>(e, &tmap_c, blocks, t_row, i_base, p.Mi, j0, p.bn, p.Nj, lane, nblk, 0, step);
                else
                    epilogue_rows_tma<2>(e, &tmap_c, blocks, t_row, i_base, p.Mi, j0, p.bn, p.Nj, lane, nblk, 0, step);
            } else {
                // with helpers the gather warps take two of every three chunks
                epilogue_rows_thread(e, t_row, i, p.Mi, j0, p.bn, p.Nj, 0, helpers ? 48 : 16);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_tempty + 8 * b);
            if (local == 0 && threadIdx.x == kEpiWarp0 * 32) trace_at(p, 35);
        }
        // the tensor stores read this warp's blocks and write C after the loop
        if (p.epi_tma && lane == 0) bulk_wait_read<0>();  // writes land before the grid completes
    } else if (GATHER) {
        // ------------------------------------------------ gather producers
        const int gtid = threadIdx.x - (kEpiWarp0 + 4) * 32;
        switch (p.gather_vec * es) {
        case 16: gather_role<16>(p, L, sbase, bar_full, bar_empty, bar_part, g_row_off, abort_flag, wc, bk, es, gtid, lane); break;
        case 8: gather_role<8>(p, L, sbase, bar_full, bar_empty, bar_part, g_row_off, abort_flag, wc, bk, es, gtid, lane); break;
        case 4: gather_role<4>(p, L, sbase, bar_full, bar_empty, bar_part, g_row_off, abort_flag, wc, bk, es, gtid, lane); break;
        case 2: gather_role<2>(p, L, sbase, bar_full, bar_empty, bar_part, g_row_off, abort_flag, wc, bk, es, gtid, lane); break;
        default: gather_role<1>(p, L, sbase, bar_full, bar_empty, bar_part, g_row_off, abort_flag, wc, bk, es, gtid, lane); break;
        }
        if (helpers) {
            // ------------------------------ gather warps as epilogue helpers
            // One tile per CTA: once its accumulator is ready, the operand ring
            // is idle, so each gather warp takes a third of the column blocks
            // of its TMEM lane quarter, staging its tensor stores in the ring
            // (or a third of the 16-column chunks, stored by its threads).
            const int hw = warp - (kEpiWarp0 + 4);  // 0..7
            const int quarter = warp & 3;
            const EpiParams e = p.epi;  // a local copy: its fields stay in registers
            uint32_t nblk = 0;
            // the ring is idle once every CTA that reads or writes it is done
            // with its last use of each stage: the empty barriers count every
            // MMA of a gather cluster, whose completion also means this CTA's
            // parts have reached the other CTAs
            bool ready = true;
            const int kbn = p.kb_total;
            for (int it = kbn > p.stages ? kbn - p.stages : 0; it < kbn && ready; ++it)
                ready = mbar_wait(bar_empty + 8 * (it % p.stages), (uint32_t)(it / p.stages) & 1u, wc);
            if (ready && mbar_wait(bar_tfull, 0u, wc)) {
                tc_fence_after();
                const TileCoord tc = unit_coord(blockIdx.x, p);
                const uint32_t blocks = sbase + (uint32_t)hw * 2u * kEpiBlockBytes;
                const uint32_t t_row = tmem_base + ((uint32_t)(quarter * 32) << 16);
                const int i_base = tc.ti * kBM + quarter * 32, j0 = tc.tj * p.bn;
                __syncwarp();
                if (!p.epi_tma)
                    epilogue_rows_thread(e, t_row, i_base + lane, p.Mi, j0, p.bn, p.Nj, 16 * (1 + hw / 4), 48);
                else if (e.c_dtype == DG_F32)
                    epilogue_rows_tma<4>(e, &tmap_c, blocks, t_row, i_base, p.Mi, j0, p.bn, p.Nj, lane, nblk,
                                         1 + hw / 4, 3);
                else
                    epilogue_rows_tma<2>(e, &tmap_c, blocks, t_row, i_base, p.Mi, j0, p.bn, p.Nj, lane, nblk,
                                         1 + hw / 4, 3);
                tc_fence_before();
            }
            if (p.epi_tma && lane == 0) bulk_wait_read<0>();  // writes land before the grid completes
        }
    }

    if (kSplit && p.split_k > 1 && p.red_add) {
        // ------------------------------------- split-K partials added into C
        // beta = 1 and FP32 C: C += alpha * s_i * s_j * partial (+ bias, by the
        // first split only) is linear in the splits, so each CTA adds its own
        // scaled partial into C with tensor reduce-adds, which the memory
        // system applies element by element.  No slices travel between the
        // CTAs and no CTA waits for another; the order of the adds, and so the
        // last bits of C, can vary from run to run.  The blocks are staged in
        // the idle operand ring: 32 x 32 FP32, laid out along C's unit-stride
        // dim (i: rows of 32 i, no swizzle; j: rows of 32 j, 128-byte swizzle).
        __syncwarp();
        if (!cluster_ready) {
            cluster_wait();  // the start-up barrier every thread arrived on
            cluster_ready = true;
        }
        if (warp >= kEpiWarp0 && warp < kEpiWarp0 + 4 && !*abort_flag) {
            tc_fence_after();
            const int quarter = warp & 3;
            const EpiParams e = p.epi;  // a local copy: its fields stay in registers
            const TileCoord tc = unit_coord(blockIdx.x, p);
            const int i_base = tc.ti * kBM + quarter * 32, i = i_base + lane;
            const int j0 = tc.tj * p.bn, Nj = p.Nj;
            const bool row_ok = i < p.Mi;
            const float asi = row_ok ? e.alpha * (e.scale_i ? e.scale_i[i] : 1.f) : 0.f;
            const bool first = tc.split == 0;  // the bias enters C once
            const float *const bias_j = first ? e.bias_j : nullptr;
            const float bi = (first && e.bias_i && row_ok) ? e.bias_i[i] : 0.f;
            const float *const scale_j = e.scale_j;
            const uint32_t t_row = tmem_base + ((uint32_t)(quarter * 32) << 16);
            const uint32_t blocks = sbase + (uint32_t)quarter * 2u * kEpiBlockBytes;
            const bool inner_i = p.red_inner_i != 0;
            uint32_t nblk = 0;
            for (int c0 = 0; c0 < p.bn && j0 + c0 < Nj; c0 += 32) {
                uint32_t r[32];
                tmem_ld16(t_row + (uint32_t)c0, *reinterpret_cast<uint32_t(*)[16]>(&r[0]));
                tmem_ld16(t_row + (uint32_t)(c0 + 16), *reinterpret_cast<uint32_t(*)[16]>(&r[16]));
                tmem_ld_wait();
                float v[32];
#pragma unroll
                for (int c = 0; c < 32; ++c) {
                    const int j = min(j0 + c0 + c, Nj - 1);  // columns past C are clipped by the copy
                    float x = (asi * (scale_j ? scale_j[j] : 1.f)) * __uint_as_float(r[c]);
                    if (bias_j) x += bias_j[j];
                    v[c] = x + bi;
                }
                const uint32_t buf = blocks + (nblk & 1u) * kEpiBlockBytes;
                if (lane == 0) bulk_wait_read<1>();  // the copy that last read this block is done with it
                __syncwarp();
                if (inner_i) {
#pragma unroll
                    for (int c = 0; c < 32; ++c) st_shared_f32(buf + (uint32_t)c * 128u + (uint32_t)lane * 4u, v[c]);
                } else {
                    const uint32_t rowa = buf + (uint32_t)lane * 128u;
#pragma unroll
                    for (int u = 0; u < 8; ++u)
                        st_shared_v4(rowa + ((uint32_t)(u ^ (lane & 7)) << 4), __float_as_uint(v[4 * u]),
                                     __float_as_uint(v[4 * u + 1]), __float_as_uint(v[4 * u + 2]),
                                     __float_as_uint(v[4 * u + 3]));
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    if (inner_i) tma_reduce_add_2d(&tmap_c, buf, i_base, j0 + c0);
                    else tma_reduce_add_2d(&tmap_c, buf, j0 + c0, i_base);
                    bulk_commit();
                }
                ++nblk;
            }
            if (lane == 0) bulk_wait_read<0>();  // the adds land before the grid completes
        }
    } else if (kSplit && p.split_k > 1) {
        // ------------------------------------------ cluster reduction of k splits
        // CTA s of the cluster owns rows [128 s / S, 128 (s+1) / S) of the
        // tile.  Once its own main loop is done (its ring is then idle), each
        // CTA writes its partial from TMEM into its ring as S slices, slice d
        // holding the rows CTA d owns (column-major), and one thread copies
        // every other slice into its owner's receive region with a bulk
        // shared-memory copy that completes on the owner's receive barrier.
        // An owner adds the S slices of its rows in rank order (its own slice
        // stays local), so the sum is deterministic, and runs the epilogue.  A
        // cluster barrier, arrived at once a CTA has received everything and
        // waited on before exit, keeps every CTA alive until all copies out of
        // its shared memory have landed.
        const int S = p.split_k;
        const int rs_max = (kBM + S - 1) / S;
        const uint32_t slice = split_slice_bytes(p.bn, S);
        const uint32_t out_slices = sbase;
        const uint32_t in_slices = sbase + L.recv_off;
        const uint32_t rank = cluster_ctarank();
        const bool epi_warp = warp >= kEpiWarp0 && warp < kEpiWarp0 + 4;
        if (threadIdx.x == kEpiWarp0 * 32) trace_at(p, 54);
        // cluster barrier operations are issued by whole, converged warps
        __syncwarp();
        if (!cluster_ready) {
            cluster_wait();  // every CTA of the cluster is initialised
            cluster_ready = true;
        }
        if (!epi_warp) cluster_arrive_relaxed();  // nothing to receive here
        if (epi_warp) {
            tc_fence_after();
            const int quarter = warp & 3;
            const int row = quarter * 32 + lane;
            int d;  // owner of this row
            if (kBM % S == 0) {
                d = row / (kBM / S);
            } else {
                d = 0;
                while (d + 1 < S && (d + 1) * kBM / S <= row) ++d;
            }
            const int rl = row - d * kBM / S;
            const uint32_t dst = out_slices + (uint32_t)d * slice + (uint32_t)rl * 4u;
            const uint32_t col_pitch = (uint32_t)rs_max * 4u;
            const uint32_t t_row = tmem_base + ((uint32_t)(quarter * 32) << 16);
            for (int c0 = 0; c0 < p.bn; c0 += 16) {
                uint32_t r[16];
                __syncwarp();
                tmem_ld16(t_row + c0, r);
                tmem_ld_wait();
#pragma unroll
                for (int c = 0; c < 16; ++c) st_shared_f32(dst + (uint32_t)(c0 + c) * col_pitch, __uint_as_float(r[c]));
            }
            if (threadIdx.x == kEpiWarp0 * 32) trace_at(p, 57);
            fence_proxy_async_smem();  // the slices are read by the bulk copies
            asm volatile("bar.sync 2, 128;" ::: "memory");
            // (test hook, stall mode 2: no slice is sent, so every owner's
            // receive wait runs out and reports the timeout)
            if (threadIdx.x == kEpiWarp0 * 32 && !*abort_flag && p.stall_loader != 2) {
                trace_at(p, 58);
                for (int q = 1; q < S; ++q) {
                    const uint32_t dr = (rank + (uint32_t)q) % (uint32_t)S;
                    bulk_copy_to_cluster(dsmem_map(in_slices + rank * slice, dr), out_slices + dr * slice, slice,
                                         dsmem_map(bar_recv, dr));
                }
                trace_at(p, 59);
            }
            // the owner's rows: everything below except the slice sums needs
            // nothing from the other CTAs
            const EpiParams e = p.epi;  // a local copy: its fields stay in registers
            const TileCoord tc = unit_coord(blockIdx.x, p);
            const int r0 = (int)(rank * kBM / S), r1 = (int)((rank + 1) * kBM / S), rs = r1 - r0;
            const int t = threadIdx.x - kEpiWarp0 * 32;
            const int bn = p.bn, Mi = p.Mi, Nj = p.Nj;
            const int i0 = tc.ti * kBM + r0, jt = tc.tj * bn;
            const float alpha = e.alpha, beta = e.beta;
            const float *const scale_i = e.scale_i, *const scale_j = e.scale_j;
            const float *const bias_i = e.bias_i, *const bias_j = e.bias_j;
            const int act = e.act;
            const bool fused = bias_i != nullptr || bias_j != nullptr || act != DG_ACT_NONE;
            char *const cbase = e.c;
            const int64_t ci = e.ci, cj = e.cj;
            const bool ci_multi = e.ci_multi != 0;
            const int cdt = e.c_dtype;
            const bool vec4 = cdt == DG_F32 && !ci_multi && ci == 4 && rs_max % 4 == 0 && rs % 4 == 0 &&
                              i0 % 4 == 0 && cj % 16 == 0 && (reinterpret_cast<uintptr_t>(cbase) & 15) == 0;
            constexpr int kB4 = 4;  // four-row groups per thread per batch (vector path)
            const int g_rows = vec4 ? rs / 4 : 1;
            // vector path: the four outputs (i .. i+3, j) of a group are
            // mul[k] * sum + beta * C + add[k]: mul = alpha * s_i * s_j, add = the
            // bias.  Their factors are loaded with the group's C, before any
            // store (a load after a store through C's pointer would wait for it).
            auto load_factors = [&](int i, int j, float (&mul)[4], float (&add)[4]) {
                const float sj = scale_j ? scale_j[j] : 1.f;
                const float bj = (fused && bias_j) ? bias_j[j] : 0.f;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const bool in = i + k < Mi;
                    mul[k] = alpha * (scale_i && in ? scale_i[i + k] : 1.f) * sj;
                    add[k] = ((fused && bias_i && in) ? bias_i[i + k] : 0.f) + bj;
                }
            };
            // vector path: C of the first batch is loaded while the slices travel
            float4 cfirst[kB4];
#pragma unroll
            for (int b = 0; b < kB4; ++b) cfirst[b] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (vec4 && beta != 0.f) {
#pragma unroll
                for (int b = 0; b < kB4; ++b) {
                    const int g = t + b * 128;
                    const int i = i0 + (g % g_rows) * 4, j = jt + g / g_rows;
                    if (g < g_rows * bn && j < Nj && i + 3 < Mi)
                        cfirst[b] = *reinterpret_cast<const float4 *>(cbase + (int64_t)i * 4 + (int64_t)j * cj);
                }
            }
            const bool received = mbar_wait(bar_recv, 0, wc);
            __syncwarp();
            // barrier 2: every copy into this CTA has landed (seen on bar_recv;
            // the arrival needs to order nothing else)
            cluster_arrive_relaxed();
            if (threadIdx.x == kEpiWarp0 * 32) trace_at(p, 55);
            if (received) {
                // slice of source q: local for this CTA's own rank
                uint32_t src[kMaxSplit];
#pragma unroll
                for (int q = 0; q < kMaxSplit; ++q)
                    src[q] = q == (int)rank ? out_slices + rank * slice : in_slices + (uint32_t)q * slice;
                if (vec4) {
                    // four consecutive rows (contiguous in C and in a slice) per
                    // thread and step; consecutive threads take consecutive rows
                    const int total = g_rows * bn;
                    constexpr int kB = kB4;
                    // group g = t + 128 n: row group g % g_rows, column g / g_rows,
                    // advanced without division
                    const int dgr = 128 % g_rows, dgc = 128 / g_rows;
                    int gr = t % g_rows, gc = t / g_rows;
                    for (int base = t; base < total; base += 128 * kB) {
                        float4 cin[kB], acc[kB];
                        float mul[kB][4], add[kB][4];
                        int rr[kB], cc[kB];
#pragma unroll
                        for (int b = 0; b < kB; ++b) {
                            const int g = base + b * 128;
                            const int r = gr * 4, c = gc;
                            rr[b] = r;
                            cc[b] = c;
                            gr += dgr;
                            gc += dgc;
                            if (gr >= g_rows) {
                                gr -= g_rows;
                                ++gc;
                            }
                            const int i = i0 + r, j = jt + c;
                            acc[b] = make_float4(0.f, 0.f, 0.f, 0.f);
                            cin[b] = acc[b];
#pragma unroll
                            for (int k = 0; k < 4; ++k) mul[b][k] = add[b][k] = 0.f;
                            if (g < total && j < Nj && i < Mi) load_factors(i, j, mul[b], add[b]);
                            if (g < total && j < Nj && i + 3 < Mi) {
                                if (beta != 0.f)
                                    cin[b] = base == t ? cfirst[b]
                                                       : *reinterpret_cast<const float4 *>(cbase + (int64_t)i * 4 +
                                                                                          (int64_t)j * cj);
                                const uint32_t off = (uint32_t)(c * rs_max + r) * 4u;
#pragma unroll
                                for (int q = 0; q < kMaxSplit; ++q) {
                                    if (q < S) {
                                        const float4 v = ld_shared_v4(src[q] + off);
                                        acc[b].x += v.x;
                                        acc[b].y += v.y;
                                        acc[b].z += v.z;
                                        acc[b].w += v.w;
                                    }
                                }
                            }
                        }
                        // the activation is picked once per batch: this code runs once per
                        // CTA, so its instruction footprint, more than its arithmetic, sets
                        // its time (C is FP32 here: the accurate tanh)
                        auto finish = [&](auto act_c) {
                            constexpr int kAct = decltype(act_c)::value;
#pragma unroll
                        for (int b = 0; b < kB; ++b) {
                            const int g = base + b * 128;
                            const int r = rr[b], c = cc[b];
                            const int i = i0 + r, j = jt + c;
                            if (!(g < total && j < Nj && i < Mi)) continue;
                            const float a4[4] = {acc[b].x, acc[b].y, acc[b].z, acc[b].w};
                            const float c4[4] = {cin[b].x, cin[b].y, cin[b].z, cin[b].w};
                            float o[4];
#pragma unroll
                            for (int k = 0; k < 4; ++k) {
                                o[k] = mul[b][k] * a4[k];
                                if (beta != 0.f) o[k] = fmaf(beta, c4[k], o[k]);
                                if (fused) o[k] = act_fn<kAct, false>(o[k] + add[b][k]);
                            }
                            char *dstc = cbase + (int64_t)i * 4 + (int64_t)j * cj;
                            if (i + 3 < Mi) {
                                *reinterpret_cast<float4 *>(dstc) = make_float4(o[0], o[1], o[2], o[3]);
                            } else {
                                // rows past C: element by element (loads too)
#pragma unroll
                                for (int k = 0; k < 4; ++k) {
                                    if (i + k >= Mi) break;
                                    float a = 0.f;
                                    const uint32_t off = (uint32_t)(c * rs_max + r + k) * 4u;
#pragma unroll
                                    for (int q = 0; q < kMaxSplit; ++q)
                                        if (q < S) a += ld_shared_f32(src[q] + off);
                                    float val = mul[b][k] * a;
                                    if (beta != 0.f) val = fmaf(beta, load_elem(dstc + k * 4, cdt), val);
                                    if (fused) val = act_fn<kAct, false>(val + add[b][k]);
                                    store_elem(dstc + k * 4, cdt, val);
                                }
                            }
                        }
                        };
                        if (act == DG_ACT_RELU) finish(std::integral_constant<int, DG_ACT_RELU>{});
                        else if (act == DG_ACT_GELU_TANH) finish(std::integral_constant<int, DG_ACT_GELU_TANH>{});
                        else finish(std::integral_constant<int, DG_ACT_NONE>{});
                    }
                } else {
                    // any C layout: element by element; consecutive threads take
                    // consecutive addresses along C's contiguous dim
                    const bool along_i = (ci == (int64_t)elem_bytes(cdt));
                    const int total = rs * bn;
                    int r = along_i ? t % rs : t / bn, c = along_i ? t / rs : t % bn;
                    const int dr = along_i ? 128 % rs : 128 / bn, dc = along_i ? 128 / rs : 128 % bn;
                    constexpr int kB = 8;  // outputs per thread per batch: their loads are in flight together
                    for (int base = t; base < total; base += 128 * kB) {
                        int ii[kB], jj[kB];
                        float acc[kB], cin[kB], sc[kB], bs[kB];
#pragma unroll
                        for (int b = 0; b < kB; ++b) {
                            const int i = i0 + r, j = jt + c;
                            const bool ok = base + b * 128 < total && i < Mi && j < Nj;
                            ii[b] = ok ? i : -1;
                            jj[b] = j;
                            float a = 0.f;
                            if (ok) {
                                const uint32_t off = (uint32_t)(c * rs_max + r) * 4u;
#pragma unroll
                                for (int q = 0; q < kMaxSplit; ++q)
                                    if (q < S) a += ld_shared_f32(src[q] + off);
                            }
                            acc[b] = a;
                            const int64_t ro = ci_multi ? epi_row_offset(e, ok ? i : 0) : (int64_t)i * ci;
                            cin[b] = (ok && beta != 0.f) ? load_elem(cbase + ro + (int64_t)j * cj, cdt) : 0.f;
                            // scales and bias loaded with the batch, before any store
                            sc[b] = ok ? alpha * (scale_i ? scale_i[i] : 1.f) * (scale_j ? scale_j[j] : 1.f) : 0.f;
                            bs[b] = ok ? (bias_i ? bias_i[i] : 0.f) + (bias_j ? bias_j[j] : 0.f) : 0.f;
                            // advance by 128 elements
                            if (along_i) {
                                r += dr;
                                c += dc;
                                if (r >= rs) { r -= rs; ++c; }
                            } else {
                                c += dc;
                                r += dr;
                                if (c >= bn) { c -= bn; ++r; }
                            }
                        }
                        // the activation and C's type are picked once per batch (a smaller
                        // instruction footprint for this once-per-CTA code; C is never E4M3)
                        auto finish = [&](auto act_c, auto cd_c) {
                            constexpr int kAct = decltype(act_c)::value, kCd = decltype(cd_c)::value;
#pragma unroll
                            for (int b = 0; b < kB; ++b) {
                                if (ii[b] < 0) continue;
                                const int i = ii[b], j = jj[b];
                                float val = sc[b] * acc[b];
                                if (beta != 0.f) val = fmaf(beta, cin[b], val);
                                if (fused) {
                                    if (bias_i || bias_j) val += bs[b];
                                    val = act_fn<kAct, kCd != DG_F32>(val);
                                }
                                const int64_t ro = ci_multi ? epi_row_offset(e, i) : (int64_t)i * ci;
                                st_out<kCd>(cbase + ro + (int64_t)j * cj, val);
                            }
                        };
                        auto finish_act = [&](auto act_c) {
                            if (cdt == DG_F32) finish(act_c, std::integral_constant<int, DG_F32>{});
                            else if (cdt == DG_BF16) finish(act_c, std::integral_constant<int, DG_BF16>{});
                            else finish(act_c, std::integral_constant<int, DG_F16>{});
                        };
                        if (act == DG_ACT_RELU) finish_act(std::integral_constant<int, DG_ACT_RELU>{});
                        else if (act == DG_ACT_GELU_TANH) finish_act(std::integral_constant<int, DG_ACT_GELU_TANH>{});
                        else finish_act(std::integral_constant<int, DG_ACT_NONE>{});
                    }
                }
            }
        }
        if (threadIdx.x == kEpiWarp0 * 32) trace_at(p, 56);
        __syncwarp();
        cluster_wait();  // barrier 2
    }

    // --------------------------------------------------------------- teardown
    if (threadIdx.x == 0) trace_at(p, 36);
    tc_fence_before();
    __syncthreads();
    // a gather cluster's CTAs copy into each other's shared memory: none leaves first
    if (G > 1) {
        __syncwarp();
        if (!cluster_ready) cluster_wait();  // warp-uniform: warp 1 waited at its start
        cluster_sync();
    }
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem_base, (uint32_t)p.tmem_cols);
    }
}

}  // namespace

}  // namespace dg
