// Paired-CTA tensor-core GEMM for sm_100a: tcgen05.mma.cta_group::2.
//
// Two CTAs of a cluster compute one 256 x bn tile of D = P Q together.  Each
// CTA loads its own 128 rows of P and its own half (bn/2 columns) of Q into
// its shared memory, holds its 128 x bn half of the accumulator in its TMEM,
// and runs its own epilogue; the even CTA of the pair issues the MMAs for
// both.  Against one CTA per 128 x bn tile this halves each SM's share of the
// Q tile: 32 KB instead of 48 KB of operands per 64-deep k step at bn = 256,
// so more stages fit in shared memory and less L2 bandwidth is needed per
// flop ("DeepGEMM deep dive", §2.1-§2.3: blocking for reuse, and overlapping
// loads with compute, taken to the pair of SMs that Blackwell's tensor core
// can drive as one).
//
// Barriers: full[s] lives in the even CTA and counts the copy bytes of both
// CTAs (each CTA's TMA loads signal it across the pair); empty[s] and the
// accumulator-ready barriers exist in both CTAs and are signalled by one
// multicast tcgen05.commit; accumulator-drained barriers live in the even CTA
// and collect the epilogue warps of both.  Every wait is bounded as in the
// single-CTA kernel.  Loads use no cluster multicast.
#include <atomic>

#include "common.cuh"
#include "sm100.cuh"
#include "umma_common.cuh"

namespace dg {

namespace {

constexpr int kHalfM = 128;   // rows of P (and TMEM lanes) per CTA
constexpr int kRowBytes = 128;

// A stage holds ksub k sub-blocks of 128 bytes per row (ksub = 1 or 2).  Its
// P part (128 rows) and Q part (bn/2 columns) are each laid out as whole
// 128-byte-swizzled boxes: K-major, one box of 128 rows (P) or bn/2 rows in
// boxes of bn/4 (Q) per sub-block, the sub-blocks one after the other;
// MN-major, one box of ksub * bk rows of k per 128-byte column group, the
// groups one after the other.  A deeper stage loads the same bytes in half as
// many boxes when Q is MN-major (the copy engine has a fixed cost per box).
struct PairLayout {
    uint32_t a_sub, b_sub;  // bytes of one k sub-block of P and of Q
    uint32_t a_bytes, b_bytes, stage_bytes, epi_off, bar_off, aux_off, total;
};

__host__ __device__ inline PairLayout pair_layout(int bn, int stages, bool epi_tma, int ksub) {
    PairLayout L;
    L.a_sub = kHalfM * kRowBytes;
    L.b_sub = (uint32_t)(bn / 2) * kRowBytes;
    L.a_bytes = (uint32_t)ksub * L.a_sub;
    L.b_bytes = (uint32_t)ksub * L.b_sub;
    L.stage_bytes = L.a_bytes + L.b_bytes;  // a multiple of 1024: bn is a multiple of 16
    L.epi_off = L.stage_bytes * stages;
    L.bar_off = L.epi_off + (epi_tma ? kEpiStoreBytes : 0u);
    // full[S], empty[S], tfull[2], tempty[2], drain
    L.aux_off = L.bar_off + 8 * (2 * stages + 5);
    L.total = L.aux_off + 16 + 1024;
    return L;
}

// Unit u of the pair schedule: whole tiles first (column-major), then each
// tile of the last, partial wave as two half-width units, so that the last
// wave takes half as long.
struct PairUnit {
    int ti, j0, w;  // tile row, first column, columns
};

__device__ __forceinline__ PairUnit pair_unit(int u, const UmmaParams &p) {
    PairUnit r;
    int t = u, half = -1;
    if (u >= p.full_units) {
        t = p.full_units + (u - p.full_units) / 2;
        half = (u - p.full_units) & 1;
    }
    r.ti = t % p.tiles_i;
    const int tj = t / p.tiles_i;
    r.w = half < 0 ? p.bn : p.bn / 2;
    r.j0 = tj * p.bn + (half > 0 ? p.bn / 2 : 0);
    return r;
}

// One unit of a pair's schedule: a tile (or half of one) and a range of its
// k blocks, with what the epilogue does with the accumulator.
enum : int {
    kWhole = 0,      // the whole k range: store C
    kSkPartial = 1,  // Stream-K, a range that ends inside the tile: leave the partial in this pair's slot
    kSkOwner = 2     // Stream-K, the range that ends the tile: add the other pairs' partials, store C
};
struct PairWork {
    int ti, j0, w;   // tile row, first column, columns
    int kb0, kb1;    // k blocks [kb0, kb1)
    int role;
    int sk_first;    // kSkOwner: the tile's first k block in the Stream-K run
};

// Pair c's share [lo, hi) of the Stream-K run of `total` k blocks.
__device__ __forceinline__ void sk_range(int64_t total, int c, int P, int64_t &lo, int64_t &hi) {
    lo = total * c / P;
    hi = total * (c + 1) / P;
}

// Unit idx of pair c of P (false past its last unit).  Without Stream-K:
// pair_unit's whole and half tiles.  With it: first the Stream-K units (the
// range that ends inside a tile, whose partial other pairs wait for, then
// the ranges that end tiles this pair owns), then the whole tiles
// c, c + P, ... below dp_tiles.  A tile's owner holds its last k blocks and
// so has the highest pair index of the tile: owners wait only on pairs with
// lower indices, which are launched no later than they are.
__device__ __forceinline__ bool pair_work(const UmmaParams &p, int c, int P, int idx, PairWork &w) {
    const int KB = p.kb_total;
    if (p.sk_tiles == 0) {
        const int u = c + idx * P;
        if (u >= p.num_units) return false;
        const PairUnit pu = pair_unit(u, p);
        w.ti = pu.ti;
        w.j0 = pu.j0;
        w.w = pu.w;
        w.kb0 = 0;
        w.kb1 = KB;
        w.role = kWhole;
        w.sk_first = 0;
        return true;
    }
    int64_t lo, hi;
    sk_range((int64_t)p.sk_tiles * KB, c, P, lo, hi);
    const int64_t ta = lo / KB, tb = hi / KB;
    const bool partial = hi > lo && hi % KB != 0;
    const int n_sk = hi > lo ? (int)(tb - ta) + (partial ? 1 : 0) : 0;
    int t;
    if (idx < n_sk) {
        int64_t ts, k0, k1;
        if (partial && idx == 0) {
            ts = tb;
            k0 = lo > tb * KB ? lo : tb * KB;
            k1 = hi;
            w.role = kSkPartial;
        } else {
            ts = ta + idx - (partial ? 1 : 0);
            k0 = lo > ts * KB ? lo : ts * KB;
            k1 = (ts + 1) * KB;
            w.role = kSkOwner;
        }
        w.kb0 = (int)(k0 - ts * KB);
        w.kb1 = (int)(k1 - ts * KB);
        w.sk_first = (int)(ts * KB);
        t = p.dp_tiles + (int)ts;
    } else {
        t = c + (idx - n_sk) * P;
        if (t >= p.dp_tiles) return false;
        w.kb0 = 0;
        w.kb1 = KB;
        w.role = kWhole;
        w.sk_first = 0;
    }
    w.ti = t % p.tiles_i;
    w.j0 = (t / p.tiles_i) * p.bn;
    w.w = p.bn;
    return true;
}

// The pairs whose partials the owner c of the Stream-K tile starting at k
// block `first` adds: q in [q0, c) with a non-empty range (every such range
// ends inside the tile).
__device__ __forceinline__ int sk_first_contributor(const UmmaParams &p, int c, int P, int first) {
    const int64_t total = (int64_t)p.sk_tiles * p.kb_total;
    int64_t lo, hi;
    sk_range(total, c, P, lo, hi);
    if (lo <= first) return c;  // this pair starts the tile: nothing to add
    int q = c;
    while (q > 0) {
        --q;
        if (total * q / P <= first) break;
    }
    return q;
}

// This CTA's slot of pair q: 128 rows x bn FP32 in groups of four columns,
// element (row, col) at [(col / 4) * 128 + row] * 4 + col % 4, so that a
// warp's 16-byte stores and loads of one column group are 512 contiguous bytes.
__device__ __forceinline__ float *sk_slot(const UmmaParams &p, int q, uint32_t rank) {
    return p.sk_part + (size_t)(q * 2 + (int)rank) * (size_t)(kHalfM * p.bn);
}

template <bool FP8, int KSUB>
__global__ void __launch_bounds__(192, 1)
    umma_pair_kernel(const __grid_constant__ CUtensorMap tmap_p, const __grid_constant__ CUtensorMap tmap_q,
                     const __grid_constant__ CUtensorMap tmap_c, const UmmaParams p) {
    if (threadIdx.x == 64) {
        // descriptor fetches start at once, while thread 0 sets up the barriers
        tma_prefetch_desc(&tmap_p);
        tma_prefetch_desc(&tmap_q);
        if (p.epi_tma) tma_prefetch_desc(&tmap_c);
    }
    if (p.pdl == 1) pdl_release();
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const PairLayout L = pair_layout(p.bn, p.stages, p.epi_tma != 0, KSUB);
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar_full = sbase + L.bar_off;
    const uint32_t bar_empty = bar_full + 8 * p.stages;
    const uint32_t bar_tfull = bar_empty + 8 * p.stages;
    const uint32_t bar_tempty = bar_tfull + 16;
    const uint32_t bar_drain = bar_tempty + 16;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L.aux_off);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L.aux_off + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int cluster_id = blockIdx.x >> 1, nclusters = gridDim.x >> 1;
    const WaitCtl wc{abort_flag, p.err_word, p.timeout_ns};

    if (threadIdx.x == 0) {
        for (int s = 0; s < p.stages; ++s) {
            mbar_init(bar_full + 8 * s, 1);
            mbar_init(bar_empty + 8 * s, 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar_tfull + 8 * b, 1);
            mbar_init(bar_tempty + 8 * b, 8);  // four epilogue warps in each CTA of the pair
        }
        mbar_init(bar_drain, 1);
        *abort_flag = 0;
        fence_barrier_init();
        fence_proxy_async_smem();
    }
    if (warp == 1) {
        tmem_alloc_pair(smem_u32(tmem_slot), (uint32_t)p.tmem_cols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();  // both CTAs' barriers exist before either signals the other's
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    // The set-up above touches only the pair's shared memory and TMEM, so it
    // runs while the previous kernel finishes; every global access below
    // waits for that kernel (programmatic dependent launch).
    pdl_wait();

    // Stream-K: the tag of this launch's partials is one more than the
    // sequence number the previous launch left (it completed before this
    // launch passed its dependency wait), so flags of earlier launches, or of
    // a launch that gave up on a wait, never match
    const uint32_t sk_tag = p.sk_tiles > 0 ? ld_acquire_gpu(p.sk_hdr) + 1u : 0u;
    const int es = FP8 ? 1 : 2;
    const int bk = p.bk;
    const int half_bn = p.bn / 2;
    constexpr int kUmmaK = FP8 ? 32 : 16;
    const int per = 128 / es;  // MN elements per 128-byte row of an MN-major box

    if (warp == 0) {
        // ------------------------------------------------ TMA producer (both CTAs)
        if (lane == 0) {
            // everything the loop needs in registers: the asynchronous copies
            // (memory clobbers) would otherwise make it re-read the parameters,
            // and stage and phase advance without division
            const int stages = p.stages, kb_total = p.kb_total, num_units = p.num_units;
            const bool stall = p.stall_loader == 1, p_mn = p.p_mn_major != 0, q_mn = p.q_mn_major != 0;
            const uint32_t stage_bytes = L.stage_bytes, a_bytes = L.a_bytes, a_sub = L.a_sub, b_sub = L.b_sub;
            constexpr int ksub = KSUB;
            const uint32_t mn_box_bytes = (uint32_t)(ksub * bk) * kRowBytes;  // an MN-major box: ksub * bk rows
            (void)num_units;
            (void)kb_total;
            int it = 0, s = 0;
            uint32_t ph = 0;
            PairWork pw;
            for (int idx = 0; !*abort_flag && pair_work(p, cluster_id, nclusters, idx, pw); ++idx) {
                const int i0 = pw.ti * 2 * kHalfM + (int)rank * kHalfM;
                const int cw = pw.w / 2;  // this CTA's columns of the unit
                const int j0 = pw.j0 + (int)rank * cw;
                // both CTAs' bytes: MN-major Q in boxes of 128-byte column groups (cw
                // columns), K-major Q in one box of the CTA's bn/2 rows per sub-block,
                // for a half-width unit too (its second half is loaded and not used)
                const uint32_t qrows = q_mn ? (uint32_t)cw : (uint32_t)half_bn;
                const uint32_t tx = 2u * (a_bytes + (uint32_t)ksub * qrows * kRowBytes);
                bool ok = true;
                for (int kb = pw.kb0; kb < pw.kb1; ++kb, ++it) {
                    if (!mbar_wait(bar_empty + 8 * s, ph ^ 1u, wc)) { ok = false; break; }
                    if (!stall) {
                        const uint32_t full_c = dsmem_map(bar_full + 8 * s, 0);
                        if (leader) mbar_arrive_expect_tx(bar_full + 8 * s, tx);
                        const uint32_t as = sbase + s * stage_bytes;
                        const uint32_t bs = as + a_bytes;
                        const int k0 = kb * ksub * bk;
                        if (p_mn) {
                            for (int c = 0; c < kHalfM / per; ++c)
                                tma_load_2d_pair(as + c * mn_box_bytes, &tmap_p, full_c, i0 + c * per, k0);
                        } else {
                            for (int j = 0; j < ksub; ++j)
                                tma_load_2d_pair(as + j * a_sub, &tmap_p, full_c, k0 + j * bk, i0);
                        }
                        if (q_mn) {
                            for (int c = 0; c < cw / per; ++c)
                                tma_load_2d_pair(bs + c * mn_box_bytes, &tmap_q, full_c, j0 + c * per, k0);
                        } else {
                            // one box of bn/2 rows per sub-block (a box's fixed cost is paid
                            // once); a half-width unit's CTA uses the first bn/4 of them
                            for (int j = 0; j < ksub; ++j)
                                tma_load_2d_pair(bs + j * b_sub, &tmap_q, full_c, k0 + j * bk, j0);
                        }
                    }
                    if (++s == stages) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                if (!ok) break;
            }
            if (!leader) pdl_release();
            // full[] of the even CTA counts both CTAs' bytes: once its last
            // phases complete, every copy of the pair has landed
            if (leader && p.stall_loader != 1)
                for (int d = 1; d <= p.stages && it - d >= 0; ++d) {
                    const int j = it - d;
                    mbar_wait_drain(bar_full + 8 * (j % p.stages), (uint32_t)(j / p.stages) & 1u, p.timeout_ns);
                }
        }
    } else if (warp == 1) {
        // ----------------------------------------- MMA issuer (even CTA only)
        if (lane == 0 && leader) {
            const int stages = p.stages, kb_total = p.kb_total, num_units = p.num_units;
            const int full_units = p.full_units, bn = p.bn;
            const uint32_t idesc_full = p.idesc, idesc_half = p.idesc_half, stage_bytes = L.stage_bytes;
            constexpr int ksub = KSUB;
            // MN-major: the next 128-byte column group is one box (ksub * bk rows) further, and
            // k advances by rows of the box; K-major: k advances within the 128-byte rows of a
            // sub-block, and the next sub-block follows the previous one
            const uint32_t p_lbo = p.p_mn_major ? (uint32_t)(ksub * bk * 128) : 16u;
            const uint32_t q_lbo = p.q_mn_major ? (uint32_t)(ksub * bk * 128) : 16u;
            const uint32_t p_kstep = p.p_mn_major ? kUmmaK * 128 : kUmmaK * es;
            const uint32_t q_kstep = p.q_mn_major ? kUmmaK * 128 : kUmmaK * es;
            const uint32_t p_sstep = p.p_mn_major ? (uint32_t)(kRowBytes / (kUmmaK * es)) * p_kstep : L.a_sub;
            const uint32_t q_sstep = p.q_mn_major ? (uint32_t)(kRowBytes / (kUmmaK * es)) * q_kstep : L.b_sub;
            // descriptors of stage 0; a stage's differ only in the start address
            // field (address >> 4, below 2^14 for any shared-memory address)
            const uint64_t da0 = make_sw128_desc(sbase, p_lbo, 1024);
            const uint64_t db0 = make_sw128_desc(sbase + L.a_bytes, q_lbo, 1024);
            (void)num_units;
            (void)kb_total;
            (void)full_units;
            int local = 0, s = 0;
            uint32_t ph = 0;
            bool ok = true;
            PairWork pw;
            for (int idx = 0; ok && pair_work(p, cluster_id, nclusters, idx, pw); ++idx, ++local) {
                const uint32_t idesc = pw.w == bn ? idesc_full : idesc_half;
                const int b = local & 1;
                const uint32_t tph = (uint32_t)(local >> 1) & 1u;
                if (!mbar_wait(bar_tempty + 8 * b, tph ^ 1u, wc)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(b * bn);
                const int kb0 = pw.kb0;
                for (int kb = kb0; kb < pw.kb1; ++kb) {
                    if (!mbar_wait(bar_full + 8 * s, ph, wc)) { ok = false; break; }
                    tc_fence_after();
                    const uint64_t soff = (uint64_t)((s * stage_bytes) >> 4);
#pragma unroll
                    for (int sub = 0; sub < ksub; ++sub) {
                        const uint64_t sa = soff + (uint64_t)((sub * p_sstep) >> 4);
                        const uint64_t sb = soff + (uint64_t)((sub * q_sstep) >> 4);
#pragma unroll
                        for (int kk = 0; kk < kRowBytes / (kUmmaK * es); ++kk) {
                            const uint64_t da = da0 + sa + (uint64_t)((kk * p_kstep) >> 4);
                            const uint64_t db = db0 + sb + (uint64_t)((kk * q_kstep) >> 4);
                            const uint32_t acc = (kb > kb0 || sub > 0 || kk > 0) ? 1u : 0u;
                            if (FP8) umma_f8_pair(d_tmem, da, db, idesc, acc);
                            else umma_f16_pair(d_tmem, da, db, idesc, acc);
                        }
                    }
                    tc_commit_pair_mc(bar_empty + 8 * s, 0x3);  // the stage is free in both CTAs
                    if (++s == stages) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                if (!ok) break;
                tc_commit_pair_mc(bar_tfull + 8 * b, 0x3);       // both halves of the accumulator are ready
            }
            pdl_release();
            tc_commit_pair_mc(bar_drain, 0x1);
            mbar_wait_drain(bar_drain, 0, p.timeout_ns);
        }
    } else {
        // ------------------------------------------- epilogue (both CTAs)
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;
        const EpiParams e = p.epi;  // a local copy: its fields stay in registers
        int local = 0;
        uint32_t nblk = 0;  // tensor-store blocks this warp has issued
        PairWork pw;
        for (int idx = 0; pair_work(p, cluster_id, nclusters, idx, pw); ++idx, ++local) {
            const int b = local & 1;
            const uint32_t tph = (uint32_t)(local >> 1) & 1u;
            if (!mbar_wait(bar_tfull + 8 * b, tph, wc)) break;
            tc_fence_after();
            const int i = pw.ti * 2 * kHalfM + (int)rank * kHalfM + row;
            const uint32_t t_row = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(b * p.bn);
            const int j0 = pw.j0;
            if (pw.role == kSkPartial) {
                // ------------------------- Stream-K: leave the partial for the tile's owner
                float4 *slot = reinterpret_cast<float4 *>(sk_slot(p, cluster_id, rank)) + row;
                for (int c0 = 0; c0 < pw.w; c0 += 16) {
                    uint32_t r[16];
                    __syncwarp();
                    tmem_ld16(t_row + c0, r);
                    tmem_ld_wait();
#pragma unroll
                    for (int g = 0; g < 4; ++g)  // column group (c0 + 4g) / 4
                        slot[((c0 >> 2) + g) * kHalfM] =
                            make_float4(__uint_as_float(r[4 * g]), __uint_as_float(r[4 * g + 1]),
                                        __uint_as_float(r[4 * g + 2]), __uint_as_float(r[4 * g + 3]));
                }
                tc_fence_before();
                __syncwarp();  // orders the warp's stores before lane 0's release below
                if (lane == 0) {
                    mbar_arrive_cluster(dsmem_map(bar_tempty + 8 * b, 0));
                    // one flag per warp (32 rows): the owner's warp of the same quarter waits on it
                    st_release_gpu(p.sk_flag + (cluster_id * 2 + (int)rank) * 4 + quarter, sk_tag);
                }
                continue;
            }
            if (pw.role == kSkOwner) {
                // ------------------------- Stream-K: add the other pairs' partials into TMEM
                // Wait (bounded) for each lower pair's flag of this warp's rows, then
                // add its partial to the accumulator in place (tcgen05.ld, add,
                // tcgen05.st), in pair order q = c-1, c-2, ...; the epilogue below
                // then reads the finished sum like any other tile.
                const int q0 = sk_first_contributor(p, cluster_id, nclusters, pw.sk_first);
                const int64_t total = (int64_t)p.sk_tiles * p.kb_total;
                bool ok = true;
                for (int q = cluster_id - 1; q >= q0 && ok; --q) {
                    if (total * q / nclusters == total * (q + 1) / nclusters) continue;  // empty range: no partial
                    const uint32_t *flag = p.sk_flag + (q * 2 + (int)rank) * 4 + quarter;
                    if (ld_acquire_gpu(flag) != sk_tag) {
                        const uint64_t t0 = globaltimer_ns();
                        while (ld_acquire_gpu(flag) != sk_tag) {
                            if (*abort_flag || globaltimer_ns() - t0 > p.timeout_ns) {
                                ok = false;
                                break;
                            }
                        }
                        if (!ok) {
                            *abort_flag = 1;
                            if (p.err_word) atomicExch(p.err_word, kErrTimeout);
                            break;
                        }
                    }
                    // 64 columns at a time: their 16 loads are in flight together, so the
                    // partial costs a few round trips to L2, not one per 16 columns
                    const float4 *src = reinterpret_cast<const float4 *>(sk_slot(p, q, rank)) + row;
                    for (int c0 = 0; c0 < pw.w; c0 += 64) {
                        float4 pv[16];
#pragma unroll
                        for (int g = 0; g < 16; ++g) pv[g] = src[((c0 >> 2) + g) * kHalfM];
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            uint32_t r[16];
                            __syncwarp();
                            tmem_ld16(t_row + c0 + 16 * k, r);
                            tmem_ld_wait();
#pragma unroll
                            for (int g = 0; g < 4; ++g) {
                                const float4 a = pv[4 * k + g];
                                r[4 * g] = __float_as_uint(__uint_as_float(r[4 * g]) + a.x);
                                r[4 * g + 1] = __float_as_uint(__uint_as_float(r[4 * g + 1]) + a.y);
                                r[4 * g + 2] = __float_as_uint(__uint_as_float(r[4 * g + 2]) + a.z);
                                r[4 * g + 3] = __float_as_uint(__uint_as_float(r[4 * g + 3]) + a.w);
                            }
                            tmem_st16(t_row + c0 + 16 * k, r);
                        }
                    }
                    tmem_st_wait();
                }
            }
            if (p.epi_tma) {
                const uint32_t blocks = sbase + L.epi_off + (uint32_t)quarter * 2u * kEpiBlockBytes;
                const int i_base = i - lane;
                __syncwarp();
                if (e.c_dtype == DG_F32)
                    epilogue_rows_tma<4>(e, &tmap_c, blocks, t_row, i_base, p.Mi, j0, pw.w, p.Nj, lane, nblk);
                else
                    epilogue_rows_tma<2>(e, &tmap_c, blocks, t_row, i_base, p.Mi, j0, pw.w, p.Nj, lane, nblk);
            } else {
                epilogue_rows_thread(e, t_row, i, p.Mi, j0, pw.w, p.Nj);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(dsmem_map(bar_tempty + 8 * b, 0));
        }
        // the tensor stores read this warp's blocks and write C after the loop
        if (p.epi_tma && lane == 0) bulk_wait_read<0>();  // writes land before the grid completes
    }

    // --------------------------------------------------------------- teardown
    tc_fence_before();
    __syncthreads();
    cluster_sync();  // neither CTA frees TMEM or exits while the pair still uses it
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, (uint32_t)p.tmem_cols);
    }
    if (p.sk_tiles > 0 && threadIdx.x == 0) {
        // the last CTA out publishes this launch's tag as the sequence number
        __threadfence();
        if (atomicAdd(p.sk_hdr + 1, 1u) == gridDim.x - 1) {
            p.sk_hdr[1] = 0;
            __threadfence();
            st_release_gpu(p.sk_hdr, sk_tag);
        }
    }
}

}  // namespace

size_t umma_pair_smem_bytes(int bn, int stages, bool epi_tma, int ksub) {
    return pair_layout(bn, stages, epi_tma, ksub).total;
}

int umma_pair_max_stages(int bn, bool epi_tma, int ksub) {
    int s = 2;
    while (s < 12 && pair_layout(bn, s + 1, epi_tma, ksub).total <= 227 * 1024) ++s;
    return s;
}

cudaError_t launch_umma_pair(const UmmaParams &p, const CUtensorMap *tp, const CUtensorMap *tq,
                             const CUtensorMap *tc, bool fp8, int grid, size_t smem, cudaStream_t s) {
    void (*kern)(const CUtensorMap, const CUtensorMap, const CUtensorMap, const UmmaParams);
    if (p.ksub != 1 && p.ksub != 2) return cudaErrorInvalidValue;
    const bool deep = p.ksub == 2;
    kern = fp8 ? (deep ? umma_pair_kernel<true, 2> : umma_pair_kernel<true, 1>)
               : (deep ? umma_pair_kernel<false, 2> : umma_pair_kernel<false, 1>);
    static SmemLimit s_limit[4];
    const cudaError_t e = s_limit[(fp8 ? 2 : 0) + (deep ? 1 : 0)].ensure(kern, smem);
    if (e != cudaSuccess) return e;
    return launch_ex(kern, dim3(grid), dim3(192), smem, s, dim3(2, 1, 1), p.pdl, *tp, *tq, *tc, p);
}

}  // namespace dg
