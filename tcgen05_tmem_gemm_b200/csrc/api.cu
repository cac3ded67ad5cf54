// C-ABI entry points of libdg: argument validation, the view-analysis
// dispatcher, per-device state and the launches.
//
// Dispatch ("DeepGEMM: a recalibration of the compute paradigm", §2.2: view
// analysis picks the tiling from the contiguous segments; "DeepGEMM deep
// dive", §4.1: compare the arithmetic intensity with the machine balance):
//   M == 0 or N == 0         -> nothing
//   alpha == 0 or K == 0     -> C = beta * C
//   M <= 8, W unit-stride    -> GEMV (HBM-bound: 2 flops per weight byte pair)
//   16-bit / E4M3 operands   -> tcgen05 tensor-core kernel; operands TMA can
//                               describe are loaded by TMA, one that it cannot
//                               (non-16-byte strides) by thread gathers; thin
//                               M (<= 64) swaps A and B so N fills the
//                               128-row tensor-core tile; few tiles -> split-K
//   anything else            -> CUDA-core tiled kernel
#include <atomic>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <vector>

#include <cudaTypedefs.h>

#include "dg_internal.h"

namespace dg {
namespace {

std::atomic<uint64_t> g_launches{0};
std::atomic<int> g_force_kind{0};
std::atomic<int64_t> g_timeout_ms{2000};
std::atomic<int> g_stall{0};
std::atomic<int> g_max_split{8};
std::atomic<int> g_pair{1};
std::atomic<int> g_pdl{3};
std::atomic<uint64_t> g_trace{0};
std::atomic<int> g_epi_tma{1};
std::atomic<int> g_gather_cluster{1};
std::atomic<int> g_pair_tail{1};
std::atomic<int> g_pair_deep{1};  // CTA-pair stages two k sub-blocks deep where they apply
std::atomic<int> g_stream_k{0};
std::atomic<int> g_deterministic{0};
std::atomic<uint32_t> g_epoch{1};  // bumped by every option change: cached launches go stale

constexpr int kMaxDevices = 64;
constexpr int kMaxCluster = 8;    // portable thread-block cluster size: the most k splits

// Stream-K workspace of one stream: partial accumulators, flags and the
// sequence header (see UmmaParams).  Kernels of one stream run one after the
// other, so a stream's launches can share it; launches on different streams
// may overlap and get their own.
struct SkWorkspace {
    cudaStream_t stream = nullptr;
    void *ptr = nullptr;
    size_t bytes = 0;
};
constexpr int kMaxSkStreams = 16;  // further streams run without Stream-K
constexpr size_t kSkHeaderBytes = 256;

struct DeviceState {
    bool ready = false;
    int num_sms = 0;
    int *err_word = nullptr;       // device: DG_ERR_TIMEOUT when a bounded wait gave up
    SkWorkspace sk[kMaxSkStreams];
    int n_sk = 0;
};

std::mutex g_mu;
DeviceState g_dev[kMaxDevices];
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

dg_status device_state(DeviceState **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return DG_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_mu);
    DeviceState &d = g_dev[dev];
    if (!d.ready) {
        if (cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return DG_ERR_CUDA;
        // a word allocated by an earlier attempt whose later steps failed is reused, not leaked
        if (!d.err_word && cudaMalloc(&d.err_word, sizeof(int)) != cudaSuccess) {
            d.err_word = nullptr;
            return DG_ERR_CUDA;
        }
        if (cudaMemset(d.err_word, 0, sizeof(int)) != cudaSuccess) return DG_ERR_CUDA;
        if (cudaDeviceSynchronize() != cudaSuccess) return DG_ERR_CUDA;
        if (!g_encode) {
            cudaDriverEntryPointQueryResult q;
            void *fn = nullptr;
            if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q) !=
                    cudaSuccess ||
                q != cudaDriverEntryPointSuccess || !fn)
                return DG_ERR_CUDA;
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
        }
        d.ready = true;
    }
    *out = &d;
    return DG_OK;
}

// Bytes of a Stream-K workspace for `pairs` CTA pairs and tiles bn wide: the
// header, one flag per (pair, CTA, epilogue warp), one 128 x bn FP32 slot per
// (pair, CTA).
size_t sk_workspace_bytes(int pairs, int bn, size_t *flag_off, size_t *part_off) {
    const size_t flags = ((size_t)pairs * 2 * 4 * sizeof(uint32_t) + 255) / 256 * 256;
    *flag_off = kSkHeaderBytes;
    *part_off = kSkHeaderBytes + flags;
    return *part_off + (size_t)pairs * 2 * 128 * (size_t)bn * sizeof(float);
}

// The Stream-K workspace of `stream` on this device, at least `need` bytes,
// or null when none can be had now: the stream is being captured into a
// graph (nothing is allocated then; calls run without Stream-K until a call
// outside the capture has allocated it) or every slot is taken.  A new or
// larger workspace is allocated with its header and flags zeroed on the
// stream; a smaller one it replaces is freed after the stream has drained,
// and cached launches that pointed at it are invalidated.
void *sk_workspace(DeviceState *ds, cudaStream_t stream, size_t need, size_t zero_bytes) {
    std::lock_guard<std::mutex> lk(g_mu);
    SkWorkspace *w = nullptr;
    for (int i = 0; i < ds->n_sk; ++i)
        if (ds->sk[i].stream == stream) w = &ds->sk[i];
    if (w && w->bytes >= need) return w->ptr;
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(stream, &cap) != cudaSuccess) {
        cudaGetLastError();
        return nullptr;
    }
    if (cap != cudaStreamCaptureStatusNone) return nullptr;
    if (!w) {
        if (ds->n_sk == kMaxSkStreams) return nullptr;
        w = &ds->sk[ds->n_sk++];
        w->stream = stream;
    } else {
        if (cudaStreamSynchronize(stream) != cudaSuccess || cudaFree(w->ptr) != cudaSuccess) {
            cudaGetLastError();
            w->ptr = nullptr;
            w->bytes = 0;
            return nullptr;
        }
        w->ptr = nullptr;
        w->bytes = 0;
        g_epoch.fetch_add(1);  // cached launches held the old pointer
    }
    void *ptr = nullptr;
    if (cudaMalloc(&ptr, need) != cudaSuccess) {
        cudaGetLastError();
        return nullptr;
    }
    if (cudaMemsetAsync(ptr, 0, zero_bytes, stream) != cudaSuccess) {
        cudaGetLastError();
        cudaFree(ptr);
        return nullptr;
    }
    w->ptr = ptr;
    w->bytes = need;
    return ptr;
}

bool device_accessible_uncached(const void *p) {
    if (!p) return false;
    cudaPointerAttributes a;
    if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    if (a.type == cudaMemoryTypeManaged) return true;
    if (a.type != cudaMemoryTypeDevice) return false;
    int dev = -1;
    cudaGetDevice(&dev);
    return a.device == dev;
}

// Recently validated device pointers (per host thread and device), so that a
// caller reusing its buffers does not pay cudaPointerGetAttributes each call.
struct PtrCache {
    int dev = -1;
    const void *ptr[16] = {};
    int next = 0;
    bool has(int d, const void *p) const {
        if (d != dev) return false;
        for (const void *q : ptr)
            if (q == p) return true;
        return false;
    }
    void add(int d, const void *p) {
        if (d != dev) {
            dev = d;
            for (auto &q : ptr) q = nullptr;
        }
        ptr[next] = p;
        next = (next + 1) % 16;
    }
};
thread_local PtrCache t_ptrs;

bool device_accessible(const void *p) {
    if (!p) return false;
    int cur = -1;
    cudaGetDevice(&cur);
    if (t_ptrs.has(cur, p)) return true;
    const bool ok = device_accessible_uncached(p);
    if (ok) t_ptrs.add(cur, p);
    return ok;
}

DevView dev_view(const dg_view *v, const ViewInfo &vi) {
    DevView d{};
    d.ptr = static_cast<const char *>(v->ptr);
    d.row = vi.row;
    d.col = vi.col;
    d.dtype = v->dtype;
    return d;
}

// stride of a group with at most one merged dim (0 when the group is empty)
int64_t axis_stride(const Axis &a) { return a.n == 1 ? a.stride[0] : 0; }

struct Plan {
    dg_plan_info info{};
    // UMMA specifics
    bool fp8 = false;
    size_t smem = 0;
};

struct Views {
    const dg_view *A, *B, *C;
    ViewInfo a, b, c;
    int act = DG_ACT_NONE;  // the call's activation: split-K partials add into C only without one
};

uint32_t make_idesc(int in_dtype, bool p_mn, bool q_mn, int bn, int m = 128) {
    uint32_t d = 0;
    d |= 1u << 4;                                    // D format: F32
    const uint32_t fmt = (in_dtype == DG_BF16) ? 1u : 0u;  // F16 = 0, BF16 = 1; E4M3 = 0 (kind::f8f6f4)
    d |= fmt << 7;                                   // A format
    d |= fmt << 10;                                  // B format
    d |= (p_mn ? 1u : 0u) << 15;                     // A major (1 = MN)
    d |= (q_mn ? 1u : 0u) << 16;                     // B major
    d |= (uint32_t)(bn >> 3) << 17;                  // N >> 3
    d |= (uint32_t)(m >> 4) << 24;                   // M >> 4 (256 for a CTA pair)
    return d;
}

bool gemv_applicable(const Views &v, int64_t M, int64_t N, int64_t K, int kind) {
    const int dt = v.A->dtype;
    if (dt != DG_F16 && dt != DG_BF16) return false;
    if (M > 8 || K > INT32_MAX || N > INT32_MAX) return false;
    if (v.c.row.n > 1 || v.c.col.n > 1) return false;
    const uintptr_t wp = reinterpret_cast<uintptr_t>(v.B->ptr);
    if (wp % 16) return false;
    const int64_t r_inst = M <= 1 ? 1 : M <= 2 ? 2 : M <= 4 ? 4 : 8;
    if (kind == DG_KIND_GEMV_N) {
        // B: columns one unit-stride dim, rows one dim with a 16-byte multiple
        // stride (a TMA map); each block's slice of x fits in shared memory
        if (!(v.b.col.n == 1 && v.b.col.stride[0] == 2 && v.b.row.n <= 1)) return false;
        if (N % 8) return false;
        if (v.b.row.n == 1 && v.b.row.stride[0] % 16) return false;
        if ((K + kMaxCluster - 1) / kMaxCluster * r_inst > 16384) return false;
        return true;
    }
    if (kind == DG_KIND_GEMV_K) {
        if (!(v.b.row.n == 1 && v.b.row.stride[0] == 2 && v.b.col.n <= 1)) return false;
        if (K % 8) return false;
        if (v.b.col.n == 1 && v.b.col.stride[0] % 16) return false;
        if (K * r_inst > 32768) return false;   // all of x staged in shared memory
        return true;
    }
    return false;
}

// A plan variant: each field replaces the dispatcher's rule for one choice
// (0 or -1: keep the rule).  dg_autotune times the variants a call admits
// and keeps the fastest per shape key; a variant the operands do not admit
// makes the planner fail, and the autotuner skips it.
struct Override {
    int bn = 0;          // tensor-core tile width
    int split = 0;       // tensor-core k splits (1 = none)
    int pair = -1;       // CTA pairs: 0 / 1
    int sk = -1;         // Stream-K tail of a CTA-pair schedule: 0 / 1
    int gcl = 0;         // gather-cluster size: 1, 2 or 4
    int epi_tma = -1;    // tensor-store epilogue: 0 / 1
    int stages = 0;      // pipeline depth (at most what shared memory holds)
    int gemv_split = 0;  // GEMV_N k splits
    int ksub = 0;        // CTA-pair stage depth in 128-byte k sub-blocks: 1 or 2
    bool any() const {
        return bn || split || pair >= 0 || sk >= 0 || gcl || epi_tma >= 0 || stages || gemv_split || ksub;
    }
};

// GEMV_N grid: 256-column strips times k splits (one cluster per strip, at
// most 8), about two blocks per SM, k ranges in whole 64-row TMA stages (so
// one split's last stage never reads the next split's rows) and each block's
// slice of x within 64 KB of shared memory.
bool gemv_n_split(int64_t M, int64_t N, int64_t K, int num_sms, dg_plan_info *in, int force_s = 0) {
    const int64_t r_inst = M <= 1 ? 1 : M <= 2 ? 2 : M <= 4 ? 4 : 8;
    const int64_t gx = (N + 255) / 256;
    int64_t S = (2 * num_sms + gx / 2) / gx;
    S = std::max<int64_t>(1, std::min<int64_t>(S, kMaxCluster));
    S = std::min<int64_t>(S, std::max<int64_t>(1, K / 64));
    if (force_s > 0) {
        if (force_s > kMaxCluster) return false;
        S = force_s;
    }
    int64_t kper = ((K + S - 1) / S + 63) / 64 * 64;
    while (kper * r_inst > 16384 && S < kMaxCluster) {
        if (force_s > 0) return false;
        ++S;
        kper = ((K + S - 1) / S + 63) / 64 * 64;
    }
    S = (K + kper - 1) / kper;
    if (force_s > 0 && S != force_s) return false;  // the k range does not split that many ways
    in->block_n = 256;
    in->block_k = (int32_t)kper;
    in->split_k = (int32_t)std::max<int64_t>(S, 1);
    in->grid = (int32_t)(gx * in->split_k);
    in->vec_bytes = 16;
    return true;
}

// Which UMMA configuration serves these views (false: none).
bool umma_plan(const Views &v, int64_t M, int64_t N, int64_t K, float beta, int num_sms, bool allow_sk, Plan *pl,
               const Override *ov = nullptr) {
    static const Override kNone;
    if (!ov) ov = &kNone;
    const int dt = v.A->dtype;
    if (dt != DG_F16 && dt != DG_BF16 && dt != DG_E4M3) return false;
    if (M > INT32_MAX || N > INT32_MAX || K > INT32_MAX) return false;
    const bool a_tma = v.a.tma_ok, b_tma = v.b.tma_ok;
    if (!a_tma && !b_tma) return false;
    const bool thin = (M <= 64 && N >= 2 * M);
    bool swap;
    if (!a_tma) swap = false;       // A is loaded by threads as the M-side operand
    else if (!b_tma) swap = true;   // B is, after the swap
    else swap = thin;
    // C: the epilogue addresses a row (i) through any number of merged dims,
    // computed once per row (a layout transform such as writing an NCHW
    // output from an [N*H*W, C] product), and walks j with one stride
    if ((swap ? v.c.row.n : v.c.col.n) > 1) return false;
    const ViewInfo &pvi = swap ? v.b : v.a;
    const bool p_tma = swap ? b_tma : a_tma;
    // unit-stride direction of P(i, k) and Q(k, j)
    // A: rows = i/m, cols = k.  B: rows = k, cols = j/n.
    bool p_mn, q_mn;
    if (!swap) {
        p_mn = (v.a.unit_dim == 2);
        q_mn = (v.b.unit_dim == 1);
    } else {
        p_mn = (v.b.unit_dim == 1);
        q_mn = (v.a.unit_dim == 2);
    }
    int gather_vec = 1;
    if (!p_tma) {
        // innermost unit-stride dim of the gathered operand decides its layout
        const Axis &ig = swap ? pvi.col : pvi.row;   // i group of P
        const Axis &kg = swap ? pvi.row : pvi.col;   // k group of P
        const int es = pvi.es;
        if (ig.n >= 1 && ig.stride[ig.n - 1] == es) p_mn = true;
        else if (kg.n >= 1 && kg.stride[kg.n - 1] == es) p_mn = false;
        else p_mn = false;
        gather_vec = pvi.vec_bytes / es;
        if (gather_vec < 1) gather_vec = 1;
        if (!(ig.n >= 1 && ig.stride[ig.n - 1] == es) && !(kg.n >= 1 && kg.stride[kg.n - 1] == es)) gather_vec = 1;
    }
    const int64_t Mi = swap ? N : M, Nj = swap ? M : N;
    const int es = elem_size(dt);
    const int bk = 128 / es;
    int bn;
    const int64_t tiles_i = (Mi + 127) / 128;
    const int64_t tiles_128 = tiles_i * ((Nj + 127) / 128), tiles_256 = tiles_i * ((Nj + 255) / 256);
    if (Nj <= 64 && !q_mn) {
        bn = (int)((Nj + 15) / 16) * 16;
    } else if (Nj >= 256 && (tiles_256 >= num_sms || tiles_128 > num_sms)) {
        // wide tiles when there are enough of them, or when they fit one wave
        // that narrower tiles would overflow
        bn = 256;
    } else if (Nj > 64) {
        bn = 128;
    } else {
        bn = 64;
    }
    if (q_mn) {
        const int per = 128 / es;  // MN elements per 128-byte box row
        bn = (int)(((bn + per - 1) / per) * per);
        if (bn > 256) return false;
    }
    if (g_pair.load() != 2 && !ov->bn) {
        // very few tiles: narrower ones put more SMs to work, each loading
        // less of Q and storing less of C (not when CTA pairs are forced:
        // they need tiles of 128 columns or more)
        const int bn_min = q_mn ? 128 / es : 32;
        while (bn / 2 >= bn_min && bn % 2 == 0 && tiles_i * ((Nj + bn / 2 - 1) / (bn / 2)) <= num_sms / 8)
            bn /= 2;
    }
    if (ov->bn) {
        bn = ov->bn;
        if (bn < 16 || bn > 256 || bn % 16 || (q_mn && bn % (128 / es))) return false;
    }
    const int64_t tiles_j = (Nj + bn - 1) / bn;
    const int64_t tiles = tiles_i * tiles_j;
    const int64_t kb_total = (K + bk - 1) / bk;
    int64_t split = 1;
    const int max_split = g_max_split.load();
    if (ov->split) {
        // every split is one CTA of a cluster and all of them resident at once
        split = ov->split;
        if (split > kMaxCluster || split > kb_total || (split > 1 && tiles * split > num_sms)) return false;
    } else if (tiles * 2 <= num_sms && kb_total >= 8 && max_split > 1) {
        // k splits of a tile form one cluster and reduce on chip
        split = std::min<int64_t>(num_sms / tiles, kb_total / 4);
        split = std::min<int64_t>(split, std::min(max_split, kMaxCluster));
        if (split < 1) split = 1;
    }
    int64_t kb_per = (kb_total + split - 1) / split;
    split = (kb_total + kb_per - 1) / kb_per;
    if (ov->split && split != ov->split) return false;  // k does not split that many ways
    const int64_t units = tiles * split;
    if (units > INT32_MAX) return false;
    // a CTA pair shares each 256 x bn tile when there are enough tiles to fill
    // the machine (or when forced); TMA operands only, no split
    const int pair_mode = g_pair.load();
    bool pair = false;
    bool pair_ok = false;  // the operands admit CTA pairs
    if (p_tma && split == 1 && bn >= 128 && num_sms >= 2) {
        const int per = 128 / es;
        // a CTA loads bn/2 columns of Q: whole 128-byte boxes (MN-major) or
        // two boxes of bn/4 rows (K-major)
        pair_ok = q_mn ? ((bn / 2) % per == 0) : ((bn / 4) % 8 == 0);
        if (pair_ok && pair_mode > 0) pair = (pair_mode == 2) || (Mi >= 256 && tiles >= num_sms);
    }
    if (ov->pair >= 0) {
        if (ov->pair && !pair_ok) return false;
        pair = ov->pair != 0;
    }
    // the epilogue stores C through tensor copies when C is row-major along j
    // with 16-byte aligned rows, is not read (beta == 0) and each tile is a
    // whole number of 128-byte blocks; split tiles use the cluster reduction
    const int ces = elem_size(v.C->dtype);
    const int blk = 128 / ces;  // columns per 128-byte block
    const bool epi_ok = !swap && split == 1 && beta == 0.f && v.c.tma_ok && v.c.unit_dim == 1 && bn % blk == 0 &&
                        Nj >= blk && Mi >= 32;
    bool epi_tma = g_epi_tma.load() != 0 && epi_ok;
    if (ov->epi_tma >= 0) {
        if (ov->epi_tma && !epi_ok) return false;
        epi_tma = ov->epi_tma != 0;
    }
    // CTA pairs: stages two 128-byte k sub-blocks deep when an operand is
    // MN-major (its copies come in half as many boxes, each twice as tall;
    // the copy engine has a fixed cost per box) and K is a whole number of
    // such stages; at least three of them must fit.  With B MN-major, a
    // 16-bit tile pair needs six boxes per two 128-byte k sub-blocks in
    // one-deep stages and four in two-deep ones, an E4M3 pair four and three
    // (4096^3 on B200: BF16 103.6 -> 96.4 us, E4M3 57.7 -> 56.8 us)
    const bool deep_ok = pair && (p_mn || q_mn) && K % (2 * bk) == 0 && umma_pair_max_stages(bn, epi_tma, 2) >= 3;
    int ksub = (deep_ok && g_pair_deep.load() != 0) ? 2 : 1;
    if (ov->ksub) {
        if (ov->ksub != 1 && (ov->ksub != 2 || !deep_ok)) return false;
        ksub = ov->ksub;
    }
    const int max_stages =
        pair ? umma_pair_max_stages(bn, epi_tma, ksub) : umma_max_stages(bn, !p_tma, epi_tma, (int)split);
    int stages = max_stages;
    if (ov->stages) {
        if (ov->stages < 2 || ov->stages > max_stages) return false;
        stages = ov->stages;
    }
    if (split > 1) {
        // the split-K reduction stages a CTA's partial in its operand ring
        const int64_t ring = (int64_t)stages * (128 * 128 + bn * 128);
        if (stages < 3 || (int64_t)umma_split_out_bytes(bn, (int)split) > ring) {
            if (ov->split > 1) return false;
            stages = umma_max_stages(bn, !p_tma, epi_tma, 1);
            split = 1;
            kb_per = kb_total;
        }
    }
    const int64_t units2 = tiles * split;
    // a gathered P tile is shared by the CTAs of its row of tiles: 2 or 4 of
    // them form a cluster and each gathers its share of every stage
    int gcl = 1;
    const bool gcl_ok = !p_tma && split == 1 && !pair && gather_vec * pvi.es >= 4;
    if (gcl_ok && g_gather_cluster.load() != 0) {
        for (int c : {4, 2})
            if (tiles_j % c == 0 && num_sms >= c) {
                gcl = c;
                break;
            }
    }
    if (ov->gcl) {
        if (ov->gcl != 1 && (!gcl_ok || (ov->gcl != 2 && ov->gcl != 4) || tiles_j % ov->gcl || num_sms < ov->gcl))
            return false;
        gcl = ov->gcl;
    }
    dg_plan_info &in = pl->info;
    in.kind = DG_KIND_UMMA;
    in.swap_ab = swap;
    in.p_gather = !p_tma;
    in.p_mn_major = p_mn;
    in.q_mn_major = q_mn;
    in.block_m = 128;
    in.block_n = bn;
    in.block_k = bk * ksub;  // k per stage
    in.stages = stages;
    in.split_k = (int32_t)split;
    in.grid = (int32_t)(split > 1 ? units2 : std::min<int64_t>(units2, num_sms));  // split: one unit per CTA
    in.vec_bytes = p_tma ? 16 : gather_vec * es;
    in.cta_pair = pair;
    in.epi_tma_store = epi_tma && split == 1;
    in.gather_cluster = gcl;
    if (gcl > 1) in.grid = (int32_t)std::min<int64_t>(units2, (num_sms / gcl) * gcl);
    // split-K with beta == 1 and FP32 C: the splits can add their partials
    // straight into C through one 2-D tensor map of C (its i group one dim)
    if (split > 1 && beta == 1.f && v.C->dtype == DG_F32 && v.c.tma_ok && g_deterministic.load() == 0 &&
        v.act == DG_ACT_NONE) {
        in.split_reduce_add = 1;
    }
    if (pair) {
        const int64_t pair_units = ((Mi + 255) / 256) * tiles_j;
        in.block_m = 256;
        const int64_t ncl = std::min<int64_t>(pair_units, num_sms / 2);
        in.grid = (int32_t)(2 * ncl);
        // the last, partial wave of tiles runs as half-width tiles (two per
        // tile), so it takes half as long; a CTA then loads bn/4 columns of Q
        const int per = 128 / es;
        const bool quarter_ok = q_mn ? ((bn / 4) % per == 0) : ((bn / 4) % 8 == 0);
        const int64_t tail = pair_units % ncl;
        // Stream-K: the tiles of the last, partial wave share their k blocks
        // out over every pair ("DeepGEMM deep dive", §5.2), when each of those
        // tiles is split among at most kMaxFix + 1 pairs and every pair gets
        // at least one k block
        const int64_t kb_all = tail * ((K + bk * ksub - 1) / (bk * ksub));  // stages of the tail's tiles
        const bool sk_ok = pair_units > ncl && tail > 0 && 7 * tail >= ncl && kb_all >= ncl;
        const bool sk = allow_sk && sk_ok && (ov->sk >= 0 ? ov->sk != 0 : g_stream_k.load() != 0);
        if (ov->sk == 1 && allow_sk && !sk_ok) return false;
        if (sk)
            in.stream_k_tiles = (int32_t)tail;
        else if (g_pair_tail.load() != 0 && quarter_ok && pair_units > ncl && tail > 0 && 2 * tail <= ncl)
            in.pair_half_tiles = (int32_t)tail;
    } else if (ov->sk == 1) {
        return false;
    }
    pl->fp8 = (dt == DG_E4M3);
    pl->smem = pair ? umma_pair_smem_bytes(bn, stages, epi_tma, ksub)
                    : umma_smem_bytes(bn, stages, !p_tma, epi_tma, in.split_reduce_add ? 1 : (int)split);
    return true;
}

// ---------------------------------------------------------------- autotune
// Tuned plan variants, keyed by everything a plan depends on except the
// addresses themselves: the three views with their pointers reduced to the
// 128-byte alignment class the planner looks at, beta == 0, alpha == 0, the
// device and its SM count.
struct TuneKey {
    dg_view A, B, C;
    int32_t beta_zero, alpha_zero, num_sms, dev;
};

TuneKey tune_key(const dg_view *A, const dg_view *B, const dg_view *C, float alpha, float beta, int num_sms) {
    TuneKey k;
    std::memset(&k, 0, sizeof(k));
    k.A = *A;
    k.B = *B;
    k.C = *C;
    for (dg_view *v : {&k.A, &k.B, &k.C}) v->ptr = reinterpret_cast<void *>(reinterpret_cast<uintptr_t>(v->ptr) & 127u);
    k.beta_zero = beta == 0.f;
    k.alpha_zero = alpha == 0.f;
    k.num_sms = num_sms;
    if (cudaGetDevice(&k.dev) != cudaSuccess) {
        cudaGetLastError();
        k.dev = -1;
    }
    return k;
}

struct TuneEntry {
    TuneKey key;
    Override ov;
};
std::mutex g_tune_mu;
std::vector<TuneEntry> g_tuned;

bool tuned_override(const TuneKey &k, Override *ov) {
    std::lock_guard<std::mutex> lk(g_tune_mu);
    for (const TuneEntry &e : g_tuned)
        if (std::memcmp(&e.key, &k, sizeof(k)) == 0) {
            *ov = e.ov;
            return true;
        }
    return false;
}

void store_tuned(const TuneKey &k, const Override &ov) {
    std::lock_guard<std::mutex> lk(g_tune_mu);
    for (TuneEntry &e : g_tuned)
        if (std::memcmp(&e.key, &k, sizeof(k)) == 0) {
            e.ov = ov;
            return;
        }
    g_tuned.push_back(TuneEntry{k, ov});
}

// `force`: plan with exactly this variant (an empty one: the rules, not the
// tuned table); null: the tuned variant for these views if there is one.
dg_status make_plan(Views &v, float alpha, float beta, int num_sms, Plan *pl, bool allow_sk = true,
                    const Override *force = nullptr) {
    (void)beta;
    dg_status st;
    if ((st = analyse(v.A, false, &v.a)) != DG_OK) return st;
    if ((st = analyse(v.B, false, &v.b)) != DG_OK) return st;
    if ((st = analyse(v.C, true, &v.c)) != DG_OK) return st;
    const int64_t M = v.a.rows, K = v.a.cols, N = v.b.cols;
    if (v.b.rows != K || v.c.rows != M || v.c.cols != N) return DG_ERR_SHAPE;
    if (v.A->dtype != v.B->dtype) return DG_ERR_DTYPE;
    if (v.C->dtype == DG_E4M3) return DG_ERR_DTYPE;
    if (!std::isfinite(alpha) || !std::isfinite(beta)) return DG_ERR_VALUE;
    dg_plan_info &in = pl->info;
    std::memset(&in, 0, sizeof(in));
    in.M = M;
    in.N = N;
    in.K = K;
    in.split_k = 1;
    if (M == 0 || N == 0) { in.kind = DG_KIND_NONE; return DG_OK; }
    if (alpha == 0.f || K == 0) { in.kind = DG_KIND_SCALE_C; return DG_OK; }
    Override tuned;
    const Override *ov = force;
    if (!ov && tuned_override(tune_key(v.A, v.B, v.C, alpha, beta, num_sms), &tuned)) ov = &tuned;
    const bool forced = force != nullptr && force->any();
    const int force_kind = g_force_kind.load();
    const bool simt_only = (v.A->dtype == DG_F32) || force_kind == DG_KIND_SIMT;
    if (!simt_only) {
        if (force_kind == DG_KIND_GEMV_N || force_kind == DG_KIND_GEMV_K) {
            if (gemv_applicable(v, M, N, K, force_kind)) {
                in.kind = force_kind;
                if (force_kind == DG_KIND_GEMV_N && !gemv_n_split(M, N, K, num_sms, &in, ov ? ov->gemv_split : 0)) {
                    if (forced) return DG_ERR_UNSUPPORTED;
                    gemv_n_split(M, N, K, num_sms, &in);
                }
                return DG_OK;
            }
        } else if (force_kind == DG_KIND_UMMA) {
            if (umma_plan(v, M, N, K, beta, num_sms, allow_sk, pl, ov)) return DG_OK;
            if (forced) return DG_ERR_UNSUPPORTED;
            if (ov && umma_plan(v, M, N, K, beta, num_sms, allow_sk, pl)) return DG_OK;
        } else {
            if (M <= 8) {
                if (gemv_applicable(v, M, N, K, DG_KIND_GEMV_N)) {
                    in.kind = DG_KIND_GEMV_N;
                    if (!gemv_n_split(M, N, K, num_sms, &in, ov ? ov->gemv_split : 0)) {
                        if (forced) return DG_ERR_UNSUPPORTED;
                        gemv_n_split(M, N, K, num_sms, &in);
                    }
                    return DG_OK;
                }
                if (gemv_applicable(v, M, N, K, DG_KIND_GEMV_K)) { in.kind = DG_KIND_GEMV_K; return DG_OK; }
            }
            if (umma_plan(v, M, N, K, beta, num_sms, allow_sk, pl, ov)) return DG_OK;
            if (forced) return DG_ERR_UNSUPPORTED;
            if (ov && umma_plan(v, M, N, K, beta, num_sms, allow_sk, pl)) return DG_OK;  // a stale variant
        }
    }
    if (M > int64_t(65535) * 64 || N > INT32_MAX || K > INT32_MAX) return DG_ERR_UNSUPPORTED;
    in.kind = DG_KIND_SIMT;
    in.block_m = 64;
    in.block_n = 64;
    in.block_k = 16;
    return DG_OK;
}

CUtensorMapDataType tma_dtype(int dt) {
    switch (dt) {
    case DG_F32: return CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
    case DG_F16: return CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    case DG_BF16: return CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    default: return CU_TENSOR_MAP_DATA_TYPE_UINT8;
    }
}

// 2-D tensor map: `inner` elements along the unit-stride dim, `outer` along
// the other (byte stride `outer_stride`), a box of box_inner x box_outer
// elements, zero fill out of bounds.  Encodings are cached per host thread:
// a caller that reuses its buffers does not re-encode.
struct MapKey {
    const void *ptr;
    int64_t inner, outer, stride;
    int dt, box_inner, box_outer, swizzle;
    bool operator==(const MapKey &o) const {
        return ptr == o.ptr && inner == o.inner && outer == o.outer && stride == o.stride && dt == o.dt &&
               box_inner == o.box_inner && box_outer == o.box_outer && swizzle == o.swizzle;
    }
};
struct MapCache {
    MapKey key[16];
    CUtensorMap map[16];
    bool used[16] = {};
    int next = 0;
};
thread_local MapCache t_maps;

bool encode_2d_box(CUtensorMap *m, int dt, const void *ptr, int64_t inner, int64_t outer, int64_t outer_stride,
                   int box_inner, int box_outer, bool swizzle128) {
    const int es = elem_size(dt);
    if (outer <= 1) outer_stride = ((inner * es + 15) / 16) * 16;  // any legal value
    if (outer_stride == 0) outer_stride = 16;
    const MapKey key{ptr, inner, outer, outer_stride, dt, box_inner, box_outer, swizzle128 ? 1 : 0};
    for (int i = 0; i < 16; ++i)
        if (t_maps.used[i] && t_maps.key[i] == key) {
            *m = t_maps.map[i];
            return true;
        }
    cuuint64_t gdim[2] = {(cuuint64_t)inner, (cuuint64_t)outer};
    cuuint64_t gstride[1] = {(cuuint64_t)outer_stride};
    cuuint32_t box[2] = {(cuuint32_t)box_inner, (cuuint32_t)box_outer};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = g_encode(m, tma_dtype(dt), 2, const_cast<void *>(ptr), gdim, gstride, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE,
                          swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return false;
    const int slot = t_maps.next;
    t_maps.key[slot] = key;
    t_maps.map[slot] = *m;
    t_maps.used[slot] = true;
    t_maps.next = (slot + 1) % 16;
    return true;
}

// Operand tiles for the tensor core: 128 bytes along the unit-stride dim,
// 128-byte swizzle.
bool encode_2d(CUtensorMap *m, int dt, const void *ptr, int64_t inner, int64_t outer, int64_t outer_stride,
               int box_outer) {
    return encode_2d_box(m, dt, ptr, inner, outer, outer_stride, 128 / elem_size(dt), box_outer, true);
}

EpiParams epi_params(const Views &v, bool swap, float alpha, float beta, const float *sa, const float *sb,
                     const float *bias, int act) {
    EpiParams e{};
    e.c = static_cast<char *>(v.C->ptr);
    const int64_t crs = axis_stride(v.c.row), ccs = axis_stride(v.c.col);
    e.ci = swap ? ccs : crs;
    e.cj = swap ? crs : ccs;
    e.c_dtype = v.C->dtype;
    const Axis &ia = swap ? v.c.col : v.c.row;
    e.ci_multi = ia.n > 1;
    e.ci_axis = ia;
    bool rows16 = true;  // every row starts 16-byte aligned
    for (int d = 0; d < ia.n; ++d) rows16 = rows16 && ia.stride[d] % 16 == 0;
    const int ces = elem_size(v.C->dtype);
    e.vec_ok = (e.cj == ces) && (reinterpret_cast<uintptr_t>(e.c) % 16 == 0) && rows16;
    e.alpha = alpha;
    e.beta = beta;
    e.scale_i = swap ? sb : sa;
    e.scale_j = swap ? sa : sb;
    // the bias belongs to the output column n: j, or i when the kernel computes C^T
    e.bias_i = swap ? bias : nullptr;
    e.bias_j = swap ? nullptr : bias;
    e.act = act;
    return e;
}

// Everything a launch needs, built once per distinct call: kernel
// parameters, tensor maps and the grid.
struct LaunchRec {
    int kind = DG_KIND_NONE;
    DevView c{};
    int64_t M = 0, N = 0;
    float beta = 0.f;
    const float *bias = nullptr;  // scale_c: the fused epilogue
    int act = DG_ACT_NONE;
    int pdl = 0;
    SimtParams simt{};
    GemvParams gemv{};
    UmmaParams umma{};
    CUtensorMap t0{}, t1{}, t2{};
    bool fp8 = false, gather = false, pair = false;
    int grid = 0;
    size_t smem = 0;
};

dg_status prepare(const Views &v, const Plan &pl, float alpha, float beta, const float *sa, const float *sb,
                  const float *bias, int act, DeviceState *ds, void *sk_ws, LaunchRec *rec) {
    const dg_plan_info &in = pl.info;
    rec->kind = in.kind;
    // early launch, mode 3: the launch-bound K-contiguous GEMV (64 blocks: the
    // next launch finds free SMs while it runs) and the tensor-core kernels
    // (released once their MMAs are issued; they wait before any memory access),
    // not the N-contiguous GEMV, whose blocks fill every SM's shared memory
    const int pdl_mode = g_pdl.load();
    rec->pdl = pdl_mode == 3 ? (in.kind == DG_KIND_GEMV_K ? 1 : in.kind == DG_KIND_UMMA ? 2 : 0) : pdl_mode;
    switch (in.kind) {
    case DG_KIND_NONE: return DG_OK;
    case DG_KIND_SCALE_C: {
        rec->c = dev_view(v.C, v.c);
        rec->M = in.M;
        rec->N = in.N;
        rec->beta = beta;
        rec->bias = bias;
        rec->act = act;
        break;
    }
    case DG_KIND_SIMT: {
        SimtParams p{};
        p.a = dev_view(v.A, v.a);
        p.b = dev_view(v.B, v.b);
        p.c = dev_view(v.C, v.c);
        p.M = (int32_t)in.M;
        p.N = (int32_t)in.N;
        p.K = (int32_t)in.K;
        p.epi = epi_params(v, false, alpha, beta, sa, sb, bias, act);
        p.pdl = rec->pdl;
        rec->simt = p;
        break;
    }
    case DG_KIND_GEMV_N:
    case DG_KIND_GEMV_K: {
        GemvParams p{};
        p.x = dev_view(v.A, v.a);
        p.w = static_cast<const char *>(v.B->ptr);
        p.w_ld = (in.kind == DG_KIND_GEMV_N) ? axis_stride(v.b.row) : axis_stride(v.b.col);
        p.R = (int32_t)in.M;
        p.K = (int32_t)in.K;
        p.N = (int32_t)in.N;
        p.in_dtype = v.A->dtype;
        p.epi = epi_params(v, false, alpha, beta, sa, sb, bias, act);
        p.err_word = ds->err_word;
        p.timeout_ns = (uint64_t)g_timeout_ms.load() * 1000000ull;
        p.pdl = rec->pdl;
        // x read with 16-byte loads when it is unit-stride along k
        const bool x_unit = v.a.col.n == 1 && v.a.col.stride[0] == 2 && v.A->dtype == v.B->dtype;
        p.x_ld = axis_stride(v.a.row);
        p.x_vec16 = x_unit && (in.K % 8 == 0) && (reinterpret_cast<uintptr_t>(v.A->ptr) % 16 == 0) &&
                    (v.a.row.n == 0 || p.x_ld % 16 == 0);
        if (in.kind == DG_KIND_GEMV_N) {
            p.kper = in.block_k;
            if (!encode_2d_box(&rec->t0, v.B->dtype, v.B->ptr, in.N, in.K, p.w_ld, 256, 64, false))
                return DG_ERR_UNSUPPORTED;
        }
        rec->gemv = p;
        break;
    }
    case DG_KIND_UMMA: {
        const bool swap = in.swap_ab != 0;
        const int dt = v.A->dtype;
        const int es = elem_size(dt);
        const int bk = 128 / es, bn = in.block_n;
        // a CTA-pair stage may be two 128-byte k sub-blocks deep (block_k = 2 * bk)
        const int ksub = in.cta_pair ? in.block_k / bk : 1;
        if (ksub < 1 || ksub > 2 || ksub * bk != in.block_k) return DG_ERR_UNSUPPORTED;
        const int mn_rows = ksub * bk;  // rows of k in an MN-major box
        const int64_t Mi = swap ? in.N : in.M, Nj = swap ? in.M : in.N;
        CUtensorMap &tp = rec->t0, &tq = rec->t1;
        // P(i, k): A (no swap) or B^T; Q(k, j): B (no swap) or A^T
        const dg_view *Pv = swap ? v.B : v.A;
        const dg_view *Qv = swap ? v.A : v.B;
        const ViewInfo &pi = swap ? v.b : v.a;
        const ViewInfo &qi = swap ? v.a : v.b;
        const Axis &p_i = swap ? pi.col : pi.row, &p_k = swap ? pi.row : pi.col;
        const Axis &q_k = swap ? qi.col : qi.row, &q_j = swap ? qi.row : qi.col;
        if (!in.p_gather) {
            const bool ok = in.p_mn_major ? encode_2d(&tp, dt, Pv->ptr, Mi, in.K, axis_stride(p_k), mn_rows)
                                          : encode_2d(&tp, dt, Pv->ptr, in.K, Mi, axis_stride(p_i), 128);
            if (!ok) return DG_ERR_UNSUPPORTED;
        }
        {
            // a CTA of a pair loads half of a tile's columns: one box of bn/2 rows when K-major
            const int q_rows = in.cta_pair ? bn / 2 : bn;
            const bool ok = in.q_mn_major ? encode_2d(&tq, dt, Qv->ptr, Nj, in.K, axis_stride(q_k), mn_rows)
                                          : encode_2d(&tq, dt, Qv->ptr, in.K, Nj, axis_stride(q_j), q_rows);
            if (!ok) return DG_ERR_UNSUPPORTED;
        }
        if (in.epi_tma_store) {
            // C(i, j) in blocks of 32 rows x 128 bytes, the epilogue's unit
            const int ces = elem_size(v.C->dtype);
            if (!encode_2d_box(&rec->t2, v.C->dtype, v.C->ptr, Nj, Mi, axis_stride(v.c.row), 128 / ces, 32, true))
                return DG_ERR_UNSUPPORTED;
        }
        UmmaParams p{};
        p.Mi = (int32_t)Mi;
        p.Nj = (int32_t)Nj;
        p.K = (int32_t)in.K;
        p.bn = bn;
        p.bk = bk;
        p.stages = in.stages;
        p.tiles_i = (int32_t)((Mi + in.block_m - 1) / in.block_m);
        p.tiles_j = (int32_t)((Nj + bn - 1) / bn);
        p.split_k = in.split_k;
        p.ksub = ksub;
        p.kb_total = (int32_t)((in.K + ksub * bk - 1) / (ksub * bk));  // stages along k
        p.kb_per_split = (p.kb_total + p.split_k - 1) / p.split_k;
        p.num_units = p.tiles_i * p.tiles_j * p.split_k;
        p.p_mn_major = in.p_mn_major;
        p.q_mn_major = in.q_mn_major;
        p.idesc = make_idesc(dt, in.p_mn_major, in.q_mn_major, bn, in.cta_pair ? 256 : 128);
        p.full_units = p.num_units;
        if (in.cta_pair) {
            // whole 256-row tiles; the last in.pair_half_tiles of them as two halves each
            const int32_t tiles = (int32_t)(((Mi + 255) / 256) * p.tiles_j);
            p.full_units = tiles - in.pair_half_tiles;
            p.num_units = p.full_units + 2 * in.pair_half_tiles;
            p.idesc_half = make_idesc(dt, in.p_mn_major, in.q_mn_major, bn / 2, 256);
            if (in.stream_k_tiles > 0) {
                // the workspace of the stream: header, flags, partial slots
                if (!sk_ws) return DG_ERR_UNSUPPORTED;
                size_t flag_off = 0, part_off = 0;
                sk_workspace_bytes(in.grid / 2, bn, &flag_off, &part_off);
                p.sk_tiles = in.stream_k_tiles;
                p.dp_tiles = tiles - in.stream_k_tiles;
                p.sk_hdr = static_cast<uint32_t *>(sk_ws);
                p.sk_flag = reinterpret_cast<uint32_t *>(static_cast<char *>(sk_ws) + flag_off);
                p.sk_part = reinterpret_cast<float *>(static_cast<char *>(sk_ws) + part_off);
            }
        }
        int tc = 32;
        while (tc < 2 * bn) tc *= 2;
        p.tmem_cols = tc;
        p.epi = epi_params(v, swap, alpha, beta, sa, sb, bias, act);
        if (in.split_reduce_add && act == DG_ACT_NONE) {
            // C as a 2-D FP32 map along its unit-stride dim, 32 x 32 boxes: i is
            // unit-stride when C's rows are (no swap) or its columns are (swap)
            const bool inner_i = swap ? v.c.unit_dim == 1 : v.c.unit_dim == 2;
            const Axis &ia = swap ? v.c.col : v.c.row, &ja = swap ? v.c.row : v.c.col;
            const bool ok = inner_i ? encode_2d_box(&rec->t2, DG_F32, v.C->ptr, Mi, Nj, axis_stride(ja), 32, 32, false)
                                    : encode_2d_box(&rec->t2, DG_F32, v.C->ptr, Nj, Mi, axis_stride(ia), 32, 32, true);
            if (!ok) return DG_ERR_UNSUPPORTED;
            p.red_add = 1;
            p.red_inner_i = inner_i;
        }
        if (in.p_gather) {
            DevView d{};
            d.ptr = static_cast<const char *>(Pv->ptr);
            d.row = p_i;
            d.col = p_k;
            d.dtype = dt;
            p.pv = d;
            p.gather_vec = in.vec_bytes / es;
        }
        p.err_word = ds->err_word;
        p.timeout_ns = (uint64_t)g_timeout_ms.load() * 1000000ull;
        p.stall_loader = g_stall.load();
        p.epi_tma = in.epi_tma_store;
        p.gather_cluster = in.gather_cluster;
        p.pdl = rec->pdl;
        p.trace = reinterpret_cast<uint64_t *>(g_trace.load());
        rec->umma = p;
        rec->pair = in.cta_pair != 0;
        rec->fp8 = pl.fp8;
        rec->gather = in.p_gather != 0;
        rec->grid = in.grid;
        // the kernel lays out its shared memory from these parameters
        rec->smem = rec->pair ? pl.smem
                              : umma_smem_bytes(p.bn, p.stages, rec->gather, p.epi_tma != 0, p.red_add ? 1 : p.split_k);
        break;
    }
    default: return DG_ERR_UNSUPPORTED;
    }
    return DG_OK;
}

// Enqueue a prepared launch on `stream`.
dg_status fire(const LaunchRec &r, cudaStream_t stream) {
    cudaError_t err = cudaSuccess;
    int grid = 0;
    switch (r.kind) {
    case DG_KIND_NONE: return DG_OK;
    case DG_KIND_SCALE_C: err = launch_scale_c(r.c, r.M, r.N, r.beta, r.bias, r.act, r.pdl, stream); break;
    case DG_KIND_SIMT: err = launch_simt(r.simt, stream); break;
    case DG_KIND_GEMV_N: err = launch_gemv_n(r.gemv, &r.t0, stream, &grid); break;
    case DG_KIND_GEMV_K: err = launch_gemv_k(r.gemv, stream, &grid); break;
    case DG_KIND_UMMA:
        err = r.pair ? launch_umma_pair(r.umma, &r.t0, &r.t1, &r.t2, r.fp8, r.grid, r.smem, stream)
                     : launch_umma(r.umma, &r.t0, &r.t1, &r.t2, r.fp8, r.gather, r.grid, r.smem, stream);
        break;
    default: return DG_ERR_UNSUPPORTED;
    }
    if (err != cudaSuccess) return DG_ERR_CUDA;
    g_launches.fetch_add(1);
    return DG_OK;
}

// The exact arguments of a dg_gemm call, with the device and the option
// epoch: equal keys mean an identical launch.
struct CallKey {
    dg_view A, B, C;
    float alpha, beta;
    const float *sa, *sb;
    const float *bias;
    int act;
    int dev;
    uint32_t epoch;
    void *stream;  // a Stream-K launch uses its stream's workspace
};

bool key_equal(const CallKey &x, const CallKey &y) { return std::memcmp(&x, &y, sizeof(CallKey)) == 0; }

struct CallCache {
    CallKey key[8];
    LaunchRec rec[8];
    bool used[8] = {};
    int next = 0;
};
thread_local CallCache t_calls;

// Check the buffers of a planned call, fetch the Stream-K workspace it needs
// and prepare its launch.  Without a workspace on this stream (e.g. during a
// graph capture) the call is planned again without Stream-K; with a forced
// variant that needs one, it is DG_ERR_UNSUPPORTED.
dg_status build_launch(Views &v, Plan &pl, float alpha, float beta, const float *scale_a, const float *scale_b,
                       const float *bias, int act, DeviceState *ds, cudaStream_t stream, const Override *force,
                       LaunchRec *rec) {
    const dg_plan_info &in = pl.info;
    // every buffer the launch touches must live on this device
    const bool use_ab = in.kind != DG_KIND_SCALE_C;
    if (use_ab && (!device_accessible(v.A->ptr) || !device_accessible(v.B->ptr))) return DG_ERR_POINTER;
    if (!device_accessible(v.C->ptr)) return DG_ERR_POINTER;
    if (use_ab && scale_a && !device_accessible(scale_a)) return DG_ERR_POINTER;
    if (use_ab && scale_b && !device_accessible(scale_b)) return DG_ERR_POINTER;
    if (bias && !device_accessible(bias)) return DG_ERR_POINTER;
    void *sk_ws = nullptr;
    if (in.stream_k_tiles > 0) {
        size_t flag_off = 0, part_off = 0;
        const size_t need = sk_workspace_bytes(in.grid / 2, in.block_n, &flag_off, &part_off);
        sk_ws = sk_workspace(ds, stream, need, part_off);
        if (!sk_ws) {
            if (force && force->any()) return DG_ERR_UNSUPPORTED;
            const dg_status st = make_plan(v, alpha, beta, ds->num_sms, &pl, false, force);
            if (st != DG_OK) return st;
        }
    }
    return prepare(v, pl, alpha, beta, use_ab ? scale_a : nullptr, use_ab ? scale_b : nullptr, bias, act, ds, sk_ws,
                   rec);
}

// The variants dg_autotune times for a call whose rule-based plan is `base`.
std::vector<Override> tune_candidates(const dg_plan_info &base) {
    std::vector<Override> c;
    c.push_back(Override{});  // the dispatcher's own rule first
    if (base.kind == DG_KIND_GEMV_N) {
        for (int s = 1; s <= kMaxCluster; ++s) {
            Override o;
            o.gemv_split = s;
            c.push_back(o);
        }
        return c;
    }
    for (int bn : {32, 64, 128, 256}) {
        for (int split : {1, 2, 3, 4, 6, 8}) {
            for (int pair : {0, 1}) {
                if (pair && split > 1) continue;
                for (int sk : {0, 1}) {
                    if (sk && !pair) continue;
                    for (int gcl : {1, 2, 4}) {
                        if (gcl > 1 && (!base.p_gather || split > 1 || pair)) continue;
                        for (int epi : {0, 1}) {
                            for (int ks : {1, 2}) {
                                if (ks == 2 && !pair) continue;
                                Override o;
                                o.bn = bn;
                                o.split = split;
                                o.pair = pair;
                                o.sk = pair ? sk : -1;
                                o.gcl = base.p_gather ? gcl : 0;
                                o.epi_tma = epi;
                                o.ksub = pair ? ks : 0;
                                c.push_back(o);
                            }
                        }
                    }
                }
            }
        }
    }
    return c;
}

}  // namespace
}  // namespace dg

using namespace dg;

extern "C" {

dg_status dg_gemm_ex(const dg_view *A, const dg_view *B, const dg_view *C, float alpha, float beta,
                     const float *scale_a, const float *scale_b, const dg_epilogue *epilogue, void *stream) {
    if (!A || !B || !C) return DG_ERR_NULL;
    const float *bias = nullptr;
    int act = DG_ACT_NONE;
    if (epilogue) {
        if (epilogue->activation < DG_ACT_NONE || epilogue->activation > DG_ACT_GELU_TANH || epilogue->reserved != 0)
            return DG_ERR_VALUE;
        bias = epilogue->bias;
        act = epilogue->activation;
    }
    // a call identical to a recent one on this thread and device reuses its
    // validated plan, parameters and tensor maps
    CallKey key;
    std::memset(&key, 0, sizeof(key));
    key.A = *A;
    key.B = *B;
    key.C = *C;
    key.alpha = alpha;
    key.beta = beta;
    key.sa = scale_a;
    key.sb = scale_b;
    key.bias = bias;
    key.act = act;
    key.epoch = g_epoch.load();
    key.stream = stream;
    if (cudaGetDevice(&key.dev) != cudaSuccess) {
        cudaGetLastError();
        key.dev = -1;
    }
    if (key.dev >= 0)
        for (int i = 0; i < 8; ++i)
            if (t_calls.used[i] && key_equal(t_calls.key[i], key))
                return fire(t_calls.rec[i], static_cast<cudaStream_t>(stream));

    Views v{A, B, C, {}, {}, {}};
    v.act = act;
    Plan pl;
    // argument errors are reported before any CUDA call
    dg_status st = make_plan(v, alpha, beta, 148, &pl);
    if (st != DG_OK) return st;
    if (pl.info.kind == DG_KIND_NONE) return DG_OK;
    DeviceState *ds = nullptr;
    st = device_state(&ds);
    if (st != DG_OK) return st;
    if (ds->num_sms != 148) {
        st = make_plan(v, alpha, beta, ds->num_sms, &pl);
        if (st != DG_OK) return st;
    }
    const int slot = t_calls.next;
    t_calls.used[slot] = false;
    st = build_launch(v, pl, alpha, beta, scale_a, scale_b, bias, act, ds, static_cast<cudaStream_t>(stream), nullptr,
                      &t_calls.rec[slot]);
    if (st != DG_OK) return st;
    key.epoch = g_epoch.load();  // a replaced Stream-K workspace invalidated the cache
    t_calls.key[slot] = key;
    t_calls.used[slot] = true;
    t_calls.next = (slot + 1) % 8;
    return fire(t_calls.rec[slot], static_cast<cudaStream_t>(stream));
}

dg_status dg_gemm(const dg_view *A, const dg_view *B, const dg_view *C, float alpha, float beta,
                  const float *scale_a, const float *scale_b, void *stream) {
    return dg_gemm_ex(A, B, C, alpha, beta, scale_a, scale_b, nullptr, stream);
}

dg_status dg_autotune(const dg_view *A, const dg_view *B, const dg_view *C, float alpha, float beta,
                      const float *scale_a, const float *scale_b, const dg_epilogue *epilogue, void *stream,
                      int reps, dg_tune_result *out) {
    if (!A || !B || !C) return DG_ERR_NULL;
    const float *bias = nullptr;
    int act = DG_ACT_NONE;
    if (epilogue) {
        if (epilogue->activation < DG_ACT_NONE || epilogue->activation > DG_ACT_GELU_TANH || epilogue->reserved != 0)
            return DG_ERR_VALUE;
        bias = epilogue->bias;
        act = epilogue->activation;
    }
    if (reps < 1 || reps > 1000) return DG_ERR_VALUE;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    Views v{A, B, C, {}, {}, {}};
    v.act = act;
    Plan base;
    const Override rule;  // the dispatcher's rules, not an earlier tuning
    dg_status st = make_plan(v, alpha, beta, 148, &base, true, &rule);
    if (st != DG_OK) return st;
    dg_tune_result res;
    std::memset(&res, 0, sizeof(res));
    if (base.info.kind == DG_KIND_NONE) {
        if (out) *out = res;
        return DG_OK;
    }
    DeviceState *ds = nullptr;
    if ((st = device_state(&ds)) != DG_OK) return st;
    if ((st = make_plan(v, alpha, beta, ds->num_sms, &base, true, &rule)) != DG_OK) return st;
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(s, &cap) != cudaSuccess) return DG_ERR_CUDA;
    if (cap != cudaStreamCaptureStatusNone) return DG_ERR_UNSUPPORTED;  // it synchronises and may allocate
    const TuneKey key = tune_key(A, B, C, alpha, beta, ds->num_sms);
    const bool tunable = base.info.kind == DG_KIND_UMMA || base.info.kind == DG_KIND_GEMV_N;
    if (tunable) {
        // with beta != 0 every trial reads and rewrites C: keep its bytes and put them back
        void *saved = nullptr;
        size_t span = 0;
        if (beta != 0.f) {
            span = (size_t)v.c.span;
            if (cudaMalloc(&saved, span) != cudaSuccess ||
                cudaMemcpyAsync(saved, C->ptr, span, cudaMemcpyDeviceToDevice, s) != cudaSuccess) {
                cudaGetLastError();
                if (saved) cudaFree(saved);
                return DG_ERR_CUDA;
            }
        }
        cudaEvent_t e0, e1;
        if (cudaEventCreate(&e0) != cudaSuccess || cudaEventCreate(&e1) != cudaSuccess) return DG_ERR_CUDA;
        std::vector<dg_plan_info> seen;
        float best = 0.f;
        Override best_ov;
        bool have = false;
        for (const Override &o : tune_candidates(base.info)) {
            Plan pl;
            if (make_plan(v, alpha, beta, ds->num_sms, &pl, true, &o) != DG_OK || pl.info.kind != base.info.kind)
                continue;  // a variant these operands do not admit
            bool dup = false;
            for (const dg_plan_info &q : seen) dup = dup || std::memcmp(&q, &pl.info, sizeof(q)) == 0;
            if (dup) continue;
            LaunchRec rec;
            if (build_launch(v, pl, alpha, beta, scale_a, scale_b, bias, act, ds, s, &o, &rec) != DG_OK) continue;
            seen.push_back(pl.info);
            bool ok = fire(rec, s) == DG_OK;  // warm-up (tensor maps, instruction cache)
            ok = ok && cudaEventRecord(e0, s) == cudaSuccess;
            for (int r = 0; ok && r < reps; ++r) ok = fire(rec, s) == DG_OK;
            ok = ok && cudaEventRecord(e1, s) == cudaSuccess && cudaEventSynchronize(e1) == cudaSuccess;
            float ms = 0.f;
            ok = ok && cudaEventElapsedTime(&ms, e0, e1) == cudaSuccess;
            if (!ok) {
                cudaGetLastError();
                continue;
            }
            const float us = ms * 1000.f / (float)reps;
            if (seen.size() == 1) res.default_us = us;
            if (!have || us < best) {
                best = us;
                best_ov = o;
                have = true;
            }
            ++res.candidates;
        }
        cudaEventDestroy(e0);
        cudaEventDestroy(e1);
        if (saved) {
            const bool ok = cudaMemcpyAsync(C->ptr, saved, span, cudaMemcpyDeviceToDevice, s) == cudaSuccess &&
                            cudaStreamSynchronize(s) == cudaSuccess;
            cudaFree(saved);
            if (!ok) return DG_ERR_CUDA;
        }
        if (have) {
            store_tuned(key, best_ov);
            g_epoch.fetch_add(1);  // cached launches of these views take the tuned plan from now on
            res.best_us = best;
        }
    }
    // the call itself, with the chosen variant
    st = dg_gemm_ex(A, B, C, alpha, beta, scale_a, scale_b, epilogue, stream);
    if (st != DG_OK) return st;
    Plan chosen;
    if (make_plan(v, alpha, beta, ds->num_sms, &chosen) == DG_OK) res.plan = chosen.info;
    if (out) *out = res;
    return DG_OK;
}

}  // extern "C"

// ------------------------------------------------ the allocation-free entry
// Some callers cannot let a library call cudaMalloc: code running inside a
// CUDA graph capture (an allocation there fails or would end the capture),
// frameworks that own every byte of device memory through their own pool and
// account for it, and real-time serving loops where an allocation's implicit
// device synchronisation is not allowed.  dg_gemm allocates twice on first use
// (the status word of the device, the Stream-K workspace of a stream); the
// entry point below allocates nothing: both live in this file-scope array,
// which the CUDA runtime places in device memory when it loads the library's
// module on a device, and which stays there until the process exits.
namespace dg {
namespace {
constexpr size_t kStaticScratchBytes = size_t(24) << 20;  // 24 MiB per device
constexpr size_t kStaticStatusBytes = 256;                 // the status word, then the Stream-K workspace
constexpr size_t kStaticZeroBytes = kStaticStatusBytes + kSkHeaderBytes + 8192;  // status, header, flags of 256 pairs
}  // namespace
}  // namespace dg

static __device__ __align__(256) unsigned char g_static_scratch[dg::kStaticScratchBytes];

namespace dg {
namespace {
struct StaticState {
    bool ready = false;
    void *scratch = nullptr;  // device address of g_static_scratch on this device
    int num_sms = 0;
};
StaticState g_static[kMaxDevices];

// Once per device, with the device current: the array's device address (in
// host code its name is only a host-side stand-in), the SM count, the tensor
// map encoder, and the words that must start at zero cleared on the stream.
dg_status static_setup(int dev, cudaStream_t stream, StaticState **out) {
    std::lock_guard<std::mutex> lk(g_mu);
    StaticState &st = g_static[dev];
    if (!st.ready) {
        void *ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_static_scratch) != cudaSuccess || !ptr) {
            cudaGetLastError();
            return DG_ERR_CUDA;
        }
        if (cudaDeviceGetAttribute(&st.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return DG_ERR_CUDA;
        if (!g_encode) {
            cudaDriverEntryPointQueryResult q;
            void *fn = nullptr;
            if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q) !=
                    cudaSuccess ||
                q != cudaDriverEntryPointSuccess || !fn)
                return DG_ERR_CUDA;
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
        }
        if (cudaMemsetAsync(ptr, 0, kStaticZeroBytes, stream) != cudaSuccess) return DG_ERR_CUDA;
        st.scratch = ptr;
        st.ready = true;
    }
    *out = &st;
    return DG_OK;
}
}  // namespace
}  // namespace dg

extern "C" {

dg_status dg_gemm_static(const dg_view *A, const dg_view *B, const dg_view *C, float alpha, float beta,
                         const float *scale_a, const float *scale_b, void *stream) {
    if (!A || !B || !C) return DG_ERR_NULL;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    Views v{A, B, C, {}, {}, {}};
    Plan pl;
    dg_status st = make_plan(v, alpha, beta, 148, &pl);
    if (st != DG_OK) return st;
    if (pl.info.kind == DG_KIND_NONE) return DG_OK;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return DG_ERR_CUDA;
    StaticState *ss = nullptr;
    if ((st = static_setup(dev, s, &ss)) != DG_OK) return st;
    if (ss->num_sms != 148 && (st = make_plan(v, alpha, beta, ss->num_sms, &pl)) != DG_OK) return st;
    const dg_plan_info &in = pl.info;
    const bool use_ab = in.kind != DG_KIND_SCALE_C;
    if (use_ab && (!device_accessible(A->ptr) || !device_accessible(B->ptr))) return DG_ERR_POINTER;
    if (!device_accessible(C->ptr)) return DG_ERR_POINTER;
    if (use_ab && scale_a && !device_accessible(scale_a)) return DG_ERR_POINTER;
    if (use_ab && scale_b && !device_accessible(scale_b)) return DG_ERR_POINTER;
    char *scratch = static_cast<char *>(ss->scratch);
    void *sk_ws = nullptr;
    if (in.stream_k_tiles > 0) {
        size_t flag_off = 0, part_off = 0;
        const size_t need = sk_workspace_bytes(in.grid / 2, in.block_n, &flag_off, &part_off);
        if (kStaticStatusBytes + need > kStaticScratchBytes || part_off > kStaticZeroBytes - kStaticStatusBytes)
            return DG_ERR_UNSUPPORTED;  // the problem's Stream-K workspace does not fit the static array
        sk_ws = scratch + kStaticStatusBytes;
    }
    DeviceState ds;  // no allocation: the status word is the array's first word
    ds.ready = true;
    ds.num_sms = ss->num_sms;
    ds.err_word = reinterpret_cast<int *>(scratch);
    LaunchRec rec;
    st = prepare(v, pl, alpha, beta, use_ab ? scale_a : nullptr, use_ab ? scale_b : nullptr, nullptr, DG_ACT_NONE,
                 &ds, sk_ws, &rec);
    if (st != DG_OK) return st;
    return fire(rec, s);
}

dg_status dg_tune_clear(void) {
    {
        std::lock_guard<std::mutex> lk(g_tune_mu);
        g_tuned.clear();
    }
    g_epoch.fetch_add(1);
    return DG_OK;
}

dg_status dg_gemv(const dg_view *x, const dg_view *W, const dg_view *y, float alpha, float beta, void *stream) {
    if (!x || !W || !y) return DG_ERR_NULL;
    ViewInfo xi;
    dg_status st = analyse(x, false, &xi);
    if (st != DG_OK) return st;
    if (xi.rows > 8) return DG_ERR_UNSUPPORTED;
    return dg_gemm(x, W, y, alpha, beta, nullptr, nullptr, stream);
}

const char *dg_status_string(dg_status s) {
    switch (s) {
    case DG_OK: return "ok";
    case DG_ERR_NULL: return "null pointer";
    case DG_ERR_NDIM: return "ndim must be 1..4 and row_dims 0..ndim";
    case DG_ERR_SHAPE: return "shape mismatch or negative size";
    case DG_ERR_DTYPE: return "unsupported element type combination";
    case DG_ERR_STRIDE: return "negative/overflowing stride or overlapping output";
    case DG_ERR_ALIGN: return "pointer or stride not a multiple of the element size";
    case DG_ERR_POINTER: return "pointer is not device memory of the current device";
    case DG_ERR_VALUE: return "alpha or beta is not finite";
    case DG_ERR_UNSUPPORTED: return "request not supported";
    case DG_ERR_CUDA: return "CUDA runtime error";
    case DG_ERR_TIMEOUT: return "a device-side wait timed out";
    default: return "unknown status";
    }
}

dg_status dg_sync_status(void *stream) {
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return DG_ERR_CUDA;
    DeviceState *ds = nullptr;
    dg_status st = device_state(&ds);
    if (st != DG_OK) return st;
    int word = 0;
    if (cudaMemcpy(&word, ds->err_word, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return DG_ERR_CUDA;
    if (word != 0) {
        if (cudaMemset(ds->err_word, 0, sizeof(int)) != cudaSuccess) return DG_ERR_CUDA;
        if (cudaDeviceSynchronize() != cudaSuccess) return DG_ERR_CUDA;
        return word == DG_ERR_TIMEOUT ? DG_ERR_TIMEOUT : DG_ERR_CUDA;
    }
    return DG_OK;
}

dg_status dg_analyse_view(const dg_view *v, dg_view_info *out);  // view.cpp

dg_status dg_plan(const dg_view *A, const dg_view *B, const dg_view *C, float alpha, float beta, int has_scales,
                  int num_sms, dg_plan_info *out) {
    (void)has_scales;
    if (!A || !B || !C || !out) return DG_ERR_NULL;
    if (num_sms <= 0) {
        int dev = 0, n = 0;
        if (cudaGetDevice(&dev) == cudaSuccess &&
            cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && n > 0)
            num_sms = n;
        else {
            cudaGetLastError();
            num_sms = 148;
        }
    }
    Views v{A, B, C, {}, {}, {}};
    Plan pl;
    dg_status st = make_plan(v, alpha, beta, num_sms, &pl);
    if (st != DG_OK) return st;
    *out = pl.info;
    return DG_OK;
}

uint64_t dg_launch_count(void) { return g_launches.load(); }

dg_status dg_set_option(int option, int64_t value) {
    g_epoch.fetch_add(1);
    switch (option) {
    case DG_OPT_FORCE_KIND:
        if (value < 0 || value > DG_KIND_UMMA) return DG_ERR_VALUE;
        g_force_kind.store((int)value);
        return DG_OK;
    case DG_OPT_WAIT_TIMEOUT_MS:
        if (value < 1 || value > 600000) return DG_ERR_VALUE;
        g_timeout_ms.store(value);
        return DG_OK;
    case DG_OPT_TEST_STALL:
        if (value < 0 || value > 2) return DG_ERR_VALUE;
        g_stall.store((int)value);
        return DG_OK;
    case DG_OPT_TRACE:
        g_trace.store((uint64_t)value);
        return DG_OK;
    case DG_OPT_EARLY_LAUNCH:
        if (value < 0 || value > 3) return DG_ERR_VALUE;
        g_pdl.store((int)value);
        return DG_OK;
    case DG_OPT_CTA_PAIR:
        if (value < 0 || value > 2) return DG_ERR_VALUE;
        g_pair.store((int)value);
        return DG_OK;
    case DG_OPT_MAX_SPLIT_K:
        if (value < 1 || value > 64) return DG_ERR_VALUE;
        g_max_split.store((int)value);
        return DG_OK;
    case DG_OPT_EPI_TMA:
        if (value < 0 || value > 1) return DG_ERR_VALUE;
        g_epi_tma.store((int)value);
        return DG_OK;
    case DG_OPT_GATHER_CLUSTER:
        if (value < 0 || value > 1) return DG_ERR_VALUE;
        g_gather_cluster.store((int)value);
        return DG_OK;
    case DG_OPT_PAIR_TAIL:
        if (value < 0 || value > 1) return DG_ERR_VALUE;
        g_pair_tail.store((int)value);
        return DG_OK;
    case DG_OPT_STREAM_K:
        if (value < 0 || value > 1) return DG_ERR_VALUE;
        g_stream_k.store((int)value);
        return DG_OK;
    case DG_OPT_DETERMINISTIC:
        if (value < 0 || value > 1) return DG_ERR_VALUE;
        g_deterministic.store((int)value);
        return DG_OK;
    case DG_OPT_PAIR_DEEP_STAGES:
        if (value < 0 || value > 1) return DG_ERR_VALUE;
        g_pair_deep.store((int)value);
        return DG_OK;
    default: return DG_ERR_VALUE;
    }
}

int dg_version(void) { return 100; }

}  // extern "C"
