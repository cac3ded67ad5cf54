"""Host-only checks of the C-ABI library: it loads, exports every entry point
include/dg.h declares, validates arguments, analyses views and takes the
dispatch decisions described in its header.  Nothing here needs a GPU:
pointers are plain aligned integers and no compute entry point runs a kernel.
"""
import ctypes
import os
import re

import pytest

import tcgen05_tmem_gemm_b200 as dg
import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dg.h")

FAKE = 1 << 40  # a 4 KiB-aligned address; only its alignment is ever looked at


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(dg_[a-z_]+)\s*\(", text)))


def test_header_symbols_exported():
    names = declared_functions()
    assert "dg_gemm" in names and "dg_gemv" in names
    for n in names:
        assert hasattr(dg.lib, n), f"libdg.so does not export {n}"


def test_version_and_status_strings():
    assert dg.dg_version() >= 100
    for s in range(12):
        assert dg.status_string(s)
    assert dg.status_string(dg.DG_ERR_TIMEOUT) == "a device-side wait timed out"


def fake_view(op: W.Operand, base=FAKE) -> dg.dg_view:
    return dg.make_view(base + op.offset, op.shape, op.stride, op.row_dims, op.dtype)


def meta_problem(name, **kw):
    """A workload's views with fake pointers (shapes/strides only, tiny tensors)."""
    return W.WORKLOADS[name](**kw)


def views(p: W.Problem, bases=(FAKE, FAKE + (1 << 32), FAKE + (2 << 32))):
    return fake_view(p.A, bases[0]), fake_view(p.B, bases[1]), fake_view(p.C, bases[2])


# ---------------------------------------------------------------- analysis

def test_analyse_row_major_and_transpose():
    info = dg.dg_analyse_view(dg.make_view(FAKE, (64, 4096), (8192, 2), 1, "bf16"))
    assert (info.rows, info.cols, info.unit_dim, info.tma_ok, info.vec_bytes) == (64, 4096, 1, 1, 16)
    info = dg.dg_analyse_view(dg.make_view(FAKE, (4096, 128), (2, 8192), 1, "bf16"))
    assert (info.rows, info.cols, info.unit_dim, info.tma_ok) == (4096, 128, 2, 1)


def test_analyse_nchw_feature_map():
    # [16,256,14,14] BF16 NCHW read as [N*H*W, C]: h and w merge into one
    # contiguous segment of 196, the channel stride (392 B) is not a multiple
    # of 16, so no TMA map covers it and thread loads of 8 bytes are the widest.
    info = dg.dg_analyse_view(dg.make_view(FAKE, (16, 14, 14, 256), (100352, 28, 2, 392), 3, "bf16"))
    assert (info.rows, info.cols) == (3136, 256)
    assert info.n_row == 2 and list(info.row_shape[:2]) == [16, 196] and list(info.row_stride[:2]) == [100352, 2]
    assert info.n_col == 1 and info.col_stride[0] == 392
    assert info.tma_ok == 0 and info.unit_dim == 0 and info.vec_bytes == 8


def test_analyse_pages_example_merges():
    # shape (1,128,7,7) with byte strides (0,196,28,4): the size-1 dim drops,
    # h and w merge into one contiguous segment of 49 FP32 elements.
    info = dg.dg_analyse_view(dg.make_view(FAKE, (1, 128, 7, 7), (0, 196, 28, 4), 2, "f32"))
    assert (info.rows, info.cols) == (128, 49)
    assert info.n_row == 1 and info.row_stride[0] == 196
    assert info.n_col == 1 and info.col_shape[0] == 49 and info.col_stride[0] == 4


@pytest.mark.parametrize("shape,stride,row_dims,dtype,status", [
    ((4, 4), (8, -2), 1, "f16", dg.DG_ERR_STRIDE),
    ((4, 4), (8, 3), 1, "f16", dg.DG_ERR_ALIGN),
    ((1 << 40, 1 << 30), (1 << 31, 2), 1, "f16", dg.DG_ERR_STRIDE),  # byte extent overflows int64
    ((4, -1), (8, 2), 1, "f16", dg.DG_ERR_SHAPE),
])
def test_analyse_rejects(shape, stride, row_dims, dtype, status):
    with pytest.raises(dg.DgError) as e:
        dg.dg_analyse_view(dg.make_view(FAKE, shape, stride, row_dims, dtype))
    assert e.value.status == status


def test_analyse_misaligned_pointer():
    with pytest.raises(dg.DgError) as e:
        dg.dg_analyse_view(dg.make_view(FAKE + 1, (4, 4), (8, 2), 1, "f16"))
    assert e.value.status == dg.DG_ERR_ALIGN


def test_ndim_checks():
    for nd, rd in ((0, 0), (5, 1), (2, 3), (2, -1)):
        v = dg.make_view(FAKE, (4,) * max(nd, 1), (2,) * max(nd, 1), 0, "f16")
        v.ndim = nd
        v.row_dims = rd
        with pytest.raises(dg.DgError) as e:
            dg.dg_analyse_view(v)
        assert e.value.status == dg.DG_ERR_NDIM


# ---------------------------------------------------------------- dispatch

def plan_of(name, **kw):
    p = meta_problem(name, **kw)
    A, B, C = views(p)
    return dg.dg_plan(A, B, C, p.alpha, p.beta, p.scale_a is not None, 148).as_dict()


def test_plan_decode_gemv():
    pl = plan_of("gemv", K=64, N=256)
    assert pl["kind_name"] == "gemv_n"
    pl = plan_of("gemv_kt", K=64, N=16)
    assert pl["kind_name"] == "gemv_k"


def test_plan_small_gemm_umma():
    pl = plan_of("small")
    assert pl["kind_name"] == "umma" and pl["swap_ab"] == 0 and pl["block_n"] == 64  # two CTAs, not one
    assert pl["p_mn_major"] == 0 and pl["q_mn_major"] == 1 and pl["split_k"] == 1
    assert pl["cta_pair"] == 0 and pl["grid"] == 2  # few tiles: no pairing
    assert pl["epi_tma_store"] == 1  # beta == 0, row-major FP32 C: tensor stores


def test_plan_thin_swaps_and_splits():
    pl = plan_of("thin", M=64, N=4096, K=4096)
    assert pl["kind_name"] == "umma" and pl["swap_ab"] == 1
    assert pl["block_n"] == 64 and pl["p_mn_major"] == 1 and pl["q_mn_major"] == 0
    assert pl["split_k"] == 4 and pl["grid"] == 128
    assert pl["epi_tma_store"] == 0  # beta == 1: split tiles reduce in the cluster


def test_plan_square_bf16_and_fp8():
    pl = plan_of("square_bf16", M=4096, N=4096, K=64)
    assert pl["kind_name"] == "umma" and pl["block_n"] == 256 and pl["grid"] == 148
    assert pl["cta_pair"] == 1 and pl["block_m"] == 256  # CTA pairs share 256-row tiles
    # 256 tiles on 74 pairs: the last 34 run as half-width tiles
    assert pl["pair_half_tiles"] == 34
    pl = plan_of("square_e4m3", M=4096, N=4096, K=64)
    assert pl["kind_name"] == "umma" and pl["block_k"] == 128 and pl["q_mn_major"] == 1


def test_plan_pair_deep_stages():
    # CTA pairs with B MN-major (row-major [K, N]) and K a multiple of 128:
    # stages two 64-deep k sub-blocks deep, three of them (64 KB each)
    pl = plan_of("square_bf16", M=4096, N=4096, K=128)
    assert pl["cta_pair"] == 1 and pl["q_mn_major"] == 1
    assert pl["block_k"] == 128 and pl["stages"] == 3
    dg.dg_set_option(dg.DG_OPT_PAIR_DEEP_STAGES, 0)
    try:
        pl = plan_of("square_bf16", M=4096, N=4096, K=128)
        assert pl["block_k"] == 64 and pl["stages"] == 6
    finally:
        dg.dg_set_option(dg.DG_OPT_PAIR_DEEP_STAGES, 1)
    # K not a whole number of deep stages: one sub-block per stage
    pl = plan_of("square_bf16", M=4096, N=4096, K=192)
    assert pl["cta_pair"] == 1 and pl["block_k"] == 64
    pl = plan_of("square_e4m3", M=4096, N=4096, K=256)
    assert pl["cta_pair"] == 1 and pl["block_k"] == 256 and pl["stages"] == 3
    with pytest.raises(dg.DgError):
        dg.dg_set_option(dg.DG_OPT_PAIR_DEEP_STAGES, 2)


def test_plan_thin_split_reduce_add():
    # beta = 1 with FP32 C: the k splits add into C unless deterministic
    p = meta_problem("thin")
    pl = dg.dg_plan(*views(p), 1.0, 1.0, False, 148).as_dict()
    assert pl["split_k"] == 4 and pl["split_reduce_add"] == 1
    assert dg.dg_plan(*views(p), 1.0, 0.5, False, 148).as_dict()["split_reduce_add"] == 0
    dg.dg_set_option(dg.DG_OPT_DETERMINISTIC, 1)
    try:
        assert dg.dg_plan(*views(p), 1.0, 1.0, False, 148).as_dict()["split_reduce_add"] == 0
    finally:
        dg.dg_set_option(dg.DG_OPT_DETERMINISTIC, 0)


def test_plan_square_stream_k_tail():
    # 256 tiles of 256 x 256 on 74 CTA pairs: 222 whole, the last 34 as
    # half-width tiles (the default), or shared out along k over every pair
    # (Stream-K, opt-in)
    p = meta_problem("square_bf16")
    pl = dg.dg_plan(*views(p), 1.0, 0.0, False, 148).as_dict()
    assert pl["cta_pair"] == 1 and pl["stream_k_tiles"] == 0 and pl["pair_half_tiles"] == 34
    dg.dg_set_option(dg.DG_OPT_STREAM_K, 1)
    try:
        pl = dg.dg_plan(*views(p), 1.0, 0.0, False, 148).as_dict()
        assert pl["stream_k_tiles"] == 34 and pl["pair_half_tiles"] == 0
    finally:
        dg.dg_set_option(dg.DG_OPT_STREAM_K, 0)
    with pytest.raises(dg.DgError):
        dg.dg_set_option(dg.DG_OPT_STREAM_K, 2)


def test_plan_strided_gathers_a():
    pl = plan_of("strided")
    assert pl["kind_name"] == "umma" and pl["p_gather"] == 1 and pl["swap_ab"] == 0
    assert pl["p_mn_major"] == 1 and pl["vec_bytes"] == 8
    assert pl["epi_tma_store"] == 1
    # the four CTAs along N that need the same A tile share its gather
    assert pl["block_n"] == 256 and pl["gather_cluster"] == 4 and pl["grid"] == 100
    dg.dg_set_option(dg.DG_OPT_GATHER_CLUSTER, 0)
    try:
        assert plan_of("strided")["gather_cluster"] == 1
    finally:
        dg.dg_set_option(dg.DG_OPT_GATHER_CLUSTER, 1)


def test_plan_edge_kinds():
    p = meta_problem("small", M=16, N=16, K=16)
    A, B, C = views(p)
    assert dg.dg_plan(A, B, C, 0.0, 1.0, False, 148).kind == dg.DG_KIND_SCALE_C
    A0 = dg.make_view(FAKE, (16, 0), (0, 2), 1, "f16")
    B0 = dg.make_view(FAKE, (0, 16), (32, 2), 1, "f16")
    assert dg.dg_plan(A0, B0, C, 1.0, 0.0, False, 148).kind == dg.DG_KIND_SCALE_C
    Ae = dg.make_view(FAKE, (0, 16), (32, 2), 1, "f16")
    Ce = dg.make_view(FAKE, (0, 16), (64, 4), 1, "f32")
    assert dg.dg_plan(Ae, B, Ce, 1.0, 0.0, False, 148).kind == dg.DG_KIND_NONE


def test_plan_f32_inputs_use_cuda_cores():
    A = dg.make_view(FAKE, (32, 32), (128, 4), 1, "f32")
    C = dg.make_view(FAKE, (32, 32), (128, 4), 1, "f32")
    assert dg.dg_plan(A, A, C, 1.0, 0.0, False, 148).kind == dg.DG_KIND_SIMT


def test_plan_rejects():
    p = meta_problem("small", M=16, N=16, K=16)
    A, B, C = views(p)
    bad_k = dg.make_view(FAKE, (17, 16), (32, 2), 1, "f16")
    for args, status in (
        ((A, bad_k, C, 1.0, 0.0), dg.DG_ERR_SHAPE),
        ((A, B, C, float("nan"), 0.0), dg.DG_ERR_VALUE),
        ((A, B, C, 1.0, float("inf")), dg.DG_ERR_VALUE),
        ((A, dg.make_view(FAKE, (16, 16), (32, 2), 1, "bf16"), C, 1.0, 0.0), dg.DG_ERR_DTYPE),
        ((A, B, dg.make_view(FAKE, (16, 16), (16, 1), 1, "e4m3"), 1.0, 0.0), dg.DG_ERR_DTYPE),
        ((A, B, dg.make_view(FAKE, (16, 16), (0, 4), 1, "f32"), 1.0, 0.0), dg.DG_ERR_STRIDE),
        ((A, B, dg.make_view(FAKE, (16, 16), (8, 4), 1, "f32"), 1.0, 0.0), dg.DG_ERR_STRIDE),
    ):
        with pytest.raises(dg.DgError) as e:
            dg.dg_plan(*args, False, 148)
        assert e.value.status == status


def test_gemm_argument_errors_need_no_device():
    # argument errors come back before any CUDA call, so they work here too
    p = meta_problem("small", M=16, N=16, K=16)
    A, B, C = views(p)
    assert dg.lib.dg_gemm(None, ctypes.byref(B), ctypes.byref(C), 1.0, 0.0, None, None, None) == dg.DG_ERR_NULL
    bad_k = dg.make_view(FAKE, (17, 16), (32, 2), 1, "f16")
    assert dg.lib.dg_gemm(ctypes.byref(A), ctypes.byref(bad_k), ctypes.byref(C), 1.0, 0.0, None, None,
                          None) == dg.DG_ERR_SHAPE
    x = dg.make_view(FAKE, (9, 16), (32, 2), 1, "f16")
    y = dg.make_view(FAKE, (9, 16), (64, 4), 1, "f32")
    assert dg.lib.dg_gemv(ctypes.byref(x), ctypes.byref(B), ctypes.byref(y), 1.0, 0.0,
                          None) == dg.DG_ERR_UNSUPPORTED


def test_gemm_ex_epilogue_errors_need_no_device():
    p = meta_problem("small", M=16, N=16, K=16)
    A, B, C = views(p)
    for act, reserved in ((3, 0), (-1, 0), (0, 1)):
        e = dg.dg_epilogue()
        e.bias = None
        e.activation = act
        e.reserved = reserved
        assert dg.lib.dg_gemm_ex(ctypes.byref(A), ctypes.byref(B), ctypes.byref(C), 1.0, 0.0, None, None,
                                 ctypes.byref(e), None) == dg.DG_ERR_VALUE
    assert dg.lib.dg_gemm_ex(None, ctypes.byref(B), ctypes.byref(C), 1.0, 0.0, None, None, None,
                             None) == dg.DG_ERR_NULL


def test_autotune_argument_errors_need_no_device():
    p = meta_problem("small", M=16, N=16, K=16)
    A, B, C = views(p)
    out = dg.dg_tune_result()
    assert dg.lib.dg_autotune(None, ctypes.byref(B), ctypes.byref(C), 1.0, 0.0, None, None, None, None, 3,
                              ctypes.byref(out)) == dg.DG_ERR_NULL
    for reps in (0, 1001):
        assert dg.lib.dg_autotune(ctypes.byref(A), ctypes.byref(B), ctypes.byref(C), 1.0, 0.0, None, None, None,
                                  None, reps, ctypes.byref(out)) == dg.DG_ERR_VALUE
    bad_k = dg.make_view(FAKE, (17, 16), (32, 2), 1, "f16")
    assert dg.lib.dg_autotune(ctypes.byref(A), ctypes.byref(bad_k), ctypes.byref(C), 1.0, 0.0, None, None, None,
                              None, 3, ctypes.byref(out)) == dg.DG_ERR_SHAPE
    assert dg.lib.dg_tune_clear() == dg.DG_OK


def test_plan_nchw_output_stays_on_tensor_cores():
    # C written as an NCHW tensor [n, N, h, w] from the [n*h*w, N] product: the
    # row index of C spans two dims (n and h*w), which the tensor-core epilogue
    # addresses per row; the column walks one stride (h*w elements)
    n, c, h, w, N = 4, 64, 7, 7, 128
    A = dg.make_view(FAKE, (n, h, w, c), (c * h * w * 2, w * 2, 2, h * w * 2), 3, "bf16")
    B = dg.make_view(FAKE, (c, N), (N * 2, 2), 1, "bf16")
    C = dg.make_view(FAKE, (n, h, w, N), (N * h * w * 4, w * 4, 4, h * w * 4), 3, "f32")
    info = dg.dg_analyse_view(C)
    assert info.n_row == 2 and info.n_col == 1
    assert dg.dg_plan(A, B, C, 1.0, 0.0, False, 148).as_dict()["kind_name"] == "umma"
    # two dims along the other index of C (j) still go to the CUDA-core kernel
    Ct = dg.make_view(FAKE, (n * h * w, 2, N // 2), (4, n * h * w * 4 * (N // 2) + 64, n * h * w * 4), 1, "f32")
    assert dg.dg_analyse_view(Ct).n_col == 2
    assert dg.dg_plan(A, B, Ct, 1.0, 0.0, False, 148).as_dict()["kind_name"] == "simt"


def test_options():
    with pytest.raises(dg.DgError):
        dg.dg_set_option(dg.DG_OPT_FORCE_KIND, 99)
    with pytest.raises(dg.DgError):
        dg.dg_set_option(12345, 0)
    dg.dg_set_option(dg.DG_OPT_FORCE_KIND, dg.DG_KIND_SIMT)
    try:
        assert plan_of("small")["kind_name"] == "simt"
    finally:
        dg.dg_set_option(dg.DG_OPT_FORCE_KIND, 0)
    assert plan_of("small")["kind_name"] == "umma"
    dg.dg_set_option(dg.DG_OPT_EPI_TMA, 0)
    try:
        assert plan_of("small")["epi_tma_store"] == 0
    finally:
        dg.dg_set_option(dg.DG_OPT_EPI_TMA, 1)
    with pytest.raises(dg.DgError):
        dg.dg_set_option(dg.DG_OPT_EPI_TMA, 2)


# ------------------------------------------------------- plan invariants
#
# Random views (layouts, paddings, 4-D feature maps, misaligned pointers) through
# dg_plan, and the launch invariants the kernels are built on: tile shapes the
# tensor core accepts, cluster sizes within the portable limit, every split
# owning some k, co-resident split-K and gather clusters, CTA pairs on whole
# pairs of SMs.

ES = {"f32": 4, "f16": 2, "bf16": 2, "e4m3": 1}
SMS = 148


def _rand_dim(rng, small=False):
    if rng.random() < 0.5:
        pool = [1, 2, 3, 4, 5, 7, 8, 9, 16, 31, 32, 63, 64, 65, 96, 127, 128, 129, 200, 255, 256,
                257, 384, 512, 1000, 1024, 2048, 3136, 4096, 8192]
        if small:
            pool = [p for p in pool if p <= 1024]
        return rng.choice(pool)
    return rng.randint(1, 1200 if small else 5000)


def _matrix_view(rng, base, rows, cols, dt, allow_t=True):
    """A [rows x cols] view: row-major or transposed storage, padded leading
    dimension, sometimes an offset start."""
    es = ES[dt]
    pad = rng.choice([0, 0, 0, 0, 8, 3, 64])
    off = rng.choice([0, 0, 0, 0, 0, 1, 8]) * es
    if allow_t and rng.random() < 0.35:       # stored [cols x rows], viewed transposed
        ld = rows + pad
        return dg.make_view(base + off, (rows, cols), (es, ld * es), 1, dt)
    ld = cols + pad
    return dg.make_view(base + off, (rows, cols), (ld * es, es), 1, dt)


def _random_problem(rng):
    dt = rng.choice(["f16", "bf16", "bf16", "e4m3", "e4m3", "f32"])
    cdt = rng.choice(["f32", "bf16", "f16"])
    if rng.random() < 0.15:
        # an NCHW feature map read in place as [N*H*W, C]
        n, hw, c = rng.randint(1, 16), rng.choice([7, 14, 28]), rng.choice([3, 64, 96, 256])
        K, N = c, _rand_dim(rng, small=True)
        M = n * hw * hw
        es = ES[dt]
        A = dg.make_view(FAKE, (n, hw, hw, c), (c * hw * hw * es, hw * es, es, hw * hw * es), 3, dt)
    else:
        M, K, N = _rand_dim(rng), _rand_dim(rng), _rand_dim(rng)
        if rng.random() < 0.3:
            M = rng.randint(1, 8)             # decode-sized
        A = _matrix_view(rng, FAKE, M, K, dt)
    B = _matrix_view(rng, FAKE * 2, K, N, dt)
    C = _matrix_view(rng, FAKE * 3, M, N, cdt, allow_t=rng.random() < 0.2)
    alpha = rng.choice([1.0, 1.0, 2.0, 0.0]) if rng.random() < 0.1 else 1.0
    beta = rng.choice([0.0, 0.0, 1.0, 0.5])
    return dt, cdt, M, N, K, A, B, C, alpha, beta


def _check_plan(p, dt, M, N, K, alpha):
    kind = p["kind_name"]
    assert (p["M"], p["N"], p["K"]) == (M, N, K)
    if M == 0 or N == 0:
        assert kind == "none"
        return
    if alpha == 0.0 or K == 0:
        assert kind == "scale_c"
        return
    if dt == "f32":
        assert kind == "simt"
    if kind == "gemv_n":
        assert dt in ("f16", "bf16") and M <= 8
        r_inst = 1 if M <= 1 else 2 if M <= 2 else 4 if M <= 4 else 8
        S, kper = p["split_k"], p["block_k"]
        assert p["block_n"] == 256 and kper % 64 == 0 and 1 <= S <= 8
        assert (S - 1) * kper < K <= S * kper          # every k split owns some k
        assert kper * r_inst <= 16384                   # its slice of x fits in shared memory
        assert p["grid"] == -(-N // 256) * S
    elif kind == "gemv_k":
        r_inst = 1 if M <= 1 else 2 if M <= 2 else 4 if M <= 4 else 8
        assert dt in ("f16", "bf16") and M <= 8 and K % 8 == 0 and K * r_inst <= 32768
    elif kind == "umma":
        es = ES[dt]
        assert dt in ("f16", "bf16", "e4m3")
        bn, split, grid = p["block_n"], p["split_k"], p["grid"]
        # k per stage: one 128-byte sub-block, or two for CTA pairs with an
        # MN-major operand and K a whole number of such stages
        if p["block_k"] != 128 // es:
            assert p["cta_pair"] and p["block_k"] == 256 // es and K % p["block_k"] == 0
            assert p["p_mn_major"] or p["q_mn_major"]
        assert 16 <= bn <= 256 and bn % 16 == 0         # N of a 128-row tcgen05.mma
        if p["q_mn_major"]:
            assert bn % (128 // es) == 0                 # whole 128-byte boxes
        assert 1 <= split <= 8 and p["stages"] >= 2
        Mi, Nj = (N, M) if p["swap_ab"] else (M, N)
        tiles_j = -(-Nj // bn)
        tiles = -(-Mi // 128) * tiles_j
        assert 1 <= grid <= SMS
        if p["split_reduce_add"]:
            assert split > 1
        if split > 1:
            assert p["stages"] >= 3 and not p["cta_pair"] and p["gather_cluster"] == 1
            assert not p["epi_tma_store"]
            assert grid == tiles * split                 # one unit per CTA, all resident
            kb_total = -(-K // p["block_k"])
            kb_per = -(-kb_total // split)
            assert (split - 1) * kb_per < kb_total       # every k split owns some k
        if p["epi_tma_store"]:
            assert split == 1 and not p["swap_ab"]
        g = p["gather_cluster"]
        assert g in (1, 2, 4)
        if g > 1:
            assert p["p_gather"] and grid % g == 0 and tiles_j % g == 0
        if p["cta_pair"]:
            assert p["block_m"] == 256 and grid % 2 == 0 and bn >= 128 and split == 1
            assert 0 <= 2 * p["pair_half_tiles"] <= grid // 2
            sk, pairs = p["stream_k_tiles"], grid // 2
            assert not (sk and p["pair_half_tiles"])      # one tail treatment at a time
            if sk:
                pair_tiles = -(-Mi // 256) * tiles_j
                kb_total = -(-K // p["block_k"])
                assert sk == pair_tiles % pairs and pair_tiles > pairs   # the last, partial wave
                assert 7 * sk >= pairs                   # a tile is split among at most 8 pairs
                assert sk * kb_total >= pairs            # every pair gets at least one k block
        else:
            assert p["block_m"] == 128 and p["pair_half_tiles"] == 0 and p["stream_k_tiles"] == 0
        assert p["vec_bytes"] in (1, 2, 4, 8, 16)
        if not p["p_gather"]:
            assert p["vec_bytes"] == 16
    else:
        assert kind == "simt", kind


def test_plan_invariants_random_views():
    import random

    rng = random.Random(20261203)
    kinds = {}
    for n in range(3000):
        dt, cdt, M, N, K, A, B, C, alpha, beta = _random_problem(rng)
        dg.dg_set_option(dg.DG_OPT_STREAM_K, n % 2)      # half the draws with the opt-in Stream-K tail
        try:
            info = dg.dg_plan(A, B, C, alpha, beta, rng.random() < 0.3, SMS)
        except dg.DgError:
            continue                                     # a view the library rejects up front
        finally:
            dg.dg_set_option(dg.DG_OPT_STREAM_K, 0)
        p = info.as_dict()
        tags = [p["kind_name"]]
        if p["kind_name"] == "umma":
            tags += ["umma/pair"] * p["cta_pair"] + ["umma/split"] * (p["split_k"] > 1)
            tags += ["umma/stream_k"] * (p["stream_k_tiles"] > 0)
            tags += ["umma/gather_cluster"] * (p["gather_cluster"] > 1)
        for t in tags:
            kinds[t] = kinds.get(t, 0) + 1
        _check_plan(p, dt, M, N, K, alpha)
    # the draw reaches every kernel family and the tensor-core variants
    for k in ("gemv_n", "gemv_k", "umma", "simt", "umma/pair", "umma/split", "umma/gather_cluster", "umma/stream_k"):
        assert kinds.get(k, 0) >= 5, kinds


def test_plan_invariant_checks_reject_broken_plans():
    # the checks above are not vacuous: valid plans with one field broken fail them
    import random

    rng = random.Random(7)
    found = {}
    for _ in range(3000):
        dt, cdt, M, N, K, A, B, C, alpha, beta = _random_problem(rng)
        try:
            p = dg.dg_plan(A, B, C, alpha, beta, False, SMS).as_dict()
        except dg.DgError:
            continue
        key = "pair" if p["cta_pair"] else "split" if p["split_k"] > 1 else p["kind_name"]
        found.setdefault(key, (p, dt, M, N, K, alpha))
    breaks = {
        "pair": [("grid", lambda v: v - 1), ("block_n", lambda v: 64)],
        "split": [("split_k", lambda v: 9), ("grid", lambda v: v + 1), ("stages", lambda v: 2)],
        "gemv_n": [("block_k", lambda v: v - 64 if v > 64 else v + 1), ("split_k", lambda v: v + 1)],
        "umma": [("block_n", lambda v: v + 8), ("block_k", lambda v: 32)],
    }
    for key, muts in breaks.items():
        assert key in found, key
        p, dt, M, N, K, alpha = found[key]
        _check_plan(p, dt, M, N, K, alpha)
        for field, f in muts:
            q = dict(p)
            q[field] = f(p[field])
            with pytest.raises(AssertionError):
                _check_plan(q, dt, M, N, K, alpha)


def _offsets_by_dims(shape, stride, idx_dims):
    """Byte offset of a flat index unflattened row-major over the given dims."""
    def off(flat):
        o = 0
        for d in reversed(idx_dims):
            o += (flat % shape[d]) * stride[d]
            flat //= shape[d]
        return o
    return off


def test_analyse_random_views_address_the_same_elements():
    # Size-1 dims dropped and neighbours merged: the merged row and column
    # groups must reach exactly the bytes the original dims do (checked by
    # brute force on sampled (row, col) pairs), and the derived facts (extent,
    # span, unit-stride direction, TMA legality) must agree with the view.
    import random

    rng = random.Random(99)
    checked = 0
    for _ in range(600):
        dt = rng.choice(["f32", "f16", "bf16", "e4m3"])
        es = ES[dt]
        nd = rng.randint(1, 4)
        shape = [rng.choice([1, 1, 2, 3, 7, 14, 16, 64, 196]) for _ in range(nd)]
        # strides: mostly packed in some dim order (so that merges happen), at
        # times padded, broadcast (0) on size-1 dims
        order = list(range(nd))
        rng.shuffle(order)
        stride = [0] * nd
        run = es
        for d in reversed(order):
            stride[d] = run if shape[d] > 1 or rng.random() < 0.5 else 0
            run *= shape[d] + (rng.choice([0, 0, 0, 1, 8]) if rng.random() < 0.3 else 0)
        row_dims = rng.randint(0, nd) if nd > 1 else rng.randint(0, 1)
        ptr = FAKE + rng.choice([0, 0, 0, es, 8, 16])
        v = dg.make_view(ptr, shape, stride, row_dims, dt)
        try:
            info = dg.dg_analyse_view(v)
        except dg.DgError:
            continue
        rows = math_prod(shape[:row_dims])
        cols = math_prod(shape[row_dims:])
        assert (info.rows, info.cols) == (rows, cols)
        orig_r = _offsets_by_dims(shape, stride, list(range(row_dims)))
        orig_c = _offsets_by_dims(shape, stride, list(range(row_dims, nd)))
        m_r = _offsets_by_dims(list(info.row_shape), list(info.row_stride), list(range(info.n_row)))
        m_c = _offsets_by_dims(list(info.col_shape), list(info.col_stride), list(range(info.n_col)))
        assert math_prod(list(info.row_shape[:info.n_row])) == rows
        assert math_prod(list(info.col_shape[:info.n_col])) == cols
        for _ in range(40):
            r, c = rng.randrange(rows), rng.randrange(cols)
            assert m_r(r) + m_c(c) == orig_r(r) + orig_c(c), (shape, stride, row_dims, r, c)
        top = sum((s - 1) * st for s, st in zip(shape, stride))
        assert info.span_bytes == top + es
        if info.unit_dim == 1:
            assert info.n_col == 1 and info.col_stride[0] == es
        if info.unit_dim == 2:
            assert info.n_row == 1 and info.row_stride[0] == es
        if info.tma_ok:
            assert ptr % 16 == 0 and info.n_row <= 1 and info.n_col <= 1 and info.unit_dim in (1, 2)
            other = info.row_stride[0] if info.unit_dim == 1 else info.col_stride[0]
            assert info.n_row == 0 or info.n_col == 0 or other % 16 == 0
        assert info.vec_bytes in (1, 2, 4, 8, 16)
        checked += 1
    assert checked > 400


def math_prod(xs):
    p = 1
    for x in xs:
        p *= int(x)
    return p
