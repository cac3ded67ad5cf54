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
