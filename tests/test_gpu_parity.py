"""GPU parity: the CUDA path through the C ABI against the FP64 oracle.

Small problems are compared element by element (they span several tiles and
end in ragged tails).  The benchmark's full-size workloads, in the launch
configuration the benchmark uses, are compared element by element too, except
the two 4096^3 products, whose tile corners and random outputs are computed
one by one by the oracle.  Index and view handling is checked bit-exactly
with identity and permutation operands.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import tcgen05_tmem_gemm_b200 as dg
import workloads as W
from harness import c_matrix, check_full, check_sampled, compare, dg_view_of, plan, run, tile_corners, tolerance

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _reset_options():
    yield
    dg.dg_set_option(dg.DG_OPT_FORCE_KIND, 0)
    dg.dg_set_option(dg.DG_OPT_TEST_STALL, 0)
    dg.dg_set_option(dg.DG_OPT_WAIT_TIMEOUT_MS, 2000)
    dg.dg_set_option(dg.DG_OPT_MAX_SPLIT_K, 8)
    dg.dg_set_option(dg.DG_OPT_CTA_PAIR, 1)
    dg.dg_set_option(dg.DG_OPT_EARLY_LAUNCH, 3)
    dg.dg_set_option(dg.DG_OPT_EPI_TMA, 1)
    dg.dg_set_option(dg.DG_OPT_GATHER_CLUSTER, 1)
    dg.dg_set_option(dg.DG_OPT_PAIR_TAIL, 1)
    dg.dg_set_option(dg.DG_OPT_DETERMINISTIC, 0)
    dg.dg_set_option(dg.DG_OPT_PAIR_DEEP_STAGES, 1)


def expect_kind(p, kind, **fields):
    pl = plan(p.to("cuda"))
    assert pl["kind_name"] == kind, pl
    for k, v in fields.items():
        assert pl[k] == v, (k, pl)
    return pl


# ------------------------------------------------------------ small, full compare

def test_small_config_full():
    p = W.cfg_small()
    expect_kind(p, "umma")
    check_full(p)


@pytest.mark.parametrize("M,N,K", [(300, 520, 200), (129, 136, 72), (16, 16, 16), (1000, 264, 1000)])
@pytest.mark.parametrize("dt,out", [("bf16", "bf16"), ("f16", "f32"), ("bf16", "f32")])
def test_umma_row_major_ragged(M, N, K, dt, out):
    g = torch.Generator().manual_seed(M * 7 + N + K)
    A = W.cast(W.normal((M, K), g), dt)
    B = W.cast(W.normal((K, N), g), dt)
    p = W.Problem(f"rm_{M}x{N}x{K}_{dt}_{out}", W.row_major(A, dt), W.row_major(B, dt), W.empty_out(M, N, out))
    expect_kind(p, "umma")
    check_full(p)


@pytest.mark.parametrize("ta,tb", [(True, False), (False, True), (True, True)])
def test_umma_transposed_operands(ta, tb):
    # A given as the transpose of an [K, M] tensor (M-major), B as the transpose of [N, K] (K-major)
    M, N, K = 264, 200, 136
    g = torch.Generator().manual_seed(17)
    a = W.cast(W.uniform((K, M) if ta else (M, K), g), "bf16")
    b = W.cast(W.uniform((N, K) if tb else (K, N), g), "bf16")
    A = W.transposed(a, "bf16") if ta else W.row_major(a, "bf16")
    B = W.transposed(b, "bf16") if tb else W.row_major(b, "bf16")
    p = W.Problem("transposed", A, B, W.empty_out(M, N, "f32"))
    expect_kind(p, "umma", p_mn_major=int(ta), q_mn_major=int(not tb))
    check_full(p)


@pytest.mark.parametrize("ta,pair", [(True, 0), (False, 0), (True, 2)])
def test_umma_mn_major_chunk_boxes(ta, pair):
    # MN-major operands in 128-byte chunk boxes whose last tiles run past M
    # and N: the trailing boxes are partly or wholly outside the tensor (zero fill).
    M, N, K = (1280, 320, 200) if pair == 0 else (320, 192, 200)
    g = torch.Generator().manual_seed(320 + int(ta) + pair)
    a = W.cast(W.uniform((K, M) if ta else (M, K), g), "bf16")
    b = W.cast(W.uniform((K, N), g), "bf16")
    A = W.transposed(a, "bf16") if ta else W.row_major(a, "bf16")
    p = W.Problem("chunks3d", A, W.row_major(b, "bf16"), W.empty_out(M, N, "f32"))
    dg.dg_set_option(dg.DG_OPT_CTA_PAIR, pair)
    expect_kind(p, "umma", p_mn_major=int(ta), q_mn_major=1, cta_pair=int(pair == 2))
    check_full(p)


@pytest.mark.parametrize("M,N,K", [(300, 384, 272), (128, 128, 128), (77, 256, 512)])
def test_umma_fp8_scaled(M, N, K):
    g = torch.Generator().manual_seed(M + N + K)
    qa, sa = W.quantise_e4m3(W.normal((M, K), g), dim=1)
    qb, sb = W.quantise_e4m3(W.normal((K, N), g), dim=0)
    p = W.Problem("fp8", W.row_major(qa, "e4m3"), W.row_major(qb, "e4m3"), W.empty_out(M, N, "bf16"),
                  1.0, 0.0, sa, sb)
    expect_kind(p, "umma", block_k=128)
    check_full(p)


def test_fp8_k_major_b():
    M, N, K = 200, 144, 256
    g = torch.Generator().manual_seed(5)
    qa, sa = W.quantise_e4m3(W.normal((M, K), g), dim=1)
    qbt, sb = W.quantise_e4m3(W.normal((N, K), g), dim=1)  # B^T stored [N, K]
    p = W.Problem("fp8_kmajor", W.row_major(qa, "e4m3"), W.transposed(qbt, "e4m3"), W.empty_out(M, N, "f32"),
                  0.5, 0.0, sa, sb)
    expect_kind(p, "umma", q_mn_major=0)
    check_full(p)


@pytest.mark.parametrize("M,N,K,dt,out,ta,tb", [
    (300, 520, 200, "bf16", "bf16", False, False),
    (1000, 264, 1000, "f16", "f32", False, False),
    (264, 200, 136, "bf16", "f32", True, False),
    (520, 256, 64, "bf16", "bf16", False, True),
    (256, 128, 16, "f16", "f16", False, False),
])
def test_umma_cta_pair_forced(M, N, K, dt, out, ta, tb):
    # two CTAs of a cluster share each 256-row tile (tcgen05 cta_group::2); pairs
    # take no split-K, so split-K is switched off for these shapes
    dg.dg_set_option(dg.DG_OPT_CTA_PAIR, 2)
    dg.dg_set_option(dg.DG_OPT_MAX_SPLIT_K, 1)
    g = torch.Generator().manual_seed(M + 3 * N + K)
    a = W.cast(W.normal((K, M) if ta else (M, K), g), dt)
    b = W.cast(W.normal((N, K) if tb else (K, N), g), dt)
    A = W.transposed(a, dt) if ta else W.row_major(a, dt)
    B = W.transposed(b, dt) if tb else W.row_major(b, dt)
    c = W.uniform((M, N), g)
    p = W.Problem("pair", A, B, W.row_major(c.to(W.TORCH_DTYPE[out]).contiguous(), out), 0.75, 0.5)
    expect_kind(p, "umma", cta_pair=1, block_m=256)
    check_full(p)


@pytest.mark.parametrize("tb", [False, True])
def test_cta_pair_half_width_tail(tb):
    # 10 x 8 = 80 pair tiles on 74 pairs: the last 6 run as 12 half-width
    # tiles.  Whole and split tails do the same arithmetic per output, so the
    # results agree bit for bit; each is also checked against the oracle.
    M, N, K = 2560, 2048, 192
    g = torch.Generator().manual_seed(2560 + int(tb))
    a = W.cast(W.normal((M, K), g), "bf16")
    b = W.cast(W.normal((N, K) if tb else (K, N), g), "bf16")
    B = W.transposed(b, "bf16") if tb else W.row_major(b, "bf16")
    p = W.Problem("pair_tail", W.row_major(a, "bf16"), B, W.empty_out(M, N, "f32"))
    if torch.cuda.get_device_properties(0).multi_processor_count != 148:
        pytest.skip("the tail size is worked out for 148 SMs")
    outs = []
    for tail in (1, 0):
        dg.dg_set_option(dg.DG_OPT_PAIR_TAIL, tail)
        expect_kind(p, "umma", cta_pair=1, pair_half_tiles=6 if tail else 0, q_mn_major=int(not tb))
        check_full(p)
        outs.append(c_matrix(run(p.to("cuda"))))
    assert np.array_equal(outs[0], outs[1])


def test_umma_cta_pair_fp8():
    dg.dg_set_option(dg.DG_OPT_CTA_PAIR, 2)
    dg.dg_set_option(dg.DG_OPT_MAX_SPLIT_K, 1)
    M, N, K = 384, 256, 384
    g = torch.Generator().manual_seed(77)
    qa, sa = W.quantise_e4m3(W.normal((M, K), g), dim=1)
    qbt, sb = W.quantise_e4m3(W.normal((N, K), g), dim=1)
    p = W.Problem("pair_fp8", W.row_major(qa, "e4m3"), W.transposed(qbt, "e4m3"), W.empty_out(M, N, "bf16"),
                  1.0, 0.0, sa, sb)
    expect_kind(p, "umma", cta_pair=1)
    check_full(p)


def _pair_deep_problem(case):
    g = torch.Generator().manual_seed(sum(map(ord, case)))
    if case == "e4m3_b_mn":
        # tiles 256 wide (a CTA's half of an MN-major E4M3 tile is one 128-byte box)
        M, N, K = 2560, 1024, 512
        qa, sa = W.quantise_e4m3(W.normal((M, K), g), dim=1)
        qb, sb = W.quantise_e4m3(W.normal((K, N), g), dim=0)
        return W.Problem(case, W.row_major(qa, "e4m3"), W.row_major(qb, "e4m3"), W.empty_out(M, N, "bf16"),
                         1.0, 0.0, sa, sb), 1
    ta = case in ("bf16_a_mn", "bf16_a_mn_b_k")
    tb = case == "bf16_a_mn_b_k"
    M, N, K = {"ragged": (300, 520, 256), "half_tail": (2560, 2048, 256)}.get(case, (512, 512, 384))
    a = W.cast(W.normal((K, M) if ta else (M, K), g), "bf16")
    b = W.cast(W.normal((N, K) if tb else (K, N), g), "bf16")
    A = W.transposed(a, "bf16") if ta else W.row_major(a, "bf16")
    B = W.transposed(b, "bf16") if tb else W.row_major(b, "bf16")
    if case == "ragged":
        c = W.uniform((M, N), g)
        return W.Problem(case, A, B, W.row_major(c.to(torch.bfloat16).contiguous(), "bf16"), 0.75, 0.5), 2
    return W.Problem(case, A, B, W.empty_out(M, N, "f32")), 2


@pytest.mark.parametrize("case", ["bf16_b_mn", "bf16_a_mn", "bf16_a_mn_b_k", "e4m3_b_mn", "ragged", "half_tail"])
def test_pair_deep_stages_match_shallow(case):
    # CTA-pair stages two 128-byte k sub-blocks deep (taller MN-major boxes)
    # issue the same MMAs in the same k order as stages one sub-block deep,
    # so the results agree bit for bit; each is also checked against the oracle
    p, es = _pair_deep_problem(case)
    if case == "half_tail":
        if torch.cuda.get_device_properties(0).multi_processor_count != 148:
            pytest.skip("the tail size is worked out for 148 SMs")
    else:
        dg.dg_set_option(dg.DG_OPT_CTA_PAIR, 2)
        dg.dg_set_option(dg.DG_OPT_MAX_SPLIT_K, 1)
    outs = []
    for deep in (1, 0):
        dg.dg_set_option(dg.DG_OPT_PAIR_DEEP_STAGES, deep)
        pl = expect_kind(p, "umma", cta_pair=1, block_k=(2 if deep else 1) * 128 // es)
        if case == "half_tail":
            assert pl["pair_half_tiles"] == 6
        check_full(p)
        outs.append(c_matrix(run(p.to("cuda"))))
    assert np.array_equal(outs[0], outs[1])


def test_thin_beta_one_split_k():
    p = W.cfg_thin(M=40, N=1000, K=784)
    pl = expect_kind(p, "umma", swap_ab=1)
    assert pl["split_k"] > 1
    check_full(p)


@pytest.mark.parametrize("deterministic", [1, 0])
@pytest.mark.parametrize("case", ["s8_ragged_rows", "s3_rows_not_multiple_of_4", "s2_bf16_out", "fp8_scales",
                                  "no_swap_row_major_c"])
def test_split_k_cluster_reduction(case, deterministic):
    # Every path of the on-chip split-K reduction: four-row vector steps with
    # a ragged last row group, the element-wise path (S = 3, BF16 output, C
    # row-major along j) and per-row / per-column scales.  With beta = 1 and
    # FP32 C the default adds the splits' partials straight into C instead
    # (tensor reduce-adds along i when swapped, along j otherwise);
    # deterministic = 1 keeps the cluster reduction for those cases too.
    dg.dg_set_option(dg.DG_OPT_DETERMINISTIC, deterministic)
    g = torch.Generator().manual_seed(len(case) * 31)
    ms, out, beta = 8, "f32", 1.0
    if case == "s8_ragged_rows":
        M, N, K = 64, 1001, 4096
    elif case == "s3_rows_not_multiple_of_4":
        M, N, K, ms = 48, 1000, 2048, 3
    elif case == "s2_bf16_out":
        M, N, K, ms, out, beta = 64, 512, 2048, 2, "bf16", 0.0
    elif case == "fp8_scales":
        M, N, K, out, beta = 32, 1024, 4096, "bf16", 0.0
    else:
        M, N, K = 256, 128, 8192
    dg.dg_set_option(dg.DG_OPT_MAX_SPLIT_K, ms)
    if case == "fp8_scales":
        qa, sa = W.quantise_e4m3(W.normal((M, K), g), dim=1)
        qb, sb = W.quantise_e4m3(W.normal((K, N), g), dim=0)
        p = W.Problem(case, W.row_major(qa, "e4m3"), W.row_major(qb, "e4m3"), W.empty_out(M, N, out),
                      1.0, beta, sa, sb)
    else:
        A = W.row_major(W.cast(W.normal((M, K), g), "f16"), "f16")
        # B read K-major from an [N, K] tensor, so N needs no alignment
        B = W.transposed(W.cast(W.normal((N, K), g, 0.05), "f16"), "f16")
        C = W.row_major(W.uniform((M, N), g), "f32") if out == "f32" else W.empty_out(M, N, out)
        p = W.Problem(case, A, B, C, 1.0, beta)
    pl = expect_kind(p, "umma")
    assert pl["split_k"] > 1 and pl["epi_tma_store"] == 0, pl
    # adding into C needs one 2-D tensor map of C (16-byte multiple row stride: not N = 1001)
    c_map_ok = dg.dg_analyse_view(dg_view_of(p.C)).tma_ok == 1
    assert pl["split_reduce_add"] == int(beta == 1.0 and out == "f32" and not deterministic and c_map_ok), pl
    if case == "s3_rows_not_multiple_of_4":
        assert pl["split_k"] == 3
    if case == "no_swap_row_major_c":
        assert pl["swap_ab"] == 0
    check_full(p)


@pytest.mark.parametrize("M,N,K", [(64, 4096, 2048), (40, 1000, 784), (7, 300, 4096)])
def test_split_k_reduce_add_into_c(M, N, K):
    # beta = 1, FP32 C: every split adds alpha * partial into C in the memory
    # system; against the oracle, and against the fixed-order cluster
    # reduction within the tolerance (the order of the adds differs)
    p = W.cfg_thin(M=M, N=N, K=K)
    pl = expect_kind(p, "umma", swap_ab=1)
    assert pl["split_k"] > 1 and pl["split_reduce_add"] == 1, pl
    check_full(p)
    a = c_matrix(run(p.to("cuda")))
    dg.dg_set_option(dg.DG_OPT_DETERMINISTIC, 1)
    assert expect_kind(p, "umma")["split_reduce_add"] == 0
    b = c_matrix(run(p.to("cuda")))
    assert np.allclose(a, b, rtol=1e-5, atol=1e-4)


def test_thin_without_split_k_matches():
    dg.dg_set_option(dg.DG_OPT_MAX_SPLIT_K, 1)
    p = W.cfg_thin(M=64, N=512, K=1024)
    expect_kind(p, "umma", swap_ab=1, split_k=1)
    check_full(p)


@pytest.mark.parametrize("n,c,h,w,N", [(3, 72, 14, 14, 200), (2, 40, 9, 11, 72), (1, 256, 14, 14, 1024)])
def test_strided_nchw_gather(n, c, h, w, N):
    p = W.cfg_strided(n=n, c=c, h=h, w=w, N=N)
    expect_kind(p, "umma", p_gather=1, p_mn_major=1)
    check_full(p)


@pytest.mark.parametrize("n,c,h,w,N,cluster", [(3, 72, 14, 14, 200, 2), (1, 256, 14, 14, 1024, 4),
                                                (2, 40, 10, 10, 1024, 4), (4, 128, 6, 6, 512, 4),
                                                (2, 64, 7, 2, 512, 4)])
def test_strided_gather_cluster_matches_single_cta_gather(n, c, h, w, N, cluster):
    # CTAs sharing an A tile each gather a k-slice of every stage and copy it
    # to the others; the tensor core then reads the same bytes as when every
    # CTA gathers the whole tile, so the outputs agree bit for bit.
    g = torch.Generator().manual_seed(n * c + N)
    x = W.cast(W.uniform((n, c, h, w), g), "bf16")
    B = W.cast(W.uniform((c, N), g), "bf16")
    p = W.Problem("nchw", W.nchw_as_rows(x, "bf16"), W.row_major(B, "bf16"), W.empty_out(n * h * w, N, "f32"))
    outs = []
    for on in (1, 0):
        dg.dg_set_option(dg.DG_OPT_GATHER_CLUSTER, on)
        expect_kind(p, "umma", p_gather=1, gather_cluster=cluster if on else 1)
        check_full(p)
        outs.append(c_matrix(run(p.to("cuda"))))
    assert np.array_equal(outs[0], outs[1])


def test_gemv_shapes():
    for p in (W.cfg_gemv(K=1000, N=1032), W.cfg_gemv(K=4096, N=4096), W.cfg_gemv(K=8, N=8)):
        expect_kind(p, "gemv_n")
        check_full(p)
    for p in (W.cfg_gemv_kt(K=1032, N=77), W.cfg_gemv_kt(K=4096, N=128)):
        expect_kind(p, "gemv_k")
        check_full(p)


@pytest.mark.parametrize("R", [2, 3, 8])
def test_gemv_multi_row(R):
    g = torch.Generator().manual_seed(R)
    x = W.cast(W.normal((R, 1536), g), "f16")
    Wt = W.cast(W.normal((1536, 520), g, 0.05), "f16")
    C = W.uniform((R, 520), g).contiguous()
    p = W.Problem("gemv_rows", W.row_major(x, "f16"), W.row_major(Wt, "f16"), W.row_major(C, "f32"), 0.5, -2.0)
    expect_kind(p, "gemv_n")
    check_full(p)


def test_dg_gemv_entry_point():
    p = W.cfg_gemv(K=512, N=256).to("cuda")
    x = dg.make_view(p.A.base.data_ptr(), (512,), (2,), 0, "bf16")  # a 1-D view is one row
    st = dg.dg_gemv(x, dg_view_of(p.B), dg_view_of(p.C), 1.0, 0.0)
    assert st == dg.DG_OK and dg.dg_sync_status() == dg.DG_OK
    ref, bound = oracle.gemm(p.to("cpu"))
    compare(p, c_matrix(p), ref, bound, where="dg_gemv")


@pytest.mark.parametrize("name", ["small", "gemv", "gemv_kt", "thin", "strided"])
def test_forced_simt_path(name):
    dg.dg_set_option(dg.DG_OPT_FORCE_KIND, dg.DG_KIND_SIMT)
    kw = {"small": {}, "gemv": {"K": 512, "N": 264}, "gemv_kt": {"K": 512, "N": 40},
          "thin": {"M": 40, "N": 264, "K": 300}, "strided": {"n": 2, "c": 40, "h": 9, "w": 11, "N": 72}}[name]
    p = W.WORKLOADS[name](**kw)
    expect_kind(p, "simt")
    check_full(p)


def test_f32_inputs_simt():
    g = torch.Generator().manual_seed(3)
    q = W.normal((128 * 49,), g)
    k = W.normal((128 * 49,), g)
    Q = W.Operand(q, (1, 128, 7, 7), (0, 196, 28, 4), 2, "f32")
    KT = W.Operand(k, (7, 7, 1, 128), (28, 4, 0, 196), 2, "f32")
    p = W.Problem("pages_strided_fp32", Q, KT, W.empty_out(128, 128, "f32"))
    expect_kind(p, "simt")
    check_full(p)


# --------------------------------------------------------------- bit-exact

def test_identity_gathers_strided_a_exactly():
    # C = A * I with A the NCHW view: products by 1 and sums with 0 are exact,
    # so the output must equal the gathered A bit for bit.
    p = W.cfg_strided(n=2, c=64, h=14, w=14, N=64)
    eye = torch.eye(64, dtype=torch.bfloat16)
    p = W.Problem("identity", p.A, W.row_major(eye, "bf16"), W.empty_out(p.M, 64, "f32"))
    expect_kind(p, "umma", p_gather=1)
    gpu = run(p.to("cuda"))
    got = c_matrix(gpu)
    x = p.A.base  # [n, c, h, w]
    want = x.permute(0, 2, 3, 1).reshape(-1, 64).to(torch.float64).numpy()
    assert np.array_equal(got, want)


@pytest.mark.parametrize("kind", ["umma", "simt"])
def test_permutation_exact(kind):
    if kind == "simt":
        dg.dg_set_option(dg.DG_OPT_FORCE_KIND, dg.DG_KIND_SIMT)
    g = torch.Generator().manual_seed(11)
    M, K = 256, 128
    a = W.cast(W.uniform((M, K), g), "bf16")
    perm = torch.randperm(K, generator=g)
    P = torch.zeros(K, K, dtype=torch.bfloat16)
    P[perm, torch.arange(K)] = 1
    p = W.Problem("perm", W.row_major(a, "bf16"), W.row_major(P, "bf16"), W.empty_out(M, K, "f32"))
    expect_kind(p, kind)
    got = c_matrix(run(p.to("cuda")))
    assert np.array_equal(got, a.to(torch.float64).numpy()[:, perm.numpy()])


# ----------------------------------------------------------------- edge cases

def test_empty_and_k_zero():
    for (M, N, K) in ((0, 16, 16), (16, 0, 16)):
        A = W.row_major(torch.zeros(M, K, dtype=torch.bfloat16), "bf16")
        B = W.row_major(torch.zeros(K, N, dtype=torch.bfloat16), "bf16")
        p = W.Problem("empty", A, B, W.empty_out(M, N, "f32")).to("cuda")
        run(p)
    c = torch.arange(48, dtype=torch.float32).reshape(6, 8)
    A = W.Operand(torch.zeros(8, dtype=torch.bfloat16), (6, 0), (0, 2), 1, "bf16")
    B = W.Operand(torch.zeros(8, dtype=torch.bfloat16), (0, 8), (16, 2), 1, "bf16")
    p = W.Problem("k0", A, B, W.row_major(c.clone(), "f32"), 1.0, 3.0).to("cuda")
    run(p)
    assert np.array_equal(c_matrix(p), 3.0 * c.double().numpy())


def test_alpha_zero_never_reads_a():
    M, N, K = 64, 96, 80
    a = torch.full((M, K), float("inf")).to(torch.bfloat16)
    b = torch.ones(K, N, dtype=torch.bfloat16)
    c = torch.arange(M * N, dtype=torch.float32).reshape(M, N) / 7
    p = W.Problem("alpha0", W.row_major(a, "bf16"), W.row_major(b, "bf16"), W.row_major(c.clone(), "f32"),
                  0.0, -0.5).to("cuda")
    run(p)
    assert np.array_equal(c_matrix(p), (-0.5 * c).double().numpy())


@pytest.mark.parametrize("kind", ["umma", "gemv_n", "simt"])
def test_beta_zero_ignores_nan_c_and_nan_propagates(kind):
    M = 4 if kind == "gemv_n" else 200
    N, K = 136, 96
    if kind == "simt":
        dg.dg_set_option(dg.DG_OPT_FORCE_KIND, dg.DG_KIND_SIMT)
    g = torch.Generator().manual_seed(1)
    a = W.cast(W.uniform((M, K), g), "bf16")
    a[1, 5] = float("nan")
    b = W.cast(W.uniform((K, N), g), "bf16")
    b[7, 3] = float("inf")
    p = W.Problem("nan", W.row_major(a, "bf16"), W.row_major(b, "bf16"), W.empty_out(M, N, "f32"))
    expect_kind(p, kind)
    check_full(p)


def test_scales_applied_once():
    M, N, K = 256, 256, 128
    a = torch.ones(M, K).to(torch.float8_e4m3fn)
    b = torch.ones(K, N).to(torch.float8_e4m3fn)
    sa = torch.tensor([2.0 ** (j % 5 - 2) for j in range(M)])
    sb = torch.tensor([2.0 ** (-(j % 3)) for j in range(N)])
    p = W.Problem("scales", W.row_major(a, "e4m3"), W.row_major(b, "e4m3"), W.empty_out(M, N, "f32"),
                  1.0, 0.0, sa, sb)
    got = c_matrix(run(p.to("cuda")))
    assert np.array_equal(got, K * np.outer(sa.numpy(), sb.numpy()))


@pytest.mark.parametrize("M,N,K,dt,out,pair", [
    (300, 520, 200, "bf16", "bf16", 0),   # ragged rows and columns, 16-bit blocks of 64 columns
    (129, 136, 72, "f16", "f32", 0),      # one row past a tile, FP32 blocks of 32 columns
    (520, 384, 128, "bf16", "f32", 2),    # CTA pairs
    (256, 256, 64, "e4m3", "bf16", 0),    # per-row / per-column scales in the block packing
])
def test_epilogue_tensor_stores_match_thread_stores(M, N, K, dt, out, pair):
    # The two epilogues do the same arithmetic in the same order, so their
    # outputs agree bit for bit; each is also checked against the oracle.
    g = torch.Generator().manual_seed(M + 3 * N + K)
    if dt == "e4m3":
        qa, sa = W.quantise_e4m3(W.normal((M, K), g), dim=1)
        qb, sb = W.quantise_e4m3(W.normal((K, N), g), dim=0)
        p = W.Problem("epi_fp8", W.row_major(qa, "e4m3"), W.row_major(qb, "e4m3"), W.empty_out(M, N, out),
                      1.5, 0.0, sa, sb)
    else:
        A = W.cast(W.normal((M, K), g), dt)
        B = W.cast(W.normal((K, N), g), dt)
        p = W.Problem("epi", W.row_major(A, dt), W.row_major(B, dt), W.empty_out(M, N, out), 0.75, 0.0)
    dg.dg_set_option(dg.DG_OPT_CTA_PAIR, pair)
    outs = []
    for tma in (1, 0):
        dg.dg_set_option(dg.DG_OPT_EPI_TMA, tma)
        expect_kind(p, "umma", epi_tma_store=tma, cta_pair=int(pair == 2))
        check_full(p)
        outs.append(c_matrix(run(p.to("cuda"))))
    assert np.array_equal(outs[0], outs[1])


def test_epilogue_tensor_stores_need_beta_zero_and_row_major_c():
    M, N, K = 256, 256, 64
    g = torch.Generator().manual_seed(5)
    A = W.row_major(W.cast(W.uniform((M, K), g), "bf16"), "bf16")
    B = W.row_major(W.cast(W.uniform((K, N), g), "bf16"), "bf16")
    c = W.uniform((M, N), g)
    expect_kind(W.Problem("b0", A, B, W.row_major(c, "f32"), 1.0, 0.0), "umma", epi_tma_store=1)
    expect_kind(W.Problem("b1", A, B, W.row_major(c, "f32"), 1.0, 1.0), "umma", epi_tma_store=0)
    expect_kind(W.Problem("ct", A, B, W.transposed(c.t().contiguous(), "f32"), 1.0, 0.0), "umma",
                epi_tma_store=0)


def test_output_guard_band_untouched():
    M, N, K = 130, 72, 64
    g = torch.Generator().manual_seed(8)
    a = W.cast(W.uniform((M, K), g), "f16")
    b = W.cast(W.uniform((K, N), g), "f16")
    ld = N + 24  # C embedded in a wider buffer, canaries on both sides
    buf = torch.full((M + 2, ld), 12345.0)
    C = W.Operand(buf, (M, N), (ld * 4, 4), 1, "f32", offset=(ld + 8) * 4)
    p = W.Problem("guard", W.row_major(a, "f16"), W.row_major(b, "f16"), C)
    gpu = run(p.to("cuda"))
    out = gpu.C.base.cpu()
    mask = torch.ones_like(out, dtype=torch.bool)
    mask[1:M + 1, 8:8 + N] = False
    assert torch.all(out[mask] == 12345.0)
    ref, bound = oracle.gemm(p)
    compare(p, c_matrix(gpu), ref, bound, where="guard")


def test_pointer_and_value_errors():
    p = W.cfg_small(M=16, N=16, K=16)
    A, B, C = (dg.make_view(o.base.data_ptr(), o.shape, o.stride, o.row_dims, o.dtype) for o in (p.A, p.B, p.C))
    assert dg.dg_gemm(A, B, C, 1.0, 0.0) == dg.DG_ERR_POINTER  # host memory
    gp = p.to("cuda")
    A, B, C = dg_view_of(gp.A), dg_view_of(gp.B), dg_view_of(gp.C)
    assert dg.dg_gemm(A, B, C, math.nan, 0.0) == dg.DG_ERR_VALUE
    assert dg.dg_sync_status() == dg.DG_OK


def test_bounded_wait_reports_timeout_and_recovers():
    # The loader issues no copies, so the MMA issuer's wait runs out after the
    # bound; the kernel records the timeout, frees TMEM and returns.
    p = W.cfg_small(M=128, N=128, K=256).to("cuda")
    dg.dg_set_option(dg.DG_OPT_WAIT_TIMEOUT_MS, 300)
    dg.dg_set_option(dg.DG_OPT_TEST_STALL, 1)
    A, B, C = dg_view_of(p.A), dg_view_of(p.B), dg_view_of(p.C)
    assert dg.dg_gemm(A, B, C, 1.0, 0.0) == dg.DG_OK
    assert dg.dg_sync_status() == dg.DG_ERR_TIMEOUT
    dg.dg_set_option(dg.DG_OPT_TEST_STALL, 0)
    check_full(W.cfg_small())


def test_split_k_exchange_wait_reports_timeout_and_recovers():
    # stall mode 2: the main loops run, but no CTA of a split-K cluster sends
    # its slices, so every owner's wait for them runs out; the kernel records
    # the timeout and every CTA still reaches the end of the kernel (no slice
    # copy is in flight), and the next call is correct
    p = W.cfg_thin(M=40, N=1000, K=784)
    pl = expect_kind(p, "umma", swap_ab=1)
    assert pl["split_k"] > 1
    dg.dg_set_option(dg.DG_OPT_DETERMINISTIC, 1)  # the cluster exchange (beta = 1 would add into C)
    assert expect_kind(p, "umma")["split_reduce_add"] == 0
    g = p.to("cuda")
    dg.dg_set_option(dg.DG_OPT_WAIT_TIMEOUT_MS, 300)
    dg.dg_set_option(dg.DG_OPT_TEST_STALL, 2)
    A, B, C = dg_view_of(g.A), dg_view_of(g.B), dg_view_of(g.C)
    assert dg.dg_gemm(A, B, C, g.alpha, g.beta) == dg.DG_OK
    assert dg.dg_sync_status() == dg.DG_ERR_TIMEOUT
    dg.dg_set_option(dg.DG_OPT_TEST_STALL, 0)
    check_full(p)


@pytest.mark.parametrize("mode", [0, 1, 2, 3])
def test_early_launch_modes_back_to_back(mode):
    # Programmatic dependent launch lets a kernel start before the previous one
    # in the stream has finished; every kernel waits for it before touching
    # memory.  Chained calls where each reads the previous one's output must
    # still see it: y1 = x W1, then C = A(y1 rows) B, then y2 = x W2 on y1's
    # buffer again, all queued back to back.
    dg.dg_set_option(dg.DG_OPT_EARLY_LAUNCH, mode)
    g = torch.Generator().manual_seed(77 + mode)
    K, N = 512, 256
    x = W.cast(W.normal((1, K), g), "bf16").cuda()
    w1 = W.cast(W.normal((K, N), g, 0.05), "bf16").cuda()
    y1 = torch.empty((1, N), dtype=torch.bfloat16, device="cuda")
    b = W.cast(W.normal((N, 64), g, 0.05), "bf16").cuda()
    c = torch.empty((1, 64), dtype=torch.float32, device="cuda")
    for _ in range(3):
        dg.gemm(x, w1, y1)           # gemv_n
        dg.gemm(y1, b, c)            # reads y1 right away (gemv_n again, N = 64)
    torch.cuda.synchronize()
    assert dg.dg_sync_status() == dg.DG_OK
    ref1 = x.double().cpu() @ w1.double().cpu()
    got1 = y1.double().cpu()
    assert torch.allclose(got1, ref1, rtol=1e-2, atol=1e-2)
    ref2 = got1 @ b.double().cpu()   # from the y1 the GPU produced (its BF16 rounding included)
    assert torch.allclose(c.double().cpu(), ref2, rtol=1e-3, atol=1e-3)


@pytest.mark.parametrize("mode", [0, 1, 2, 3])
def test_early_launch_tensor_core_chain(mode):
    # The same for the tensor-core kernels: a CTA-pair GEMM, split-K clusters
    # and a single-CTA GEMM, each reading an output of the calls just before
    # it, and the first operand written by a torch kernel right before the
    # first call.  The buffers are rewritten every round while the calls of
    # the round before may still be in flight; the rounds scale A by 1, 2 and
    # 4 (exact in BF16), so a stale operand is off by a factor of two.
    dg.dg_set_option(dg.DG_OPT_EARLY_LAUNCH, mode)
    g = torch.Generator().manual_seed(123 + mode)
    bf = torch.bfloat16
    a = W.cast(W.normal((2048, 1024), g), "bf16").cuda()
    b1 = W.cast(W.normal((1024, 4096), g, 0.05), "bf16").cuda()
    b2 = W.cast(W.normal((4096, 2048), g, 0.05), "bf16").cuda()
    b3 = W.cast(W.normal((256, 512), g, 0.05), "bf16").cuda()
    b4 = W.cast(W.normal((2048, 256), g, 0.05), "bf16").cuda()
    a_r = torch.empty_like(a)
    c1 = torch.empty((2048, 4096), dtype=bf, device="cuda")
    c2 = torch.empty((64, 2048), dtype=bf, device="cuda")
    plans = [dg.dg_plan(dg.view(x), dg.view(y), dg.view(z)).as_dict() for x, y, z in
             [(a_r, b1, c1), (c1[:64], b2, c2), (c1[:512, :256], b3, torch.empty((512, 512), device="cuda")),
              (c2, b4, torch.empty((64, 256), device="cuda"))]]
    assert plans[0]["cta_pair"] == 1 and plans[1]["split_k"] > 1 and plans[3]["split_k"] > 1
    assert plans[2]["cta_pair"] == 0 and plans[2]["split_k"] == 1
    outs = []
    for r in range(3):
        torch.mul(a, float(2 ** r), out=a_r)
        dg.gemm(a_r, b1, c1)                     # CTA pair, reads a_r at once
        dg.gemm(c1[:64], b2, c2)                 # split-K cluster, reads c1 at once
        c3 = torch.empty((512, 512), dtype=torch.float32, device="cuda")
        dg.gemm(c1[:512, :256], b3, c3)          # single CTA, reads c1 in place
        c4 = torch.empty((64, 256), dtype=torch.float32, device="cuda")
        dg.gemm(c2, b4, c4)                      # split-K cluster, reads c2 at once
        outs.append((float(2 ** r), c1.clone(), c2.clone(), c3, c4))
    torch.cuda.synchronize()
    assert dg.dg_sync_status() == dg.DG_OK

    def check(got, x, y, out):
        # the parity suite's bound: S = |x| |y| summed over k
        ref, bound = (x @ y).numpy(), (x.abs() @ y.abs()).numpy()
        err = np.abs(got.double().cpu().numpy() - ref)
        assert (err <= tolerance(out, ref, bound, np.zeros_like(ref))).all(), float(err.max())

    a_d, b1_d, b2_d, b3_d, b4_d = (t.double().cpu() for t in (a, b1, b2, b3, b4))
    for f, g1, g2, g3, g4 in outs:
        g1d, g2d = g1.double().cpu(), g2.double().cpu()
        check(g1, a_d * f, b1_d, "bf16")
        # each later product from the values the GPU produced (their BF16 rounding included)
        check(g2, g1d[:64], b2_d, "bf16")
        check(g3, g1d[:512, :256], b3_d, "f32")
        check(g4, g2d, b4_d, "f32")


def test_streams_and_launch_count():
    s = torch.cuda.Stream()
    n0 = dg.dg_launch_count()
    with torch.cuda.stream(s):
        check_full(W.cfg_small(M=256, N=128, K=64), stream=s)
    assert dg.dg_launch_count() == n0 + 1


# ------------------------------------------------------------- full size
# The benchmark's workloads at their full sizes, in the launch configuration
# the benchmark times (the plans are asserted).  Every output is compared with
# the oracle where the oracle finishes in seconds (the decode GEMVs, the thin
# projection and the strided view); the 4096^3 products are compared on the
# four corners of every 128 x 128 block (each tile of either kernel shape has
# its corners among them) plus 3000 random outputs.

def _assert_bench_plan(name, pl):
    if name == "thin":
        assert pl["swap_ab"] == 1 and pl["split_k"] == 4, pl
    if name == "strided":
        assert pl["p_gather"] == 1 and pl["gather_cluster"] == 4, pl
    if name.startswith("square"):
        assert pl["cta_pair"] == 1, pl


@pytest.mark.parametrize("name", ["gemv", "gemv_kt", "thin", "strided"])
def test_full_size_every_output(name):
    p = W.WORKLOADS[name]()
    pl = expect_kind(p, {"gemv": "gemv_n", "gemv_kt": "gemv_k"}.get(name, "umma"))
    _assert_bench_plan(name, pl)
    check_full(p)


@pytest.mark.parametrize("name", ["square_bf16", "square_e4m3"])
def test_full_size_square_tile_corners(name):
    p = W.WORKLOADS[name]()
    pl = expect_kind(p, "umma")
    _assert_bench_plan(name, pl)
    check_sampled(p, npts=3000, extra=tile_corners(p.M, p.N, 128, 128))


@pytest.mark.parametrize("tma", [1, 0])
def test_output_past_4_gib(tma):
    # C of 8 GiB (65536 x 32768 FP32): the byte offsets of its last rows pass
    # 2^32, through the tensor-store and the thread-store epilogues.  The
    # oracle evaluates the sampled outputs on the sub-problem of their rows of
    # A and columns of B (the same data, the same definition).
    dg.dg_set_option(dg.DG_OPT_EPI_TMA, tma)
    M, N, K = 65536, 32768, 16
    g = torch.Generator().manual_seed(65536)
    a = W.cast(W.normal((M, K), g), "bf16")
    b = W.cast(W.normal((K, N), g), "bf16")
    c = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    p = W.Problem("past_4gib", W.row_major(a, "bf16"), W.row_major(b, "bf16"), W.row_major(c, "f32"))
    pl = plan(p)
    assert pl["kind_name"] == "umma" and pl["epi_tma_store"] == tma, pl
    ga, gb = a.to("cuda"), b.to("cuda")
    A = dg.make_view(ga.data_ptr(), (M, K), (2 * K, 2), 1, "bf16")
    B = dg.make_view(gb.data_ptr(), (K, N), (2 * N, 2), 1, "bf16")
    C = dg.make_view(c.data_ptr(), (M, N), (4 * N, 4), 1, "f32")
    assert dg.dg_gemm(A, B, C, 1.0, 0.0) == dg.DG_OK
    assert dg.dg_sync_status() == dg.DG_OK
    rng = np.random.default_rng(7)
    ms = np.concatenate([rng.integers(0, M, 200), np.full(40, M - 1), rng.integers(M - 128, M, 40), [0, M - 1]])
    ns = np.concatenate([rng.integers(0, N, 200), rng.integers(0, N, 40), np.full(40, N - 1), [N - 1, 0]])
    got = c[torch.as_tensor(ms, device="cuda"), torch.as_tensor(ns, device="cuda")].double().cpu().numpy()
    n = len(ms)
    sub = W.Problem("past_4gib_rows_cols", W.row_major(a[torch.as_tensor(ms)].contiguous(), "bf16"),
                    W.row_major(b[:, torch.as_tensor(ns)].contiguous(), "bf16"), W.empty_out(n, n, "f32"))
    ref, bound = oracle.gemm_points(sub, np.arange(n), np.arange(n))
    compare(sub, got, ref, bound, np.zeros(n), "past_4gib")
    del c
    torch.cuda.empty_cache()


def test_gathered_operand_past_2_gib():
    # An NCHW feature map of 2.5 GB (x[48, 256, 320, 320] BF16) read in place
    # as [n*h*w, c]: the gather's byte offsets pass 2^31.  Sampled outputs,
    # the last rows among them, against the oracle on their sub-problem.
    n, c, h, w, N = 48, 256, 320, 320, 32
    x = W.pattern((n, c, h, w), "bf16", device="cuda")
    g = torch.Generator().manual_seed(2 ** 31 % 1000)
    b = W.cast(W.uniform((c, N), g), "bf16")
    M = n * h * w
    cmat = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    A = W.nchw_as_rows(x, "bf16")
    p = W.Problem("nchw_past_2gib", A, W.row_major(b, "bf16"), W.row_major(cmat, "f32"))
    assert plan(p)["p_gather"] == 1
    gb = b.to("cuda")
    Av = dg.make_view(x.data_ptr(), A.shape, A.stride, A.row_dims, "bf16")
    Bv = dg.make_view(gb.data_ptr(), (c, N), (2 * N, 2), 1, "bf16")
    Cv = dg.make_view(cmat.data_ptr(), (M, N), (4 * N, 4), 1, "f32")
    assert dg.dg_gemm(Av, Bv, Cv, 1.0, 0.0) == dg.DG_OK
    assert dg.dg_sync_status() == dg.DG_OK
    rng = np.random.default_rng(31)
    ms = np.concatenate([rng.integers(0, M, 200), rng.integers(M - 4096, M, 60), [0, M - 1]])
    ns = np.concatenate([rng.integers(0, N, 200), rng.integers(0, N, 60), [N - 1, 0]])
    got = cmat[torch.as_tensor(ms, device="cuda"), torch.as_tensor(ns, device="cuda")].double().cpu().numpy()
    mi = torch.as_tensor(ms, device="cuda")
    rows = x.view(n, c, h * w)[mi // (h * w), :, mi % (h * w)].cpu().contiguous()  # [len(ms), c]
    k = len(ms)
    sub = W.Problem("nchw_past_2gib_rows_cols", W.row_major(rows, "bf16"),
                    W.row_major(b[:, torch.as_tensor(ns)].contiguous(), "bf16"), W.empty_out(k, k, "f32"))
    ref, bound = oracle.gemm_points(sub, np.arange(k), np.arange(k))
    compare(sub, got, ref, bound, np.zeros(k), "nchw_past_2gib")
    del x, cmat
    torch.cuda.empty_cache()


def _sampled_against_subproblem(a_rows, b_cols, got, name, out, alpha=1.0):
    """The oracle on the sub-problem made of the sampled outputs' rows of A
    ([k, K]) and columns of B ([K, k]): output i is (i, i); `out` is the real
    output's dtype, which sets the tolerance."""
    k = a_rows.shape[0]
    dt = {torch.bfloat16: "bf16", torch.float16: "f16"}[a_rows.dtype]
    sub = W.Problem(name, W.row_major(a_rows.contiguous(), dt), W.row_major(b_cols.contiguous(), dt),
                    W.empty_out(k, k, out), alpha)
    ref, bound = oracle.gemm_points(sub, np.arange(k), np.arange(k))
    compare(sub, got, ref, bound, np.zeros(k), name)


def test_gemv_weight_past_4_gib():
    # Decode GEMV on W[65536 x 40960] BF16 (5.4 GB, 2.7e9 elements, made on
    # the device): TMA coordinates and k splits far past the benchmark's.
    K, N = 65536, 40960
    Wt = W.pattern((K, N), "bf16", device="cuda")
    g = torch.Generator().manual_seed(40960)
    x = W.cast(W.normal((1, K), g, 0.02), "bf16")
    y = torch.full((1, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    p = W.Problem("gemv_past_4gib", W.row_major(x, "bf16"), W.row_major(Wt, "bf16"), W.row_major(y, "bf16"))
    assert plan(p)["kind_name"] == "gemv_n"
    gx = x.to("cuda")
    X = dg.make_view(gx.data_ptr(), (1, K), (2 * K, 2), 1, "bf16")
    Wv = dg.make_view(Wt.data_ptr(), (K, N), (2 * N, 2), 1, "bf16")
    Y = dg.make_view(y.data_ptr(), (1, N), (2 * N, 2), 1, "bf16")
    assert dg.dg_gemm(X, Wv, Y, 1.0, 0.0) == dg.DG_OK
    assert dg.dg_sync_status() == dg.DG_OK
    ns = np.concatenate([np.random.default_rng(5).integers(0, N, 96), [0, N - 1, N - 2]])
    ni = torch.as_tensor(ns, device="cuda")
    got = y[0, ni].double().cpu().numpy()
    cols = Wt[:, ni].cpu()  # [K, k]
    _sampled_against_subproblem(x.expand(len(ns), K), cols, got, "gemv_past_4gib", "bf16")
    del Wt
    torch.cuda.empty_cache()


def test_square_16384_many_pair_tiles():
    # 16384 x 16384 x 1024 BF16 on CTA pairs: 4096 tiles on 74 pairs, the
    # persistent schedule's later waves and last half-width tiles; the tile
    # corners of a band of tiles and random outputs against the oracle.
    M = N = 16384
    K = 1024
    g = torch.Generator().manual_seed(16384)
    a = W.cast(W.normal((M, K), g), "bf16")
    b = W.cast(W.normal((K, N), g), "bf16")
    cmat = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    p = W.Problem("square_16384", W.row_major(a, "bf16"), W.row_major(b, "bf16"), W.row_major(cmat, "bf16"))
    pl = plan(p)
    assert pl["kind_name"] == "umma" and pl["cta_pair"] == 1, pl
    ga, gb = a.to("cuda"), b.to("cuda")
    A = dg.make_view(ga.data_ptr(), (M, K), (2 * K, 2), 1, "bf16")
    B = dg.make_view(gb.data_ptr(), (K, N), (2 * N, 2), 1, "bf16")
    C = dg.make_view(cmat.data_ptr(), (M, N), (2 * N, 2), 1, "bf16")
    assert dg.dg_gemm(A, B, C, 1.0, 0.0) == dg.DG_OK
    assert dg.dg_sync_status() == dg.DG_OK
    cm, cn = tile_corners(M, N, 256, pl["block_n"])
    band = [(m, n) for m, n in zip(cm, cn) if m >= M - 1024]  # the last rows of tiles
    rng = np.random.default_rng(3)
    ms = np.array([m for m, _ in band] + list(rng.integers(0, M, 300)))
    ns = np.array([n for _, n in band] + list(rng.integers(0, N, 300)))
    got = cmat[torch.as_tensor(ms, device="cuda"), torch.as_tensor(ns, device="cuda")].double().cpu().numpy()
    _sampled_against_subproblem(a[torch.as_tensor(ms)], b[:, torch.as_tensor(ns)], got, "square_16384", "bf16")
    del cmat
    torch.cuda.empty_cache()
