"""GPU parity of the fused epilogue (dg_gemm_ex) against the FP64 oracle.

out = act(alpha * sa * sb * sum_k a b + beta * C + bias[n]), the GEMM + BiasAdd
+ GeLU fusion of "DeepGEMM is not a new model: the inner discipline of GPU
matrix multiplication", §3.3 ("DeepGEMM deep dive", §5.1), on every kernel
path the dispatcher can take: tensor-core tiles with tensor stores or thread
stores, CTA pairs, split-K clusters with swapped operands (the bias then runs
along the tensor core's M side), gathered operands, the GEMVs, the CUDA-core
kernel and the alpha = 0 / K = 0 path; plus the layout transform of the
fusion, an NCHW output written straight from an [N*H*W, C] product.
"""
import numpy as np
import pytest
import torch

import tcgen05_tmem_gemm_b200 as dg
import workloads as W
from harness import c_matrix, check_full, check_sampled, plan, run, tile_corners

pytestmark = pytest.mark.gpu

ACTS = ["relu", "gelu_tanh"]


@pytest.fixture(autouse=True)
def _reset_options():
    yield
    dg.dg_set_option(dg.DG_OPT_FORCE_KIND, 0)
    dg.dg_set_option(dg.DG_OPT_MAX_SPLIT_K, 8)
    dg.dg_set_option(dg.DG_OPT_CTA_PAIR, 1)
    dg.dg_set_option(dg.DG_OPT_EPI_TMA, 1)
    dg.dg_set_option(dg.DG_OPT_GATHER_CLUSTER, 1)
    dg.dg_set_option(dg.DG_OPT_DETERMINISTIC, 0)


def expect(p, kind, **fields):
    pl = plan(p.to("cuda"))
    assert pl["kind_name"] == kind, pl
    for k, v in fields.items():
        assert pl[k] == v, (k, pl)
    return pl


def _rm(M, N, K, dt, out, seed, beta=0.0, alpha=1.0):
    g = torch.Generator().manual_seed(seed)
    A = W.cast(W.normal((M, K), g), dt)
    B = W.cast(W.normal((K, N), g), dt)
    C = W.row_major(W.uniform((M, N), g).to(W.TORCH_DTYPE[out]).contiguous(), out) if beta != 0 \
        else W.empty_out(M, N, out)
    return W.Problem(f"rm_{M}x{N}x{K}", W.row_major(A, dt), W.row_major(B, dt), C, alpha, beta)


@pytest.mark.parametrize("act", ACTS + ["none"])
def test_tensor_store_epilogue(act):
    # beta = 0, row-major C: 32-row x 128-byte blocks through tensor stores
    p = W.with_epilogue(_rm(300, 520, 200, "bf16", "bf16", 1), act)
    expect(p, "umma", epi_tma_store=1, split_k=1)
    check_full(p)


@pytest.mark.parametrize("act", ACTS)
def test_thread_store_epilogue_beta(act):
    # beta != 0: C is read, so the thread-store epilogue; the activation sees beta*C too
    p = W.with_epilogue(_rm(129, 136, 72, "f16", "f32", 2, beta=0.5, alpha=0.75), act)
    expect(p, "umma", epi_tma_store=0)
    check_full(p)


@pytest.mark.parametrize("act", ACTS)
def test_tensor_and_thread_stores_agree(act):
    # the two epilogues do the same arithmetic in the same order: equal bits
    p = W.with_epilogue(_rm(256, 384, 128, "bf16", "f32", 3, alpha=1.5), act)
    outs = []
    for tma in (1, 0):
        dg.dg_set_option(dg.DG_OPT_EPI_TMA, tma)
        expect(p, "umma", epi_tma_store=tma)
        check_full(p)
        outs.append(c_matrix(run(p.to("cuda"))))
    assert np.array_equal(outs[0], outs[1])


@pytest.mark.parametrize("act", ACTS)
def test_cta_pair_epilogue(act):
    dg.dg_set_option(dg.DG_OPT_CTA_PAIR, 2)
    dg.dg_set_option(dg.DG_OPT_MAX_SPLIT_K, 1)
    p = W.with_epilogue(_rm(520, 256, 64, "bf16", "bf16", 4), act)
    expect(p, "umma", cta_pair=1)
    check_full(p)


@pytest.mark.parametrize("act", ACTS)
def test_split_k_swapped_bias_along_i(act):
    # thin M: the kernel computes C^T, so the per-column bias runs along the
    # tensor core's rows; split-K clusters reduce on chip, beta = 1
    p = W.with_epilogue(W.cfg_thin(M=40, N=1000, K=784), act)
    pl = expect(p, "umma", swap_ab=1)
    assert pl["split_k"] > 1
    check_full(p)


def test_split_k_reduce_add_bias_once():
    # beta = 1, FP32 C, a bias and no activation: the splits add their partials
    # into C and only the first adds the bias
    p = W.with_epilogue(W.cfg_thin(M=48, N=1024, K=2048), "none")
    pl = expect(p, "umma", swap_ab=1)
    assert pl["split_k"] > 1 and pl["split_reduce_add"] == 1, pl
    check_full(p)


def test_split_k_element_path_no_swap():
    # split-K without a swap: the owner's element-by-element epilogue
    dg.dg_set_option(dg.DG_OPT_MAX_SPLIT_K, 3)
    g = torch.Generator().manual_seed(6)
    M, N, K = 256, 128, 6144
    A = W.row_major(W.cast(W.normal((M, K), g), "f16"), "f16")
    B = W.transposed(W.cast(W.normal((N, K), g, 0.05), "f16"), "f16")
    p = W.with_epilogue(W.Problem("sk", A, B, W.row_major(W.uniform((M, N), g), "f32"), 1.0, 1.0), "gelu_tanh")
    pl = expect(p, "umma", swap_ab=0)
    assert pl["split_k"] == 3
    check_full(p)


@pytest.mark.parametrize("act", ACTS)
def test_fp8_scales_bias(act):
    g = torch.Generator().manual_seed(7)
    M, N, K = 300, 384, 272
    qa, sa = W.quantise_e4m3(W.normal((M, K), g), dim=1)
    qb, sb = W.quantise_e4m3(W.normal((K, N), g), dim=0)
    p = W.with_epilogue(W.Problem("fp8", W.row_major(qa, "e4m3"), W.row_major(qb, "e4m3"), W.empty_out(M, N, "bf16"),
                                  1.0, 0.0, sa, sb), act)
    expect(p, "umma")
    check_full(p)


@pytest.mark.parametrize("act", ACTS)
def test_gathered_operand_epilogue(act):
    p = W.with_epilogue(W.cfg_strided(n=2, c=40, h=9, w=11, N=72), act)
    expect(p, "umma", p_gather=1)
    check_full(p)


@pytest.mark.parametrize("cluster", [1, 0])
def test_nchw_output_layout_transform(cluster):
    # The strided workload's product [n*h*w, N] written as an NCHW tensor
    # [n, N, h, w] by the epilogue (bias + ReLU fused).  The arithmetic is the
    # same as for a row-major output, so the two agree bit for bit once the
    # NCHW tensor is permuted back.
    dg.dg_set_option(dg.DG_OPT_GATHER_CLUSTER, cluster)
    n, c, h, w, N = 4, 128, 14, 14, 512
    base = W.with_epilogue(W.cfg_strided(n=n, c=c, h=h, w=w, N=N), "relu")
    p = W.Problem("nchw_out", base.A, base.B, W.nchw_out(n, N, h, w), 1.0, 0.0, bias=base.bias, act="relu")
    expect(p, "umma", p_gather=1, epi_tma_store=0)
    check_full(p)
    gpu = run(p.to("cuda"))
    rm = run(base.to("cuda"))
    nchw = gpu.C.base.cpu()  # [n, N, h, w]
    assert np.array_equal(nchw.permute(0, 2, 3, 1).reshape(n * h * w, N).double().numpy(), c_matrix(rm))


def test_nchw_output_from_row_major_operands():
    # a layout transform with TMA operands and a CTA-pair-sized problem
    n, h, w, N, K = 8, 16, 16, 256, 192
    g = torch.Generator().manual_seed(8)
    A = W.row_major(W.cast(W.normal((n * h * w, K), g), "bf16"), "bf16")
    B = W.row_major(W.cast(W.normal((K, N), g), "bf16"), "bf16")
    p = W.with_epilogue(W.Problem("nchw_rm", A, B, W.nchw_out(n, N, h, w, "bf16")), "gelu_tanh")
    expect(p, "umma")
    check_full(p)


@pytest.mark.parametrize("act", ACTS)
def test_gemv_epilogues(act):
    p = W.with_epilogue(W.cfg_gemv(K=1024, N=1032), act)
    expect(p, "gemv_n")
    check_full(p)
    q = W.with_epilogue(W.cfg_gemv_kt(K=1032, N=77), act)
    expect(q, "gemv_k")
    check_full(q)


@pytest.mark.parametrize("act", ACTS)
def test_simt_epilogue(act):
    dg.dg_set_option(dg.DG_OPT_FORCE_KIND, dg.DG_KIND_SIMT)
    p = W.with_epilogue(W.cfg_strided(n=2, c=40, h=9, w=11, N=72), act)
    expect(p, "simt")
    check_full(p)


def test_alpha_zero_and_k_zero_apply_bias_and_activation():
    M, N, K = 64, 96, 80
    g = torch.Generator().manual_seed(9)
    a = torch.full((M, K), float("inf")).to(torch.bfloat16)
    b = torch.ones(K, N, dtype=torch.bfloat16)
    c = W.uniform((M, N), g)
    p = W.with_epilogue(W.Problem("alpha0", W.row_major(a, "bf16"), W.row_major(b, "bf16"),
                                  W.row_major(c.clone(), "f32"), 0.0, -0.5), "gelu_tanh")
    expect(p, "scale_c")
    check_full(p)
    A = W.Operand(torch.zeros(8, dtype=torch.bfloat16), (6, 0), (0, 2), 1, "bf16")
    B = W.Operand(torch.zeros(8, dtype=torch.bfloat16), (0, 8), (16, 2), 1, "bf16")
    q = W.with_epilogue(W.Problem("k0", A, B, W.row_major(c[:6, :8].contiguous(), "f32"), 1.0, 3.0), "relu")
    check_full(q)


def test_epilogue_none_is_dg_gemm():
    # an epilogue with no bias and the identity is exactly dg_gemm: equal bits
    p = _rm(200, 264, 136, "bf16", "bf16", 10)
    q = W.Problem(p.name, p.A, p.B, p.C, bias=None, act="none")
    a = c_matrix(run(p.to("cuda")))
    gq = q.to("cuda")
    A, B, C = (dg.make_view(o.base.data_ptr() + o.offset, o.shape, o.stride, o.row_dims, o.dtype)
               for o in (gq.A, gq.B, gq.C))
    assert dg.dg_gemm_ex(A, B, C, 1.0, 0.0, None, None, dg.epilogue(None, "none")) == dg.DG_OK
    assert dg.dg_sync_status() == dg.DG_OK
    assert np.array_equal(a, c_matrix(gq))


def test_bias_must_be_device_memory():
    p = W.with_epilogue(_rm(128, 128, 64, "bf16", "bf16", 11), "relu").to("cuda")
    A, B, C = (dg.make_view(o.base.data_ptr() + o.offset, o.shape, o.stride, o.row_dims, o.dtype)
               for o in (p.A, p.B, p.C))
    host_bias = torch.zeros(128)
    assert dg.dg_gemm_ex(A, B, C, 1.0, 0.0, None, None, dg.epilogue(host_bias, "relu")) == dg.DG_ERR_POINTER
    assert dg.dg_sync_status() == dg.DG_OK


@pytest.mark.parametrize("name", ["square_bf16", "thin"])
def test_full_size_fused(name):
    # the benchmark's fused rows: 4096^3 BF16 with bias + GeLU (CTA pairs,
    # tensor-store epilogue), and the thin projection with bias + GeLU (split-K,
    # swapped, beta = 1), in the plans the benchmark times
    p = W.with_epilogue(W.WORKLOADS[name](), "gelu_tanh")
    pl = expect(p, "umma")
    if name == "thin":
        assert pl["swap_ab"] == 1 and pl["split_k"] == 4
        check_full(p)
    else:
        assert pl["cta_pair"] == 1
        check_sampled(p, npts=3000, extra=tile_corners(p.M, p.N, 128, 128))


def _off_16(t: torch.Tensor) -> torch.Tensor:
    """A device copy of 1-D t whose first element sits 4 bytes past a 16-byte
    boundary, so that no 16-byte vector load of it is legal."""
    big = torch.empty(t.numel() + 4, dtype=t.dtype, device="cuda")
    v = big[1:1 + t.numel()]
    v.copy_(t.to("cuda"))
    assert v.data_ptr() % 16 == 4
    return v


def _fp8_problem(M, N, K, seed, k_major_b=False):
    g = torch.Generator().manual_seed(seed)
    qa, sa = W.quantise_e4m3(W.normal((M, K), g), dim=1)
    if k_major_b:  # B read K-major from an [N, K] tensor (CTA pairs need it for FP8)
        qbt, sb = W.quantise_e4m3(W.normal((N, K), g), dim=1)
        B = W.transposed(qbt, "e4m3")
    else:
        qb, sb = W.quantise_e4m3(W.normal((K, N), g), dim=0)
        B = W.row_major(qb, "e4m3")
    return W.Problem("fp8_off16", W.row_major(qa, "e4m3"), B, W.empty_out(M, N, "bf16"), 1.0, 0.0, sa, sb)


@pytest.mark.parametrize("case", ["tensor_store_bf16", "tensor_store_f32", "thread_store_beta", "pair_fp8",
                                  "umma_fp8", "gemv"])
def test_bias_and_scales_off_16_byte_boundaries(case):
    # The epilogues read the bias and the column scales as 16-byte vectors only
    # when the array allows it; arrays 4 bytes past a 16-byte boundary take the
    # element loads, with the same results.
    from harness import _bias_abs, beta_c_of, compare
    import oracle

    if case == "tensor_store_bf16":
        p, kind = W.with_epilogue(_rm(300, 520, 200, "bf16", "bf16", 21), "gelu_tanh"), dict(epi_tma_store=1)
    elif case == "tensor_store_f32":
        p, kind = W.with_epilogue(_rm(300, 520, 200, "bf16", "f32", 22), "relu"), dict(epi_tma_store=1)
    elif case == "thread_store_beta":
        p, kind = W.with_epilogue(_rm(300, 520, 200, "bf16", "f32", 23, beta=0.5), "gelu_tanh"), \
            dict(epi_tma_store=0)
    elif case == "pair_fp8":
        dg.dg_set_option(dg.DG_OPT_CTA_PAIR, 2)
        dg.dg_set_option(dg.DG_OPT_MAX_SPLIT_K, 1)
        p, kind = W.with_epilogue(_fp8_problem(512, 512, 512, 24, k_major_b=True), "gelu_tanh"), dict(cta_pair=1)
    elif case == "umma_fp8":
        p, kind = W.with_epilogue(_fp8_problem(300, 400, 256, 25), "relu"), dict(cta_pair=0)
    else:
        g = torch.Generator().manual_seed(26)
        x = W.cast(W.normal((1, 1024), g, 0.02), "bf16")
        Wt = W.cast(W.normal((1024, 2056), g, 0.02), "bf16")
        p = W.with_epilogue(W.Problem("gemv_off16", W.row_major(x, "bf16"), W.row_major(Wt, "bf16"),
                                      W.empty_out(1, 2056, "bf16")), "gelu_tanh")
        kind = {}
    pl = expect(p, "gemv_n" if case == "gemv" else "umma", **kind)
    ref, bound, pre = oracle.gemm(p, want_pre=True)
    gp = p.to("cuda")
    gp.bias = _off_16(p.bias)
    if p.scale_a is not None:
        gp.scale_a = _off_16(p.scale_a)
        gp.scale_b = _off_16(p.scale_b)
    run(gp)
    compare(p, c_matrix(gp), ref, bound, beta_c_of(p), f"{case} {pl['kind_name']}", pre, _bias_abs(p))
