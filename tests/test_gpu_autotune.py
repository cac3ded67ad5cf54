"""GPU checks of the shape-keyed autotuner (dg_autotune).

"DeepGEMM deep dive", §5.3: the best tile and pipeline settings depend on the
shape and are found by measuring; "DeepGEMM: a recalibration of the compute
paradigm", §6.1: the chosen configuration is cached per problem.  The
autotuner times the kernel variants a call admits on the caller's operands,
keeps the fastest per shape key, and runs the call; later calls with the same
key take the tuned plan.  Whatever it picks, the result must match the oracle
(C restored when beta != 0, so C is read exactly once).
"""
import numpy as np
import pytest
import torch

import oracle
import tcgen05_tmem_gemm_b200 as dg
import workloads as W
from harness import _bias_abs, beta_c_of, c_matrix, compare, dg_view_of, fused, plan

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _clear():
    dg.dg_tune_clear()
    yield
    dg.dg_tune_clear()


def _autotune_and_check(p_cpu, reps=3):
    ref, bound, pre = oracle.gemm(p_cpu, want_pre=True)
    bc = beta_c_of(p_cpu)
    p = p_cpu.to("cuda")
    A, B, C = (dg_view_of(o) for o in (p.A, p.B, p.C))
    epi = dg.epilogue(p.bias, p.act) if fused(p) else None
    st, res = dg.dg_autotune(A, B, C, p.alpha, p.beta, p.scale_a, p.scale_b, epi, None, reps)
    assert st == dg.DG_OK, dg.status_string(st)
    assert dg.dg_sync_status() == dg.DG_OK
    compare(p_cpu, c_matrix(p), ref, bound, bc, p_cpu.name + "/autotune", pre if fused(p_cpu) else None,
            _bias_abs(p_cpu))
    return p, res


@pytest.mark.parametrize("name,kw", [("thin", {"M": 64, "N": 1024, "K": 2048}),
                                      ("strided", {"n": 4, "c": 128, "h": 14, "w": 14, "N": 512}),
                                      ("small", {}),
                                      ("gemv", {"K": 2048, "N": 4096})])
def test_autotune_correct_and_cached(name, kw):
    p_cpu = W.WORKLOADS[name](**kw)
    p, res = _autotune_and_check(p_cpu)
    assert res.candidates >= 2 and res.best_us > 0 and res.best_us <= res.default_us * 1.0001
    # the table now answers for these views: the plan is the chosen one
    chosen = res.plan
    now = plan(p)
    for f in ("kind", "block_n", "split_k", "cta_pair", "gather_cluster", "epi_tma_store", "stream_k_tiles", "grid"):
        assert now[f] == getattr(chosen, f), (f, now, chosen.as_dict())
    # and a plain dg_gemm with the tuned plan is still right
    from harness import check_full
    check_full(p_cpu)


def test_autotune_beta_keeps_c_and_epilogue():
    # beta = 1: C is saved before the trials and put back before the final call
    p_cpu = W.with_epilogue(W.cfg_thin(M=48, N=768, K=1536), "gelu_tanh")
    _autotune_and_check(p_cpu)


def test_autotune_square_variants():
    if torch.cuda.get_device_properties(0).multi_processor_count != 148:
        pytest.skip("the variants are worked out for 148 SMs")
    g = torch.Generator().manual_seed(40)
    M, N, K = 4096, 3072, 256
    a = W.cast(W.normal((M, K), g), "bf16")
    b = W.cast(W.normal((K, N), g), "bf16")
    p_cpu = W.Problem("tune_sq", W.row_major(a, "bf16"), W.row_major(b, "bf16"), W.empty_out(M, N, "bf16"))
    _, res = _autotune_and_check(p_cpu, reps=2)
    assert res.candidates >= 4
