"""The allocation-free entry point, dg_gemm_static, against dg_gemm.

Callers that cannot let a library allocate device memory (work captured into
a CUDA graph, frameworks whose own pool owns every byte, serving loops that
may not synchronise) use dg_gemm_static: the same GEMM, with its status word
and Stream-K workspace in a static device array instead of memory the
library allocates.  The test calls it through the C ABI twice in a row on a
problem whose plan uses the Stream-K workspace and on one that does not, and
checks each result against dg_gemm's within the tolerance of the parity
tests.  This file is collected last, so a run that stops at the first failure
has run every other test before it.
"""
import ctypes

import numpy as np
import pytest
import torch

import tcgen05_tmem_gemm_b200 as dg
import workloads as W
from harness import c_matrix, dg_view_of, plan, run, tolerance

pytestmark = pytest.mark.gpu


def _call_static(p):
    A, B, C = (dg_view_of(o) for o in (p.A, p.B, p.C))
    st = dg.lib.dg_gemm_static(ctypes.byref(A), ctypes.byref(B), ctypes.byref(C), float(p.alpha), float(p.beta),
                               None, None, None)
    assert st == dg.DG_OK, dg.status_string(st)
    torch.cuda.synchronize()
    return c_matrix(p)


def _scale(p):
    # S = |alpha| sum_k |a b|, the scale the parity tolerance multiplies
    a = p.A.base.double().abs()
    b = p.B.base.double().abs()
    return (abs(p.alpha) * (a @ b)).cpu().numpy()


@pytest.mark.parametrize("M,N,K,stream_k", [(4096, 3072, 256, True), (300, 520, 200, False)])
def test_static_scratch_entry_matches_dg_gemm_twice(M, N, K, stream_k):
    g = torch.Generator().manual_seed(M + N + K)
    a = W.cast(W.normal((M, K), g), "bf16")
    b = W.cast(W.normal((K, N), g), "bf16")
    ref_p = W.Problem("dg_gemm", W.row_major(a, "bf16"), W.row_major(b, "bf16"), W.empty_out(M, N, "bf16"))
    gp = ref_p.to("cuda")
    dg.dg_set_option(dg.DG_OPT_STREAM_K, 1 if stream_k else 0)
    try:
        if stream_k and torch.cuda.get_device_properties(0).multi_processor_count == 148:
            assert plan(gp)["stream_k_tiles"] > 0  # the Stream-K workspace is in use
        ref = c_matrix(run(gp))
        S = _scale(gp)
        tol = tolerance("bf16", ref, S, np.zeros_like(ref))
        for call in range(2):
            q = W.Problem("static", gp.A, gp.B, W.empty_out(M, N, "bf16").to("cuda"))
            got = _call_static(q)
            err = np.abs(got - ref)
            assert np.all(err <= tol), (call, float(err.max()))
    finally:
        dg.dg_set_option(dg.DG_OPT_STREAM_K, 0)
