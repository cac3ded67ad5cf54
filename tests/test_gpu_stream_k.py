"""GPU parity of the Stream-K schedule of the CTA-pair kernel.

When the 256-row tiles leave a last, partial wave (4096^3 is 256 tiles on
74 pairs), the k blocks of those tiles are shared out evenly over all pairs
("DeepGEMM deep dive", §5.2: Stream-K as the load-balanced successor of
split-K).  A pair whose range ends inside a tile leaves its partial
accumulator in a workspace; the tile's owner (the pair holding its last k
blocks) adds the partials in pair order and runs the epilogue.  The sum order
is fixed by the schedule, so repeated runs agree bit for bit; against the
whole-tile schedule the results differ only by rounding.
"""
import numpy as np
import pytest
import torch

import tcgen05_tmem_gemm_b200 as dg
import workloads as W
from harness import c_matrix, check_full, dg_view_of, plan, run

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _reset_options():
    dg.dg_set_option(dg.DG_OPT_STREAM_K, 1)  # opt-in: the half-width tail is the default
    yield
    dg.dg_set_option(dg.DG_OPT_STREAM_K, 0)
    dg.dg_set_option(dg.DG_OPT_TEST_STALL, 0)
    dg.dg_set_option(dg.DG_OPT_WAIT_TIMEOUT_MS, 2000)
    dg.dg_set_option(dg.DG_OPT_PAIR_TAIL, 1)
    dg.dg_set_option(dg.DG_OPT_PAIR_DEEP_STAGES, 1)


def _needs_148():
    if torch.cuda.get_device_properties(0).multi_processor_count != 148:
        pytest.skip("the schedule sizes are worked out for 148 SMs")


def _bf16(M, N, K, seed, tb=False, out="bf16", beta=0.0):
    g = torch.Generator().manual_seed(seed)
    a = W.cast(W.normal((M, K), g), "bf16")
    b = W.cast(W.normal((N, K) if tb else (K, N), g), "bf16")
    B = W.transposed(b, "bf16") if tb else W.row_major(b, "bf16")
    C = W.row_major(W.uniform((M, N), g).to(W.TORCH_DTYPE[out]).contiguous(), out) if beta else W.empty_out(M, N, out)
    return W.Problem(f"sk_{M}x{N}x{K}", W.row_major(a, "bf16"), B, C, 1.0, beta)


@pytest.mark.parametrize("tb", [False, True])
def test_stream_k_matches_oracle_and_is_deterministic(tb):
    _needs_148()
    # 16 x 12 = 192 tiles on 74 pairs: 148 whole, 44 shared out (176 k blocks
    # of 64, or 88 stages two k blocks deep when B is MN-major)
    p = _bf16(4096, 3072, 256, 31 + int(tb), tb)
    pl = plan(p.to("cuda"))
    assert pl["cta_pair"] == 1 and pl["stream_k_tiles"] == 44 and pl["pair_half_tiles"] == 0, pl
    assert pl["block_k"] == (64 if tb else 128), pl
    check_full(p)
    a = c_matrix(run(p.to("cuda")))
    b = c_matrix(run(p.to("cuda")))
    assert np.array_equal(a, b)
    # the whole-tile schedule computes the same product (rounding apart)
    dg.dg_set_option(dg.DG_OPT_STREAM_K, 0)
    assert plan(p.to("cuda"))["stream_k_tiles"] == 0
    c = c_matrix(run(p.to("cuda")))
    assert np.allclose(a, c, rtol=2e-2, atol=2e-2)


def test_stream_k_many_pairs_per_tile():
    _needs_148()
    # 17 x 5 = 85 tiles: 11 shared out as 88 k blocks over 74 pairs, so a tile's
    # 8 k blocks are split among up to 7 pairs (the owner adds up to 6 partials);
    # stages one k block deep (two-deep stages would leave 44 for 74 pairs)
    dg.dg_set_option(dg.DG_OPT_PAIR_DEEP_STAGES, 0)
    p = _bf16(4352, 1280, 512, 33, out="f32")
    pl = plan(p.to("cuda"))
    assert pl["stream_k_tiles"] == 11, pl
    check_full(p)


def test_stream_k_beta_bias_gelu_thread_stores():
    _needs_148()
    # beta != 0: the thread-store epilogue adds the partials; bias + GeLU after
    p = W.with_epilogue(_bf16(4096, 3072, 192, 34, beta=0.5, out="f32"), "gelu_tanh")
    pl = plan(p.to("cuda"))
    assert pl["stream_k_tiles"] == 44 and pl["epi_tma_store"] == 0, pl
    check_full(p)


def test_stream_k_fp8():
    _needs_148()
    g = torch.Generator().manual_seed(35)
    M, N, K = 4096, 3072, 512
    qa, sa = W.quantise_e4m3(W.normal((M, K), g), dim=1)
    qb, sb = W.quantise_e4m3(W.normal((K, N), g), dim=0)
    p = W.Problem("sk_fp8", W.row_major(qa, "e4m3"), W.row_major(qb, "e4m3"), W.empty_out(M, N, "bf16"),
                  1.0, 0.0, sa, sb)
    pl = plan(p.to("cuda"))
    assert pl["cta_pair"] == 1 and pl["stream_k_tiles"] == 44, pl
    check_full(p)


def test_stream_k_graph_replay_and_second_stream():
    _needs_148()
    # The workspace's sequence tags live in device memory, so replays of a
    # captured launch do not see the flags of the replay before; a second
    # stream gets a workspace of its own.
    p = _bf16(4096, 3072, 256, 36).to("cuda")
    q = _bf16(4096, 3072, 256, 37).to("cuda")
    ref_p = c_matrix(run(p))
    ref_q = c_matrix(run(q))
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    vp = [dg_view_of(o) for o in (p.A, p.B, p.C)]
    vq = [dg_view_of(o) for o in (q.A, q.B, q.C)]
    for s, v in ((s1, vp), (s2, vq)):  # outside capture: each stream's workspace is allocated here
        assert dg.dg_gemm(*v, 1.0, 0.0, None, None, s) == dg.DG_OK
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s1):
        assert dg.dg_gemm(*vp, 1.0, 0.0, None, None, s1) == dg.DG_OK
    for _ in range(3):
        p.C.base.fill_(float("nan"))
        g.replay()
        with torch.cuda.stream(s2):  # concurrently, the other product on its own stream
            assert dg.dg_gemm(*vq, 1.0, 0.0, None, None, s2) == dg.DG_OK
        torch.cuda.synchronize()
        assert dg.dg_sync_status(s1) == dg.DG_OK
        assert np.array_equal(c_matrix(p), ref_p)
        assert np.array_equal(c_matrix(q), ref_q)
    del g


def test_stream_k_timeout_then_correct():
    _needs_148()
    # a launch whose waits run out leaves flags of its own tag behind; the
    # next launch's tag differs, so it is correct (stages one k block deep:
    # K = 128 in two-deep stages would leave 44 stages for 74 pairs)
    dg.dg_set_option(dg.DG_OPT_PAIR_DEEP_STAGES, 0)
    p = _bf16(4096, 3072, 128, 38)
    dg.dg_set_option(dg.DG_OPT_WAIT_TIMEOUT_MS, 300)
    dg.dg_set_option(dg.DG_OPT_TEST_STALL, 1)
    gp = p.to("cuda")
    A, B, C = (dg_view_of(o) for o in (gp.A, gp.B, gp.C))
    assert dg.dg_gemm(A, B, C, 1.0, 0.0) == dg.DG_OK
    assert dg.dg_sync_status() == dg.DG_ERR_TIMEOUT
    dg.dg_set_option(dg.DG_OPT_TEST_STALL, 0)
    assert plan(p.to("cuda"))["stream_k_tiles"] == 44
    check_full(p)
