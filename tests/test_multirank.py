"""World-size-2 checks of the multi-GPU host logic on CPU (gloo).

The benchmark scales by running one replica of the step per GPU (weak
scaling, no collective on the data path) and reports the slowest rank's
time; a single GEMM can also be split over GPUs by columns of B and C with A
replicated (tcgen05_tmem_gemm_b200.shard: independent blocks, then one
all-gather to assemble C).  Both are exercised here with two gloo ranks on
127.0.0.1 and the CPU oracle standing in for the per-block kernel.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import sys

    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        import oracle
        import workloads as W

        # the slowest rank's time wins
        elapsed = 1.0 + rank
        mx = bench.max_over_ranks(elapsed, world, torch.device("cpu"))
        value = bench.whole_job_value(100.0, 10, world, mx)

        # one GEMM split by columns across the ranks
        p = W.cfg_strided(n=2, c=24, h=5, w=7, N=50)
        lo, hi = bench.shard_columns(p.N, rank, world)
        B = W.Operand(p.B.base, (p.K, hi - lo), p.B.stride, 1, p.B.dtype, offset=lo * 2)
        part = oracle.gemm(W.Problem("shard", p.A, B, W.empty_out(p.M, hi - lo, "f32")), want_bound=False)
        width = torch.tensor([hi - lo])
        widths = [torch.zeros(1, dtype=torch.int64) for _ in range(world)]
        dist.all_gather(widths, width)
        maxw = int(max(w.item() for w in widths))
        buf = torch.zeros(p.M, maxw, dtype=torch.float64)
        buf[:, : hi - lo] = torch.from_numpy(part)
        bufs = [torch.zeros_like(buf) for _ in range(world)]
        dist.all_gather(bufs, buf)
        full = torch.cat([b[:, : int(w.item())] for b, w in zip(bufs, widths)], dim=1).numpy()
        ref = oracle.gemm(p, want_bound=False)
        q.put((rank, mx, value, bool(np.array_equal(full, ref))))
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_and_column_shards():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for pr in procs:
        pr.start()
    for pr in procs:
        pr.join(timeout=120)
        assert pr.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, mx, value, same in res:
        assert mx == 2.0  # both ranks see the slower rank's time
        assert value == pytest.approx(100.0 * 10 * 2 / 2.0 / 1e9)
        assert same  # gathered column shards reproduce the single-process result


def _shard_worker(rank, world, port, q):
    import sys

    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        import workloads as W
        from tcgen05_tmem_gemm_b200 import shard

        # the library's column sharding and NCCL-style gather, with the oracle
        # standing in for the per-block kernel (no GPU here): each rank holds A,
        # its block of B, C and the bias; the gathered C equals the whole product
        g = torch.Generator().manual_seed(4)
        M, K, N = 9, 40, 53                       # N not a multiple of the world size
        a = W.cast(W.normal((M, K), g), "bf16")
        b = W.cast(W.normal((K, N), g), "bf16")
        c = W.uniform((M, N), g)
        bias = W.normal((N,), g)

        def ref_gemm(A, Bv, Cv, alpha, beta, bias_v, act):
            # the block views read through contiguous copies (the oracle's operands own their bytes)
            p = W.Problem("block", W.row_major(A.contiguous(), "bf16"), W.row_major(Bv.contiguous(), "bf16"),
                          W.row_major(Cv.contiguous(), "f32"), alpha, beta,
                          bias=None if bias_v is None else bias_v.contiguous(), act=act)
            Cv.copy_(torch.from_numpy(oracle.gemm(p, want_bound=False)).float())

        B_blk = shard.local_block(b, rank, world)
        C_blk = shard.local_block(c, rank, world)
        bias_blk = shard.local_block(bias[None, :], rank, world)[0]
        shard.gemm_block(a, B_blk, C_blk, N, rank, world, 0.5, 1.0, bias_blk, "gelu_tanh", gemm=ref_gemm)
        full = shard.assemble(C_blk, N)
        whole = W.Problem("whole", W.row_major(a, "bf16"), W.row_major(b, "bf16"), W.row_major(c.clone(), "f32"),
                          0.5, 1.0, bias=bias, act="gelu_tanh")
        ref = oracle.gemm(whole, want_bound=False)
        q.put((rank, tuple(full.shape), bool(np.allclose(full.double().numpy(), ref, rtol=1e-6, atol=1e-6))))
    finally:
        dist.destroy_process_group()


def test_two_rank_column_sharded_gemm_and_gather():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_shard_worker, args=(r, 2, port, q)) for r in range(2)]
    for pr in procs:
        pr.start()
    for pr in procs:
        pr.join(timeout=120)
        assert pr.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, shape, same in res:
        assert shape == (9, 53) and same


def test_library_column_ranges():
    from tcgen05_tmem_gemm_b200 import shard

    for n in (0, 1, 7, 53, 4096, 14336):
        for world in (1, 2, 3, 8):
            w = shard.shard_width(n, world)
            spans = [shard.column_range(n, r, world) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == n
            for (a, b), (c, d) in zip(spans, spans[1:]):
                assert b == c and 0 <= b - a <= w
            assert sum(b - a for a, b in spans) == n


def test_shard_columns_cover_exactly():
    import bench

    for n in (1, 7, 50, 4096):
        for world in (1, 2, 3, 8):
            spans = [bench.shard_columns(n, r, world) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == n
            for (a, b), (c, d) in zip(spans, spans[1:]):
                assert b == c and a <= b
