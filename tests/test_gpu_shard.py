"""The column-sharded GEMM (tcgen05_tmem_gemm_b200.shard) on one GPU.

Every rank's block runs in libdg's kernels on its own GPU's memory; one NCCL
all-gather assembles C.  With one GPU available, the real path runs as a
one-rank NCCL group, and a four-way split is emulated on the one GPU by
computing every rank's block in turn and assembling them as the all-gather
lays them out; both are compared with the oracle.
"""
import os
import socket

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from harness import compare
from tcgen05_tmem_gemm_b200 import shard

pytestmark = pytest.mark.gpu


def _problem(seed=50, M=64, K=1024, N=1000):
    g = torch.Generator().manual_seed(seed)
    a = W.cast(W.normal((M, K), g), "bf16")
    b = W.cast(W.normal((K, N), g, 0.05), "bf16")
    c = W.uniform((M, N), g)
    bias = W.normal((N,), g)
    p = W.Problem("sharded", W.row_major(a, "bf16"), W.row_major(b, "bf16"), W.row_major(c.clone(), "f32"),
                  1.0, 0.5, bias=bias, act="gelu_tanh")
    return p, a, b, c, bias


def _check(p, full):
    ref, bound, pre = oracle.gemm(p, want_pre=True)
    bc = 0.5 * p.C.base.double().numpy()
    compare(p, full.double().cpu().numpy(), ref, bound, bc, "sharded", pre, np.abs(p.bias.double().numpy()))


def test_four_way_split_emulated_on_one_gpu():
    p, a, b, c, bias = _problem()
    world, N = 4, p.N
    blocks = []
    for r in range(world):
        Bb = shard.local_block(b, r, world, "cuda")
        Cb = shard.local_block(c, r, world, "cuda")
        bb = shard.local_block(bias[None, :], r, world, "cuda")[0].contiguous()
        shard.gemm_block(a.cuda(), Bb, Cb, N, r, world, 1.0, 0.5, bb, "gelu_tanh")
        blocks.append(Cb)
    torch.cuda.synchronize()
    # the all-gather's layout: [world, rows, width], then the padding dropped
    out = torch.stack(blocks).permute(1, 0, 2).reshape(p.M, -1)[:, :N]
    _check(p, out)


def test_one_rank_nccl_group():
    import torch.distributed as dist

    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1)
    try:
        p, a, b, c, bias = _problem(51)
        Bb = shard.local_block(b, 0, 1, "cuda")
        Cb = shard.local_block(c, 0, 1, "cuda")
        bb = shard.local_block(bias[None, :], 0, 1, "cuda")[0].contiguous()
        shard.gemm_block(a.cuda(), Bb, Cb, p.N, 0, 1, 1.0, 0.5, bb, "gelu_tanh")
        full = shard.assemble(Cb, p.N)
        torch.cuda.synchronize()
        _check(p, full)
    finally:
        dist.destroy_process_group()
