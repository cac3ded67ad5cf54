"""Column-sharded GEMM over the GPUs of one node, one process per GPU.

C = alpha * A B + beta * C splits by columns of B and C with A replicated:
rank r computes  C[:, cols_r] = alpha * A B[:, cols_r] + beta * C[:, cols_r]
with dg_gemm on its own GPU's memory, and no data crosses between GPUs while
it does.  Every rank's block has the same width, ceil(N / world) (the last
blocks may be short or empty), so the blocks can be gathered with one NCCL
all-gather over NVLink / NVSwitch when every rank needs the whole C
(assemble()).  No kernel reads another GPU's memory: the gathered blocks land
in local memory before anything reads them, so no TMA load, with or without
cluster multicast, is ever given a peer's address.

torch.distributed is the plumbing (process group, all-gather); the product of
each block runs in libdg's kernels.
"""
from __future__ import annotations

import torch

from . import DG_OK, DgError, dg_gemm, dg_gemm_ex, epilogue, status_string, view


def shard_width(n: int, world: int) -> int:
    """Columns in every rank's block: the same for all ranks."""
    return -(-n // world) if n > 0 else 0


def column_range(n: int, rank: int, world: int):
    """Columns [lo, hi) of an n-wide matrix that `rank` owns (hi - lo may be
    smaller than shard_width for the last ranks, or zero)."""
    w = shard_width(n, world)
    lo = min(n, rank * w)
    return lo, min(n, lo + w)


def local_block(full: torch.Tensor, rank: int, world: int, device=None) -> torch.Tensor:
    """This rank's [rows x shard_width] block of a [rows x n] matrix, copied
    into a contiguous tensor on `device` (the columns past n are zero)."""
    rows, n = full.shape
    lo, hi = column_range(n, rank, world)
    out = torch.zeros(rows, shard_width(n, world), dtype=full.dtype, device=device or full.device)
    out[:, : hi - lo] = full[:, lo:hi]
    return out


def gemm_block(A: torch.Tensor, B_block: torch.Tensor, C_block: torch.Tensor, n: int, rank: int, world: int,
               alpha: float = 1.0, beta: float = 0.0, bias_block=None, act: str = "none", stream=None,
               gemm=None) -> torch.Tensor:
    """This rank's block of C = act(alpha A B + beta C + bias): the valid
    columns of the padded blocks, through dg_gemm / dg_gemm_ex (or `gemm`,
    a callable with the same arguments, e.g. a reference on the CPU)."""
    lo, hi = column_range(n, rank, world)
    w = hi - lo
    if w == 0:
        return C_block
    Bv, Cv = B_block[:, :w], C_block[:, :w]
    if gemm is not None:
        gemm(A, Bv, Cv, alpha, beta, None if bias_block is None else bias_block[:w], act)
        return C_block
    if bias_block is None and act == "none":
        st = dg_gemm(view(A), view(Bv), view(Cv), alpha, beta, None, None, stream)
    else:
        st = dg_gemm_ex(view(A), view(Bv), view(Cv), alpha, beta, None, None,
                        epilogue(None if bias_block is None else bias_block[:w], act), stream)
    if st != DG_OK:
        raise DgError(st, "dg_gemm (column block): " + status_string(st))
    return C_block


def assemble(C_block: torch.Tensor, n: int, group=None) -> torch.Tensor:
    """The whole [rows x n] C on every rank: one all-gather of the equal-width
    blocks into local memory, then a view that drops the padding columns."""
    import torch.distributed as dist

    world = dist.get_world_size(group)
    rows, width = C_block.shape
    block = C_block.contiguous()
    out = torch.empty(world * rows, width, dtype=block.dtype, device=block.device)
    try:
        dist.all_gather_into_tensor(out, block, group=group)
    except (RuntimeError, NotImplementedError, AttributeError):
        # backends without the single-tensor form (older gloo): the list form
        parts = list(out.chunk(world, dim=0))
        dist.all_gather(parts, block, group=group)
    full = out.view(world, rows, width).permute(1, 0, 2).reshape(rows, world * width)
    return full[:, :n]
