"""Seeded synthetic inputs for the strided-view GEMM  C = alpha*A*B + beta*C.

This module only *draws* inputs: it holds none of the GEMM arithmetic. Both
the CUDA path (through the C-ABI) and the CPU oracle consume what it returns,
so the two sides always see the same bytes.

An operand is described the way the strided "view" API describes it
("DeepGEMM: a recalibration of the compute paradigm", §3.2 view struct):
a base tensor that owns the bytes, up to four dims, byte strides, and a
``row_dims`` split that says which leading dims flatten (row-major) into the
matrix rows; the remaining dims flatten into the columns.

Workloads (shapes, dtypes, value distributions) are the five synthetic
configurations of the benchmark: a 128x256x128 FP16 GEMM, the decode GEMV
x[1x4096]*W[4096x14336] plus x*K^T with K[128x4096], the thin FP16 projection
A[64x4096]*B[4096x4096] with beta=1, the 4096^3 square GEMM in BF16 and in
FP8 E4M3 with per-row / per-column scales, and the NCHW feature map
[16,256,14,14] read in place as a [3136x256] operand.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional

import torch

ELEM_SIZE = {"f32": 4, "f16": 2, "bf16": 2, "e4m3": 1}
TORCH_DTYPE = {
    "f32": torch.float32,
    "f16": torch.float16,
    "bf16": torch.bfloat16,
    "e4m3": torch.float8_e4m3fn,
}
E4M3_MAX = 448.0


@dataclass
class Operand:
    """A strided view over the bytes of ``base``.

    ``offset`` is the byte offset of element (0,...,0) inside ``base``;
    ``shape``/``stride`` have up to four entries, strides in BYTES;
    the first ``row_dims`` dims are the matrix rows, the rest the columns.
    """

    base: torch.Tensor
    shape: tuple
    stride: tuple
    row_dims: int
    dtype: str
    offset: int = 0

    @property
    def rows(self) -> int:
        r = 1
        for s in self.shape[: self.row_dims]:
            r *= int(s)
        return r

    @property
    def cols(self) -> int:
        c = 1
        for s in self.shape[self.row_dims:]:
            c *= int(s)
        return c

    def to(self, device) -> "Operand":
        return Operand(self.base.to(device), self.shape, self.stride,
                       self.row_dims, self.dtype, self.offset)


@dataclass
class Problem:
    name: str
    A: Operand
    B: Operand
    C: Operand
    alpha: float = 1.0
    beta: float = 0.0
    scale_a: Optional[torch.Tensor] = None  # float32 [M] or None
    scale_b: Optional[torch.Tensor] = None  # float32 [N] or None
    note: str = ""
    extra: dict = field(default_factory=dict)
    bias: Optional[torch.Tensor] = None     # float32 [N] or None (fused epilogue)
    act: str = "none"                       # "none", "relu" or "gelu_tanh" (fused epilogue)

    @property
    def M(self) -> int:
        return self.A.rows

    @property
    def K(self) -> int:
        return self.A.cols

    @property
    def N(self) -> int:
        return self.B.cols

    def to(self, device) -> "Problem":
        return Problem(self.name, self.A.to(device), self.B.to(device), self.C.to(device),
                       self.alpha, self.beta,
                       None if self.scale_a is None else self.scale_a.to(device),
                       None if self.scale_b is None else self.scale_b.to(device),
                       self.note, dict(self.extra),
                       None if self.bias is None else self.bias.to(device), self.act)


def row_major(t: torch.Tensor, dtype: str, row_dims: int = 1) -> Operand:
    """Operand over a contiguous tensor, strides taken from the tensor itself."""
    es = ELEM_SIZE[dtype]
    return Operand(t, tuple(t.shape), tuple(s * es for s in t.stride()), row_dims, dtype)


def transposed(t: torch.Tensor, dtype: str) -> Operand:
    """The 2-D transpose of a contiguous [R, C] tensor as a no-copy view [C, R]."""
    es = ELEM_SIZE[dtype]
    r, c = t.shape
    return Operand(t, (c, r), (t.stride(1) * es, t.stride(0) * es), 1, dtype)


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator()
    g.manual_seed(seed)
    return g


def uniform(shape, g, lo=-1.0, hi=1.0) -> torch.Tensor:
    return torch.rand(shape, generator=g, dtype=torch.float32) * (hi - lo) + lo


def normal(shape, g, std=1.0) -> torch.Tensor:
    return torch.randn(shape, generator=g, dtype=torch.float32) * std


def cast(x: torch.Tensor, dtype: str) -> torch.Tensor:
    return x.to(TORCH_DTYPE[dtype]).contiguous()


def quantise_e4m3(x: torch.Tensor, dim: int):
    """Per-row (dim=1) or per-column (dim=0) E4M3 quantisation of float32 data.

    scale = amax/448 over the reduced dim (1 where the amax is 0), q = x/scale
    clamped to the finite range and rounded by torch's float8_e4m3fn cast.
    Returns (q as float8_e4m3fn, scale as float32 with the kept dim's length).
    """
    amax = x.abs().amax(dim=dim)
    scale = torch.where(amax > 0, amax / E4M3_MAX, torch.ones_like(amax)).to(torch.float32)
    s = scale.unsqueeze(dim)
    q = (x / s).clamp(-E4M3_MAX, E4M3_MAX).to(torch.float8_e4m3fn).contiguous()
    return q, scale.contiguous()


def pattern(shape, dtype: str = "bf16", device="cpu") -> torch.Tensor:
    """A deterministic tensor ((i mod 251) - 125) / 128 over the flat index i,
    made where it will live (on the device for operands too large to draw on
    the host).  Every value is a multiple of 1/128 below 1 in magnitude, exact
    in F16 and BF16."""
    numel = 1
    for s in shape:
        numel *= int(s)
    i = torch.arange(numel, device=device, dtype=torch.int64)
    v = ((i % 251) - 125).to(torch.float32) / 128.0
    return v.to(TORCH_DTYPE[dtype]).reshape(tuple(shape))


def empty_out(M: int, N: int, dtype: str, fill=float("nan")) -> Operand:
    t = torch.full((M, N), fill, dtype=torch.float32).to(TORCH_DTYPE[dtype])
    return row_major(t, dtype)


# ---------------------------------------------------------------- workloads

def cfg_small(seed: int = 1001, M=128, N=128, K=256, dtype="f16", out="f32") -> Problem:
    """FP16 A[128x256] * B[256x128] row-major -> FP32 C, alpha=1, beta=0, U[-1,1]."""
    g = _gen(seed)
    A = cast(uniform((M, K), g), dtype)
    B = cast(uniform((K, N), g), dtype)
    return Problem("small_f16_128x128x256", row_major(A, dtype), row_major(B, dtype),
                   empty_out(M, N, out), 1.0, 0.0)


def cfg_gemv(seed: int = 1002, K=4096, N=14336, dtype="bf16") -> Problem:
    """Decode GEMV x[1xK] * W[KxN] row-major, N(0, 0.02^2), BF16 out."""
    g = _gen(seed)
    x = cast(normal((1, K), g, 0.02), dtype)
    W = cast(normal((K, N), g, 0.02), dtype)
    return Problem(f"gemv_bf16_1x{N}x{K}", row_major(x, dtype), row_major(W, dtype),
                   empty_out(1, N, dtype), 1.0, 0.0)


def cfg_gemv_kt(seed: int = 1012, K=4096, N=128, dtype="bf16") -> Problem:
    """x[1xK] * K^T with the key matrix Kmat[NxK] row-major read as a [KxN] view."""
    g = _gen(seed)
    x = cast(normal((1, K), g, 0.02), dtype)
    Kmat = cast(normal((N, K), g, 0.02), dtype)
    return Problem(f"gemv_kt_bf16_1x{N}x{K}", row_major(x, dtype), transposed(Kmat, dtype),
                   empty_out(1, N, dtype), 1.0, 0.0)


def cfg_thin(seed: int = 1003, M=64, N=4096, K=4096, dtype="f16") -> Problem:
    """Thin projection A[64x4096]~N(0,1) * B[4096x4096]~N(0,0.02^2), FP32 C~U[-1,1] in/out, beta=1."""
    g = _gen(seed)
    A = cast(normal((M, K), g, 1.0), dtype)
    B = cast(normal((K, N), g, 0.02), dtype)
    C = uniform((M, N), g).contiguous()
    return Problem(f"thin_f16_{M}x{N}x{K}_beta1", row_major(A, dtype), row_major(B, dtype),
                   row_major(C, "f32"), 1.0, 1.0)


def cfg_square_bf16(seed: int = 1004, M=4096, N=4096, K=4096) -> Problem:
    """Square GEMM, BF16 in (N(0,1)), FP32 accumulate, BF16 out."""
    g = _gen(seed)
    A = cast(normal((M, K), g), "bf16")
    B = cast(normal((K, N), g), "bf16")
    return Problem(f"square_bf16_{M}x{N}x{K}", row_major(A, "bf16"), row_major(B, "bf16"),
                   empty_out(M, N, "bf16"), 1.0, 0.0)


def cfg_square_e4m3(seed: int = 1005, M=4096, N=4096, K=4096) -> Problem:
    """Square GEMM, E4M3 A (per-row scale) and B (per-column scale) from N(0,1), BF16 out."""
    g = _gen(seed)
    a = normal((M, K), g)
    b = normal((K, N), g)
    qa, sa = quantise_e4m3(a, dim=1)
    qb, sb = quantise_e4m3(b, dim=0)
    return Problem(f"square_e4m3_{M}x{N}x{K}", row_major(qa, "e4m3"), row_major(qb, "e4m3"),
                   empty_out(M, N, "bf16"), 1.0, 0.0, sa, sb)


def nchw_as_rows(t: torch.Tensor, dtype: str) -> Operand:
    """An NCHW tensor [n,c,h,w] read in place as a [n*h*w, c] matrix (no copy).

    Rows are (n, h, w) in that order, columns are channels; byte strides come
    from the NCHW tensor.
    """
    es = ELEM_SIZE[dtype]
    n, c, h, w = t.shape
    sn, sc, sh, sw = (s * es for s in t.stride())
    return Operand(t, (n, h, w, c), (sn, sh, sw, sc), 3, dtype)


def cfg_strided(seed: int = 1006, n=16, c=256, h=14, w=14, N=1024) -> Problem:
    """NCHW BF16 [16,256,14,14] as A[3136x256] in place, times B[256x1024] -> FP32, U[-1,1]."""
    g = _gen(seed)
    x = cast(uniform((n, c, h, w), g), "bf16")
    B = cast(uniform((c, N), g), "bf16")
    return Problem(f"strided_nchw_bf16_{n * h * w}x{N}x{c}", nchw_as_rows(x, "bf16"),
                   row_major(B, "bf16"), empty_out(n * h * w, N, "f32"), 1.0, 0.0)


def with_epilogue(p: Problem, act: str = "gelu_tanh", seed: int = 2001, bias: bool = True) -> Problem:
    """The same problem with a fused epilogue: a bias per output column drawn
    from N(0, 1) (seeded) and an activation ("none", "relu", "gelu_tanh")."""
    g = _gen(seed)
    b = normal((p.N,), g).contiguous() if bias else None
    return Problem(f"{p.name}_{'bias_' if bias else ''}{act}", p.A, p.B, p.C, p.alpha, p.beta,
                   p.scale_a, p.scale_b, p.note, dict(p.extra), b, act)


def nchw_out(n: int, c: int, h: int, w: int, dtype: str = "f32") -> Operand:
    """An output written as an NCHW tensor [n, c, h, w] (NaN-filled) and
    addressed as the [n*h*w, c] product it receives: the epilogue's layout
    transform from rows of (n, h, w) to channel planes."""
    t = torch.full((n, c, h, w), float("nan"), dtype=torch.float32).to(TORCH_DTYPE[dtype])
    return nchw_as_rows(t, dtype)


WORKLOADS = {
    "small": cfg_small,
    "gemv": cfg_gemv,
    "gemv_kt": cfg_gemv_kt,
    "thin": cfg_thin,
    "square_bf16": cfg_square_bf16,
    "square_e4m3": cfg_square_e4m3,
    "strided": cfg_strided,
}
