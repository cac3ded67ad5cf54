"""Shared helpers of the GPU parity tests: run a workload through the C ABI
and compare it with the FP64 oracle element by element.

Tolerances (from the accuracy targets of the benchmark definition; the pages
themselves only quote a 1e-4 check, "DeepGEMM: a recalibration of the compute
paradigm", §4.3):
  with S = |alpha * sa * sb| * sum_k |a b|  (the scale of the rounding error),
  FP32 output: |got - r| <= 5e-4 * S + 2^-22 * (|r| + |beta c|)
  BF16 output: |got - r| <= 4e-3 * |r| + 5e-4 * S
  FP16 output: |got - r| <= 2e-3 * |r| + 5e-4 * S + 2^-24
The 16-bit bounds have two terms: the rounding of the output to 16 bits is
relative to the result itself (half an ulp is 2^-9 |r| for BF16 and 2^-11 |r|
for FP16, so 4e-3 and 2e-3 leave a factor of two), and the FP32 accumulation
error is relative to S, with the same 5e-4 as for FP32 output.  A wrong value
on one entry is then held to the result's own size, not to S (which is about
sqrt(K) times larger for random data).
With the fused epilogue out = act(z), z = alpha*s*acc + beta*c + bias, the
FP32 error of z is 5e-4 * S + 2^-22 * (|z| + |beta c| + |bias|); the
activation passes it on multiplied by at most its largest slope (1 for ReLU,
1.129 for GeLU in its tanh form) and GeLU's evaluation adds at most 2^-20 |z|
for FP32 outputs (accurate tanh; near -1, 1 + tanh loses low bits) or 2^-11 |z|
for 16-bit outputs (the hardware tanh approximation); 16-bit outputs then add
their rounding relative to the result as above.
NaN positions must agree exactly; infinities must agree in sign and place.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
import tcgen05_tmem_gemm_b200 as dg
import workloads as W


def dg_view_of(op: W.Operand) -> dg.dg_view:
    return dg.make_view(op.base.data_ptr() + op.offset, op.shape, op.stride, op.row_dims, op.dtype)


def fused(problem: W.Problem) -> bool:
    return problem.bias is not None or problem.act != "none"


def run(problem: W.Problem, stream=None, check_status=True) -> W.Problem:
    """Enqueue dg_gemm (dg_gemm_ex for a fused epilogue) for a
    device-resident problem and wait for it."""
    A, B, C = dg_view_of(problem.A), dg_view_of(problem.B), dg_view_of(problem.C)
    if fused(problem):
        st = dg.dg_gemm_ex(A, B, C, problem.alpha, problem.beta, problem.scale_a, problem.scale_b,
                           dg.epilogue(problem.bias, problem.act), stream)
    else:
        st = dg.dg_gemm(A, B, C, problem.alpha, problem.beta, problem.scale_a, problem.scale_b, stream)
    if check_status:
        assert st == dg.DG_OK, dg.status_string(st)
    sst = dg.dg_sync_status(stream)
    if check_status:
        assert sst == dg.DG_OK, dg.status_string(sst)
    return problem


def plan(problem: W.Problem) -> dict:
    A, B, C = dg_view_of(problem.A), dg_view_of(problem.B), dg_view_of(problem.C)
    return dg.dg_plan(A, B, C, problem.alpha, problem.beta, problem.scale_a is not None).as_dict()


def c_matrix(problem: W.Problem) -> np.ndarray:
    """C as an [M, N] float64 array, read through its view on the host."""
    op = problem.C
    base = op.base.detach().cpu()
    flat = base.reshape(-1).view(torch.uint8)
    es = W.ELEM_SIZE[op.dtype]
    M, N = problem.M, problem.N
    out = np.empty((M, N), dtype=np.float64)
    # generic gather through the view (C views are small in tests or 2-D)
    t = torch.as_strided(base.reshape(-1).view(W.TORCH_DTYPE[op.dtype]),
                         size=op.shape, stride=[s // es for s in op.stride],
                         storage_offset=op.offset // es)
    out[:] = t.to(torch.float64).reshape(M, N).numpy()
    del flat
    return out


ACT_SLOPE = {"none": 1.0, "relu": 1.0, "gelu_tanh": 1.13}


def tolerance(out_dtype: str, ref, bound, beta_c, pre=None, bias_abs=None, act="none"):
    ref = np.abs(ref)
    if pre is None and bias_abs is None and act == "none":
        # plain GEMM: out = z
        if out_dtype == "f32":
            return 5e-4 * bound + 2.0 ** -22 * (ref + np.abs(beta_c))
        if out_dtype == "bf16":
            return 4e-3 * ref + 5e-4 * bound
        if out_dtype == "f16":
            return 2e-3 * ref + 5e-4 * bound + 2.0 ** -24
        raise ValueError(out_dtype)
    z = np.abs(pre) if pre is not None else ref
    b = bias_abs if bias_abs is not None else 0.0
    tz = ACT_SLOPE[act] * (5e-4 * bound + 2.0 ** -22 * (z + np.abs(beta_c) + b))
    if act == "gelu_tanh":
        # FP32 outputs evaluate tanh accurately; 16-bit outputs with the
        # hardware approximation (relative error about 2^-11 of the tanh, so at
        # most 2^-12 |z| in the output), below their own rounding
        tz = tz + (2.0 ** -20 if out_dtype == "f32" else 2.0 ** -11) * z
    if out_dtype == "f32":
        return tz
    if out_dtype == "bf16":
        return 4e-3 * ref + tz
    if out_dtype == "f16":
        return 2e-3 * ref + tz + 2.0 ** -24
    raise ValueError(out_dtype)


def compare(problem: W.Problem, got, ref, bound, beta_c=None, where="", pre=None, bias_abs=None):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if beta_c is None:
        beta_c = np.zeros_like(ref)
    nan_g, nan_r = np.isnan(got), np.isnan(ref)
    assert np.array_equal(nan_g, nan_r), f"{where}: NaN positions differ ({nan_g.sum()} vs {nan_r.sum()})"
    inf_r = np.isinf(ref)
    assert np.array_equal(np.isinf(got), inf_r), f"{where}: Inf positions differ"
    assert np.array_equal(got[inf_r], ref[inf_r]), f"{where}: Inf signs differ"
    fin = ~(nan_r | inf_r)
    err = np.abs(got[fin] - ref[fin])
    tol = tolerance(problem.C.dtype, ref[fin], bound[fin], beta_c[fin],
                    None if pre is None else np.asarray(pre)[fin],
                    None if bias_abs is None else np.broadcast_to(bias_abs, ref.shape)[fin], problem.act)
    bad = err > tol
    if bad.any():
        idx = np.argmax(err - tol)
        raise AssertionError(f"{where}: {bad.sum()} of {err.size} outside tolerance; worst err "
                             f"{err[idx]:.3e} tol {tol[idx]:.3e} ref {ref[fin][idx]:.6e} got {got[fin][idx]:.6e}")
    scale = np.maximum(bound[fin], 1e-30)
    norm = err / scale
    return {"max": float(norm.max(initial=0)), "mean": float(norm.mean()) if norm.size else 0.0,
            "rms": float(np.sqrt((norm ** 2).mean())) if norm.size else 0.0}


def beta_c_of(problem: W.Problem) -> np.ndarray:
    if problem.beta == 0:
        return np.zeros((problem.M, problem.N))
    return problem.beta * c_matrix(problem)


def _bias_abs(problem: W.Problem, ns=None):
    if problem.bias is None:
        return None
    b = np.abs(problem.bias.detach().cpu().double().numpy())
    return b if ns is None else b[ns]


def check_full(problem_cpu: W.Problem, stream=None) -> dict:
    """Run on the GPU and compare every output with the full oracle."""
    if fused(problem_cpu):
        ref, bound, pre = oracle.gemm(problem_cpu, want_pre=True)
    else:
        (ref, bound), pre = oracle.gemm(problem_cpu), None
    bc = beta_c_of(problem_cpu)
    gpu = problem_cpu.to("cuda")
    run(gpu, stream)
    got = c_matrix(gpu)
    return compare(problem_cpu, got, ref, bound, bc, problem_cpu.name, pre, _bias_abs(problem_cpu))


def tile_corners(M: int, N: int, bm: int, bn: int):
    """The four corner outputs of every bm x bn tile of an M x N output."""
    ms, ns = [], []
    for i0 in range(0, M, bm):
        for j0 in range(0, N, bn):
            i1, j1 = min(M, i0 + bm) - 1, min(N, j0 + bn) - 1
            ms += [i0, i0, i1, i1]
            ns += [j0, j1, j0, j1]
    return ms, ns


def check_sampled(problem_cpu: W.Problem, npts=2048, seed=0, gpu=None, extra=None) -> dict:
    """Run (unless `gpu` already ran) and compare sampled outputs with the
    one-by-one oracle: random points, the four corners, the last row and
    column, and the (ms, ns) lists in `extra`."""
    M, N = problem_cpu.M, problem_cpu.N
    rng = np.random.default_rng(seed)
    ms = list(rng.integers(0, M, npts)) + [0, 0, M - 1, M - 1] + [M - 1] * 16 + list(rng.integers(0, M, 16))
    ns = list(rng.integers(0, N, npts)) + [0, N - 1, 0, N - 1] + list(rng.integers(0, N, 16)) + [N - 1] * 16
    if extra is not None:
        ms += list(extra[0])
        ns += list(extra[1])
    ms, ns = np.array(ms), np.array(ns)
    ref, bound, pre = oracle.gemm_points(problem_cpu, ms, ns, want_pre=True)
    bc = problem_cpu.beta * c_matrix(problem_cpu)[ms, ns] if problem_cpu.beta != 0 else np.zeros(len(ms))
    if gpu is None:
        gpu = problem_cpu.to("cuda")
        run(gpu)
    got = c_matrix(gpu)[ms, ns]
    return compare(problem_cpu, got, ref, bound, bc, problem_cpu.name,
                   pre if fused(problem_cpu) else None, _bias_abs(problem_cpu, ns))
