"""Python front of the FP64 CPU oracle (``dg_oracle.c``).

TEST INFRASTRUCTURE ONLY: imported by the test suite, the smoke check and the
benchmark's CPU-baseline / reference leg, never by the library it checks.
It shares no code with the CUDA path; both sides only share the seeded input
generators in ``workloads.py``.

The oracle computes, in FP64,
    z[m, n] = alpha * sa[m] * sb[n] * sum_k a(m, k) b(k, n) + beta * c(m, n) + bias[n]
    r[m, n] = act(z[m, n])      (identity, ReLU or GeLU in its tanh form)
over byte-strided views ("DeepGEMM: a recalibration of the compute paradigm",
§2.3 address formula and §3.2 view struct), decoding FP8 E4M3 from its bits
("DeepGEMM deep dive", §2.4), with the fused bias and activation of "DeepGEMM is
not a new model: the inner discipline of GPU matrix multiplication", §3.3.
See ``dg_oracle.c`` for the readings it takes
where the pages are silent.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dg_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

DTYPE_CODE = {"f32": 0, "f16": 1, "bf16": 2, "e4m3": 3}
ACT_CODE = {"none": 0, "relu": 1, "gelu_tanh": 2}


class OView(ctypes.Structure):
    _fields_ = [
        ("base", ctypes.c_void_p),
        ("ndim", ctypes.c_int32),
        ("row_dims", ctypes.c_int32),
        ("dtype", ctypes.c_int32),
        ("pad_", ctypes.c_int32),
        ("shape", ctypes.c_int64 * 4),
        ("stride", ctypes.c_int64 * 4),
    ]


def build(force: bool = False, src: str = _SRC, out: str = _LIB) -> str:
    """Compile the oracle with gcc (-O2, OpenMP). Returns the library path."""
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c99", src, "-o", out, "-lm"]
        subprocess.run(cmd, check=True)
    return out


class Oracle:
    """A loaded copy of the oracle library (``path`` defaults to the built one)."""

    def __init__(self, path: str | None = None):
        if path is None:
            path = build()
        L = ctypes.CDLL(path)
        P = ctypes.POINTER
        L.dgo_gemm.argtypes = [P(OView), P(OView), P(OView), ctypes.c_double, ctypes.c_double,
                               ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
                               ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]
        L.dgo_gemm.restype = ctypes.c_int
        L.dgo_gemm_points.argtypes = [P(OView), P(OView), P(OView), ctypes.c_double,
                                      ctypes.c_double, ctypes.c_void_p, ctypes.c_void_p,
                                      ctypes.c_void_p, ctypes.c_int,
                                      ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64,
                                      ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]
        L.dgo_gemm_points.restype = ctypes.c_int
        L.dgo_activation.argtypes = [ctypes.c_int, ctypes.c_double]
        L.dgo_activation.restype = ctypes.c_double
        L.dgo_decode_e4m3.argtypes = [ctypes.c_uint]
        L.dgo_decode_e4m3.restype = ctypes.c_double
        L.dgo_decode.argtypes = [ctypes.c_int, ctypes.c_void_p]
        L.dgo_decode.restype = ctypes.c_double
        L.dgo_offset.argtypes = [P(OView), ctypes.c_int64, ctypes.c_int64]
        L.dgo_offset.restype = ctypes.c_int64
        L.dgo_max_threads.restype = ctypes.c_int
        self.L = L

    def gemm(self, problem, want_bound: bool = True, nthreads: int = 0, want_pre: bool = False):
        """Full FP64 result as an [M, N] float64 array; with want_bound also the
        rounding scale S, with want_pre also the value before the activation."""
        keep = []
        ops = (problem.A, problem.B, problem.C)
        bufs = [_Bytes(o) for o in ops]
        va, vb, vc = (b.view(o) for b, o in zip(bufs, ops))
        M, N = problem.M, problem.N
        out = np.empty((M, N), dtype=np.float64)
        bound = np.empty((M, N), dtype=np.float64) if want_bound else None
        pre = np.empty((M, N), dtype=np.float64) if want_pre else None
        st = self.L.dgo_gemm(ctypes.byref(va), ctypes.byref(vb), ctypes.byref(vc),
                             float(problem.alpha), float(problem.beta),
                             _scale_ptr(problem.scale_a, keep), _scale_ptr(problem.scale_b, keep),
                             _scale_ptr(getattr(problem, "bias", None), keep),
                             ACT_CODE[getattr(problem, "act", "none")],
                             out.ctypes.data, None if bound is None else bound.ctypes.data,
                             None if pre is None else pre.ctypes.data, nthreads)
        if st != 0:
            raise ValueError(f"oracle rejected the problem (status {st})")
        res = (out,) + ((bound,) if want_bound else ()) + ((pre,) if want_pre else ())
        return res if len(res) > 1 else out

    def gemm_points(self, problem, ms, ns, nthreads: int = 0, want_pre: bool = False):
        """The definition evaluated at the sampled outputs (ms[i], ns[i]):
        (out, bound) or, with want_pre, (out, bound, pre)."""
        keep = []
        ops = (problem.A, problem.B, problem.C)
        bufs = [_Bytes(o) for o in ops]
        va, vb, vc = (b.view(o) for b, o in zip(bufs, ops))
        ms = np.ascontiguousarray(np.asarray(ms, dtype=np.int64))
        ns = np.ascontiguousarray(np.asarray(ns, dtype=np.int64))
        out = np.empty(len(ms), dtype=np.float64)
        bound = np.empty(len(ms), dtype=np.float64)
        pre = np.empty(len(ms), dtype=np.float64)
        st = self.L.dgo_gemm_points(ctypes.byref(va), ctypes.byref(vb), ctypes.byref(vc),
                                    float(problem.alpha), float(problem.beta),
                                    _scale_ptr(problem.scale_a, keep),
                                    _scale_ptr(problem.scale_b, keep),
                                    _scale_ptr(getattr(problem, "bias", None), keep),
                                    ACT_CODE[getattr(problem, "act", "none")],
                                    ms.ctypes.data, ns.ctypes.data, len(ms),
                                    out.ctypes.data, bound.ctypes.data, pre.ctypes.data, nthreads)
        if st != 0:
            raise ValueError(f"oracle rejected the problem (status {st})")
        return (out, bound, pre) if want_pre else (out, bound)

    def activation(self, act: str, z: float) -> float:
        """The epilogue's activation applied to one FP64 value."""
        return self.L.dgo_activation(ACT_CODE[act], float(z))

    def decode_e4m3(self, code: int) -> float:
        return self.L.dgo_decode_e4m3(code)

    def decode(self, dtype: str, raw: bytes) -> float:
        buf = ctypes.create_string_buffer(bytes(raw), len(raw))
        return self.L.dgo_decode(DTYPE_CODE[dtype], ctypes.cast(buf, ctypes.c_void_p))

    def offset(self, operand, r: int, c: int) -> int:
        """Byte offset of matrix element (r, c) of a view, per the oracle's addressing."""
        b = _Bytes(operand)
        v = b.view(operand)
        return self.L.dgo_offset(ctypes.byref(v), r, c)

    def max_threads(self) -> int:
        return self.L.dgo_max_threads()


_default = None


def default() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle()
    return _default


class _Bytes:
    """Keeps a host byte buffer alive while an OView points into it."""

    def __init__(self, operand):
        t = operand.base
        if t.device.type != "cpu":
            t = t.cpu()
        if not t.is_contiguous():
            raise ValueError("operand base must own contiguous storage")
        self.buf = t.reshape(-1).view(torch.uint8).numpy()
        self.ptr = self.buf.ctypes.data + int(operand.offset)

    def view(self, operand) -> OView:
        v = OView()
        v.base = self.ptr
        v.ndim = len(operand.shape)
        v.row_dims = operand.row_dims
        v.dtype = DTYPE_CODE[operand.dtype]
        for i in range(4):
            v.shape[i] = int(operand.shape[i]) if i < v.ndim else 1
            v.stride[i] = int(operand.stride[i]) if i < v.ndim else 0
        return v


def _scale_ptr(s, keep):
    if s is None:
        return None
    a = np.ascontiguousarray(s.detach().cpu().numpy().astype(np.float32))
    keep.append(a)
    return a.ctypes.data


def gemm(problem, want_bound: bool = True, nthreads: int = 0, want_pre: bool = False):
    return default().gemm(problem, want_bound, nthreads, want_pre)


def gemm_points(problem, ms, ns, nthreads: int = 0, want_pre: bool = False):
    return default().gemm_points(problem, ms, ns, nthreads, want_pre)


def activation(act: str, z: float) -> float:
    return default().activation(act, z)


def decode_e4m3(code: int) -> float:
    return default().decode_e4m3(code)


def decode(dtype: str, raw: bytes) -> float:
    return default().decode(dtype, raw)


def offset(operand, r: int, c: int) -> int:
    return default().offset(operand, r, c)


def max_threads() -> int:
    return default().max_threads()
