"""Python binding of libdg, the B200 (sm_100a) strided-view GEMM library.

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind the C ABI declared in include/dg.h.  The names mirror the C
entry points (dg_gemm, dg_gemm_ex, dg_gemv, dg_sync_status, ...).  PyTorch is used by
callers for device memory and streams; a torch tensor can be turned into a
view with `view()`.

The library must have been built (``python tcgen05_tmem_gemm_b200/build.py``
or ``__graft_entry__.build()``); importing this package without it raises.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdg.so")

DG_F32, DG_F16, DG_BF16, DG_E4M3 = 0, 1, 2, 3
DTYPE = {"f32": DG_F32, "f16": DG_F16, "bf16": DG_BF16, "e4m3": DG_E4M3}
ELEM_SIZE = {DG_F32: 4, DG_F16: 2, DG_BF16: 2, DG_E4M3: 1}

(DG_OK, DG_ERR_NULL, DG_ERR_NDIM, DG_ERR_SHAPE, DG_ERR_DTYPE, DG_ERR_STRIDE, DG_ERR_ALIGN,
 DG_ERR_POINTER, DG_ERR_VALUE, DG_ERR_UNSUPPORTED, DG_ERR_CUDA, DG_ERR_TIMEOUT) = range(12)

(DG_KIND_NONE, DG_KIND_SCALE_C, DG_KIND_SIMT, DG_KIND_GEMV_N, DG_KIND_GEMV_K,
 DG_KIND_UMMA) = range(6)
KIND_NAME = {0: "none", 1: "scale_c", 2: "simt", 3: "gemv_n", 4: "gemv_k", 5: "umma"}

DG_ACT_NONE, DG_ACT_RELU, DG_ACT_GELU_TANH = 0, 1, 2
ACT = {"none": DG_ACT_NONE, "relu": DG_ACT_RELU, "gelu_tanh": DG_ACT_GELU_TANH}

(DG_OPT_FORCE_KIND, DG_OPT_WAIT_TIMEOUT_MS, DG_OPT_TEST_STALL, DG_OPT_MAX_SPLIT_K, DG_OPT_CTA_PAIR,
 DG_OPT_EARLY_LAUNCH, DG_OPT_TRACE, DG_OPT_EPI_TMA, DG_OPT_GATHER_CLUSTER,
 DG_OPT_PAIR_TAIL, DG_OPT_STREAM_K, DG_OPT_DETERMINISTIC,
 DG_OPT_PAIR_DEEP_STAGES) = 1, 2, 3, 4, 5, 6, 7, 8, 9, 10, 11, 12, 13


class dg_view(ctypes.Structure):
    _fields_ = [
        ("ptr", ctypes.c_void_p),
        ("ndim", ctypes.c_int32),
        ("row_dims", ctypes.c_int32),
        ("shape", ctypes.c_int64 * 4),
        ("stride", ctypes.c_int64 * 4),
        ("dtype", ctypes.c_int32),
        ("reserved", ctypes.c_int32),
    ]


class dg_epilogue(ctypes.Structure):
    _fields_ = [
        ("bias", ctypes.c_void_p),
        ("activation", ctypes.c_int32),
        ("reserved", ctypes.c_int32),
    ]


class dg_view_info(ctypes.Structure):
    _fields_ = [
        ("rows", ctypes.c_int64), ("cols", ctypes.c_int64),
        ("n_row", ctypes.c_int32), ("n_col", ctypes.c_int32),
        ("row_shape", ctypes.c_int64 * 4), ("row_stride", ctypes.c_int64 * 4),
        ("col_shape", ctypes.c_int64 * 4), ("col_stride", ctypes.c_int64 * 4),
        ("unit_dim", ctypes.c_int32), ("tma_ok", ctypes.c_int32),
        ("span_bytes", ctypes.c_int64),
        ("vec_bytes", ctypes.c_int32), ("reserved", ctypes.c_int32),
    ]


class dg_plan_info(ctypes.Structure):
    _fields_ = [
        ("kind", ctypes.c_int32), ("swap_ab", ctypes.c_int32), ("p_gather", ctypes.c_int32),
        ("p_mn_major", ctypes.c_int32), ("q_mn_major", ctypes.c_int32),
        ("block_m", ctypes.c_int32), ("block_n", ctypes.c_int32), ("block_k", ctypes.c_int32),
        ("stages", ctypes.c_int32), ("split_k", ctypes.c_int32), ("grid", ctypes.c_int32),
        ("vec_bytes", ctypes.c_int32),
        ("M", ctypes.c_int64), ("N", ctypes.c_int64), ("K", ctypes.c_int64),
        ("cta_pair", ctypes.c_int32), ("epi_tma_store", ctypes.c_int32),
        ("gather_cluster", ctypes.c_int32), ("pair_half_tiles", ctypes.c_int32),
        ("stream_k_tiles", ctypes.c_int32), ("split_reduce_add", ctypes.c_int32),
    ]

    def as_dict(self) -> dict:
        d = {name: getattr(self, name) for name, _ in self._fields_}
        d["kind_name"] = KIND_NAME.get(self.kind, "?")
        return d


class dg_tune_result(ctypes.Structure):
    _fields_ = [
        ("candidates", ctypes.c_int32), ("reserved", ctypes.c_int32),
        ("default_us", ctypes.c_float), ("best_us", ctypes.c_float),
        ("plan", dg_plan_info),
    ]


class DgError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libdg.so is not built ({LIB_PATH}); run python tcgen05_tmem_gemm_b200/build.py")
    L = ctypes.CDLL(LIB_PATH)
    P = ctypes.POINTER
    V = P(dg_view)
    L.dg_gemm.argtypes = [V, V, V, ctypes.c_float, ctypes.c_float, ctypes.c_void_p, ctypes.c_void_p,
                          ctypes.c_void_p]
    L.dg_gemm.restype = ctypes.c_int
    L.dg_gemm_ex.argtypes = [V, V, V, ctypes.c_float, ctypes.c_float, ctypes.c_void_p, ctypes.c_void_p,
                             P(dg_epilogue), ctypes.c_void_p]
    L.dg_gemm_ex.restype = ctypes.c_int
    L.dg_gemv.argtypes = [V, V, V, ctypes.c_float, ctypes.c_float, ctypes.c_void_p]
    L.dg_gemv.restype = ctypes.c_int
    L.dg_status_string.argtypes = [ctypes.c_int]
    L.dg_status_string.restype = ctypes.c_char_p
    L.dg_sync_status.argtypes = [ctypes.c_void_p]
    L.dg_sync_status.restype = ctypes.c_int
    L.dg_analyse_view.argtypes = [V, P(dg_view_info)]
    L.dg_analyse_view.restype = ctypes.c_int
    L.dg_plan.argtypes = [V, V, V, ctypes.c_float, ctypes.c_float, ctypes.c_int, ctypes.c_int,
                          P(dg_plan_info)]
    L.dg_plan.restype = ctypes.c_int
    L.dg_autotune.argtypes = [V, V, V, ctypes.c_float, ctypes.c_float, ctypes.c_void_p, ctypes.c_void_p,
                              P(dg_epilogue), ctypes.c_void_p, ctypes.c_int, P(dg_tune_result)]
    L.dg_autotune.restype = ctypes.c_int
    L.dg_gemm_static.argtypes = [V, V, V, ctypes.c_float, ctypes.c_float, ctypes.c_void_p, ctypes.c_void_p,
                                 ctypes.c_void_p]
    L.dg_gemm_static.restype = ctypes.c_int
    L.dg_tune_clear.argtypes = []
    L.dg_tune_clear.restype = ctypes.c_int
    L.dg_launch_count.argtypes = []
    L.dg_launch_count.restype = ctypes.c_uint64
    L.dg_set_option.argtypes = [ctypes.c_int, ctypes.c_int64]
    L.dg_set_option.restype = ctypes.c_int
    L.dg_version.argtypes = []
    L.dg_version.restype = ctypes.c_int
    return L


lib = _load()


# ------------------------------------------------------------------ views

def make_view(ptr: int, shape, stride_bytes, row_dims: int, dtype) -> dg_view:
    """A dg_view from a raw device address, up to 4 dims, BYTE strides."""
    if isinstance(dtype, str):
        dtype = DTYPE[dtype]
    v = dg_view()
    v.ptr = ctypes.c_void_p(int(ptr))
    v.ndim = len(shape)
    v.row_dims = int(row_dims)
    for i in range(4):
        v.shape[i] = int(shape[i]) if i < len(shape) else 1
        v.stride[i] = int(stride_bytes[i]) if i < len(shape) else 0
    v.dtype = int(dtype)
    v.reserved = 0
    return v


_TORCH_DT = None


def _torch_dtype_code(t) -> int:
    global _TORCH_DT
    import torch

    if _TORCH_DT is None:
        _TORCH_DT = {torch.float32: DG_F32, torch.float16: DG_F16, torch.bfloat16: DG_BF16,
                     torch.float8_e4m3fn: DG_E4M3}
    if t.dtype not in _TORCH_DT:
        raise TypeError(f"unsupported tensor dtype {t.dtype}")
    return _TORCH_DT[t.dtype]


def view(t, row_dims: int = 1) -> dg_view:
    """A dg_view of a torch tensor in place (its strides, in bytes, as they are)."""
    code = _torch_dtype_code(t)
    es = t.element_size()
    shape = tuple(t.shape) if t.dim() > 0 else (1,)
    stride = tuple(s * es for s in t.stride()) if t.dim() > 0 else (es,)
    if len(shape) > 4:
        raise ValueError("views have at most 4 dims")
    return make_view(t.data_ptr(), shape, stride, row_dims, code)


def _as_view(x, row_dims=1):
    return x if isinstance(x, dg_view) else view(x, row_dims)


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream_ptr(stream):
    if stream is None:
        import torch

        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


# --------------------------------------------------------------- entry points

def status_string(status: int) -> str:
    return lib.dg_status_string(int(status)).decode()


def dg_gemm(A: dg_view, B: dg_view, C: dg_view, alpha: float, beta: float,
            scale_a=None, scale_b=None, stream=None) -> int:
    """C = alpha * diag(scale_a) A B diag(scale_b) + beta * C on `stream`; returns the status."""
    return lib.dg_gemm(ctypes.byref(A), ctypes.byref(B), ctypes.byref(C), float(alpha), float(beta),
                       _ptr(scale_a), _ptr(scale_b), _stream_ptr(stream))


def epilogue(bias=None, act="none") -> dg_epilogue:
    """A dg_epilogue: bias (device float32[N] tensor, address or None) and activation."""
    e = dg_epilogue()
    e.bias = ctypes.c_void_p(_ptr(bias) or 0)
    e.activation = ACT[act] if isinstance(act, str) else int(act)
    e.reserved = 0
    return e


def dg_gemm_ex(A: dg_view, B: dg_view, C: dg_view, alpha: float, beta: float,
               scale_a=None, scale_b=None, epi=None, stream=None) -> int:
    """dg_gemm with a fused epilogue C = act(... + beta * C + bias); returns the status."""
    return lib.dg_gemm_ex(ctypes.byref(A), ctypes.byref(B), ctypes.byref(C), float(alpha), float(beta),
                          _ptr(scale_a), _ptr(scale_b), None if epi is None else ctypes.byref(epi),
                          _stream_ptr(stream))


def dg_gemv(x: dg_view, W: dg_view, y: dg_view, alpha: float, beta: float, stream=None) -> int:
    return lib.dg_gemv(ctypes.byref(x), ctypes.byref(W), ctypes.byref(y), float(alpha), float(beta),
                       _stream_ptr(stream))


def dg_sync_status(stream=None) -> int:
    return lib.dg_sync_status(_stream_ptr(stream))


def dg_analyse_view(v: dg_view) -> dg_view_info:
    out = dg_view_info()
    st = lib.dg_analyse_view(ctypes.byref(v), ctypes.byref(out))
    if st != DG_OK:
        raise DgError(st, "dg_analyse_view")
    return out


def dg_plan(A: dg_view, B: dg_view, C: dg_view, alpha=1.0, beta=0.0, has_scales=False,
            num_sms: int = 0) -> dg_plan_info:
    out = dg_plan_info()
    st = lib.dg_plan(ctypes.byref(A), ctypes.byref(B), ctypes.byref(C), float(alpha), float(beta),
                     int(bool(has_scales)), int(num_sms), ctypes.byref(out))
    if st != DG_OK:
        raise DgError(st, "dg_plan")
    return out


def dg_autotune(A: dg_view, B: dg_view, C: dg_view, alpha: float, beta: float, scale_a=None, scale_b=None,
                epi=None, stream=None, reps: int = 5):
    """Time the kernel variants for this call, keep the fastest for its shape
    key, and run the call: returns (status, dg_tune_result)."""
    out = dg_tune_result()
    st = lib.dg_autotune(ctypes.byref(A), ctypes.byref(B), ctypes.byref(C), float(alpha), float(beta),
                         _ptr(scale_a), _ptr(scale_b), None if epi is None else ctypes.byref(epi),
                         _stream_ptr(stream), int(reps), ctypes.byref(out))
    return st, out


def dg_tune_clear() -> None:
    lib.dg_tune_clear()


def dg_launch_count() -> int:
    return int(lib.dg_launch_count())


def dg_set_option(option: int, value: int) -> None:
    st = lib.dg_set_option(int(option), int(value))
    if st != DG_OK:
        raise DgError(st, "dg_set_option")


def dg_version() -> int:
    return int(lib.dg_version())


# ----------------------------------------------------------- conveniences

def gemm(A, B, C, alpha: float = 1.0, beta: float = 0.0, scale_a=None, scale_b=None,
         stream=None, a_row_dims: int = 1, b_row_dims: int = 1, c_row_dims: int = 1,
         bias=None, act="none"):
    """dg_gemm (dg_gemm_ex when a bias or activation is given) on torch tensors
    or dg_view objects; raises DgError on a bad status."""
    if bias is None and act in ("none", DG_ACT_NONE):
        st = dg_gemm(_as_view(A, a_row_dims), _as_view(B, b_row_dims), _as_view(C, c_row_dims),
                     alpha, beta, scale_a, scale_b, stream)
    else:
        st = dg_gemm_ex(_as_view(A, a_row_dims), _as_view(B, b_row_dims), _as_view(C, c_row_dims),
                        alpha, beta, scale_a, scale_b, epilogue(bias, act), stream)
    if st != DG_OK:
        raise DgError(st, "dg_gemm")
    return C


def gemv(x, W, y, alpha: float = 1.0, beta: float = 0.0, stream=None):
    st = dg_gemv(_as_view(x, 1), _as_view(W, 1), _as_view(y, 1), alpha, beta, stream)
    if st != DG_OK:
        raise DgError(st, "dg_gemv")
    return y
