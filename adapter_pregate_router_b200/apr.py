"""Python binding of libapr (include/apr.h): argument marshalling only.

Every function takes torch tensors that already live where the C ABI wants
them, passes their pointers and the current CUDA stream, and raises
``AprError`` on a non-OK status.  All computation happens in libapr's CUDA
kernels; there is no Python or CPU fallback, and importing this module fails
if the library is missing.
"""
from __future__ import annotations

import ctypes
import os

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libapr.so")

APR_OK = 0
APR_ERR_INVALID_ARG = 1
APR_ERR_UNSUPPORTED = 2
APR_ERR_WORKSPACE = 3
APR_ERR_CUDA = 4
APR_ERR_DEVICE_INDEX = 5
APR_ERR_TIMEOUT = 6

APR_F32 = 0
APR_BF16 = 1

SGMM_AUTO = 0
SGMM_SKINNY = 1
SGMM_TENSOR = 2
SGMM_DENSE = 3

MAX_E = 1024
MAX_K = 8
MAX_RANK = 128
MAX_PROJ = 4


class AprError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{_status_name(status)}: {message}")
        self.status = status


if not os.path.exists(LIB_PATH):
    raise ImportError(f"libapr.so is not built ({LIB_PATH}); run adapter_pregate_router_b200.build")

_lib = ctypes.CDLL(LIB_PATH)
_vp = ctypes.c_void_p
_i = ctypes.c_int
_sz = ctypes.c_size_t


class Proj(ctypes.Structure):
    """apr_proj"""
    _fields_ = [("y", _vp), ("y_base", _vp), ("d_out", _i), ("A", _vp), ("B", _vp)]


class MergeProj(ctypes.Structure):
    """apr_merge_proj"""
    _fields_ = [("W", _vp), ("Wp", _vp), ("d_in", _i), ("d_out", _i), ("A", _vp), ("B", _vp)]


def _sig(name, res, args):
    f = getattr(_lib, name)
    f.restype = res
    f.argtypes = args
    return f


_workspace_size = _sig("apr_workspace_size", _sz, [_i, _i, _i, _i, _i])
_workspace_init = _sig("apr_workspace_init", _i, [_vp, _sz, _vp])
_pregate_route = _sig("apr_pregate_route", _i, [_vp, _vp, _i, _i, _i, _i, _i, _vp, _vp, _vp, _sz, _vp])
_pregate_route_noalloc = _sig("apr_pregate_route_noalloc", _i, [_vp, _vp, _i, _i, _i, _i, _i, _vp, _vp, _vp])
_segment_tokens = _sig("apr_segment_tokens", _i, [_vp, _i, _i, _i, _vp, _vp, _vp, _sz, _vp])
_sgmm = _sig("apr_sgmm_shrink_expand", _i,
             [_vp, _i, ctypes.POINTER(Proj), _i, _i, _i, _i, _i, _vp, _i, _vp, _vp, _vp, _vp, _vp, _sz, _i, _vp])
_merge = _sig("apr_merge_adapters", _i, [_vp, _i, _i, _i, _vp, _vp, _i, _vp, _sz, _vp])
_merge_plan_size = _sig("apr_merge_plan_size", _sz, [_i])
_merge_plan_init = _sig("apr_merge_plan_init", _i, [_vp, _i, _vp, _sz])
_merge_planned = _sig("apr_merge_adapters_planned", _i, [_vp, _vp, _i, _i, _i, _vp, _vp, _i, _vp, _sz, _vp])
_gemv = _sig("apr_gemv", _i, [_vp, _vp, _vp, _i, _i, _vp])
_stream_status = _sig("apr_stream_status", _i, [_vp, _vp])
_last_error = _sig("apr_last_error", ctypes.c_char_p, [])
_status_string = _sig("apr_status_string", ctypes.c_char_p, [_i])
_kernel_launches = _sig("apr_kernel_launches", ctypes.c_uint64, [])

EXPORTED = ("apr_workspace_size", "apr_workspace_init", "apr_pregate_route", "apr_pregate_route_noalloc",
            "apr_segment_tokens",
            "apr_sgmm_shrink_expand", "apr_merge_adapters", "apr_merge_plan_size", "apr_merge_plan_init",
            "apr_merge_adapters_planned", "apr_gemv", "apr_stream_status",
            "apr_last_error", "apr_status_string", "apr_kernel_launches")


def _status_name(s: int) -> str:
    return _status_string(int(s)).decode()


def _check(status: int):
    if status != APR_OK:
        raise AprError(status, _last_error().decode())


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        if not torch.cuda.is_available():
            return None
        stream = torch.cuda.current_stream()
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return APR_BF16
    if t.dtype == torch.float32:
        return APR_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def last_error() -> str:
    return _last_error().decode()


def status_string(s: int) -> str:
    return _status_name(s)


def kernel_launches() -> int:
    return int(_kernel_launches())


def workspace_size(T: int, k: int, E: int, max_rank: int, max_d_in: int) -> int:
    return int(_workspace_size(T, k, E, max_rank, max_d_in))


def workspace(T: int, k: int, E: int, max_rank: int, max_d_in: int, device="cuda", stream=None):
    """Allocate (with torch) and initialise a workspace for these maxima."""
    n = workspace_size(T, k, E, max_rank, max_d_in)
    if n == 0:
        raise AprError(APR_ERR_INVALID_ARG, "workspace_size: arguments out of range")
    ws = torch.empty(n, dtype=torch.uint8, device=device)
    _check(_workspace_init(ws.data_ptr(), n, _stream(stream)))
    return ws


def pregate_route(h, Wr, k, idx, gate, ws, stream=None):
    T, d = h.shape
    E = Wr.shape[0]
    _check(_pregate_route(_ptr(h), _ptr(Wr), _dtype_code(h), T, d, E, k, _ptr(idx), _ptr(gate),
                          _ptr(ws), ws.numel(), _stream(stream)))


def pregate_route_noalloc(h, Wr, k, idx, gate, stream=None):
    """``pregate_route`` for callers that cannot allocate a workspace (library-owned scratch)."""
    T, d = h.shape
    E = Wr.shape[0]
    _check(_pregate_route_noalloc(_ptr(h), _ptr(Wr), _dtype_code(h), T, d, E, k, _ptr(idx), _ptr(gate),
                                  _stream(stream)))


def segment_tokens(idx, E, seg_off, perm, ws, stream=None):
    T, k = idx.shape
    _check(_segment_tokens(_ptr(idx), T, k, E, _ptr(seg_off), _ptr(perm), _ptr(ws), ws.numel(),
                           _stream(stream)))


def ptr_array(tensors, device="cuda") -> torch.Tensor:
    """Device array of device pointers (int64), as the A/B tables of the ABI want."""
    return torch.tensor([t.data_ptr() for t in tensors], dtype=torch.int64, device=device)


def make_proj(y, y_base, A_table, B_table) -> Proj:
    return Proj(_ptr(y), _ptr(y_base), int(y_base.shape[-1]), _ptr(A_table), _ptr(B_table))


def sgmm_shrink_expand(x, projs, k, E, ranks, max_rank, idx, gate, seg_off, perm, ws,
                       kernel=SGMM_AUTO, stream=None):
    """projs: a sequence of ``Proj`` (see ``make_proj``) sharing input ``x``."""
    T, d_in = x.shape
    arr = (Proj * len(projs))(*projs)
    _check(_sgmm(_ptr(x), d_in, arr, len(projs), _dtype_code(x), T, k, E, _ptr(ranks), max_rank,
                 _ptr(idx), _ptr(gate), _ptr(seg_off), _ptr(perm), _ptr(ws), ws.numel(), kernel,
                 _stream(stream)))


def _merge_host_table(entries):
    n = len(entries)
    arr = (MergeProj * n)()
    for i, (W, Wp, At, Bt) in enumerate(entries):
        arr[i] = MergeProj(_ptr(W), _ptr(Wp), int(W.shape[1]), int(W.shape[0]), _ptr(At), _ptr(Bt))
    return arr


def merge_table(entries, device="cuda") -> torch.Tensor:
    """Device array of apr_merge_proj from (W, Wp, A_table, B_table) tuples."""
    raw = bytes(memoryview(_merge_host_table(entries)).cast("B"))
    host = torch.frombuffer(bytearray(raw), dtype=torch.uint8)
    return host.to(device)


def merge_plan(entries, device="cuda") -> torch.Tensor:
    """TMA descriptors of the weights in ``entries`` (same order as ``merge_table``)."""
    n = len(entries)
    size = int(_merge_plan_size(n))
    if size == 0:
        raise AprError(APR_ERR_INVALID_ARG, "merge_plan_size: nproj out of range")
    plan = torch.empty(size + 128, dtype=torch.uint8, device=device)
    off = (-plan.data_ptr()) % 128
    plan = plan[off:off + size]
    _check(_merge_plan_init(_merge_host_table(entries), n, plan.data_ptr(), size))
    return plan


def merge_adapters_planned(table, plan, nproj, E, r, idx, gate, k, ws, stream=None):
    _check(_merge_planned(_ptr(table), _ptr(plan), nproj, E, r, _ptr(idx), _ptr(gate), k, _ptr(ws), ws.numel(),
                          _stream(stream)))


def merge_adapters(table, nproj, E, r, idx, gate, k, ws, stream=None):
    _check(_merge(_ptr(table), nproj, E, r, _ptr(idx), _ptr(gate), k, _ptr(ws), ws.numel(), _stream(stream)))


def gemv(W, x, y, stream=None):
    d_out, d_in = W.shape
    _check(_gemv(_ptr(W), _ptr(x), _ptr(y), d_in, d_out, _stream(stream)))


def stream_status(ws, stream=None):
    """Synchronise, then raise if a kernel recorded a device-side fault in ``ws``."""
    _check(_stream_status(_ptr(ws), _stream(stream)))


def raw_stream_status(ws, stream=None) -> int:
    return int(_stream_status(_ptr(ws), _stream(stream)))
