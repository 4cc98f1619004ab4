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
SGMM_BANK = 4

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


class LinearProj(ctypes.Structure):
    """apr_linear_proj"""
    _fields_ = [("W", _vp), ("y", _vp), ("d_out", _i), ("A", _vp), ("B", _vp)]


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
_linear = _sig("apr_linear_lora", _i,
                [_vp, _i, ctypes.POINTER(LinearProj), _i, _i, _i, _i, _vp, _i, _vp, _vp, _vp, _vp, _vp, _sz, _vp])
_linear_workspace_size = _sig("apr_linear_workspace_size", _sz, [_i, _i, _i, _i, _i, _i, ctypes.c_long])
_merge = _sig("apr_merge_adapters", _i, [_vp, _i, _i, _i, _vp, _vp, _i, _vp, _sz, _vp])
_pool_state_bytes = _sig("apr_adapter_pool_state_bytes", _sz, [_i, _i])
_pool_init = _sig("apr_adapter_pool_init", _i,
                  [_vp, _sz, _i, _i, ctypes.POINTER(_vp), _sz, _vp, _vp, _sz, _vp, _vp, _i, _vp])
_pool_page_in = _sig("apr_adapter_pool_page_in", _i,
                     [_vp, _sz, _i, _i, _vp, _i, _i, _vp, _sz, _vp, _sz, _vp, _vp, _i, _vp, _sz, _vp])
_merge_escape_bytes = _sig("apr_merge_escape_bytes", _sz, [ctypes.c_long])
_merge_residual_bytes = _sig("apr_merge_residual_bytes", _sz, [_i, _i])
_merge_inplace = _sig("apr_merge_adapters_inplace", _i, [_vp, _i, _i, _i, _vp, _vp, _i, _vp, _sz, _vp, _sz, _vp])
_unmerge_inplace = _sig("apr_unmerge_adapters_inplace", _i, [_vp, _i, _i, _i, _vp, _vp, _i, _vp, _sz, _vp, _sz, _vp])
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
            "apr_sgmm_shrink_expand", "apr_linear_lora", "apr_linear_workspace_size", "apr_adapter_pool_state_bytes", "apr_adapter_pool_init", "apr_adapter_pool_page_in",
            "apr_merge_adapters", "apr_merge_escape_bytes", "apr_merge_residual_bytes", "apr_merge_adapters_inplace",
            "apr_unmerge_adapters_inplace", "apr_merge_plan_size", "apr_merge_plan_init",
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


def _need(t, name, dtypes=None, shape=None, ndim=None, min_numel=None):
    """Validate one tensor argument before its pointer crosses the ABI: a torch tensor of an
    accepted dtype and shape, contiguous.  The library reads raw memory, so a wrong dtype or
    shape here would become an out-of-bounds device access there."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor, got {type(t).__name__}")
    if dtypes is not None and t.dtype not in dtypes:
        raise TypeError(f"{name} has dtype {t.dtype}, expected {' or '.join(str(d) for d in dtypes)}")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dimensions, got shape {tuple(t.shape)}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if min_numel is not None and t.numel() < min_numel:
        raise ValueError(f"{name} has {t.numel()} elements, needs at least {min_numel}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _same_device(*named):
    """Every tensor argument lives on one CUDA device (checked after dtypes and shapes)."""
    for n, t in named:
        if not t.is_cuda:
            raise ValueError(f"{n} must be a CUDA tensor, got device {t.device}")
    devs = {t.device for _, t in named}
    if len(devs) > 1:
        raise ValueError("tensors on different devices: " + ", ".join(f"{n}={t.device}" for n, t in named))


_ACT = (torch.float32, torch.bfloat16)


def _need_ws(ws):
    _need(ws, "ws", (torch.uint8,), ndim=1)


def workspace(T: int, k: int, E: int, max_rank: int, max_d_in: int, device="cuda", stream=None):
    """Allocate (with torch) and initialise a workspace for these maxima."""
    n = workspace_size(T, k, E, max_rank, max_d_in)
    if n == 0:
        raise AprError(APR_ERR_INVALID_ARG, "workspace_size: arguments out of range")
    ws = torch.empty(n, dtype=torch.uint8, device=device)
    _check(_workspace_init(ws.data_ptr(), n, _stream(stream)))
    return ws


def _check_route_args(h, Wr, k, idx, gate):
    _need(h, "h", _ACT, ndim=2)
    T, d = h.shape
    _need(Wr, "Wr", (h.dtype,), ndim=2)
    if Wr.shape[1] != d:
        raise ValueError(f"Wr has {Wr.shape[1]} columns, h has {d}")
    _need(idx, "idx", (torch.int32,), shape=(T, k))
    _need(gate, "gate", (torch.float32,), shape=(T, k))
    return T, d, Wr.shape[0]


def pregate_route(h, Wr, k, idx, gate, ws, stream=None):
    T, d, E = _check_route_args(h, Wr, k, idx, gate)
    _need_ws(ws)
    _same_device(("h", h), ("Wr", Wr), ("idx", idx), ("gate", gate), ("ws", ws))
    _check(_pregate_route(_ptr(h), _ptr(Wr), _dtype_code(h), T, d, E, k, _ptr(idx), _ptr(gate),
                          _ptr(ws), ws.numel(), _stream(stream)))


def pregate_route_noalloc(h, Wr, k, idx, gate, stream=None):
    """``pregate_route`` for callers that cannot allocate a workspace (library-owned scratch)."""
    T, d, E = _check_route_args(h, Wr, k, idx, gate)
    _same_device(("h", h), ("Wr", Wr), ("idx", idx), ("gate", gate))
    _check(_pregate_route_noalloc(_ptr(h), _ptr(Wr), _dtype_code(h), T, d, E, k, _ptr(idx), _ptr(gate),
                                  _stream(stream)))


def segment_tokens(idx, E, seg_off, perm, ws, stream=None):
    _need(idx, "idx", (torch.int32,), ndim=2)
    T, k = idx.shape
    _need(seg_off, "seg_off", (torch.int32,), shape=(E + 1,))
    _need(perm, "perm", (torch.int32,), ndim=1, min_numel=T * k)
    _need_ws(ws)
    _same_device(("idx", idx), ("seg_off", seg_off), ("perm", perm), ("ws", ws))
    _check(_segment_tokens(_ptr(idx), T, k, E, _ptr(seg_off), _ptr(perm), _ptr(ws), ws.numel(),
                           _stream(stream)))


def ptr_array(tensors, device="cuda") -> torch.Tensor:
    """Device array of device pointers (int64), as the A/B tables of the ABI want."""
    return torch.tensor([t.data_ptr() for t in tensors], dtype=torch.int64, device=device)


def make_proj(y, y_base, A_table, B_table) -> Proj:
    """One projection of a shared-input group: y [T, d_out] (may be y_base itself), y_base
    [T, d_out] of the group's dtype, and the device tables of A and B pointers (int64 [E])."""
    _need(y_base, "y_base", _ACT, ndim=2)
    _need(y, "y", (y_base.dtype,), shape=tuple(y_base.shape))
    _need(A_table, "A_table", (torch.int64,), ndim=1)
    _need(B_table, "B_table", (torch.int64,), shape=tuple(A_table.shape))
    _same_device(("y", y), ("y_base", y_base), ("A_table", A_table), ("B_table", B_table))
    p = Proj(_ptr(y), _ptr(y_base), int(y_base.shape[-1]), _ptr(A_table), _ptr(B_table))
    p.meta = (y_base.dtype, int(y_base.shape[0]), int(A_table.shape[0]), y_base.device)
    return p


def sgmm_shrink_expand(x, projs, k, E, ranks, max_rank, idx, gate, seg_off, perm, ws,
                       kernel=SGMM_AUTO, stream=None):
    """projs: a sequence of ``Proj`` (see ``make_proj``) sharing input ``x``."""
    _need(x, "x", _ACT, ndim=2)
    T, d_in = x.shape
    for i, pj in enumerate(projs):
        meta = getattr(pj, "meta", None)
        if meta is None:
            raise TypeError(f"projs[{i}] was not made by make_proj")
        dt, t_rows, e_tab, pdev = meta
        if dt != x.dtype or t_rows != T or e_tab < E or pdev != x.device:
            raise ValueError(f"projs[{i}]: {dt} [{t_rows}, :] with {e_tab} adapters on {pdev} does not fit "
                             f"x {x.dtype} [{T}, {d_in}] with E={E} on {x.device}")
    _need(ranks, "ranks", (torch.int32,), shape=(E,))
    _need(idx, "idx", (torch.int32,), shape=(T, k))
    _need(gate, "gate", (torch.float32,), shape=(T, k))
    _need(seg_off, "seg_off", (torch.int32,), shape=(E + 1,))
    _need(perm, "perm", (torch.int32,), ndim=1, min_numel=T * k)
    _need_ws(ws)
    _same_device(("x", x), ("ranks", ranks), ("idx", idx), ("gate", gate), ("seg_off", seg_off),
                 ("perm", perm), ("ws", ws))
    arr = (Proj * len(projs))(*projs)
    _check(_sgmm(_ptr(x), d_in, arr, len(projs), _dtype_code(x), T, k, E, _ptr(ranks), max_rank,
                 _ptr(idx), _ptr(gate), _ptr(seg_off), _ptr(perm), _ptr(ws), ws.numel(), kernel,
                 _stream(stream)))


def linear_workspace_size(T: int, k: int, E: int, max_rank: int, max_d_in: int, nproj: int,
                          sum_d_out: int) -> int:
    return int(_linear_workspace_size(T, k, E, max_rank, max_d_in, nproj, sum_d_out))


def linear_workspace(T: int, k: int, E: int, max_rank: int, max_d_in: int, nproj: int, sum_d_out: int,
                     device="cuda", stream=None):
    """Allocate (with torch) and initialise a workspace that also serves ``linear_lora`` on
    groups of up to ``nproj`` projections whose output widths add up to ``sum_d_out``."""
    n = linear_workspace_size(T, k, E, max_rank, max_d_in, nproj, sum_d_out)
    if n == 0:
        raise AprError(APR_ERR_INVALID_ARG, "linear_workspace_size: arguments out of range")
    ws = torch.empty(n, dtype=torch.uint8, device=device)
    _check(_workspace_init(ws.data_ptr(), n, _stream(stream)))
    return ws


def make_linear_proj(W, y, A_table, B_table) -> LinearProj:
    """One projection of a fused group: base weight W [d_out, d_in] bf16, output y [T, d_out]
    bf16, and the device tables of A and B pointers (int64 [E])."""
    _need(W, "W", (torch.bfloat16,), ndim=2)
    d_out, d_in = W.shape
    _need(y, "y", (torch.bfloat16,), ndim=2)
    if y.shape[1] != d_out:
        raise ValueError(f"y has {y.shape[1]} columns, W has {d_out} rows")
    _need(A_table, "A_table", (torch.int64,), ndim=1)
    _need(B_table, "B_table", (torch.int64,), shape=tuple(A_table.shape))
    _same_device(("W", W), ("y", y), ("A_table", A_table), ("B_table", B_table))
    p = LinearProj(_ptr(W), _ptr(y), int(d_out), _ptr(A_table), _ptr(B_table))
    p.meta = (int(y.shape[0]), int(d_in), int(A_table.shape[0]), W.device)
    return p


def linear_lora(x, projs, k, E, ranks, max_rank, idx, gate, seg_off, perm, ws, stream=None):
    """projs: a sequence of ``LinearProj`` (see ``make_linear_proj``) sharing input ``x``:
    ``y_p = x W_p^T + sum_j gate B_e (A_e x)`` in one contraction per projection."""
    _need(x, "x", (torch.bfloat16,), ndim=2)
    T, d_in = x.shape
    for i, pj in enumerate(projs):
        meta = getattr(pj, "meta", None)
        if meta is None:
            raise TypeError(f"projs[{i}] was not made by make_linear_proj")
        t_rows, w_in, e_tab, pdev = meta
        if t_rows != T or w_in != d_in or e_tab < E or pdev != x.device:
            raise ValueError(f"projs[{i}]: y with {t_rows} rows, W with {w_in} columns, {e_tab} adapters on "
                             f"{pdev} does not fit x [{T}, {d_in}] with E={E} on {x.device}")
    _need(ranks, "ranks", (torch.int32,), shape=(E,))
    _need(idx, "idx", (torch.int32,), shape=(T, k))
    _need(gate, "gate", (torch.float32,), shape=(T, k))
    _need(seg_off, "seg_off", (torch.int32,), shape=(E + 1,))
    _need(perm, "perm", (torch.int32,), ndim=1, min_numel=T * k)
    _need_ws(ws)
    _same_device(("x", x), ("ranks", ranks), ("idx", idx), ("gate", gate), ("seg_off", seg_off),
                 ("perm", perm), ("ws", ws))
    arr = (LinearProj * len(projs))(*projs)
    _check(_linear(_ptr(x), d_in, arr, len(projs), T, k, E, _ptr(ranks), max_rank, _ptr(idx), _ptr(gate),
                   _ptr(seg_off), _ptr(perm), _ptr(ws), ws.numel(), _stream(stream)))


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


def _check_merge_args(table, nproj, idx, gate, k, ws):
    _need(table, "table", (torch.uint8,), ndim=1, min_numel=nproj * ctypes.sizeof(MergeProj))
    _need(idx, "idx", (torch.int32,), min_numel=k)
    _need(gate, "gate", (torch.float32,), min_numel=k)
    _need_ws(ws)
    _same_device(("table", table), ("idx", idx), ("gate", gate), ("ws", ws))


def merge_adapters_planned(table, plan, nproj, E, r, idx, gate, k, ws, stream=None):
    _check_merge_args(table, nproj, idx, gate, k, ws)
    _need(plan, "plan", (torch.uint8,), ndim=1, min_numel=int(_merge_plan_size(nproj)))
    _check(_merge_planned(_ptr(table), _ptr(plan), nproj, E, r, _ptr(idx), _ptr(gate), k, _ptr(ws), ws.numel(),
                          _stream(stream)))


def merge_adapters(table, nproj, E, r, idx, gate, k, ws, stream=None):
    _check_merge_args(table, nproj, idx, gate, k, ws)
    _check(_merge(_ptr(table), nproj, E, r, _ptr(idx), _ptr(gate), k, _ptr(ws), ws.numel(), _stream(stream)))


class AdapterPool:
    """Adapters in pinned host memory, ``n_slots`` of them resident on the device at a time
    (``apr_adapter_pool_*``).  ``host_buffers``: pinned uint8 CPU tensors of ``adapter_bytes``
    each (one per adapter, the layout given by ``offsets``); ``tables``: int64 device tensors
    [n_adapters] (the A/B pointer tables the SGMM calls take), each with the byte offset of its
    matrix inside an adapter."""

    def __init__(self, host_buffers, n_slots, tables, offsets, device="cuda", stream=None):
        self.n_adapters = len(host_buffers)
        self.n_slots = int(n_slots)
        sizes = {int(b.numel() * b.element_size()) for b in host_buffers}
        if len(sizes) != 1:
            raise ValueError("every adapter buffer must have the same size")
        self.adapter_bytes = sizes.pop()
        for i, b in enumerate(host_buffers):
            if b.is_cuda or not b.is_pinned() or not b.is_contiguous():
                raise ValueError(f"host_buffers[{i}] must be a contiguous pinned CPU tensor")
        if len(tables) != len(offsets):
            raise ValueError("one offset per table")
        for i, t in enumerate(tables):
            _need(t, f"tables[{i}]", (torch.int64,), shape=(self.n_adapters,))
        n = int(_pool_state_bytes(self.n_adapters, self.n_slots))
        if n == 0:
            raise AprError(APR_ERR_INVALID_ARG, "adapter_pool_state_bytes: arguments out of range")
        self.state = torch.empty(n, dtype=torch.uint8, device=device)
        self.pool = torch.empty(self.n_slots * self.adapter_bytes, dtype=torch.uint8, device=device)
        self.src_table = torch.empty(self.n_adapters, dtype=torch.int64, device=device)
        self.tables = list(tables)
        self.table_ptrs = torch.tensor([t.data_ptr() for t in tables], dtype=torch.int64, device=device)
        self.offsets = torch.tensor([int(o) for o in offsets], dtype=torch.int64, device=device)
        self.host_buffers = list(host_buffers)
        srcs = (_vp * self.n_adapters)(*[b.data_ptr() for b in host_buffers])
        _check(_pool_init(_ptr(self.state), n, self.n_adapters, self.n_slots, srcs, self.adapter_bytes,
                          _ptr(self.src_table), _ptr(self.pool), self.pool.numel(), _ptr(self.offsets),
                          _ptr(self.table_ptrs), len(self.tables), _stream(stream)))

    def page_in(self, idx, ws, stream=None):
        """Make every adapter ``idx`` [T, k] selects resident and point the tables at it."""
        _need(idx, "idx", (torch.int32,), ndim=2)
        _need_ws(ws)
        _same_device(("idx", idx), ("ws", ws), ("state", self.state))
        T, k = idx.shape
        _check(_pool_page_in(_ptr(self.state), self.state.numel(), self.n_adapters, self.n_slots, _ptr(idx), T, k,
                             _ptr(self.src_table), self.adapter_bytes, _ptr(self.pool), self.pool.numel(),
                             _ptr(self.offsets), _ptr(self.table_ptrs), len(self.tables), _ptr(ws), ws.numel(),
                             _stream(stream)))

    def stats(self):
        """(page-in calls, adapters copied in so far), synchronising."""
        h = self.state[:64].cpu()
        step = int(h[16:24].view(torch.int64).item())
        copies = int(h[24:32].view(torch.int64).item())
        return step, copies

    def slot_ptr(self, slot: int) -> int:
        return self.pool.data_ptr() + slot * self.adapter_bytes


def merge_escape_bytes(capacity: int) -> int:
    return int(_merge_escape_bytes(capacity))


def merge_residual(W: torch.Tensor) -> torch.Tensor:
    """The residual-code buffer of one weight for an in-place merge (int8, on W's device)."""
    _need(W, "W", (torch.bfloat16,), ndim=2)
    n = int(_merge_residual_bytes(int(W.shape[0]), int(W.shape[1])))
    if n == 0:
        raise AprError(APR_ERR_INVALID_ARG, "merge_residual_bytes: shape out of range")
    return torch.empty(n, dtype=torch.int8, device=W.device)


def merge_escapes(capacity: int, device="cuda") -> torch.Tensor:
    """A device buffer for ``capacity`` escapes of an in-place merge (uint8, 16-byte aligned)."""
    return torch.zeros(merge_escape_bytes(capacity), dtype=torch.uint8, device=device)


def _check_inplace_args(table, nproj, idx, gate, k, escapes, ws):
    _check_merge_args(table, nproj, idx, gate, k, ws)
    _need(escapes, "escapes", (torch.uint8,), ndim=1, min_numel=merge_escape_bytes(0))
    _same_device(("table", table), ("escapes", escapes), ("ws", ws))


def merge_adapters_inplace(table, nproj, E, r, idx, gate, k, escapes, ws, stream=None):
    """W <- rn(W + sum g B A) in place for every entry of ``table`` (see ``merge_table``: each
    entry's Wp is the int8 [d_out, d_in] residual-code buffer of that weight)."""
    _check_inplace_args(table, nproj, idx, gate, k, escapes, ws)
    _check(_merge_inplace(_ptr(table), nproj, E, r, _ptr(idx), _ptr(gate), k, _ptr(escapes), escapes.numel(),
                          _ptr(ws), ws.numel(), _stream(stream)))


def unmerge_adapters_inplace(table, nproj, E, r, idx, gate, k, escapes, ws, stream=None):
    """Restore every W of ``table`` bit for bit after ``merge_adapters_inplace`` (same routing)."""
    _check_inplace_args(table, nproj, idx, gate, k, escapes, ws)
    _check(_unmerge_inplace(_ptr(table), nproj, E, r, _ptr(idx), _ptr(gate), k, _ptr(escapes), escapes.numel(),
                            _ptr(ws), ws.numel(), _stream(stream)))


def gemv(W, x, y, stream=None):
    _need(W, "W", (torch.bfloat16,), ndim=2)
    d_out, d_in = W.shape
    _need(x, "x", (torch.bfloat16,), shape=(d_in,))
    _need(y, "y", (torch.bfloat16,), shape=(d_out,))
    _same_device(("W", W), ("x", x), ("y", y))
    _check(_gemv(_ptr(W), _ptr(x), _ptr(y), d_in, d_out, _stream(stream)))


def stream_status(ws, stream=None):
    """Synchronise, then raise if a kernel recorded a device-side fault in ``ws``."""
    _check(_stream_status(_ptr(ws), _stream(stream)))


def raw_stream_status(ws, stream=None) -> int:
    return int(_stream_status(_ptr(ws), _stream(stream)))
