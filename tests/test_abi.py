"""The C ABI library: it builds, loads without a GPU, exports every declared
symbol, and rejects bad arguments on the host before launching anything."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def apr():
    from adapter_pregate_router_b200 import build
    build.build()
    from adapter_pregate_router_b200 import apr as mod
    return mod


def declared_symbols():
    names = []
    for h in os.listdir(os.path.join(ROOT, "include")):
        if not h.endswith(".h"):
            continue
        text = open(os.path.join(ROOT, "include", h)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names += re.findall(r"\b(apr_[a-z0-9_]+)\s*\(", text)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(apr):
    lib = ctypes.CDLL(apr.LIB_PATH)
    names = declared_symbols()
    assert "apr_sgmm_shrink_expand" in names and "apr_pregate_route" in names
    for n in names:
        assert hasattr(lib, n), f"{n} declared in include/ but not exported"
    assert set(apr.EXPORTED) <= set(names)


def test_library_has_no_libcuda_dependency(apr):
    import subprocess
    out = subprocess.run(["ldd", apr.LIB_PATH], capture_output=True, text=True).stdout
    assert "libcuda.so" not in out and "libcudart.so" not in out


def test_workspace_size(apr):
    assert apr.workspace_size(32, 2, 8, 16, 11008) > 0
    assert apr.workspace_size(32, 2, 8, 12, 4096) == 0          # rank not a multiple of 8
    assert apr.workspace_size(32, 9, 16, 16, 4096) == 0          # k > 8
    assert apr.workspace_size(32, 2, 2048, 16, 4096) == 0        # E too large
    a = apr.workspace_size(8192, 2, 16, 16, 11008)
    b = apr.workspace_size(8192, 2, 16, 64, 11008)
    assert b > a


def test_status_strings(apr):
    assert apr.status_string(0) == "APR_OK"
    assert apr.status_string(5) == "APR_ERR_DEVICE_INDEX"
    assert apr.status_string(99) == "APR_ERR_UNKNOWN"


def _route(apr, **kw):
    args = dict(h=0x1000, Wr=0x1000, dtype=1, T=4, d=64, E=8, k=2, idx=0x1000, gate=0x1000,
                ws=0x100000, ws_bytes=1 << 30, stream=None)
    args.update(kw)
    return apr._pregate_route(*args.values())


def test_route_host_validation(apr):
    assert _route(apr, k=9) == apr.APR_ERR_INVALID_ARG
    assert _route(apr, k=0) == apr.APR_ERR_INVALID_ARG
    assert _route(apr, E=4, k=5) == apr.APR_ERR_INVALID_ARG
    assert _route(apr, E=2000) == apr.APR_ERR_INVALID_ARG
    assert _route(apr, d=60) == apr.APR_ERR_INVALID_ARG
    assert _route(apr, dtype=7) == apr.APR_ERR_INVALID_ARG
    assert _route(apr, h=None) == apr.APR_ERR_INVALID_ARG
    assert _route(apr, h=0x1008) == apr.APR_ERR_INVALID_ARG       # not 16-byte aligned
    assert _route(apr, ws=None) == apr.APR_ERR_WORKSPACE
    assert _route(apr, ws=0x100010) == apr.APR_ERR_WORKSPACE      # not 256-byte aligned
    assert _route(apr, ws_bytes=16) == apr.APR_ERR_WORKSPACE
    assert _route(apr, T=0, h=None, idx=None) == apr.APR_OK        # empty batch: no-op
    assert "k=9" in (_route(apr, k=9) and apr.last_error())


def test_sgmm_host_validation(apr):
    P = apr.Proj(0x1000, 0x1000, 64, 0x1000, 0x1000)
    arr = (apr.Proj * 1)(P)

    def call(**kw):
        a = dict(x=0x1000, d_in=64, projs=arr, nproj=1, dtype=1, T=4, k=2, E=8, ranks=0x1000,
                 max_rank=16, idx=0x1000, gate=0x1000, seg_off=0x1000, perm=0x1000, ws=0x100000,
                 ws_bytes=1 << 30, kernel=0, stream=None)
        a.update(kw)
        return apr._sgmm(*a.values())

    assert call(nproj=0) == apr.APR_ERR_INVALID_ARG
    assert call(nproj=5) == apr.APR_ERR_INVALID_ARG
    assert call(max_rank=12) == apr.APR_ERR_INVALID_ARG
    assert call(max_rank=136) == apr.APR_ERR_INVALID_ARG
    assert call(d_in=20) == apr.APR_ERR_INVALID_ARG
    assert call(kernel=5) == apr.APR_ERR_INVALID_ARG
    assert call(x=None) == apr.APR_ERR_INVALID_ARG
    assert call(ws_bytes=256) == apr.APR_ERR_WORKSPACE
    bad = (apr.Proj * 1)(apr.Proj(0x1000, 0x1000, 60, 0x1000, 0x1000))
    assert call(projs=bad) == apr.APR_ERR_INVALID_ARG
    assert call(T=0) == apr.APR_OK
    assert call(T=-1) == apr.APR_ERR_INVALID_ARG
    assert call(k=9, E=16) == apr.APR_ERR_INVALID_ARG                   # k above the maximum of 8
    assert call(k=3, E=2) == apr.APR_ERR_INVALID_ARG                    # k above E
    assert call(E=1025) == apr.APR_ERR_INVALID_ARG
    assert call(dtype=2) == apr.APR_ERR_INVALID_ARG
    assert call(x=0x1008) == apr.APR_ERR_INVALID_ARG                    # x not 16-byte aligned
    for y, yb in ((0x1004, 0x1000), (0x1000, 0x1002)):                  # y or y_base misaligned
        mis = (apr.Proj * 1)(apr.Proj(y, yb, 64, 0x1000, 0x1000))
        assert call(projs=mis) == apr.APR_ERR_INVALID_ARG
    nul = (apr.Proj * 1)(apr.Proj(0x1000, 0x1000, 64, None, 0x1000))   # no A table
    assert call(projs=nul) == apr.APR_ERR_INVALID_ARG
    assert call(projs=nul, T=0) == apr.APR_OK                          # nothing to do, nothing read
    assert call(ws=None) == apr.APR_ERR_WORKSPACE
    assert call(ws=0x100010) == apr.APR_ERR_WORKSPACE                   # not 256-byte aligned
    for name in ("ranks", "idx", "gate", "seg_off", "perm"):
        assert call(**{name: None}) == apr.APR_ERR_INVALID_ARG, name
    assert "sgmm" in apr.last_error()
    # the tensor-core kernel refuses shapes outside its limits before launching
    assert call(kernel=2, dtype=0) == apr.APR_ERR_UNSUPPORTED
    # so does the dense kernel (fp32, or more than 64 tokens)
    assert call(kernel=3, dtype=0) == apr.APR_ERR_UNSUPPORTED
    assert call(kernel=3, T=65) == apr.APR_ERR_UNSUPPORTED
    # and the bank kernel: fp32, E * R16 > 256, k > 4, k * R16 > 64, rank slot 128, d_in % 64 != 0
    assert call(kernel=4, dtype=0) == apr.APR_ERR_UNSUPPORTED
    assert call(kernel=4, E=17) == apr.APR_ERR_UNSUPPORTED
    assert call(kernel=4, k=5) == apr.APR_ERR_UNSUPPORTED
    assert call(kernel=4, k=3, max_rank=32) == apr.APR_ERR_UNSUPPORTED
    assert call(kernel=4, E=2, max_rank=128) == apr.APR_ERR_UNSUPPORTED
    assert call(kernel=4, d_in=72) == apr.APR_ERR_UNSUPPORTED


def test_merge_and_gemv_host_validation(apr):
    assert apr._merge(0x1000, 0, 8, 16, 0x1000, 0x1000, 2, 0x100000, 1 << 20, None) == apr.APR_ERR_INVALID_ARG
    assert apr._merge(0x1000, 4, 8, 12, 0x1000, 0x1000, 2, 0x100000, 1 << 20, None) == apr.APR_ERR_INVALID_ARG
    assert apr._merge(0x1000, 4, 8, 64, 0x1000, 0x1000, 2, 0x100000, 1 << 20, None) == apr.APR_ERR_UNSUPPORTED
    assert apr._merge(0x1000, 4, 8, 16, 0x1000, 0x1000, 2, None, 1 << 20, None) == apr.APR_ERR_WORKSPACE
    assert apr._gemv(0x1000, 0x1000, 0x1000, 60, 8, None) == apr.APR_ERR_INVALID_ARG
    assert apr._gemv(0x1000, 0x1000, 0x1000, 64, 0, None) == apr.APR_OK
    assert apr._gemv(None, 0x1000, 0x1000, 64, 8, None) == apr.APR_ERR_INVALID_ARG


def test_merge_plan_host_validation(apr):
    """The plan set-up checks its arguments on the host before touching the GPU."""
    assert apr._merge_plan_size(0) == 0
    assert apr._merge_plan_size(224) == 224 * 2 * 128
    one = (apr.MergeProj * 1)(apr.MergeProj(0x1000, 0x2000, 64, 32, 0x3000, 0x4000))
    assert apr._merge_plan_init(one, 0, 0x10000, 1 << 20) == apr.APR_ERR_INVALID_ARG
    assert apr._merge_plan_init(one, 1, None, 1 << 20) == apr.APR_ERR_INVALID_ARG
    assert apr._merge_plan_init(one, 1, 0x10040, 1 << 20) == apr.APR_ERR_INVALID_ARG     # not 128-byte aligned
    assert apr._merge_plan_init(one, 1, 0x10000, 64) == apr.APR_ERR_WORKSPACE
    bad = (apr.MergeProj * 1)(apr.MergeProj(0x1001, 0x2000, 64, 32, 0x3000, 0x4000))
    assert apr._merge_plan_init(bad, 1, 0x10000, 1 << 20) == apr.APR_ERR_INVALID_ARG       # W not 16-byte aligned
    odd = (apr.MergeProj * 1)(apr.MergeProj(0x1000, 0x2000, 60, 32, 0x3000, 0x4000))
    assert apr._merge_plan_init(odd, 1, 0x10000, 1 << 20) == apr.APR_ERR_INVALID_ARG       # d_in % 8 != 0
    # the planned merge refuses what the tensor-core merge cannot do, before launching
    assert apr._merge_planned(0x1000, 0x10000, 1, 8, 32, 0x1000, 0x1000, 3, 0x100000, 1 << 20, None) == \
        apr.APR_ERR_UNSUPPORTED



def test_segment_and_noalloc_host_validation(apr):
    def seg(**kw):
        a = dict(idx=0x1000, T=4, k=2, E=8, seg_off=0x1000, perm=0x1000, ws=0x100000, ws_bytes=1 << 30, stream=None)
        a.update(kw)
        return apr._segment_tokens(*a.values())

    assert seg(k=9, E=16) == apr.APR_ERR_INVALID_ARG
    assert seg(k=3, E=2) == apr.APR_ERR_INVALID_ARG
    assert seg(T=-2) == apr.APR_ERR_INVALID_ARG
    assert seg(seg_off=None) == apr.APR_ERR_INVALID_ARG
    assert seg(idx=None) == apr.APR_ERR_INVALID_ARG
    assert seg(perm=None) == apr.APR_ERR_INVALID_ARG
    assert seg(ws=None) == apr.APR_ERR_WORKSPACE
    assert seg(ws=0x100080) == apr.APR_ERR_WORKSPACE
    assert seg(ws_bytes=64) == apr.APR_ERR_WORKSPACE

    def noalloc(**kw):
        a = dict(h=0x1000, Wr=0x1000, dtype=1, T=4, d=64, E=8, k=2, idx=0x1000, gate=0x1000, stream=None)
        a.update(kw)
        return apr._pregate_route_noalloc(*a.values())

    assert noalloc(E=4, k=5) == apr.APR_ERR_INVALID_ARG
    assert noalloc(d=60) == apr.APR_ERR_INVALID_ARG
    assert noalloc(dtype=3) == apr.APR_ERR_INVALID_ARG
    assert noalloc(Wr=None) == apr.APR_ERR_INVALID_ARG
    assert noalloc(Wr=0x1004) == apr.APR_ERR_INVALID_ARG
    assert noalloc(T=1 << 21) == apr.APR_ERR_UNSUPPORTED          # T*E above the fixed scratch
    assert noalloc(T=0, h=None, Wr=None) == apr.APR_OK


def test_workspace_init_host_validation(apr):
    assert apr._workspace_init(None, 1 << 20, None) == apr.APR_ERR_WORKSPACE
    assert apr._workspace_init(0x100000, 8, None) == apr.APR_ERR_WORKSPACE
    assert apr._workspace_init(0x100040, 1 << 20, None) == apr.APR_ERR_WORKSPACE


def test_binding_rejects_mismatched_tensors(apr):
    """The Python binding checks dtypes, shapes and contiguity before a pointer crosses the ABI
    (a bf16 router weight under an fp32 router input would otherwise be read at twice its size)."""
    import torch
    f32, bf16, i32 = torch.float32, torch.bfloat16, torch.int32
    T, d, E, k = 4, 64, 8, 2
    h = torch.zeros((T, d), dtype=f32)
    idx = torch.zeros((T, k), dtype=i32)
    gate = torch.zeros((T, k), dtype=f32)
    ws = torch.zeros(1 << 20, dtype=torch.uint8)
    with pytest.raises(TypeError, match="Wr has dtype"):
        apr.pregate_route(h, torch.zeros((E, d), dtype=bf16), k, idx, gate, ws)
    with pytest.raises(ValueError, match="columns"):
        apr.pregate_route(h, torch.zeros((E, d + 8), dtype=f32), k, idx, gate, ws)
    with pytest.raises(TypeError, match="idx has dtype"):
        apr.pregate_route_noalloc(h, torch.zeros((E, d), dtype=f32), k, idx.long(), gate)
    with pytest.raises(ValueError, match="gate has shape"):
        apr.pregate_route(h, torch.zeros((E, d), dtype=f32), k, idx, gate[:, :1], ws)
    with pytest.raises(TypeError, match="h has dtype"):
        apr.pregate_route(h.double(), torch.zeros((E, d), dtype=torch.float64), k, idx, gate, ws)
    with pytest.raises(ValueError, match="contiguous"):
        apr.pregate_route(torch.zeros((d, T), dtype=f32).t(), torch.zeros((E, T), dtype=f32), k,
                          idx, gate, ws)
    with pytest.raises(ValueError, match="CUDA tensor"):          # everything right but the device
        apr.pregate_route(h, torch.zeros((E, d), dtype=f32), k, idx, gate, ws)
    with pytest.raises(ValueError, match="seg_off has shape"):
        apr.segment_tokens(idx, E, torch.zeros(E, dtype=i32), torch.zeros(T * k, dtype=i32), ws)
    with pytest.raises(ValueError, match="perm has"):
        apr.segment_tokens(idx, E, torch.zeros(E + 1, dtype=i32), torch.zeros(T * k - 1, dtype=i32), ws)
    # SGMM: projections must match x's dtype and rows
    tabs = torch.zeros(E, dtype=torch.int64)
    with pytest.raises(TypeError, match="y has dtype"):
        apr.make_proj(torch.zeros((T, 16), dtype=f32), torch.zeros((T, 16), dtype=bf16), tabs, tabs)
    with pytest.raises(ValueError, match="B_table has shape"):
        apr.make_proj(torch.zeros((T, 16), dtype=f32), torch.zeros((T, 16), dtype=f32), tabs, tabs[:3])
    yb = torch.zeros((T, 16), dtype=bf16)
    with pytest.raises(ValueError, match="CUDA tensor"):
        apr.make_proj(yb, yb, tabs, tabs)
    p = apr.Proj(0, 0, 16, 0, 0)
    p.meta = (bf16, T, E, torch.device("cpu"))
    x = torch.zeros((T, 64), dtype=f32)
    args = (k, E, torch.zeros(E, dtype=i32), 16, idx, gate, torch.zeros(E + 1, dtype=i32),
            torch.zeros(T * k, dtype=i32), ws)
    with pytest.raises(ValueError, match="does not fit"):
        apr.sgmm_shrink_expand(x, [p], *args)
    with pytest.raises(TypeError, match="not made by make_proj"):
        apr.sgmm_shrink_expand(x, [apr.Proj(0, 0, 16, 0, 0)], *args)
    with pytest.raises(TypeError, match="W has dtype"):
        apr.gemv(torch.zeros((8, 8), dtype=f32), torch.zeros(8, dtype=bf16), torch.zeros(8, dtype=bf16))
    with pytest.raises(ValueError, match="x has shape"):
        apr.gemv(torch.zeros((8, 16), dtype=bf16), torch.zeros(8, dtype=bf16), torch.zeros(8, dtype=bf16))
