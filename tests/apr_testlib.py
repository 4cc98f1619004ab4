"""Helpers shared by the GPU parity tests: run explicit small cases through the
C ABI and compare them with the fp64 oracle."""
from __future__ import annotations

import numpy as np
import torch

from oracle import apr_oracle as O

# Tolerances for floating outputs (per tensor): relative Frobenius error and
# max-abs error relative to the largest reference magnitude.
REL_FRO = 5e-3
MAX_ABS_REL = 1e-2
GATE_ATOL = 1e-6


def close(got, ref, what=""):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    fro = O.rel_frobenius(got, ref)
    scale = float(np.abs(ref).max()) if ref.size else 0.0
    mabs = float(np.abs(got - ref).max()) if ref.size else 0.0
    assert fro <= REL_FRO, f"{what}: relative Frobenius error {fro:.3e} > {REL_FRO}"
    assert mabs <= MAX_ABS_REL * max(scale, 1e-30), f"{what}: max abs error {mabs:.3e} > {MAX_ABS_REL}*{scale:.3e}"
    return fro, mabs


def dev(a, dtype):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to("cuda").to(dtype)


def to_np(t):
    return t.float().cpu().numpy().astype(np.float64)


def run_route(apr, h, Wr, k, dtype):
    T, d = h.shape
    E = Wr.shape[0]
    ws = apr.workspace(max(T, 1), k, E, 8, 8)
    idx = torch.full((T, k), -7, dtype=torch.int32, device="cuda")
    gate = torch.full((T, k), -1.0, dtype=torch.float32, device="cuda")
    apr.pregate_route(dev(h, dtype), dev(Wr, dtype), k, idx, gate, ws)
    apr.stream_status(ws)
    return idx.cpu().numpy(), gate.cpu().numpy().astype(np.float64)


def run_segment(apr, idx_np, E):
    T, k = idx_np.shape
    ws = apr.workspace(max(T, 1), k, E, 8, 8)
    idx = torch.from_numpy(np.ascontiguousarray(idx_np, dtype=np.int32)).cuda()
    seg_off = torch.full((E + 1,), -3, dtype=torch.int32, device="cuda")
    perm = torch.full((max(T * k, 1),), -3, dtype=torch.int32, device="cuda")
    apr.segment_tokens(idx, E, seg_off, perm, ws)
    apr.stream_status(ws)
    return seg_off.cpu().numpy(), perm.cpu().numpy()[: T * k], ws


# Guard bands around every SGMM output and y_base: GUARD elements on each side
# (128 or 256 bytes, so the views keep 16-byte alignment) filled with SENTINEL
# and compared bit for bit after the call: a write outside y, or into y_base
# when the call is out of place, fails the test.
GUARD = 64
SENTINEL = -31.25


def guarded(values, dtype):
    """(buffer, view): ``values`` on the device inside a buffer with sentinel bands."""
    n = values.size
    buf = torch.full((n + 2 * GUARD,), SENTINEL, dtype=dtype, device="cuda")
    view = buf[GUARD:GUARD + n].view(values.shape)
    view.copy_(dev(values, dtype))
    return buf, view


def check_guards(buf, what):
    band = torch.full((GUARD,), SENTINEL, dtype=buf.dtype, device=buf.device)
    assert torch.equal(buf[:GUARD], band) and torch.equal(buf[-GUARD:], band), f"{what}: write outside the tensor"


def run_sgmm(apr, x, As, Bs, idx_np, gate_np, ybases, dtype, kernel=0, in_place=False, ranks=None,
             max_rank=None, return_ws=False):
    """One shared-input group: ``As[p][e]``, ``Bs[p][e]`` numpy; returns list of y (fp64).
    Outputs and y_base sit inside guard bands that are checked after the call; out of place,
    y_base must come back unchanged."""
    T, d_in = x.shape
    k = idx_np.shape[1]
    E = len(As[0])
    if ranks is None:
        ranks = np.array([a.shape[0] for a in As[0]], dtype=np.int32)
    if max_rank is None:
        max_rank = int(max(ranks.max(), 8))
        max_rank = (max_rank + 7) // 8 * 8
    ws = apr.workspace(max(T, 1), k, E, max_rank, d_in)
    idx = torch.from_numpy(np.ascontiguousarray(idx_np, dtype=np.int32)).cuda()
    gate = torch.from_numpy(np.ascontiguousarray(gate_np, dtype=np.float32)).cuda()
    seg_off = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(max(T * k, 1), dtype=torch.int32, device="cuda")
    apr.segment_tokens(idx, E, seg_off, perm, ws)
    xd = dev(x, dtype)
    keep, projs, ys, bands, inputs = [], [], [], [], []
    for p in range(len(As)):
        A = [dev(a, dtype) for a in As[p]]
        B = [dev(b, dtype) for b in Bs[p]]
        At, Bt = apr.ptr_array(A), apr.ptr_array(B)
        ybuf, yb = guarded(np.asarray(ybases[p], dtype=np.float32), dtype)
        bands.append((ybuf, f"y_base {p}"))
        if in_place:
            y = yb
        else:
            inputs.append((ybuf, ybuf.clone(), p))
            ybuf2, y = guarded(np.full(np.shape(ybases[p]), np.nan, np.float32), dtype)
            bands.append((ybuf2, f"y {p}"))
        keep += [A, B, At, Bt, yb]
        projs.append(apr.make_proj(y, yb, At, Bt))
        ys.append(y)
    rk = torch.from_numpy(np.ascontiguousarray(ranks, dtype=np.int32)).cuda()
    apr.sgmm_shrink_expand(xd, projs, k, E, rk, max_rank, idx, gate, seg_off, perm, ws, kernel)
    apr.stream_status(ws)
    for buf, what in bands:
        check_guards(buf, what)
    for buf, before, p in inputs:
        assert torch.equal(buf, before), f"y_base {p} written by an out-of-place call"
    out = [to_np(y) for y in ys]
    if return_ws:
        return out, ws
    return out


def bf16_exact(a):
    """Round fp32 values to bf16 the way the device sees them."""
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16).float().numpy()


def oracle_group(x, As, Bs, idx, gate, ybases):
    return [O.sgmm_shrink_expand(x, As[p], Bs[p], idx, gate, ybases[p]) for p in range(len(As))]
