"""In-place merge and exact unmerge (merge, run, unmerge for the next token) through the C ABI:
the merged weights equal the out-of-place merge bit for bit and the unmerge gives every original
bit back, including elements whose restoration needs an escape and elements left unmerged when
the escape list is full."""
import numpy as np
import pytest
import torch

from apr_testlib import dev, to_np
from oracle import apr_oracle as O

pytestmark = pytest.mark.gpu
BF16 = torch.bfloat16


@pytest.fixture(scope="module")
def apr():
    from adapter_pregate_router_b200 import build
    build.build()
    from adapter_pregate_router_b200 import apr as mod
    assert torch.cuda.is_available()
    return mod


def _weights(rng, shapes, E, r, hard_fraction=0.0):
    """W ~ N(0, 0.02) with a fraction of hard elements (exact zeros and values far below the
    delta, of either sign); adapters ~ N(0, 0.02) (A 0.2 so that the delta is not tiny)."""
    Ws, As, Bs = [], [], []
    for d_out, d_in in shapes:
        w = (0.02 * rng.normal(size=(d_out, d_in))).astype(np.float32)
        if hard_fraction:
            m = rng.random(size=w.shape) < hard_fraction
            w[m] = rng.choice([0.0, 1e-6, -1e-6, 3e-8], size=int(m.sum()))
        Ws.append(w)
        As.append([(0.2 * rng.normal(size=(r, d_in))).astype(np.float32) for _ in range(E)])
        Bs.append([(0.02 * rng.normal(size=(d_out, r))).astype(np.float32) for _ in range(E)])
    return Ws, As, Bs


def _setup(apr, Ws, As, Bs):
    W = [dev(w, BF16) for w in Ws]
    A = [[dev(a, BF16) for a in P] for P in As]
    B = [[dev(b, BF16) for b in P] for P in Bs]
    At = [apr.ptr_array(P) for P in A]
    Bt = [apr.ptr_array(P) for P in B]
    return W, A, B, At, Bt


def _run(apr, Ws, As, Bs, idx1, gate1, capacity, unmerge_gate=None):
    E, r = len(As[0]), As[0][0].shape[0]
    k = len(idx1)
    W, A, B, At, Bt = _setup(apr, Ws, As, Bs)
    W0 = [w.clone() for w in W]
    Wp = [torch.empty_like(w) for w in W]
    R = [apr.merge_residual(w).fill_(99) for w in W]
    ws = apr.workspace(1, k, E, r, 8)
    idx = torch.tensor(idx1, dtype=torch.int32, device="cuda")
    gate = torch.tensor(gate1, dtype=torch.float32, device="cuda")
    n = len(W)
    # out of place (the reference for the merged values)
    tab_out = apr.merge_table([(W[p], Wp[p], At[p], Bt[p]) for p in range(n)])
    apr.merge_adapters(tab_out, n, E, r, idx, gate, k, ws)
    apr.stream_status(ws)
    # in place
    esc = apr.merge_escapes(capacity)
    tab_in = apr.merge_table([(W[p], R[p], At[p], Bt[p]) for p in range(n)])
    merge_err = None
    apr.merge_adapters_inplace(tab_in, n, E, r, idx, gate, k, esc, ws)
    try:
        apr.stream_status(ws)
    except apr.AprError as e:
        merge_err = e.status
    merged = [w.clone() for w in W]
    count = int(esc[:4].view(torch.int32).item())
    ugate = gate if unmerge_gate is None else torch.tensor(unmerge_gate, dtype=torch.float32, device="cuda")
    unmerge_err = None
    apr.unmerge_adapters_inplace(tab_in, n, E, r, idx, ugate, k, esc, ws)
    try:
        apr.stream_status(ws)
    except apr.AprError as e:
        unmerge_err = e.status
    return dict(W0=W0, Wp=Wp, merged=merged, restored=W, count=count, merge_err=merge_err,
                unmerge_err=unmerge_err, keep=(A, B, At, Bt, R, esc))


def _bits(t):
    return t.view(torch.int16)


@pytest.mark.parametrize("shapes,hard", [
    (((264, 136), (128, 4096), (1000, 520)), 0.0),
    (((264, 136), (128, 4096), (1000, 520)), 0.02),
    (((4096, 4096), (11008, 4096)), 0.001),
])
def test_merge_inplace_matches_out_of_place_and_unmerge_is_exact(apr, shapes, hard):
    rng = np.random.default_rng(sum(d for s in shapes for d in s) + int(hard * 1000))
    Ws, As, Bs = _weights(rng, shapes, 8, 16, hard)
    out = _run(apr, Ws, As, Bs, [5, 2], [0.625, 0.375], capacity=1 << 20)
    assert out["merge_err"] is None and out["unmerge_err"] is None
    for p in range(len(shapes)):
        assert torch.equal(_bits(out["merged"][p]), _bits(out["Wp"][p])), f"weight {p}: in place != out of place"
        assert torch.equal(_bits(out["restored"][p]), _bits(out["W0"][p])), f"weight {p}: not restored"
    if hard:
        assert out["count"] > 0, "the hard elements should need escapes"
    # the merged values themselves against the oracle (sampled rows)
    w0 = to_np(out["W0"][0])
    ref = O.merge_adapters(w0, [to_np(dev(a, BF16)) for a in As[0]], [to_np(dev(b, BF16)) for b in Bs[0]],
                           [5, 2], [0.625, 0.375])
    got = to_np(out["merged"][0])
    assert np.abs(got - ref).max() <= 1e-2 * np.abs(ref).max()


def test_escape_overflow_leaves_elements_unmerged_and_stays_exact(apr):
    rng = np.random.default_rng(91)
    Ws, As, Bs = _weights(rng, ((264, 136), (520, 256)), 4, 16, 0.05)
    out = _run(apr, Ws, As, Bs, [1, 3], [0.5, 0.5], capacity=3)
    assert out["merge_err"] == apr.APR_ERR_WORKSPACE
    assert out["count"] > 3
    for p in range(2):
        m, ref, w0 = _bits(out["merged"][p]), _bits(out["Wp"][p]), _bits(out["W0"][p])
        differs = m != ref
        # where the merge is incomplete the element is the original one
        assert torch.equal(m[differs], w0[differs])
        assert torch.equal(_bits(out["restored"][p]), w0), f"weight {p}: not restored"


def test_unmerge_with_another_routing_is_refused(apr):
    rng = np.random.default_rng(92)
    Ws, As, Bs = _weights(rng, ((264, 136),), 4, 16)
    out = _run(apr, Ws, As, Bs, [0, 2], [0.5, 0.5], capacity=1024, unmerge_gate=[0.75, 0.25])
    assert out["merge_err"] is None
    assert out["unmerge_err"] == apr.APR_ERR_INVALID_ARG
    assert torch.equal(_bits(out["restored"][0]), _bits(out["merged"][0])), "a refused unmerge wrote W"


def test_inplace_limits(apr):
    ws = apr.workspace(1, 2, 8, 64, 8)
    tab = torch.zeros(64, dtype=torch.uint8, device="cuda")
    idx = torch.zeros(2, dtype=torch.int32, device="cuda")
    gate = torch.zeros(2, dtype=torch.float32, device="cuda")
    with pytest.raises(apr.AprError) as ei:                   # k * round16(r) > 64
        apr.merge_adapters_inplace(tab, 1, 8, 64, idx, gate, 2, apr.merge_escapes(4), ws)
    assert ei.value.status == apr.APR_ERR_UNSUPPORTED
    with pytest.raises(ValueError):                            # escape buffer below its header
        apr.merge_adapters_inplace(tab, 1, 8, 16, idx, gate, 2, torch.zeros(64, dtype=torch.uint8, device="cuda"), ws)
