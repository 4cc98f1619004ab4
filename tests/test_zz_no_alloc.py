"""apr_pregate_route_noalloc: the router entry point for callers that cannot
allocate device memory (no allocator of their own, or no tolerance for the
synchronisation cudaMalloc can cause).  It must give the same routing as
apr_pregate_route, which runs on a caller-provided workspace, on two calls in
a row (the second call sees the scratch the first one left behind), and must
refuse sizes beyond its fixed scratch; on exact router inputs it must also equal
the fp64 oracle.  Kept in a file that pytest collects
last, so a failure here comes after every other test has run.
"""
import numpy as np
import pytest
import torch

from adapter_pregate_router_b200 import workloads as W
from oracle import apr_oracle as O

pytestmark = pytest.mark.gpu

GATE_ATOL = 1e-6


@pytest.fixture(scope="module")
def apr():
    from adapter_pregate_router_b200 import build
    build.build()
    from adapter_pregate_router_b200 import apr as mod
    assert torch.cuda.is_available()
    return mod


def _cases():
    # forced, exact-logit router inputs of two workloads (exact: the oracle decides them too),
    # then free float inputs (fp32 sums: compared with the workspace router only)
    out = []
    for name in ("prefill", "decode"):
        cfg = W.CONFIGS[name]
        h, Wr, _ = W.router_inputs(cfg)
        out.append((h, Wr, cfg.k, torch.bfloat16, True))
    rng = np.random.default_rng(5)
    out.append((rng.normal(size=(700, 512)).astype(np.float32),
                rng.normal(size=(64, 512)).astype(np.float32), 3, torch.float32, False))
    return out


def _route_both(apr, h, Wr, k, dt):
    T, E = h.shape[0], Wr.shape[0]
    hd = torch.from_numpy(h).cuda().to(dt)
    wd = torch.from_numpy(Wr).cuda().to(dt)
    ws = apr.workspace(T, k, E, 8, 8)
    idx_ref = torch.empty((T, k), dtype=torch.int32, device="cuda")
    gate_ref = torch.empty((T, k), dtype=torch.float32, device="cuda")
    apr.pregate_route(hd, wd, k, idx_ref, gate_ref, ws)
    idx = torch.full((T, k), -1, dtype=torch.int32, device="cuda")
    gate = torch.full((T, k), -1.0, dtype=torch.float32, device="cuda")
    apr.pregate_route_noalloc(hd, wd, k, idx, gate)
    apr.stream_status(ws)
    return idx.cpu().numpy(), gate.cpu().numpy(), idx_ref.cpu().numpy(), gate_ref.cpu().numpy()


def test_noalloc_route_matches_workspace_route_on_consecutive_calls(apr):
    cases = _cases()
    # two rounds over different inputs: every call follows another call's scratch
    for _ in range(2):
        for h, Wr, k, dt, exact in cases:
            idx, gate, idx_ref, gate_ref = _route_both(apr, h, Wr, k, dt)
            assert np.array_equal(idx, idx_ref)
            assert np.abs(gate - gate_ref).max() <= GATE_ATOL
            if exact:
                oidx, ogate, _ = O.pregate_route(h, Wr, k)
                assert np.array_equal(idx, oidx)
                assert np.abs(gate - ogate).max() <= GATE_ATOL


def test_noalloc_route_rejects_sizes_beyond_its_scratch(apr):
    T, E, d = 8192, 512, 64          # T * E above the 2,097,088 partial logits the scratch holds
    h = torch.zeros((T, d), dtype=torch.float32, device="cuda")
    Wr = torch.zeros((E, d), dtype=torch.float32, device="cuda")
    idx = torch.empty((T, 2), dtype=torch.int32, device="cuda")
    gate = torch.empty((T, 2), dtype=torch.float32, device="cuda")
    with pytest.raises(apr.AprError) as ei:
        apr.pregate_route_noalloc(h, Wr, 2, idx, gate)
    assert ei.value.status == apr.APR_ERR_UNSUPPORTED
