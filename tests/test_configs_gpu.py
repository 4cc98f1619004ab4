"""GPU parity on the five named workloads at their full sizes, through the same
step the benchmark times (``pipeline.Step``).

Routing and segments are compared in full, bit for bit.  Projection outputs
are compared in full for the small workloads and on a seeded sample of tokens
(every layer, every projection, every output column) for the large ones; the
oracle computes the sampled tokens one by one.
"""
import gc

import numpy as np
import pytest
import torch

from oracle import apr_oracle as O
from adapter_pregate_router_b200 import workloads as W
from tests.apr_testlib import GATE_ATOL, close, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mods():
    from adapter_pregate_router_b200 import build
    build.build()
    from adapter_pregate_router_b200 import apr, pipeline
    return apr, pipeline


def _sample_rows(T, n, seed):
    if T <= n:
        return np.arange(T)
    rng = np.random.default_rng(seed)
    rows = set(rng.choice(T, size=n - 2, replace=False).tolist()) | {0, T - 1}
    return np.array(sorted(rows))


def _check_routing(step, cfg):
    h, Wr, forced = W.router_inputs(cfg)
    ridx, rgate, _ = O.pregate_route(h, Wr, cfg.k)
    idx = step.idx.cpu().numpy()
    assert np.array_equal(idx, ridx)
    assert np.abs(step.gate.cpu().numpy() - rgate).max() <= GATE_ATOL
    rs, rp = O.segment_tokens(ridx, cfg.E)
    assert np.array_equal(step.seg_off.cpu().numpy(), rs)
    assert np.array_equal(step.perm.cpu().numpy(), rp)
    return ridx, rgate


def _check_sgmm_outputs(step, cfg, ridx, rgate, rows, zero_y_base):
    ranks = W.ranks(cfg)
    worst = 0.0
    for l in step.layers:
        for g in cfg.groups:
            xr = W.host_rows(cfg, W.x_key(l, g.name), (cfg.T, g.d_in), rows)
            for p, d_out in zip(g.proj_names, g.d_outs):
                used = sorted(set(ridx[rows].reshape(-1).tolist()))
                A = [None] * cfg.E
                B = [None] * cfg.E
                for e in used:
                    A[e] = W.host_tensor(cfg, W.a_key(l, g.name, p, e), (int(ranks[e]), g.d_in))
                    B[e] = W.host_tensor(cfg, W.b_key(l, g.name, p, e), (d_out, int(ranks[e])))
                if zero_y_base:
                    ybr = np.zeros((len(rows), d_out))
                else:
                    ybr = W.host_rows(cfg, W.ybase_key(l, g.name, p), (cfg.T, d_out), rows)
                ref = O.sgmm_shrink_expand(xr, A, B, ridx[rows], rgate[rows], ybr)
                y, _ = step.outputs[(l, g.name, p)]
                got = to_np(y[torch.from_numpy(rows).to(y.device)])
                fro, _ = close(got, ref, f"{cfg.name} layer {l} {p} zero_ybase={zero_y_base}")
                worst = max(worst, fro)
    return worst


@pytest.mark.parametrize("name,nrows", [("tiny", 64), ("decode", 32), ("multitenant", 24), ("prefill", 24)])
def test_config_parity(mods, name, nrows):
    apr, pipeline = mods
    cfg = W.CONFIGS[name]
    rows = _sample_rows(cfg.T, nrows, 17)
    for zero in (False, True):
        layers = None if (not zero or cfg.T <= 64) else [0, cfg.layers - 1]
        step = pipeline.Step(cfg, layers=layers, zero_y_base=zero)
        step.run()
        apr.stream_status(step.ws)
        ridx, rgate = _check_routing(step, cfg)
        _check_sgmm_outputs(step, cfg, ridx, rgate, rows, zero)
        del step
        gc.collect()
        torch.cuda.empty_cache()


def test_config_parity_merge(mods):
    """Every one of the 224 weights: the merged weight on 64 sampled rows (all rows for two
    layers) and the whole GEMV output, against the oracle's fp64 W' = W + sum g B A and its
    product with x.  The device GEMV reads W' after its one rounding to bf16; that rounding
    moves each output by about 2^-9 / sqrt(3) of its magnitude in relative Frobenius norm,
    inside the 5e-3 bound."""
    apr, pipeline = mods
    cfg = W.CONFIGS["merge"]
    step = pipeline.Step(cfg)
    step.run()
    apr.stream_status(step.ws)
    ridx, rgate = _check_routing(step, cfg)
    ranks = W.ranks(cfg)
    e_sel = ridx[0]
    rng = np.random.default_rng(3)
    full_layers = {0, 25}
    checked = 0
    for (l, g, p), (Wt, Wp, x, y) in step.weights.items():
        d_out, d_in = Wt.shape
        Wfull = W.host_tensor(cfg, W.w_key(l, g, p), (d_out, d_in))
        A = [W.host_tensor(cfg, W.a_key(l, g, p, e), (int(ranks[e]), d_in)) if e in e_sel else None
             for e in range(cfg.E)]
        B = [W.host_tensor(cfg, W.b_key(l, g, p, e), (d_out, int(ranks[e]))) if e in e_sel else None
             for e in range(cfg.E)]
        ref_W = O.merge_adapters(Wfull, A, B, e_sel, rgate[0])
        rows = np.arange(d_out) if l in full_layers else np.sort(rng.choice(d_out, size=64, replace=False))
        got = to_np(Wp[torch.from_numpy(rows).to(Wp.device)])
        close(got, ref_W[rows], f"merged {l}/{p}")
        xv = W.host_tensor(cfg, W.xm_key(l, g, p), (d_in,))
        close(to_np(y), O.gemv(ref_W, xv), f"gemv {l}/{p}")
        checked += 1
    assert checked == 224


def test_graph_replay_matches_eager(mods):
    apr, pipeline = mods
    cfg = W.CONFIGS["decode"]
    step = pipeline.Step(cfg, layers=[0, 1])
    step.run()
    torch.cuda.synchronize()
    eager = {k: v[0].clone() for k, v in step.outputs.items()}
    for v in step.outputs.values():
        v[0].fill_(0)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        step.run()                      # warm-up on the capture stream
        s.synchronize()
        with torch.cuda.graph(g, stream=s):
            step.run()
    for v in step.outputs.values():
        v[0].fill_(0)
    g.replay()
    torch.cuda.synchronize()
    apr.stream_status(step.ws)
    for key, ref in eager.items():
        assert torch.equal(step.outputs[key][0], ref), key


@pytest.mark.parametrize("name", ["decode", "prefill", "multitenant"])
def test_step_reruns_agree_bit_for_bit(mods, name):
    """Two layers of the workload run four times: every output bit is the same each time (the
    kernels have one writer per element and a fixed summation order, so a difference means a
    race, e.g. a staged operand read before its copy landed)."""
    apr, pipeline = mods
    step = pipeline.Step(W.CONFIGS[name], layers=[0, 1])
    ref = None
    for _ in range(4):
        step.act_out.fill_(float("nan"))
        step.run()
        apr.stream_status(step.ws)
        if ref is None:
            ref = step.act_out.clone()
        assert torch.equal(step.act_out.view(torch.int16), ref.view(torch.int16))
    del step
    gc.collect()
    torch.cuda.empty_cache()
