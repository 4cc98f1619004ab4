"""One step of the pre-gated mixture-of-LoRA hot path on device buffers.

A ``Step`` holds the device tensors of one named workload (see ``workloads``)
and runs, through the C ABI only:

* ``apr_pregate_route``   once per step (the router of the first adapted layer
  fixes every layer's adapters, AdaFuse summary §2.A);
* ``apr_segment_tokens``  once per step;
* ``apr_sgmm_shrink_expand`` once per (layer, shared-input group);

or, for the batch-1 merge workload, the route, one ``apr_merge_adapters_planned``
over every weight (its TMA plan built once with the weights) and one ``apr_gemv``
per weight (§2.B steps 1-5).

With ``base="fused"`` every (layer, group) call is instead ``apr_linear_lora``:
the base projection ``x W^T`` and the adapters in one contraction, so there is
no y_base.  With ``base="cublas"`` the same base product comes from
``torch.matmul`` (a plain library GEMM into y_base) followed by the SGMM call
adding the adapters in place: the unfused pipeline the fused call replaces.

Tensors are built once from the seeded pools (``workloads.device_tensor``) and
stay resident; ``run()`` enqueues the step on the current stream.
"""
from __future__ import annotations

import numpy as np
import torch

from . import apr
from . import workloads as W


def _dt(cfg):
    return torch.bfloat16 if cfg.dtype == "bf16" else torch.float32


class Step:
    def __init__(self, cfg: W.Config, device="cuda", layers=None, zero_y_base=False,
                 kernel=apr.SGMM_AUTO, out_of_place=True, base=None):
        if base not in (None, "fused", "cublas"):
            raise ValueError(f"base must be None, 'fused' or 'cublas', got {base!r}")
        if base is not None and (cfg.merge or cfg.dtype != "bf16"):
            raise ValueError("a base projection runs on bf16 SGMM workloads only")
        self.cfg = cfg
        self.device = device
        self.kernel = kernel
        self.base = base
        self.layers = list(range(cfg.layers)) if layers is None else list(layers)
        dt = _dt(cfg)
        T, E, k = cfg.T, cfg.E, cfg.k
        self.ranks_np = W.ranks(cfg)
        self.max_rank = int(self.ranks_np.max())
        self.ranks = torch.from_numpy(self.ranks_np).to(device)
        h, Wr, self.forced = W.router_inputs(cfg)
        self.h = torch.from_numpy(h).to(device=device, dtype=dt)
        self.Wr = torch.from_numpy(Wr).to(device=device, dtype=dt)
        self.idx = torch.empty((T, k), dtype=torch.int32, device=device)
        self.gate = torch.empty((T, k), dtype=torch.float32, device=device)
        self.seg_off = torch.empty(E + 1, dtype=torch.int32, device=device)
        self.perm = torch.empty(T * k, dtype=torch.int32, device=device)
        max_d_in = max(g.d_in for g in cfg.groups)
        if base == "fused":
            self.ws = apr.linear_workspace(T, k, E, self.max_rank, max_d_in, max(len(g.d_outs) for g in cfg.groups),
                                           max(sum(g.d_outs) for g in cfg.groups), device=device)
        else:
            self.ws = apr.workspace(T, k, E, self.max_rank, max_d_in, device=device)
        self.keep = []
        if cfg.merge:
            self._build_merge(dt)
        elif base is not None:
            self._build_base(dt)
        else:
            self._build_sgmm(dt, zero_y_base, out_of_place)

    # ------------------------------------------------------------ SGMM workload
    def _build_sgmm(self, dt, zero_y_base, out_of_place):
        cfg, dev = self.cfg, self.device
        T = cfg.T
        self.calls = []          # (x, [Proj...], (l, g))
        self.outputs = {}        # (l, g, p) -> (y, y_base)
        self.adapters = {}       # (l, g, p) -> (A list, B list)
        # Activations live in two flat arenas so that a step's inputs (router
        # hidden, x, y_base) and outputs (y) move host<->device in one copy each.
        n_in = T * cfg.d_router
        n_out = 0
        for _ in self.layers:
            for g in cfg.groups:
                n_in += T * g.d_in + sum(T * d for d in g.d_outs)
                n_out += sum(T * d for d in g.d_outs)
        self.act_in = torch.empty(n_in, dtype=dt, device=dev)
        self.act_out = self.act_in if not out_of_place else torch.empty(n_out, dtype=dt, device=dev)
        pos_in = [0]

        def take_in(shape):
            n = int(np.prod(shape))
            v = self.act_in[pos_in[0]:pos_in[0] + n].view(shape)
            pos_in[0] += n
            return v
        h = take_in(tuple(self.h.shape))
        h.copy_(self.h)
        self.h = h
        pos_out = 0
        self.layer_in = {}       # l -> (start, end) of the layer's inputs (x, y_base) in act_in
        self.layer_out = {}      # l -> (start, end) of the layer's outputs in act_out
        for l in self.layers:
            in0, out0 = pos_in[0], pos_out
            for g in cfg.groups:
                x = take_in((T, g.d_in))
                x.copy_(W.device_tensor(cfg, W.x_key(l, g.name), (T, g.d_in), dev))
                projs = []
                for p, d_out in zip(g.proj_names, g.d_outs):
                    A = [W.device_tensor(cfg, W.a_key(l, g.name, p, e), (int(self.ranks_np[e]), g.d_in), dev)
                         for e in range(cfg.E)]
                    B = [W.device_tensor(cfg, W.b_key(l, g.name, p, e), (d_out, int(self.ranks_np[e])), dev)
                         for e in range(cfg.E)]
                    At, Bt = apr.ptr_array(A, dev), apr.ptr_array(B, dev)
                    yb = take_in((T, d_out))
                    if zero_y_base:
                        yb.zero_()
                    else:
                        yb.copy_(W.device_tensor(cfg, W.ybase_key(l, g.name, p), (T, d_out), dev))
                    if out_of_place:
                        y = self.act_out[pos_out:pos_out + T * d_out].view(T, d_out)
                        pos_out += T * d_out
                    else:
                        y = yb
                    projs.append(apr.make_proj(y, yb, At, Bt))
                    self.outputs[(l, g.name, p)] = (y, yb)
                    self.adapters[(l, g.name, p)] = (A, B)
                    self.keep += [At, Bt]
                self.calls.append((x, projs, (l, g.name)))
            self.layer_in[l] = (in0, pos_in[0])
            self.layer_out[l] = (out0, pos_out) if out_of_place else (in0, pos_in[0])
        W.clear_device_pools()

    # ------------------------------------------------------------ base projection + adapters
    def _build_base(self, dt):
        cfg, dev = self.cfg, self.device
        T = cfg.T
        self.calls = []          # (x, [LinearProj...] or [(W, Proj)...], (l, g))
        self.outputs = {}        # (l, g, p) -> (y, W)
        self.adapters = {}
        n_in = T * cfg.d_router + sum(T * g.d_in for g in cfg.groups) * len(self.layers)
        n_out = sum(T * sum(g.d_outs) for g in cfg.groups) * len(self.layers)
        self.act_in = torch.empty(n_in, dtype=dt, device=dev)
        self.act_out = torch.empty(n_out, dtype=dt, device=dev)
        h = self.act_in[:T * cfg.d_router].view(tuple(self.h.shape))
        h.copy_(self.h)
        self.h = h
        pos_in, pos_out = T * cfg.d_router, 0
        self.layer_in, self.layer_out = {}, {}
        for l in self.layers:
            in0, out0 = pos_in, pos_out
            for g in cfg.groups:
                x = self.act_in[pos_in:pos_in + T * g.d_in].view(T, g.d_in)
                pos_in += T * g.d_in
                x.copy_(W.device_tensor(cfg, W.x_key(l, g.name), (T, g.d_in), dev))
                projs = []
                for p, d_out in zip(g.proj_names, g.d_outs):
                    Wt = W.device_tensor(cfg, W.w_key(l, g.name, p), (d_out, g.d_in), dev)
                    A = [W.device_tensor(cfg, W.a_key(l, g.name, p, e), (int(self.ranks_np[e]), g.d_in), dev)
                         for e in range(cfg.E)]
                    B = [W.device_tensor(cfg, W.b_key(l, g.name, p, e), (d_out, int(self.ranks_np[e])), dev)
                         for e in range(cfg.E)]
                    At, Bt = apr.ptr_array(A, dev), apr.ptr_array(B, dev)
                    y = self.act_out[pos_out:pos_out + T * d_out].view(T, d_out)
                    pos_out += T * d_out
                    if self.base == "fused":
                        projs.append(apr.make_linear_proj(Wt, y, At, Bt))
                    else:
                        projs.append((Wt, apr.make_proj(y, y, At, Bt), y))
                    self.outputs[(l, g.name, p)] = (y, Wt)
                    self.adapters[(l, g.name, p)] = (A, B)
                    self.keep += [At, Bt, Wt]
                self.calls.append((x, projs, (l, g.name)))
            self.layer_in[l] = (in0, pos_in)
            self.layer_out[l] = (out0, pos_out)
        W.clear_device_pools()

    # ------------------------------------------------------------ merge workload
    def _build_merge(self, dt):
        cfg, dev = self.cfg, self.device
        entries = []
        self.weights = {}    # (l, g, p) -> (W, Wp, x, y)
        self.adapters = {}
        # the token's activations: router hidden and every weight's GEMV input in one arena, every
        # GEMV output in another (the weights themselves stay resident from token to token)
        n_in = cfg.d_router + sum(g.d_in * len(g.d_outs) for g in cfg.groups) * len(self.layers)
        n_out = sum(sum(g.d_outs) for g in cfg.groups) * len(self.layers)
        self.act_in = torch.empty(n_in, dtype=dt, device=dev)
        self.act_out = torch.empty(n_out, dtype=dt, device=dev)
        h = self.act_in[:cfg.d_router].view(1, cfg.d_router)
        h.copy_(self.h)
        self.h = h
        pos_in, pos_out = cfg.d_router, 0
        self.layer_in, self.layer_out = {}, {}
        for l in self.layers:
            in0, out0 = pos_in, pos_out
            for g in cfg.groups:
                for p, d_out in zip(g.proj_names, g.d_outs):
                    Wt = W.device_tensor(cfg, W.w_key(l, g.name, p), (d_out, g.d_in), dev)
                    Wp = torch.empty_like(Wt)
                    A = [W.device_tensor(cfg, W.a_key(l, g.name, p, e), (int(self.ranks_np[e]), g.d_in), dev)
                         for e in range(cfg.E)]
                    B = [W.device_tensor(cfg, W.b_key(l, g.name, p, e), (d_out, int(self.ranks_np[e])), dev)
                         for e in range(cfg.E)]
                    At, Bt = apr.ptr_array(A, dev), apr.ptr_array(B, dev)
                    x = self.act_in[pos_in:pos_in + g.d_in]
                    x.copy_(W.device_tensor(cfg, W.xm_key(l, g.name, p), (g.d_in,), dev))
                    pos_in += g.d_in
                    y = self.act_out[pos_out:pos_out + d_out]
                    pos_out += d_out
                    entries.append((Wt, Wp, At, Bt))
                    self.weights[(l, g.name, p)] = (Wt, Wp, x, y)
                    self.adapters[(l, g.name, p)] = (A, B)
                    self.keep += [At, Bt]
            self.layer_in[l] = (in0, pos_in)
            self.layer_out[l] = (out0, pos_out)
        self.merge_tab = apr.merge_table(entries, dev)
        self.nmerge = len(entries)
        # TMA descriptors of the weights: built once, reused by every token's merge
        self.merge_plan = apr.merge_plan(entries, dev) if cfg.k * ((self.max_rank + 15) // 16 * 16) <= 64 else None
        W.clear_device_pools()

    # ------------------------------------------------------------ running
    def route(self, stream=None):
        cfg = self.cfg
        apr.pregate_route(self.h, self.Wr, cfg.k, self.idx, self.gate, self.ws, stream)
        apr.segment_tokens(self.idx, cfg.E, self.seg_off, self.perm, self.ws, stream)

    def merge_all(self, stream=None):
        """Merge workload: one launch merging the token's adapters into every weight."""
        cfg = self.cfg
        if self.merge_plan is not None:
            apr.merge_adapters_planned(self.merge_tab, self.merge_plan, self.nmerge, cfg.E, self.max_rank,
                                       self.idx, self.gate, cfg.k, self.ws, stream)
        else:
            apr.merge_adapters(self.merge_tab, self.nmerge, cfg.E, self.max_rank, self.idx, self.gate,
                               cfg.k, self.ws, stream)

    def run_layer(self, l, stream=None):
        """The calls of one layer: its SGMM calls, or (merge workload) its GEMVs on the merged
        weights, which ``merge_all`` must have written first."""
        cfg = self.cfg
        if cfg.merge:
            for (ll, _, _), (Wt, Wp, x, y) in self.weights.items():
                if ll == l:
                    apr.gemv(Wp, x, y, stream)
            return
        for x, projs, (ll, _) in self.calls:
            if ll != l:
                continue
            if self.base == "fused":
                apr.linear_lora(x, projs, cfg.k, cfg.E, self.ranks, self.max_rank, self.idx, self.gate,
                                self.seg_off, self.perm, self.ws, stream)
            elif self.base == "cublas":
                for Wt, _, y in projs:
                    torch.matmul(x, Wt.t(), out=y)
                apr.sgmm_shrink_expand(x, [pj for _, pj, _ in projs], cfg.k, cfg.E, self.ranks, self.max_rank,
                                       self.idx, self.gate, self.seg_off, self.perm, self.ws, self.kernel, stream)
            else:
                apr.sgmm_shrink_expand(x, projs, cfg.k, cfg.E, self.ranks, self.max_rank, self.idx,
                                       self.gate, self.seg_off, self.perm, self.ws, self.kernel, stream)

    def layers_only(self, stream=None):
        if self.cfg.merge:
            self.merge_all(stream)
        for l in self.layers:
            self.run_layer(l, stream)

    def run(self, stream=None):
        self.route(stream)
        self.layers_only(stream)

    def launches_per_step(self) -> int:
        before = apr.kernel_launches()
        s = torch.cuda.Stream()
        with torch.cuda.stream(s):
            self.run()
        s.synchronize()
        return apr.kernel_launches() - before

    # ------------------------------------------------------------ bytes moved
    def algorithmic_bytes(self, idx_np=None) -> int:
        """Bytes the step must move at least once (inputs read once, outputs written once)."""
        if idx_np is None:
            idx_np = self.idx.cpu().numpy()
        return algorithmic_bytes(self.cfg, self.layers, self.ranks_np, idx_np, base=self.base is not None)

    def flops(self) -> float:
        """Multiply-adds x 2 of the layer calls: the base products (when the step has them) and
        the adapters (shrink and expand of every token's k adapters)."""
        cfg, T = self.cfg, self.cfg.T
        r_mean = float(np.mean([self.ranks_np[e] for e in range(cfg.E)]))
        f = 0.0
        for _ in self.layers:
            for g in cfg.groups:
                for d_out in g.d_outs:
                    if self.base is not None:
                        f += 2.0 * T * g.d_in * d_out
                    f += 2.0 * T * cfg.k * r_mean * (g.d_in + d_out)
        return f


def algorithmic_bytes(cfg: W.Config, layers, ranks_np, idx_np, base=False) -> int:
    """Bytes a step must move at least once: the router's h and Wr; per shared-input group its x
    once; per projection the A and B of every adapter some token selected, and y_base read plus y
    written (SGMM), or W read and y written (base projection and adapters in one pass); or, for
    the merge, W read, W' written, the selected adapters and the GEMV's W', x and y."""
    el = 2 if cfg.dtype == "bf16" else 4
    T = cfg.T
    touched = np.unique(np.asarray(idx_np).reshape(-1))
    b = T * cfg.d_router * el + cfg.E * cfg.d_router * el                 # router h, Wr
    for _ in layers:
        for g in cfg.groups:
            if cfg.merge:
                for d_out in g.d_outs:
                    b += 2 * d_out * g.d_in * el                              # W read, W' written
                    b += sum(int(ranks_np[e]) * (g.d_in + d_out) * el for e in touched)
                    b += d_out * g.d_in * el + g.d_in * el + d_out * el       # GEMV
                continue
            b += T * g.d_in * el                                               # x once per group
            for d_out in g.d_outs:
                b += sum(int(ranks_np[e]) * (g.d_in + d_out) * el for e in touched)
                if base:
                    b += d_out * g.d_in * el + T * d_out * el                  # W read, y written
                else:
                    b += 2 * T * d_out * el                                    # y_base read, y written
    return b
