"""Plain fp64 CPU reference for the token-level pre-gated mixture-of-LoRA path.

TEST INFRASTRUCTURE.  Only the tests, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may import this module.  It shares no code with
the CUDA library and imports nothing from it; both sides take their inputs
from ``adapter_pregate_router_b200.workloads``.

What it computes follows the AdaFuse summary ("AdaFuse: Accelerating Dynamic
Adapter Inference via Token-Level Pre-Gating and Fused Kernel Optimization",
gist.science, Resumen técnico):

* §2.A, token-level pre-gating: one light router at the first adapted layer
  decides, once per token, which adapters every later layer of that token uses.
* §2.B, decoding process steps 1-2: the token goes through the router once and
  the top-K experts are selected.
* §2.B, SGMM (Segmented Gather Matrix Multiplication): one batched product over
  the tokens gathered per adapter applies the selected low-rank adapters.
* §2.B, steps 3-5: the selected adapters are merged into the backbone, the
  base model runs, and the adapters are unmerged for the next token.

Where the summary is silent this module takes the plainest reading:

* the router is a linear map without bias or temperature: ``L = h Wr^T``;
* top-k takes the k largest logits, ties going to the lower adapter index;
* gates are the softmax over the k selected logits (they sum to one);
* every layer and projection reuses the same adapters and gates;
* a LoRA adapter e of a projection is ``A_e`` [r_e, d_in] and ``B_e``
  [d_out, r_e]; its delta on a token row x is ``B_e (A_e x)`` with scale 1;
* token order inside an adapter's segment is ascending (t, then slot j);
* the merged weight is written out of place, so unmerging is leaving W as is.

Every function evaluates in float64 from the exact input values.  The
pinning tests compare these functions with closed forms, brute force and
hand-checked integer examples.  Parity against a printed result of the pages
is unpinned: the pages print no worked example and no intermediate value.
"""
from __future__ import annotations

import numpy as np

F64 = np.float64


def router_logits(h, Wr):
    """Router logits ``L[t, e] = sum_i h[t, i] * Wr[e, i]`` (§2.A, one router pass per token)."""
    h = np.asarray(h, dtype=F64)
    Wr = np.asarray(Wr, dtype=F64)
    return h @ Wr.T


def select_topk(L, k):
    """Indices of the k largest logits per token, ties to the lower index (§2.B step 2).

    A full sort of every row by the key (-L[t, e], e); the first k entries.
    """
    L = np.asarray(L, dtype=F64)
    T, E = L.shape
    if not 1 <= k <= E:
        raise ValueError("need 1 <= k <= E")
    adapter = np.broadcast_to(np.arange(E), (T, E))
    order = np.lexsort((adapter, -L), axis=-1)      # primary: -L, secondary: e
    return order[:, :k].astype(np.int32)


def gates(L, idx):
    """Softmax over the selected logits of each token: the k gates sum to one."""
    L = np.asarray(L, dtype=F64)
    sel = np.take_along_axis(L, np.asarray(idx, dtype=np.int64), axis=1)
    m = sel.max(axis=1, keepdims=True)
    w = np.exp(sel - m)
    return w / w.sum(axis=1, keepdims=True)


def pregate_route(h, Wr, k):
    """Token-level pre-gate: (idx [T, k] int32, gate [T, k] fp64, logits [T, E])."""
    L = router_logits(h, Wr)
    idx = select_topk(L, k)
    return idx, gates(L, idx), L


def segment_tokens(idx, E):
    """Group the (token, slot) pairs by adapter: (seg_off [E+1], perm [T*k]).

    Pair ``q = t*k + j`` belongs to adapter ``idx[t, j]``.  ``seg_off`` is the
    exclusive prefix sum of the per-adapter pair counts; ``perm`` lists the
    pairs of adapter 0, then adapter 1, ..., each segment in ascending q
    (the gather order of §2.B's segmented product).
    """
    flat = np.asarray(idx, dtype=np.int64).reshape(-1)
    if flat.size and (flat.min() < 0 or flat.max() >= E):
        raise ValueError("adapter index out of range")
    counts = np.bincount(flat, minlength=E)
    seg_off = np.zeros(E + 1, dtype=np.int64)
    seg_off[1:] = np.cumsum(counts)
    perm = np.argsort(flat, kind="stable")
    return seg_off.astype(np.int32), perm.astype(np.int32)


def lora_delta(x_row, A_e, B_e):
    """One adapter's low-rank delta on one token row: ``B_e (A_e x)``."""
    return np.asarray(B_e, dtype=F64) @ (np.asarray(A_e, dtype=F64) @ np.asarray(x_row, dtype=F64))


def sgmm_shrink_expand(x, A, B, idx, gate, y_base):
    """Per-token mixture-of-LoRA output for one projection (§2.B, SGMM).

    ``y[t] = y_base[t] + sum_j gate[t, j] * B_e (A_e x[t])`` with ``e = idx[t, j]``.
    ``A`` and ``B`` are sequences indexed by adapter.
    """
    x = np.asarray(x, dtype=F64)
    y = np.array(y_base, dtype=F64, copy=True)
    T, k = np.asarray(idx).shape
    for t in range(T):
        for j in range(k):
            e = int(idx[t, j])
            y[t] += float(gate[t, j]) * lora_delta(x[t], A[e], B[e])
    return y


def linear_lora(x, W, A, B, idx, gate):
    """Base projection with the selected adapters fused into it (§2.B: the experts are fused
    into the backbone in a single pass): ``y[t] = W x[t] + sum_j gate[t, j] * B_e (A_e x[t])``.
    W is [d_out, d_in]."""
    x = np.asarray(x, dtype=F64)
    base = x @ np.asarray(W, dtype=F64).T
    return sgmm_shrink_expand(x, A, B, idx, gate, base)


def merge_adapters(W, A, B, idx1, gate1):
    """Merged weight for one token (§2.B step 3): ``W' = W + sum_j g_j B_{e_j} A_{e_j}``."""
    Wp = np.array(W, dtype=F64, copy=True)
    for j in range(len(idx1)):
        e = int(idx1[j])
        Wp += float(gate1[j]) * (np.asarray(B[e], dtype=F64) @ np.asarray(A[e], dtype=F64))
    return Wp


def gemv(W, x):
    """Base inference on the merged weight (§2.B step 4): ``y = W x``."""
    return np.asarray(W, dtype=F64) @ np.asarray(x, dtype=F64)


def rel_frobenius(got, ref):
    got = np.asarray(got, dtype=F64)
    ref = np.asarray(ref, dtype=F64)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(got - ref) / (den if den > 0 else 1.0))
