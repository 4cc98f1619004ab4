"""Adapter paging (adapters in pinned host memory, a few device slots, paged in on the device
between the router and the SGMM calls): outputs against the fp64 oracle over a sequence of
steps whose adapter sets change, the number of adapters copied against a model of the slot
policy (empty slots, then least recently used), and the capacity error."""
import numpy as np
import pytest
import torch

from apr_testlib import bf16_exact, close, dev, to_np
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


def _policy(steps, n_slots):
    """Adapters copied per step under the documented policy: the missing adapters in ascending
    id take, in order, the slots this step does not need, emptiest / least recently used first
    (ties by slot index)."""
    id_of = [-1] * n_slots
    last = [0] * n_slots
    copies = []
    for s, need in enumerate(steps, start=1):
        need = sorted(set(need))
        resident = {i: sl for sl, i in enumerate(id_of) if i >= 0}
        missing = [i for i in need if i not in resident]
        cand = sorted((last[sl], sl) for sl in range(n_slots) if id_of[sl] < 0 or id_of[sl] not in need)
        for i, (_, sl) in zip(missing, cand):
            id_of[sl] = i
        for sl in range(n_slots):
            if id_of[sl] in need:
                last[sl] = s
        copies.append(len(missing))
    return copies


def test_paging_over_steps_matches_oracle_and_policy(apr):
    rng = np.random.default_rng(101)
    N, S, T, k, d_in, d_outs, r_max = 10, 4, 48, 2, 256, (264, 128), 16
    ranks = rng.choice([8, 16], size=N).astype(np.int32)
    A = [[bf16_exact(0.05 * rng.normal(size=(int(ranks[e]), d_in))) for e in range(N)] for _ in d_outs]
    B = [[bf16_exact(0.05 * rng.normal(size=(d, int(ranks[e])))) for e in range(N)] for d in d_outs]
    # one pinned host buffer per adapter: [A_0 | B_0 | A_1 | B_1], each region sized for r_max
    offs, off = [], 0
    for d in d_outs:
        offs += [off, off + r_max * d_in * 2]
        off += r_max * d_in * 2 + d * r_max * 2
    adapter_bytes = off
    bufs = []
    for e in range(N):
        b = torch.zeros(adapter_bytes, dtype=torch.uint8).pin_memory()
        for p, d in enumerate(d_outs):
            a_bytes = torch.from_numpy(A[p][e]).to(BF16).view(torch.uint8).reshape(-1)
            b_bytes = torch.from_numpy(B[p][e]).to(BF16).view(torch.uint8).reshape(-1)
            b[offs[2 * p]:offs[2 * p] + a_bytes.numel()] = a_bytes
            b[offs[2 * p + 1]:offs[2 * p + 1] + b_bytes.numel()] = b_bytes
        bufs.append(b)
    tables = [torch.zeros(N, dtype=torch.int64, device="cuda") for _ in range(2 * len(d_outs))]
    pool = apr.AdapterPool(bufs, S, tables, offs)
    ws = apr.workspace(T, k, N, r_max, d_in)
    rk = torch.from_numpy(ranks).cuda()
    sets = [[0, 1, 2], [1, 2, 3, 4], [5, 6], [1, 5, 7, 8], [9, 0], [9, 0, 6, 2], [3, 4, 5, 6]]
    for step, chosen in enumerate(sets):
        idx_np = np.stack([rng.choice(chosen, size=k, replace=False) for _ in range(T)]).astype(np.int32)
        gate_np = rng.dirichlet(np.ones(k), size=T).astype(np.float32)
        idx = torch.from_numpy(idx_np).cuda()
        gate = torch.from_numpy(gate_np).cuda()
        pool.page_in(idx, ws)
        seg_off = torch.empty(N + 1, dtype=torch.int32, device="cuda")
        perm = torch.empty(T * k, dtype=torch.int32, device="cuda")
        apr.segment_tokens(idx, N, seg_off, perm, ws)
        x_np = bf16_exact(rng.normal(size=(T, d_in)))
        x = dev(x_np, BF16)
        ys, projs = [], []
        for p, d in enumerate(d_outs):
            y = torch.zeros(T, d, dtype=BF16, device="cuda")
            projs.append(apr.make_proj(y, y, tables[2 * p], tables[2 * p + 1]))
            ys.append(y)
        apr.sgmm_shrink_expand(x, projs, k, N, rk, r_max, idx, gate, seg_off, perm, ws)
        apr.stream_status(ws)
        for p, d in enumerate(d_outs):
            ref = O.sgmm_shrink_expand(x_np, A[p], B[p], idx_np, gate_np.astype(np.float64), np.zeros((T, d)))
            close(to_np(ys[p]), ref, f"step {step} proj {p}")
    steps, copies = pool.stats()
    assert steps == len(sets)
    assert copies == sum(_policy(sets, S)), (copies, _policy(sets, S))


def test_paging_capacity_error_changes_nothing(apr):
    N, S = 6, 2
    bufs = [torch.full((64,), e, dtype=torch.uint8).pin_memory() for e in range(N)]
    tab = torch.zeros(N, dtype=torch.int64, device="cuda")
    pool = apr.AdapterPool(bufs, S, [tab], [0])
    ws = apr.workspace(4, 1, N, 8, 8)
    pool.page_in(torch.tensor([[0], [1]], dtype=torch.int32, device="cuda"), ws)
    apr.stream_status(ws)
    before = (pool.stats(), tab.clone(), pool.pool.clone())
    with pytest.raises(apr.AprError) as ei:                    # three distinct adapters, two slots
        pool.page_in(torch.tensor([[2], [3], [4]], dtype=torch.int32, device="cuda"), ws)
        apr.stream_status(ws)
    assert ei.value.status == apr.APR_ERR_WORKSPACE
    assert pool.stats() == before[0]
    assert torch.equal(tab, before[1]) and torch.equal(pool.pool, before[2])
    # the slots hold adapters 0 and 1 byte for byte, and the table points at them
    for e in (0, 1):
        ptr = int(tab[e].item())
        slot = (ptr - pool.pool.data_ptr()) // pool.adapter_bytes
        assert torch.equal(pool.pool[slot * 64:(slot + 1) * 64].cpu(), bufs[e])


def test_paging_rejects_pageable_sources(apr):
    bufs = [torch.zeros(64, dtype=torch.uint8) for _ in range(3)]
    with pytest.raises(ValueError):
        apr.AdapterPool(bufs, 2, [torch.zeros(3, dtype=torch.int64, device="cuda")], [0])
