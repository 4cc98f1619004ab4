"""Pins for the fp64 oracle, independent of the oracle itself (CPU only).

Each check uses something other than the oracle's own formula: hand-computed
integer examples, brute force, exact integer arithmetic, closed forms and
invariants.  They are chosen so that a dropped term, a wrong index, a
transposed operand or a broken tie rule in the oracle fails at least one.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest

from oracle import apr_oracle as O
from adapter_pregate_router_b200 import workloads as W


def _load(golden_dir, name):
    with open(os.path.join(golden_dir, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------- router / top-k


def test_route_golden(golden_dir):
    g = _load(golden_dir, "route_example.json")
    idx, gate, L = O.pregate_route(np.array(g["h"]), np.array(g["Wr"]), g["k"])
    assert np.array_equal(L, np.array(g["logits"], dtype=float))
    assert np.array_equal(idx, np.array(g["idx"]))
    assert np.allclose(gate, np.array(g["gate"]), rtol=0, atol=1e-15)
    seg_off, perm = O.segment_tokens(idx, len(g["Wr"]))
    assert seg_off.tolist() == g["seg_off"]
    assert perm.tolist() == g["perm"]


def _bruteforce_topk(row, k):
    """k passes of a linear scan: largest value, first (lowest) index on ties."""
    chosen = []
    for _ in range(k):
        best = None
        for e, v in enumerate(row):
            if e in chosen:
                continue
            if best is None or v > row[best]:
                best = e
        chosen.append(best)
    return chosen


@pytest.mark.parametrize("E,k,vals", [(8, 2, 3), (16, 3, 2), (5, 5, 2), (33, 1, 4), (256, 2, 7)])
def test_topk_matches_bruteforce_with_ties(E, k, vals):
    rng = np.random.default_rng(E * 100 + k)
    L = rng.integers(0, vals, size=(200, E)).astype(float)   # few distinct values: many ties
    idx = O.select_topk(L, k)
    for t in range(L.shape[0]):
        assert idx[t].tolist() == _bruteforce_topk(L[t].tolist(), k)


def test_topk_all_equal_logits_picks_lowest_indices():
    idx = O.select_topk(np.zeros((3, 6)), 4)
    assert idx.tolist() == [[0, 1, 2, 3]] * 3


def test_gates_closed_forms():
    rng = np.random.default_rng(1)
    L = rng.normal(size=(64, 10)) * 3
    idx = O.select_topk(L, 2)
    g = O.gates(L, idx)
    l0 = L[np.arange(64), idx[:, 0]]
    l1 = L[np.arange(64), idx[:, 1]]
    # k = 2: the first gate is the logistic function of the logit gap
    assert np.allclose(g[:, 0], 1.0 / (1.0 + np.exp(l1 - l0)), rtol=0, atol=1e-15)
    assert np.allclose(g.sum(axis=1), 1.0, rtol=0, atol=1e-15)
    assert np.all(g[:, 0] >= g[:, 1])
    # k = 1: the gate is exactly one
    i1 = O.select_topk(L, 1)
    assert np.all(O.gates(L, i1) == 1.0)
    # equal selected logits: exactly 1/k
    Z = np.zeros((2, 4))
    Z[:, :3] = 5.0
    assert np.all(O.gates(Z, O.select_topk(Z, 2)) == 0.5)
    assert np.all(O.gates(Z, O.select_topk(Z, 3)) == 1.0 / 3.0) or np.allclose(
        O.gates(Z, O.select_topk(Z, 3)), 1.0 / 3.0, rtol=0, atol=1e-16)


def test_gates_three_way_closed_form():
    L = np.array([[2.0, 0.0, 1.0, -7.0]])
    idx = O.select_topk(L, 3)
    assert idx.tolist() == [[0, 2, 1]]
    z = 1 + math.exp(-1) + math.exp(-2)
    assert np.allclose(O.gates(L, idx), [[1 / z, math.exp(-1) / z, math.exp(-2) / z]], rtol=0, atol=1e-15)


def test_logits_exact_against_integer_arithmetic():
    cfg = W.scaled(W.CONFIGS["decode"], T=6)
    h, Wr, _ = W.router_inputs(cfg)
    L = O.router_logits(h, Wr)
    sh, sw = 2 ** W.H_SHIFT, 2 ** W.W_SHIFT
    for t in range(cfg.T):
        for e in range(cfg.E):
            exact = sum(int(a * sh) * int(b * sw) for a, b in zip(h[t], Wr[e]))
            assert L[t, e] * sh * sw == exact


@pytest.mark.parametrize("name", ["decode", "prefill", "multitenant", "merge"])
def test_forced_router_inputs_give_the_drawn_tuples(name):
    cfg = W.CONFIGS[name]
    T = min(cfg.T, 512)
    h, Wr, tuples = W.router_inputs(cfg, T=T)
    idx, gate, L = O.pregate_route(h, Wr, cfg.k)
    assert np.array_equal(idx, tuples)
    # strict margin: no tie touches the selected set
    s = np.sort(L, axis=1)[:, ::-1]
    assert np.all(s[:, : cfg.k] > s[:, 1: cfg.k + 1])
    # logits are integers times 2^-(H+W): exact in fp32
    assert np.array_equal(L.astype(np.float32).astype(np.float64), L)


# ---------------------------------------------------------------- segments


@pytest.mark.parametrize("T,k,E", [(1, 1, 1), (7, 2, 3), (64, 2, 8), (100, 3, 40), (50, 1, 256)])
def test_segments_bruteforce_and_invariants(T, k, E):
    rng = np.random.default_rng(T + k + E)
    idx = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    seg_off, perm = O.segment_tokens(idx, E)
    flat = idx.reshape(-1)
    expect = [q for e in range(E) for q in range(T * k) if flat[q] == e]
    assert perm.tolist() == expect
    assert seg_off[0] == 0 and seg_off[-1] == T * k
    for e in range(E):
        assert seg_off[e + 1] - seg_off[e] == sum(1 for q in range(T * k) if flat[q] == e)
    assert sorted(perm.tolist()) == list(range(T * k))
    assert np.all(np.diff(flat[perm]) >= 0)


def test_segments_empty_adapters_and_bad_index():
    idx = np.array([[3, 3], [3, 0]], dtype=np.int32)
    seg_off, perm = O.segment_tokens(idx, 6)
    assert seg_off.tolist() == [0, 1, 1, 1, 4, 4, 4]
    assert perm.tolist() == [3, 0, 1, 2]
    with pytest.raises(ValueError):
        O.segment_tokens(np.array([[6]]), 6)


# ---------------------------------------------------------------- SGMM


def test_sgmm_golden(golden_dir):
    g = _load(golden_dir, "sgmm_merge_example.json")
    A = [np.array(a, dtype=float) for a in g["A"]]
    B = [np.array(b, dtype=float) for b in g["B"]]
    y = O.sgmm_shrink_expand(np.array(g["x"]), A, B, np.array(g["idx"]), np.array(g["gate"]),
                             np.array(g["y_base"], dtype=float))
    assert np.array_equal(y, np.array(g["y"], dtype=float))


def _random_case(rng, T=24, d_in=40, d_out=28, E=5, k=2, ranks=(4, 8, 4, 12, 8)):
    A = [rng.normal(size=(r, d_in)) for r in ranks[:E]]
    B = [rng.normal(size=(d_out, r)) for r in ranks[:E]]
    x = rng.normal(size=(T, d_in))
    idx = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    gate = rng.dirichlet(np.ones(k), size=T)
    yb = rng.normal(size=(T, d_out))
    return x, A, B, idx, gate, yb


def test_sgmm_equals_dense_low_rank_product():
    rng = np.random.default_rng(7)
    x, A, B, idx, gate, yb = _random_case(rng)
    y = O.sgmm_shrink_expand(x, A, B, idx, gate, yb)
    dense = [B[e] @ A[e] for e in range(len(A))]           # d_out x d_in, formed first
    ref = yb.copy()
    for t in range(x.shape[0]):
        for j in range(idx.shape[1]):
            ref[t] += gate[t, j] * (dense[idx[t, j]] @ x[t])
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-12)
    # and the whole delta as one dense matrix product per adapter over all tokens
    D = np.zeros_like(yb)
    for e in range(len(A)):
        G = np.where(idx == e, gate, 0.0).sum(axis=1)
        D += G[:, None] * (x @ dense[e].T)
    assert np.allclose(y - yb, D, rtol=1e-11, atol=1e-11)


def test_sgmm_zero_B_gives_base_exactly():
    rng = np.random.default_rng(8)
    x, A, B, idx, gate, yb = _random_case(rng)
    Bz = [np.zeros_like(b) for b in B]
    assert np.array_equal(O.sgmm_shrink_expand(x, A, Bz, idx, gate, yb), yb)


def test_sgmm_token_permutation_equivariance():
    rng = np.random.default_rng(9)
    x, A, B, idx, gate, yb = _random_case(rng)
    y = O.sgmm_shrink_expand(x, A, B, idx, gate, yb)
    p = rng.permutation(x.shape[0])
    yp = O.sgmm_shrink_expand(x[p], A, B, idx[p], gate[p], yb[p])
    assert np.array_equal(yp, y[p])


def test_sgmm_linear_in_gates_and_slot_order_free():
    rng = np.random.default_rng(10)
    x, A, B, idx, gate, yb = _random_case(rng)
    zero = np.zeros_like(yb)
    d1 = O.sgmm_shrink_expand(x, A, B, idx, gate, zero)
    d2 = O.sgmm_shrink_expand(x, A, B, idx, 2 * gate, zero)
    assert np.array_equal(d2, 2 * d1)
    # swapping the slots of every token (with their gates) changes nothing
    d3 = O.sgmm_shrink_expand(x, A, B, idx[:, ::-1].copy(), gate[:, ::-1].copy(), zero)
    assert np.allclose(d3, d1, rtol=1e-13, atol=1e-13)
    # one adapter at a time sums to the whole
    parts = sum(O.sgmm_shrink_expand(x, A, B, idx[:, j:j + 1], gate[:, j:j + 1], zero) for j in range(2))
    assert np.allclose(parts, d1, rtol=1e-13, atol=1e-13)


def test_single_adapter_equals_merged_weight_gemm():
    rng = np.random.default_rng(11)
    T, d_in, d_out, r = 9, 30, 20, 6
    Wt = rng.normal(size=(d_out, d_in))
    A = [rng.normal(size=(r, d_in))]
    B = [rng.normal(size=(d_out, r))]
    x = rng.normal(size=(T, d_in))
    idx = np.zeros((T, 1), dtype=np.int32)
    gate = np.ones((T, 1))
    y = O.sgmm_shrink_expand(x, A, B, idx, gate, x @ Wt.T)
    assert np.allclose(y, x @ (Wt + B[0] @ A[0]).T, rtol=1e-12, atol=1e-12)


def test_sgmm_rank_and_index_sensitivity():
    """Transposed or mis-indexed operands change the integer example's answer."""
    A = [np.array([[1.0, 0, 1], [0, 1, 0]]), np.array([[1.0, 1, 1], [2, 0, 0]])]
    B = [np.array([[1.0, 0], [0, 2]]), np.array([[0.0, 1], [1, 0]])]
    x = np.array([[1.0, 2, 3]])
    y0 = O.sgmm_shrink_expand(x, A, B, np.array([[0]]), np.array([[1.0]]), np.zeros((1, 2)))
    y1 = O.sgmm_shrink_expand(x, A, B, np.array([[1]]), np.array([[1.0]]), np.zeros((1, 2)))
    assert y0.tolist() == [[4.0, 4.0]] and y1.tolist() == [[2.0, 6.0]]


# ---------------------------------------------------------------- merge / GEMV


def test_merge_and_gemv_golden(golden_dir):
    g = _load(golden_dir, "sgmm_merge_example.json")
    A = [np.array(a, dtype=float) for a in g["A"]]
    B = [np.array(b, dtype=float) for b in g["B"]]
    Wp = O.merge_adapters(np.array(g["W"], dtype=float), A, B, g["merge_idx"], g["merge_gate"])
    assert np.array_equal(Wp, np.array(g["W_merged"], dtype=float))
    assert np.array_equal(O.gemv(Wp, np.array(g["gemv_x"], dtype=float)), np.array(g["gemv_y"], dtype=float))


def test_merge_zero_B_is_identity_and_matches_unmerged_path():
    rng = np.random.default_rng(12)
    d_out, d_in, r, E = 12, 16, 4, 3
    Wt = rng.normal(size=(d_out, d_in))
    A = [rng.normal(size=(r, d_in)) for _ in range(E)]
    B = [rng.normal(size=(d_out, r)) for _ in range(E)]
    assert np.array_equal(O.merge_adapters(Wt, A, [np.zeros_like(b) for b in B], [2, 0], [0.6, 0.4]), Wt)
    # merged GEMV == base GEMV + the unmerged SGMM delta for the same token
    x = rng.normal(size=d_in)
    Wp = O.merge_adapters(Wt, A, B, [2, 0], [0.6, 0.4])
    y_sgmm = O.sgmm_shrink_expand(x[None], A, B, np.array([[2, 0]]), np.array([[0.6, 0.4]]), (Wt @ x)[None])
    assert np.allclose(O.gemv(Wp, x), y_sgmm[0], rtol=1e-12, atol=1e-12)


def test_gemv_bruteforce():
    rng = np.random.default_rng(13)
    Wt = rng.integers(-5, 6, size=(7, 9)).astype(float)
    x = rng.integers(-5, 6, size=9).astype(float)
    expect = [sum(Wt[i, j] * x[j] for j in range(9)) for i in range(7)]
    assert O.gemv(Wt, x).tolist() == expect


def test_rel_frobenius():
    assert O.rel_frobenius([3.0, 4.0], [3.0, 4.0]) == 0.0
    assert abs(O.rel_frobenius([3.0, 4.0], [0.0, 5.0]) - math.sqrt(10) / 5) < 1e-15


def test_all_k_subsets_bruteforce_small():
    """top-k as the lexicographically best k-subset under (sum of ranks) ordering."""
    rng = np.random.default_rng(14)
    for _ in range(50):
        row = rng.integers(0, 3, size=6).astype(float)
        idx = O.select_topk(row[None], 3)[0]
        # the chosen set must dominate: no unchosen adapter beats a chosen one,
        # and on equal values the unchosen one has a larger index
        for c in idx:
            for u in set(range(6)) - set(idx.tolist()):
                assert row[c] > row[u] or (row[c] == row[u] and c < u)
        # within the selection: descending value, ascending index on ties
        for a, b in itertools.pairwise(idx.tolist()):
            assert row[a] > row[b] or (row[a] == row[b] and a < b)


# ---------------------------------------------------------------- base projection + adapters in one pass


def test_linear_lora_hand_example():
    """Worked by hand: W = [[1, 2], [3, 4]], one rank-1 adapter A = [[1, 0]], B = [[1], [2]].
    Token 0, x = (1, 1): W x = (3, 7), A x = 1, B (A x) = (1, 2), so y = (4, 9).
    Token 1, x = (2, 0) with gate 0.5: W x = (2, 6), A x = 2, 0.5 * B (A x) = (1, 2), so y = (3, 8)."""
    Wt = np.array([[1.0, 2.0], [3.0, 4.0]])
    A = [np.array([[1.0, 0.0]])]
    B = [np.array([[1.0], [2.0]])]
    x = np.array([[1.0, 1.0], [2.0, 0.0]])
    idx = np.zeros((2, 1), dtype=np.int32)
    gate = np.array([[1.0], [0.5]])
    assert np.array_equal(O.linear_lora(x, Wt, A, B, idx, gate), np.array([[4.0, 9.0], [3.0, 8.0]]))


def test_linear_lora_zero_adapters_is_the_plain_product_by_loops():
    """With every B zero the result is x W^T, here summed term by term on small integers."""
    rng = np.random.default_rng(31)
    T, d_in, d_out, E, k, r = 5, 7, 6, 3, 2, 4
    x = rng.integers(-3, 4, size=(T, d_in)).astype(np.float64)
    Wt = rng.integers(-3, 4, size=(d_out, d_in)).astype(np.float64)
    A = [rng.normal(size=(r, d_in)) for _ in range(E)]
    B = [np.zeros((d_out, r)) for _ in range(E)]
    idx = np.array([rng.permutation(E)[:k] for _ in range(T)], dtype=np.int32)
    gate = rng.random((T, k))
    ref = np.zeros((T, d_out))
    for t in range(T):
        for n in range(d_out):
            for i in range(d_in):
                ref[t, n] += x[t, i] * Wt[n, i]
    assert np.array_equal(O.linear_lora(x, Wt, A, B, idx, gate), ref)


def test_linear_lora_single_adapter_equals_merged_weight_gemm():
    """E = 1, k = 1, gate 1: the fused result is the textbook GEMM with W + B A."""
    rng = np.random.default_rng(32)
    T, d_in, d_out, r = 11, 24, 18, 5
    Wt = rng.normal(size=(d_out, d_in))
    A = [rng.normal(size=(r, d_in))]
    B = [rng.normal(size=(d_out, r))]
    x = rng.normal(size=(T, d_in))
    y = O.linear_lora(x, Wt, A, B, np.zeros((T, 1), dtype=np.int32), np.ones((T, 1)))
    assert np.allclose(y, x @ (Wt + B[0] @ A[0]).T, rtol=1e-12, atol=1e-12)


def test_linear_lora_transposed_weight_changes_the_answer():
    """x W^T, not x W: a square non-symmetric W tells the two apart on the integer example."""
    Wt = np.array([[1.0, 2.0], [3.0, 4.0]])
    x = np.array([[1.0, 0.0]])
    A = [np.zeros((1, 2))]
    B = [np.zeros((2, 1))]
    y = O.linear_lora(x, Wt, A, B, np.zeros((1, 1), dtype=np.int32), np.ones((1, 1)))
    assert np.array_equal(y, np.array([[1.0, 3.0]]))
