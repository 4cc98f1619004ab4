"""GPU parity: every entry point of the C ABI against the fp64 oracle.

Indices, offsets and permutations must match bit for bit; gates within 1e-6;
floating outputs within relative Frobenius 5e-3 and max-abs 1e-2*max|ref| per
tensor; small-integer cases must be exact.
"""
import numpy as np
import pytest
import torch

from oracle import apr_oracle as O
from adapter_pregate_router_b200 import workloads as W
from tests.apr_testlib import (GATE_ATOL, bf16_exact, check_guards, close, guarded, oracle_group, run_route,
                               run_segment, run_sgmm, to_np)

pytestmark = pytest.mark.gpu

BF16, F32 = torch.bfloat16, torch.float32


@pytest.fixture(scope="module")
def apr():
    from adapter_pregate_router_b200 import build
    build.build()
    from adapter_pregate_router_b200 import apr as mod
    assert torch.cuda.is_available()
    return mod


# ------------------------------------------------------------------ router


@pytest.mark.parametrize("name", ["tiny", "decode", "prefill", "multitenant", "merge"])
def test_route_configs_bit_exact(apr, name):
    cfg = W.CONFIGS[name]
    h, Wr, forced = W.router_inputs(cfg)
    dt = BF16 if cfg.dtype == "bf16" else F32
    idx, gate = run_route(apr, h, Wr, cfg.k, dt)
    ridx, rgate, _ = O.pregate_route(h, Wr, cfg.k)
    assert np.array_equal(idx, ridx)
    assert np.abs(gate - rgate).max() <= GATE_ATOL
    if forced is not None:
        assert np.array_equal(idx, forced)


@pytest.mark.parametrize("E,k,d,T", [(8, 2, 64, 100), (5, 5, 32, 33), (256, 3, 256, 70), (1024, 8, 128, 40),
                                     (33, 1, 512, 1), (64, 4, 4096, 300)])
def test_route_ties_and_shapes(apr, E, k, d, T):
    rng = np.random.default_rng(E + k + d)
    # few distinct integer values -> many exact ties among logits
    h = rng.integers(-1, 2, size=(T, d)).astype(np.float32)
    Wr = rng.integers(-1, 2, size=(E, d)).astype(np.float32)
    Wr[E // 2] = Wr[0]                         # two identical adapters: always tied
    for dt in (F32, BF16):
        idx, gate = run_route(apr, h, Wr, k, dt)
        ridx, rgate, L = O.pregate_route(h, Wr, k)
        assert np.array_equal(idx, ridx)
        assert np.abs(gate - rgate).max() <= GATE_ATOL
        assert np.allclose(gate.sum(axis=1), 1.0, atol=1e-6)


def test_route_equal_logits_give_half_gates(apr):
    h = np.ones((4, 16), np.float32)
    Wr = np.zeros((6, 16), np.float32)
    Wr[2] = 1.0
    Wr[4] = 1.0
    idx, gate = run_route(apr, h, Wr, 2, F32)
    assert idx.tolist() == [[2, 4]] * 4
    assert np.all(gate == 0.5)
    idx1, gate1 = run_route(apr, h, Wr, 1, F32)
    assert idx1.tolist() == [[2]] * 4 and np.all(gate1 == 1.0)


# ------------------------------------------------------------------ segments


@pytest.mark.parametrize("T,k,E", [(1, 1, 1), (7, 2, 3), (64, 2, 8), (1000, 3, 40), (4096, 1, 256),
                                   (8192, 2, 16), (333, 8, 1024), (5000, 2, 2), (1025, 1, 1024),
                                   (40000, 2, 64), (20000, 3, 1024)])   # the last two: plan not staged in shared memory
def test_segments_bit_exact(apr, T, k, E):
    rng = np.random.default_rng(T * 7 + k + E)
    idx = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    seg_off, perm, _ = run_segment(apr, idx, E)
    rs, rp = O.segment_tokens(idx, E)
    assert np.array_equal(seg_off, rs)
    assert np.array_equal(perm, rp)


@pytest.mark.parametrize("kernel", ["tensor", "skinny"])
def test_sgmm_large_batch_unstaged_plan(apr, kernel):
    """40000 tokens: the segment kernel keeps idx and the token order in global memory (too
    large for shared memory); the gathered kernels read that plan."""
    rng = np.random.default_rng(71)
    idx = _zipf_idx(rng, 40000, 24, 2)
    x, As, Bs, idx, gate, ybs = _case(rng, 40000, 64, (64,), (16,) * 24, 2, dist=idx)
    x, As, Bs, ybs = _rounded(x, As, Bs, ybs)
    kern = apr.SGMM_TENSOR if kernel == "tensor" else apr.SGMM_SKINNY
    got = run_sgmm(apr, x, As, Bs, idx, gate, ybs, BF16, kernel=kern)
    close(got[0], oracle_group(x, As, Bs, idx, gate.astype(np.float64), ybs)[0], f"{kernel} T=40000")


def test_segments_first_call_in_a_fresh_process(apr):
    """The segment kernel's shared-memory limit must be set by the call that needs it, not left
    over from an earlier, larger call in the same process (2500 tokens x 2: the staged plan plus
    the kernel's static shared memory pass the 48 KB default while the dynamic part alone does not)."""
    import subprocess
    import sys
    import os
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    code = (
        "import numpy as np, torch\n"
        "from adapter_pregate_router_b200 import apr\n"
        "from oracle import apr_oracle as O\n"
        "rng = np.random.default_rng(3)\n"
        "idx = np.stack([rng.permutation(12)[:2] for _ in range(2500)]).astype(np.int32)\n"
        "ws = apr.workspace(2500, 2, 12, 16, 64)\n"
        "seg = torch.empty(13, dtype=torch.int32, device='cuda')\n"
        "perm = torch.empty(5000, dtype=torch.int32, device='cuda')\n"
        "apr.segment_tokens(torch.from_numpy(idx).cuda(), 12, seg, perm, ws)\n"
        "apr.stream_status(ws)\n"
        "rs, rp = O.segment_tokens(idx, 12)\n"
        "assert np.array_equal(seg.cpu().numpy(), rs) and np.array_equal(perm.cpu().numpy(), rp)\n"
        "print('ok')\n")
    r = subprocess.run([sys.executable, "-c", code], cwd=root, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip().endswith("ok"), r.stderr[-2000:]


def test_segments_skewed_and_empty(apr):
    # one adapter takes almost everything, several are empty
    idx = np.zeros((3000, 1), np.int32)
    idx[::97] = 5
    idx[1] = 9
    seg_off, perm, _ = run_segment(apr, idx, 12)
    rs, rp = O.segment_tokens(idx, 12)
    assert np.array_equal(seg_off, rs) and np.array_equal(perm, rp)


def test_segment_rejects_out_of_range_index(apr):
    idx = np.array([[0, 1], [2, 7]], np.int32)
    T, k, E = 2, 2, 4
    ws = apr.workspace(T, k, E, 8, 8)
    d_idx = torch.from_numpy(idx).cuda()
    seg_off = torch.full((E + 1,), 5, dtype=torch.int32, device="cuda")
    perm = torch.zeros(4, dtype=torch.int32, device="cuda")
    apr.segment_tokens(d_idx, E, seg_off, perm, ws)
    assert apr.raw_stream_status(ws) == apr.APR_ERR_DEVICE_INDEX
    assert seg_off.cpu().tolist() == [0] * (E + 1)
    assert apr.raw_stream_status(ws) == apr.APR_OK          # the error word was cleared


# ------------------------------------------------------------------ SGMM, explicit cases


def _case(rng, T, d_in, d_outs, ranks, k, dist="uniform", pool=None, ints=False):
    E = len(ranks)
    if pool is None:
        pool = np.arange(E)
    if isinstance(dist, str):
        idx = np.stack([rng.choice(pool, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    else:
        idx = dist
    if ints:
        x = rng.integers(-1, 2, size=(T, d_in)).astype(np.float32)
        As = [[rng.integers(-1, 2, size=(r, d_in)).astype(np.float32) for r in ranks] for _ in d_outs]
        Bs = [[rng.integers(-1, 2, size=(d, r)).astype(np.float32) for r in ranks] for d in d_outs]
        gate = np.full((T, k), 1.0 / k, np.float32)
        ybs = [rng.integers(-4, 5, size=(T, d)).astype(np.float32) for d in d_outs]
    else:
        x = rng.normal(size=(T, d_in)).astype(np.float32)
        As = [[(0.02 * rng.normal(size=(r, d_in))).astype(np.float32) for r in ranks] for _ in d_outs]
        Bs = [[(0.02 * rng.normal(size=(d, r))).astype(np.float32) for r in ranks] for d in d_outs]
        gate = rng.dirichlet(np.ones(k), size=T).astype(np.float32)
        ybs = [rng.normal(size=(T, d)).astype(np.float32) for d in d_outs]
    return x, As, Bs, idx, gate, ybs


def _rounded(x, As, Bs, ybs):
    return (bf16_exact(x), [[bf16_exact(a) for a in P] for P in As], [[bf16_exact(b) for b in P] for P in Bs],
            [bf16_exact(y) for y in ybs])


@pytest.mark.parametrize("dtype", [F32, BF16])
@pytest.mark.parametrize("T,d_in,d_outs,ranks,k", [
    (64, 256, (256,), (8,) * 8, 2),                       # the tiny shape
    (32, 4096, (4096, 4096, 4096), (16,) * 8, 2),         # a decode qkv group
    (37, 1000, (1000, 520), (8, 16, 32, 64, 128, 8), 2),  # ragged widths, every rank
    (129, 4104, (136,), (16, 24, 40), 1),                 # three column chunks, odd ranks
    (300, 512, (256,), (16,) * 5, 3),
    (16, 64, (64,), (8,) * 16, 8),                        # k = 8
    (1, 2048, (4096,), (16,) * 8, 2),                     # one token
])
def test_sgmm_skinny_parity(apr, dtype, T, d_in, d_outs, ranks, k):
    rng = np.random.default_rng(T + d_in + k)
    x, As, Bs, idx, gate, ybs = _case(rng, T, d_in, d_outs, ranks, k)
    if dtype == BF16:
        x, As, Bs, ybs = _rounded(x, As, Bs, ybs)
    for zero in (True, False):
        yb = [np.zeros_like(y) for y in ybs] if zero else ybs
        got = run_sgmm(apr, x, As, Bs, idx, gate, yb, dtype, kernel=apr.SGMM_SKINNY)
        ref = oracle_group(x, As, Bs, idx, gate.astype(np.float64), yb)
        for p in range(len(d_outs)):
            close(got[p], ref[p], f"proj {p} zero_ybase={zero}")


def test_sgmm_adversarial_segments(apr):
    """Empty, size-1 and 127/128/129-pair segments; one huge segment; ragged T."""
    rng = np.random.default_rng(5)
    counts = {1: 1, 2: 127, 3: 128, 4: 129, 5: 2000}
    idx = np.concatenate([np.full(c, e, np.int32) for e, c in counts.items()])
    rng.shuffle(idx)
    idx = idx[:, None]
    T = idx.shape[0]
    ranks = (16, 8, 16, 32, 64, 16, 8)           # adapters 0 and 6 are empty
    x, As, Bs, _, _, ybs = _case(rng, T, 512, (328,), ranks, 1)
    gate = np.ones((T, 1), np.float32)
    x, As, Bs, ybs = _rounded(x, As, Bs, ybs)
    got = run_sgmm(apr, x, As, Bs, idx, gate, ybs, BF16, kernel=apr.SGMM_SKINNY)
    ref = oracle_group(x, As, Bs, idx, gate.astype(np.float64), ybs)
    close(got[0], ref[0], "adversarial")


def test_sgmm_all_tokens_one_adapter_pair(apr):
    rng = np.random.default_rng(6)
    T = 777
    idx = np.tile(np.array([[3, 1]], np.int32), (T, 1))
    x, As, Bs, _, gate, ybs = _case(rng, T, 256, (264,), (16,) * 4, 2)
    x, As, Bs, ybs = _rounded(x, As, Bs, ybs)
    got = run_sgmm(apr, x, As, Bs, idx, gate, ybs, BF16, kernel=apr.SGMM_SKINNY)
    close(got[0], oracle_group(x, As, Bs, idx, gate.astype(np.float64), ybs)[0], "one pair")


@pytest.mark.parametrize("dtype", [F32, BF16])
def test_sgmm_integer_inputs_exact(apr, dtype):
    """Small integers and gates of 1/2: every product and sum is exact in fp32,
    so the device result must equal the oracle's exact value rounded once to the
    output type, bit for bit (pins the gather/scatter indexing)."""
    rng = np.random.default_rng(7)
    x, As, Bs, idx, gate, ybs = _case(rng, 150, 1000, (72, 40), (8, 16, 8, 24), 2, ints=True)
    got = run_sgmm(apr, x, As, Bs, idx, gate, ybs, dtype, kernel=apr.SGMM_SKINNY)
    ref = oracle_group(x, As, Bs, idx, gate.astype(np.float64), ybs)
    for p in range(2):
        want = ref[p] if dtype == F32 else bf16_exact(ref[p]).astype(np.float64)
        assert np.array_equal(got[p], want), f"proj {p}: max diff {np.abs(got[p] - want).max()}"


def test_sgmm_zero_B_leaves_base_bit_exact(apr):
    rng = np.random.default_rng(8)
    x, As, Bs, idx, gate, ybs = _case(rng, 40, 512, (256,), (16,) * 6, 2)
    x, As, Bs, ybs = _rounded(x, As, Bs, ybs)
    Bz = [[np.zeros_like(b) for b in P] for P in Bs]
    got = run_sgmm(apr, x, As, Bz, idx, gate, ybs, BF16, kernel=apr.SGMM_SKINNY)
    assert np.array_equal(got[0], ybs[0].astype(np.float64))


def test_sgmm_in_place_and_token_order(apr):
    rng = np.random.default_rng(9)
    x, As, Bs, idx, gate, ybs = _case(rng, 90, 256, (128,), (16,) * 5, 2)
    x, As, Bs, ybs = _rounded(x, As, Bs, ybs)
    a = run_sgmm(apr, x, As, Bs, idx, gate, ybs, BF16, kernel=apr.SGMM_SKINNY, in_place=True)[0]
    b = run_sgmm(apr, x, As, Bs, idx, gate, ybs, BF16, kernel=apr.SGMM_SKINNY)[0]
    assert np.array_equal(a, b)
    p = rng.permutation(90)
    c = run_sgmm(apr, x[p], As, Bs, idx[p], gate[p], [ybs[0][p]], BF16, kernel=apr.SGMM_SKINNY)[0]
    assert np.array_equal(c, b[p])                 # the same bits: no order dependence


def test_sgmm_deterministic(apr):
    rng = np.random.default_rng(10)
    x, As, Bs, idx, gate, ybs = _case(rng, 200, 4096, (512,), (16,) * 8, 2)
    x, As, Bs, ybs = _rounded(x, As, Bs, ybs)
    a = run_sgmm(apr, x, As, Bs, idx, gate, ybs, BF16, kernel=apr.SGMM_SKINNY)[0]
    b = run_sgmm(apr, x, As, Bs, idx, gate, ybs, BF16, kernel=apr.SGMM_SKINNY)[0]
    assert np.array_equal(a, b)


def test_sgmm_device_index_fault_is_reported(apr):
    """A rank above the declared maximum is caught on the device: error word, no trap."""
    rng = np.random.default_rng(11)
    x, As, Bs, idx, gate, ybs = _case(rng, 20, 256, (128,), (16, 16, 32), 2)
    x, As, Bs, ybs = _rounded(x, As, Bs, ybs)
    with pytest.raises(apr.AprError) as ei:
        run_sgmm(apr, x, As, Bs, idx, gate, ybs, BF16, kernel=apr.SGMM_SKINNY, max_rank=16)
    assert ei.value.status == apr.APR_ERR_DEVICE_INDEX
    # the context is still usable afterwards
    ok = run_sgmm(apr, x, As, Bs, idx, gate, ybs, BF16, kernel=apr.SGMM_SKINNY)
    close(ok[0], oracle_group(x, As, Bs, idx, gate.astype(np.float64), ybs)[0], "after fault")


# ------------------------------------------------------------------ merge and GEMV


@pytest.mark.parametrize("E,r,k", [(5, 16, 2), (8, 8, 5), (4, 32, 2), (3, 8, 1)])
def test_merge_and_gemv_small(apr, E, r, k):
    """Tensor-core merge (k * rank <= 64 after rounding the rank to 16) and the
    CUDA-core merge (k=5, rank 8), on ragged weight shapes."""
    rng = np.random.default_rng(12 + E + r + k)
    shapes = [(264, 136), (40, 1000), (1000, 64)]
    Ws = [bf16_exact(0.02 * rng.normal(size=s)) for s in shapes]
    As = [[bf16_exact(0.02 * rng.normal(size=(r, s[1]))) for _ in range(E)] for s in shapes]
    Bs = [[bf16_exact(0.02 * rng.normal(size=(s[0], r))) for _ in range(E)] for s in shapes]
    xs = [bf16_exact(rng.normal(size=s[1])) for s in shapes]
    idx1 = rng.permutation(E)[:k].astype(np.int32)
    g1 = rng.dirichlet(np.ones(k)).astype(np.float32)
    dW = [torch.from_numpy(w).cuda().to(BF16) for w in Ws]
    dW_in = [w.clone() for w in dW]
    wp_bufs = [guarded(np.full(s, np.nan, np.float32), BF16) for s in shapes]   # W' inside guard bands
    dWp = [v for _, v in wp_bufs]
    keep = []
    entries = []
    for p in range(len(shapes)):
        A = [torch.from_numpy(a).cuda().to(BF16) for a in As[p]]
        B = [torch.from_numpy(b).cuda().to(BF16) for b in Bs[p]]
        At, Bt = apr.ptr_array(A), apr.ptr_array(B)
        keep += [A, B, At, Bt]
        entries.append((dW[p], dWp[p], At, Bt))
    tab = apr.merge_table(entries)
    ws = apr.workspace(1, k, E, r, 8)
    apr.merge_adapters(tab, len(shapes), E, r, torch.from_numpy(idx1).cuda(), torch.from_numpy(g1).cuda(), k, ws)
    ys, y_bufs = [], []
    for p in range(len(shapes)):
        ybuf, y = guarded(np.full(shapes[p][0], np.nan, np.float32), BF16)
        apr.gemv(dWp[p], torch.from_numpy(xs[p]).cuda().to(BF16), y)
        ys.append(y)
        y_bufs.append(ybuf)
    apr.stream_status(ws)
    for p in range(len(shapes)):
        check_guards(wp_bufs[p][0], f"merged weight {p}")
        check_guards(y_bufs[p], f"gemv {p}")
        assert torch.equal(dW[p], dW_in[p]), f"weight {p} written by the out-of-place merge"
    for p in range(len(shapes)):
        ref = O.merge_adapters(Ws[p], As[p], Bs[p], idx1, g1.astype(np.float64))
        close(to_np(dWp[p]), ref, f"merged weight {p}")
        close(to_np(ys[p]), O.gemv(ref, xs[p]), f"gemv {p}")
    # the planned (TMA) merge gives the same bits where the tensor-core merge applies
    first = [w.clone() for w in dWp]
    for w in dWp:
        w.fill_(float("nan"))
    plan = apr.merge_plan(entries)
    args = (tab, plan, len(shapes), E, r, torch.from_numpy(idx1).cuda(), torch.from_numpy(g1).cuda(), k, ws)
    if k * ((r + 15) // 16 * 16) <= 64:
        apr.merge_adapters_planned(*args)
        apr.stream_status(ws)
        for p in range(len(shapes)):
            assert torch.equal(dWp[p], first[p]), f"planned merge differs on weight {p}"
            check_guards(wp_bufs[p][0], f"planned merged weight {p}")
            assert torch.equal(dW[p], dW_in[p]), f"weight {p} written by the planned merge"
    else:
        with pytest.raises(apr.AprError) as ei:
            apr.merge_adapters_planned(*args)
        assert ei.value.status == apr.APR_ERR_UNSUPPORTED


def test_merge_zero_B_is_bit_exact_copy(apr):
    rng = np.random.default_rng(13)
    E, r = 3, 16
    Wt = bf16_exact(0.02 * rng.normal(size=(96, 512)))
    A = [torch.from_numpy(bf16_exact(rng.normal(size=(r, 512)))).cuda().to(BF16) for _ in range(E)]
    B = [torch.zeros((96, r), dtype=BF16, device="cuda") for _ in range(E)]
    At, Bt = apr.ptr_array(A), apr.ptr_array(B)
    dW = torch.from_numpy(Wt).cuda().to(BF16)
    dWp = torch.empty_like(dW)
    tab = apr.merge_table([(dW, dWp, At, Bt)])
    ws = apr.workspace(1, 2, E, r, 8)
    apr.merge_adapters(tab, 1, E, r, torch.tensor([2, 0], dtype=torch.int32, device="cuda"),
                       torch.tensor([0.7, 0.3], dtype=torch.float32, device="cuda"), 2, ws)
    apr.stream_status(ws)
    assert torch.equal(dWp, dW)
    dWp.zero_()
    plan = apr.merge_plan([(dW, dWp, At, Bt)])
    apr.merge_adapters_planned(tab, plan, 1, E, r, torch.tensor([2, 0], dtype=torch.int32, device="cuda"),
                               torch.tensor([0.7, 0.3], dtype=torch.float32, device="cuda"), 2, ws)
    apr.stream_status(ws)
    assert torch.equal(dWp, dW)


@pytest.mark.parametrize("d_out,d_in", [(4096, 4096), (11008, 4096), (4096, 11008), (37, 72)])
def test_gemv_parity(apr, d_out, d_in):
    rng = np.random.default_rng(d_out + d_in)
    Wt = bf16_exact(0.02 * rng.normal(size=(d_out, d_in)))
    x = bf16_exact(rng.normal(size=d_in))
    ybuf, y = guarded(np.full(d_out, np.nan, np.float32), BF16)
    apr.gemv(torch.from_numpy(Wt).cuda().to(BF16), torch.from_numpy(x).cuda().to(BF16), y)
    torch.cuda.synchronize()
    check_guards(ybuf, "gemv")
    close(to_np(y), O.gemv(Wt, x), "gemv")


# ------------------------------------------------------------------ SGMM, tensor-core kernel


def _zipf_idx(rng, T, E, k, s=1.1):
    p = 1.0 / np.arange(1, E + 1) ** s
    p /= p.sum()
    return np.stack([rng.choice(E, size=k, replace=False, p=p) for _ in range(T)]).astype(np.int32)


@pytest.mark.parametrize("T,d_in,d_outs,ranks,k,zipf", [
    (300, 512, (256,), (16,) * 4, 2, False),               # many small sets, partial tiles
    (1000, 1024, (512, 1008), (16,) * 6, 2, True),         # sets longer than one tile, ragged d_out
    (700, 256, (128,), (8, 16, 32, 64), 1, False),         # top-1, every rank up to 64
    (517, 4096, (4096,), (16,) * 16, 2, True),             # prefill-shaped projection
    (129, 192, (64, 64, 64, 64), (32,) * 3, 2, False),     # four projections, k * rank = 64
    (1, 128, (16,), (16, 16), 2, False),                   # one token
    (600, 256, (128, 64), (16, 8, 16, 16, 8, 16), 1, True),  # top-1 with rank slots of 16: mixed tiles of one-adapter sets
    (2500, 512, (256,), (16,) * 12, 2, True),               # many sets, mixed tiles split long sets
])
def test_sgmm_tensor_parity(apr, T, d_in, d_outs, ranks, k, zipf):
    rng = np.random.default_rng(T + d_in + k + 1)
    idx = _zipf_idx(rng, T, len(ranks), k) if zipf else "uniform"
    x, As, Bs, idx, gate, ybs = _case(rng, T, d_in, d_outs, ranks, k, dist=idx)
    x, As, Bs, ybs = _rounded(x, As, Bs, ybs)
    for zero in (True, False):
        yb = [np.zeros_like(y) for y in ybs] if zero else ybs
        got = run_sgmm(apr, x, As, Bs, idx, gate, yb, BF16, kernel=apr.SGMM_TENSOR)
        ref = oracle_group(x, As, Bs, idx, gate.astype(np.float64), yb)
        for p in range(len(d_outs)):
            close(got[p], ref[p], f"tensor proj {p} zero_ybase={zero}")


def test_sgmm_tensor_integer_inputs_exact(apr):
    """Small integers, gates of 1/2: the tensor-core result is the exact value
    rounded once to bf16."""
    rng = np.random.default_rng(21)
    x, As, Bs, idx, gate, ybs = _case(rng, 400, 512, (128, 256), (16, 16, 16, 16, 16), 2, ints=True)
    got = run_sgmm(apr, x, As, Bs, idx, gate, ybs, BF16, kernel=apr.SGMM_TENSOR)
    ref = oracle_group(x, As, Bs, idx, gate.astype(np.float64), ybs)
    for p in range(2):
        want = bf16_exact(ref[p]).astype(np.float64)
        assert np.array_equal(got[p], want), f"proj {p}: max diff {np.abs(got[p] - want).max()}"


def test_sgmm_tensor_properties(apr):
    """Zero B leaves y_base bit-exact; in place equals out of place; a token
    permutation permutes the output bits (ragged d_out: the last tile's second
    half is partly past the end)."""
    rng = np.random.default_rng(24)
    idx = _zipf_idx(rng, 900, 6, 2)
    x, As, Bs, idx, gate, ybs = _case(rng, 900, 512, (1008, 80), (16,) * 6, 2, dist=idx)
    x, As, Bs, ybs = _rounded(x, As, Bs, ybs)
    Bz = [[np.zeros_like(b) for b in P] for P in Bs]
    z = run_sgmm(apr, x, As, Bz, idx, gate, ybs, BF16, kernel=apr.SGMM_TENSOR)
    for p in range(2):
        assert np.array_equal(z[p], ybs[p].astype(np.float64))
    a = run_sgmm(apr, x, As, Bs, idx, gate, ybs, BF16, kernel=apr.SGMM_TENSOR, in_place=True)
    b = run_sgmm(apr, x, As, Bs, idx, gate, ybs, BF16, kernel=apr.SGMM_TENSOR)
    for p in range(2):
        assert np.array_equal(a[p], b[p])
    perm = rng.permutation(900)
    d = run_sgmm(apr, x[perm], As, Bs, idx[perm], gate[perm], [y[perm] for y in ybs], BF16, kernel=apr.SGMM_TENSOR)
    for p in range(2):
        assert np.array_equal(d[p], b[p][perm])


def test_sgmm_tensor_matches_skinny(apr):
    rng = np.random.default_rng(22)
    idx = _zipf_idx(rng, 2000, 8, 2)
    x, As, Bs, idx, gate, ybs = _case(rng, 2000, 1024, (512,), (16,) * 8, 2, dist=idx)
    x, As, Bs, ybs = _rounded(x, As, Bs, ybs)
    a = run_sgmm(apr, x, As, Bs, idx, gate, ybs, BF16, kernel=apr.SGMM_TENSOR)[0]
    b = run_sgmm(apr, x, As, Bs, idx, gate, ybs, BF16, kernel=apr.SGMM_SKINNY)[0]
    # both within one bf16 rounding of each other almost everywhere
    assert np.mean(a == b) > 0.95
    close(a, b, "tensor vs skinny")


def test_sgmm_tensor_rejects_unsupported(apr):
    rng = np.random.default_rng(23)
    x, As, Bs, idx, gate, ybs = _case(rng, 50, 100 * 8, (64,), (16,) * 4, 2)   # d_in % 64 != 0
    x, As, Bs, ybs = _rounded(x, As, Bs, ybs)
    with pytest.raises(apr.AprError) as ei:
        run_sgmm(apr, x, As, Bs, idx, gate, ybs, BF16, kernel=apr.SGMM_TENSOR)
    assert ei.value.status == apr.APR_ERR_UNSUPPORTED


def test_sgmm_tensor_plan_reuse_across_calls(apr):
    """Top-2 gathered calls that share one workspace: the set and mixed tiles are built by the
    first call after a plan and reused by the next; a new plan (another routing, other token
    count) rebuilds them.  Every call is checked against the oracle."""
    rng = np.random.default_rng(61)
    E, ranks = 12, (16,) * 12
    ws = apr.workspace(1500, 2, E, 16, 512)
    for T, reps in ((1000, 2), (1500, 2), (700, 1)):
        idx = _zipf_idx(rng, T, E, 2)
        x, As, Bs, idx, gate, ybs = _case(rng, T, 512, (256, 144), ranks, 2, dist=idx)
        x, As, Bs, ybs = _rounded(x, As, Bs, ybs)
        idx_d = torch.from_numpy(np.ascontiguousarray(idx, dtype=np.int32)).cuda()
        gate_d = torch.from_numpy(np.ascontiguousarray(gate, dtype=np.float32)).cuda()
        seg_off = torch.empty(E + 1, dtype=torch.int32, device="cuda")
        perm = torch.empty(T * 2, dtype=torch.int32, device="cuda")
        apr.segment_tokens(idx_d, E, seg_off, perm, ws)
        xd = torch.from_numpy(x).cuda().to(BF16)
        keep = []
        tabs = []
        for p in range(2):
            A = [torch.from_numpy(a).cuda().to(BF16) for a in As[p]]
            B = [torch.from_numpy(b).cuda().to(BF16) for b in Bs[p]]
            keep += [A, B]
            tabs.append((apr.ptr_array(A), apr.ptr_array(B)))
        rk = torch.full((E,), 16, dtype=torch.int32, device="cuda")
        ref = oracle_group(x, As, Bs, idx, gate.astype(np.float64), ybs)
        for _ in range(reps):
            ys = [torch.full_like(torch.from_numpy(y), float("nan")).cuda().to(BF16) for y in ybs]
            yb = [torch.from_numpy(y).cuda().to(BF16) for y in ybs]
            projs = [apr.make_proj(ys[p], yb[p], tabs[p][0], tabs[p][1]) for p in range(2)]
            apr.sgmm_shrink_expand(xd, projs, 2, E, rk, 16, idx_d, gate_d, seg_off, perm, ws, apr.SGMM_TENSOR)
            apr.stream_status(ws)
            for p in range(2):
                close(to_np(ys[p]), ref[p], f"T={T} proj {p}")


# ------------------------------------------------------------------ SGMM, ragged many-tenant tiles (top-1)

_RANKS_8_128 = tuple(range(8, 136, 8))


def _ragged_case(rng, T, d_in, d_outs, E, rank_set, dist, ints=False):
    ranks = tuple(int(r) for r in rng.choice(np.asarray(rank_set), size=E))
    if dist == "zipf":
        idx = _zipf_idx(rng, T, E, 1)
    elif dist == "one":
        idx = np.full((T, 1), E // 2, np.int32)
    else:
        idx = np.asarray(rng.integers(0, E, size=(T, 1)), np.int32)
    return ranks, _case(rng, T, d_in, d_outs, ranks, 1, dist=idx, ints=ints)


@pytest.mark.parametrize("T,d_in,d_outs,E,rank_set,dist", [
    (1500, 512, (256, 200), 64, _RANKS_8_128, "uniform"),     # every rank 8..128; a 72-column last block
    (700, 256, (128,), 300, (8, 16), "uniform"),               # 1-6 tokens per adapter: tiles close on 16 adapters
    (900, 256, (136, 64), 40, (64, 96, 128), "zipf"),          # tiles close on 256 rank rows; long segments split
    (1000, 512, (256,), 3, (128,), "one"),                     # one adapter of rank 128 takes every token
    (4096, 1024, (1024, 1024), 256, (8, 16, 32, 64), "uniform"),   # the many-tenant routing, narrower projections
    (130, 64, (16,), 2, (8, 24), "uniform"),                   # d_out of one 16-column block
])
def test_sgmm_ragged_parity(apr, T, d_in, d_outs, E, rank_set, dist):
    """Top-1 calls on the tensor-core path go through ragged tiles (<= 128 tokens of <= 16
    adapters, rank slots adding up to <= 256): every rank up to 128, tiles that close on the
    token, adapter and rank-row limits, and an adapter split over many tiles."""
    rng = np.random.default_rng(T + d_in + E + 7)
    ranks, (x, As, Bs, idx, gate, ybs) = _ragged_case(rng, T, d_in, d_outs, E, rank_set, dist)
    x, As, Bs, ybs = _rounded(x, As, Bs, ybs)
    for zero in (True, False):
        yb = [np.zeros_like(y) for y in ybs] if zero else ybs
        got = run_sgmm(apr, x, As, Bs, idx, gate, yb, BF16, kernel=apr.SGMM_TENSOR)
        ref = oracle_group(x, As, Bs, idx, gate.astype(np.float64), yb)
        for p in range(len(d_outs)):
            close(got[p], ref[p], f"ragged proj {p} zero_ybase={zero}")


def test_sgmm_ragged_integer_inputs_exact(apr):
    """Small integers (|v| <= 128, exact in bf16) and ranks 8..128: the result is the exact value
    rounded once to bf16 (pins each adapter's slot offset and width in V and Bcat)."""
    rng = np.random.default_rng(31)
    ranks, (x, As, Bs, idx, gate, ybs) = _ragged_case(rng, 800, 128, (264, 128), 48, _RANKS_8_128, "uniform",
                                                      ints=True)
    got = run_sgmm(apr, x, As, Bs, idx, gate, ybs, BF16, kernel=apr.SGMM_TENSOR)
    ref = oracle_group(x, As, Bs, idx, gate.astype(np.float64), ybs)
    for p in range(2):
        want = bf16_exact(ref[p]).astype(np.float64)
        assert np.array_equal(got[p], want), f"proj {p}: max diff {np.abs(got[p] - want).max()}"


def test_sgmm_ragged_properties(apr):
    """Zero B leaves y_base bit-exact; in place equals out of place; two runs agree bit for bit;
    a token permutation permutes the output bits."""
    rng = np.random.default_rng(32)
    ranks, (x, As, Bs, idx, gate, ybs) = _ragged_case(rng, 1200, 256, (520, 136), 96, (8, 16, 32, 64, 128),
                                                      "uniform")
    x, As, Bs, ybs = _rounded(x, As, Bs, ybs)
    Bz = [[np.zeros_like(b) for b in P] for P in Bs]
    z = run_sgmm(apr, x, As, Bz, idx, gate, ybs, BF16, kernel=apr.SGMM_TENSOR)
    for p in range(2):
        assert np.array_equal(z[p], ybs[p].astype(np.float64))
    a = run_sgmm(apr, x, As, Bs, idx, gate, ybs, BF16, kernel=apr.SGMM_TENSOR, in_place=True)
    b = run_sgmm(apr, x, As, Bs, idx, gate, ybs, BF16, kernel=apr.SGMM_TENSOR)
    c = run_sgmm(apr, x, As, Bs, idx, gate, ybs, BF16, kernel=apr.SGMM_TENSOR)
    for p in range(2):
        assert np.array_equal(a[p], b[p]) and np.array_equal(b[p], c[p])
    perm = rng.permutation(1200)
    d = run_sgmm(apr, x[perm], As, Bs, idx[perm], gate[perm], [y[perm] for y in ybs], BF16, kernel=apr.SGMM_TENSOR)
    for p in range(2):
        assert np.array_equal(d[p], b[p][perm])


def test_sgmm_ragged_rank_fault_is_reported(apr):
    """A rank above the declared maximum on the ragged path: error word, no trap, context usable."""
    rng = np.random.default_rng(33)
    ranks, (x, As, Bs, idx, gate, ybs) = _ragged_case(rng, 600, 128, (128,), 20, (16, 32, 64), "uniform")
    x, As, Bs, ybs = _rounded(x, As, Bs, ybs)
    with pytest.raises(apr.AprError) as ei:
        run_sgmm(apr, x, As, Bs, idx, gate, ybs, BF16, kernel=apr.SGMM_TENSOR, max_rank=32)
    assert ei.value.status == apr.APR_ERR_DEVICE_INDEX
    ok = run_sgmm(apr, x, As, Bs, idx, gate, ybs, BF16, kernel=apr.SGMM_TENSOR)
    close(ok[0], oracle_group(x, As, Bs, idx, gate.astype(np.float64), ybs)[0], "ragged after fault")


# ------------------------------------------------------------------ SGMM, dense small-batch kernel


@pytest.mark.parametrize("T,d_in,d_outs,ranks,k", [
    (32, 4096, (4096, 4096, 4096), (16,) * 8, 2),          # a decode qkv group
    (32, 11008, (4096,), (16,) * 8, 2),                    # the down projection: six clusters, the last ragged
    (32, 4096, (11008, 11008), (16,) * 8, 2),              # gate/up: a ragged last output tile
    (1, 2048, (136,), (8, 16, 24, 16), 2),                 # one token, mixed ranks, an 8-column tail tile
    (64, 200, (72,), (16,) * 16, 3),                       # 256 rank rows (two M tiles); d_in not a multiple of 64
    (17, 520, (264, 8), (64, 32, 8, 64), 1),               # rank slots of 64, k = 1, an 8-wide projection
    (50, 1024, (128,), (128, 8), 2),                       # rank 128: two adapters fill 256 rows
    (5, 64, (16,), (8,) * 3, 3),                           # k = E, fewer rank rows than one M tile
    (16, 5000, (256,), (16,) * 16, 2),                     # 256 rank rows over three clusters, ragged
    (24, 4104, (384,), (32,) * 4, 2),                      # one M tile, two wide clusters (the second 8 columns)
])
def test_sgmm_dense_parity(apr, T, d_in, d_outs, ranks, k):
    rng = np.random.default_rng(T + d_in + k + 3)
    x, As, Bs, idx, gate, ybs = _case(rng, T, d_in, d_outs, ranks, k)
    x, As, Bs, ybs = _rounded(x, As, Bs, ybs)
    for zero in (True, False):
        yb = [np.zeros_like(y) for y in ybs] if zero else ybs
        got = run_sgmm(apr, x, As, Bs, idx, gate, yb, BF16, kernel=apr.SGMM_DENSE)
        ref = oracle_group(x, As, Bs, idx, gate.astype(np.float64), yb)
        for p in range(len(d_outs)):
            close(got[p], ref[p], f"dense proj {p} zero_ybase={zero}")


@pytest.mark.parametrize("d_in,ranks", [
    (2560, (8, 16, 8, 24, 16)),      # 160 rank rows: partials per cluster, summed by the expand
    (4096, (8, 16, 8, 16)),          # 64 rank rows: one cluster spans d_in and writes the final V
])
def test_sgmm_dense_integer_inputs_exact(apr, d_in, ranks):
    """Small integers, gates of 1/2: the dense result is the exact value rounded
    once to bf16 (pins the adapter-slot and token indexing of both products)."""
    rng = np.random.default_rng(31)
    x, As, Bs, idx, gate, ybs = _case(rng, 40, d_in, (72, 136), ranks, 2, ints=True)
    got = run_sgmm(apr, x, As, Bs, idx, gate, ybs, BF16, kernel=apr.SGMM_DENSE)
    ref = oracle_group(x, As, Bs, idx, gate.astype(np.float64), ybs)
    for p in range(2):
        want = bf16_exact(ref[p]).astype(np.float64)
        assert np.array_equal(got[p], want), f"proj {p}: max diff {np.abs(got[p] - want).max()}"


def test_sgmm_dense_properties(apr):
    """Zero B leaves y_base bit-exact; in place equals out of place; a token
    permutation permutes the output bits; two runs agree bit for bit; the dense
    and CUDA-core kernels agree within one bf16 rounding."""
    rng = np.random.default_rng(32)
    x, As, Bs, idx, gate, ybs = _case(rng, 50, 4096, (512,), (16,) * 8, 2)
    x, As, Bs, ybs = _rounded(x, As, Bs, ybs)
    Bz = [[np.zeros_like(b) for b in P] for P in Bs]
    z = run_sgmm(apr, x, As, Bz, idx, gate, ybs, BF16, kernel=apr.SGMM_DENSE)[0]
    assert np.array_equal(z, ybs[0].astype(np.float64))
    a = run_sgmm(apr, x, As, Bs, idx, gate, ybs, BF16, kernel=apr.SGMM_DENSE, in_place=True)[0]
    b = run_sgmm(apr, x, As, Bs, idx, gate, ybs, BF16, kernel=apr.SGMM_DENSE)[0]
    c = run_sgmm(apr, x, As, Bs, idx, gate, ybs, BF16, kernel=apr.SGMM_DENSE)[0]
    assert np.array_equal(a, b) and np.array_equal(b, c)
    p = rng.permutation(50)
    d = run_sgmm(apr, x[p], As, Bs, idx[p], gate[p], [ybs[0][p]], BF16, kernel=apr.SGMM_DENSE)[0]
    assert np.array_equal(d, b[p])
    s = run_sgmm(apr, x, As, Bs, idx, gate, ybs, BF16, kernel=apr.SGMM_SKINNY)[0]
    assert np.mean(s == b) > 0.95
    close(b, s, "dense vs skinny")


def test_sgmm_dense_faults_and_limits(apr):
    rng = np.random.default_rng(33)
    x, As, Bs, idx, gate, ybs = _case(rng, 20, 256, (128,), (16, 16, 32), 2)
    x, As, Bs, ybs = _rounded(x, As, Bs, ybs)
    with pytest.raises(apr.AprError) as ei:                   # a rank above max_rank, caught on the device
        run_sgmm(apr, x, As, Bs, idx, gate, ybs, BF16, kernel=apr.SGMM_DENSE, max_rank=16)
    assert ei.value.status == apr.APR_ERR_DEVICE_INDEX
    ok = run_sgmm(apr, x, As, Bs, idx, gate, ybs, BF16, kernel=apr.SGMM_DENSE)
    close(ok[0], oracle_group(x, As, Bs, idx, gate.astype(np.float64), ybs)[0], "dense after fault")
    x2, As2, Bs2, idx2, gate2, ybs2 = _case(rng, 65, 256, (128,), (16,) * 4, 2)   # T above the dense limit
    x2, As2, Bs2, ybs2 = _rounded(x2, As2, Bs2, ybs2)
    with pytest.raises(apr.AprError) as ei:
        run_sgmm(apr, x2, As2, Bs2, idx2, gate2, ybs2, BF16, kernel=apr.SGMM_DENSE)
    assert ei.value.status == apr.APR_ERR_UNSUPPORTED


# ------------------------------------------------------------------ edge cases on every kernel class


def _seg_counts_idx(rng, counts, k):
    """idx [T, k] whose adapter segments hold exactly ``counts[e]`` pairs (adapters absent from
    ``counts`` are empty).  The pairs sorted by adapter are dealt slot by slot (token t takes
    positions t, t + T, ...), so a token never holds one adapter twice while every count is at
    most T; then tokens and each token's slots are shuffled."""
    pairs = np.concatenate([np.full(c, e, np.int32) for e, c in sorted(counts.items())])
    T = len(pairs) // k
    assert T * k == len(pairs) and max(counts.values()) <= T
    idx = np.stack([pairs[j * T:(j + 1) * T] for j in range(k)], axis=1)
    idx = idx[rng.permutation(T)]
    for t in range(T):
        idx[t] = idx[t][rng.permutation(k)]
    assert all(len(set(r)) == k for r in idx.tolist())
    return np.ascontiguousarray(idx)


# pair counts per adapter: empty adapters (0 and the last), a one-pair segment, 127/128/129-pair
# segments and segments of thousands of pairs
_EDGE_K1 = {1: 1, 2: 127, 3: 128, 4: 129, 5: 2001}                      # 7 adapters, T = 2386
_EDGE_K2 = {1: 1, 2: 127, 3: 128, 4: 129, 5: 1000, 6: 1001}             # 8 adapters, T = 1193


@pytest.mark.parametrize("kernel,k,ranks,d_in,d_out", [
    ("tensor", 1, (16, 8, 16, 32, 64, 16, 8), 512, 336),     # top-1, every rank slot up to 64
    ("tensor", 2, (16,) * 8, 512, 336),                       # k = 2: mixed tiles (4 adapters x 16)
    ("tensor", 2, (32, 24, 32, 16, 32, 32, 8, 32), 256, 144), # k = 2, rank slots of 32: set tiles
    ("bank", 1, (16, 8, 16, 16, 16, 16, 8), 512, 336),
    ("bank", 2, (16,) * 8, 512, 336),
    ("bank", 2, (32, 24, 32, 16, 32, 32, 8, 32), 256, 136),   # d_out with an 8-column last tile
    ("skinny", 1, (16, 8, 16, 32, 64, 16, 8), 512, 328),
    ("skinny", 2, (16, 8, 16, 32, 64, 16, 8, 16), 512, 328),
])
def test_sgmm_edge_segments_every_kernel(apr, kernel, k, ranks, d_in, d_out):
    """Empty adapters, a one-pair segment, 127/128/129-pair segments and segments of 1000-2001
    pairs through each gathered or bank kernel class, against the oracle."""
    rng = np.random.default_rng(40 + k + len(ranks) + d_out)
    E = len(ranks)
    idx = _seg_counts_idx(rng, _EDGE_K1 if k == 1 else _EDGE_K2, k)
    T = idx.shape[0]
    x, As, Bs, _, gate, ybs = _case(rng, T, d_in, (d_out,), ranks, k, dist=idx)
    x, As, Bs, ybs = _rounded(x, As, Bs, ybs)
    kern = {"tensor": apr.SGMM_TENSOR, "bank": apr.SGMM_BANK, "skinny": apr.SGMM_SKINNY}[kernel]
    seg, _, _ = run_segment(apr, idx, E)
    sizes = np.diff(seg)
    assert sizes[0] == 0 and sizes[E - 1] == 0 and {1, 127, 128, 129} <= set(sizes.tolist())
    for zero in (True, False):
        yb = [np.zeros_like(y) for y in ybs] if zero else ybs
        got = run_sgmm(apr, x, As, Bs, idx, gate, yb, BF16, kernel=kern)
        ref = oracle_group(x, As, Bs, idx, gate.astype(np.float64), yb)
        close(got[0], ref[0], f"{kernel} k={k} zero_ybase={zero}")


@pytest.mark.parametrize("T,k,counts", [
    (64, 1, {1: 1, 2: 60, 4: 3}),
    (33, 2, {1: 1, 3: 33, 4: 29, 6: 3}),
    (64, 2, {1: 1, 3: 64, 4: 60, 6: 3}),
])
def test_sgmm_dense_edge_segments(apr, T, k, counts):
    """The dense decode kernel with empty adapters, a one-pair segment and an adapter that
    every token selected (T <= 64)."""
    rng = np.random.default_rng(50 + T + k)
    ranks = (16, 8, 16, 16, 8, 16, 16, 16)
    idx = _seg_counts_idx(rng, counts, k)
    assert idx.shape == (T, k)
    x, As, Bs, _, gate, ybs = _case(rng, T, 4096, (4096, 264), ranks, k, dist=idx)
    x, As, Bs, ybs = _rounded(x, As, Bs, ybs)
    for zero in (True, False):
        yb = [np.zeros_like(y) for y in ybs] if zero else ybs
        got = run_sgmm(apr, x, As, Bs, idx, gate, yb, BF16, kernel=apr.SGMM_DENSE)
        ref = oracle_group(x, As, Bs, idx, gate.astype(np.float64), yb)
        for p in range(2):
            close(got[p], ref[p], f"dense T={T} k={k} proj {p} zero_ybase={zero}")


# ------------------------------------------------------------------ SGMM, bank (token-order) kernel


@pytest.mark.parametrize("T,d_in,d_outs,ranks,k,zipf", [
    (517, 4096, (4096,), (16,) * 16, 2, True),              # prefill-shaped projection, ragged last row tile
    (1000, 1024, (512, 1008), (16,) * 6, 2, True),          # two projections, ragged d_out
    (129, 192 * 2, (64, 64, 64, 64), (32,) * 3, 2, False),  # four projections, rank slots of 32
    (300, 256, (136,), (8, 16, 8, 16), 4, False),           # k = 4, an 8-wide last column tile
    (700, 256, (128,), (40, 64, 56, 48), 1, False),         # rank slots of 64, k = 1
    (65, 512, (256,), (16,) * 16, 3, False),                # one token past a tile, k = 3
    (1, 128, (16,), (16, 16), 2, False),                    # one token
    (8192, 512, (128,), (16,) * 16, 2, True),               # 64 full row tiles
])
def test_sgmm_bank_parity(apr, T, d_in, d_outs, ranks, k, zipf):
    rng = np.random.default_rng(T + d_in + k + 11)
    idx = _zipf_idx(rng, T, len(ranks), k) if zipf else "uniform"
    x, As, Bs, idx, gate, ybs = _case(rng, T, d_in, d_outs, ranks, k, dist=idx)
    x, As, Bs, ybs = _rounded(x, As, Bs, ybs)
    for zero in (True, False):
        yb = [np.zeros_like(y) for y in ybs] if zero else ybs
        got = run_sgmm(apr, x, As, Bs, idx, gate, yb, BF16, kernel=apr.SGMM_BANK)
        ref = oracle_group(x, As, Bs, idx, gate.astype(np.float64), yb)
        for p in range(len(d_outs)):
            close(got[p], ref[p], f"bank proj {p} zero_ybase={zero}")


def test_sgmm_bank_integer_inputs_exact(apr):
    """Small integers, gates of 1/2: the bank result is the exact value rounded once to bf16
    (pins the rank-slot placement of V, the Bcat layout and the row/column tiling)."""
    rng = np.random.default_rng(61)
    x, As, Bs, idx, gate, ybs = _case(rng, 400, 512, (128, 264), (16, 8, 16, 16, 8), 2, ints=True)
    got = run_sgmm(apr, x, As, Bs, idx, gate, ybs, BF16, kernel=apr.SGMM_BANK)
    ref = oracle_group(x, As, Bs, idx, gate.astype(np.float64), ybs)
    for p in range(2):
        want = bf16_exact(ref[p]).astype(np.float64)
        assert np.array_equal(got[p], want), f"proj {p}: max diff {np.abs(got[p] - want).max()}"


def test_sgmm_bank_properties(apr):
    """Zero B leaves y_base bit-exact; in place equals out of place; a token permutation
    permutes the output bits; two runs agree; AUTO takes the bank kernel here."""
    rng = np.random.default_rng(62)
    idx = _zipf_idx(rng, 900, 6, 2)
    x, As, Bs, idx, gate, ybs = _case(rng, 900, 512, (1008, 80), (16,) * 6, 2, dist=idx)
    x, As, Bs, ybs = _rounded(x, As, Bs, ybs)
    Bz = [[np.zeros_like(b) for b in P] for P in Bs]
    z = run_sgmm(apr, x, As, Bz, idx, gate, ybs, BF16, kernel=apr.SGMM_BANK)
    for p in range(2):
        assert np.array_equal(z[p], ybs[p].astype(np.float64))
    a = run_sgmm(apr, x, As, Bs, idx, gate, ybs, BF16, kernel=apr.SGMM_BANK, in_place=True)
    b = run_sgmm(apr, x, As, Bs, idx, gate, ybs, BF16, kernel=apr.SGMM_BANK)
    c = run_sgmm(apr, x, As, Bs, idx, gate, ybs, BF16)
    for p in range(2):
        assert np.array_equal(a[p], b[p]) and np.array_equal(b[p], c[p])
    perm = rng.permutation(900)
    d = run_sgmm(apr, x[perm], As, Bs, idx[perm], gate[perm], [y[perm] for y in ybs], BF16, kernel=apr.SGMM_BANK)
    for p in range(2):
        assert np.array_equal(d[p], b[p][perm])


def test_sgmm_bank_faults_and_limits(apr):
    rng = np.random.default_rng(63)
    x, As, Bs, idx, gate, ybs = _case(rng, 200, 256, (128,), (16, 16, 32), 2)
    x, As, Bs, ybs = _rounded(x, As, Bs, ybs)
    with pytest.raises(apr.AprError) as ei:                   # a rank above max_rank, caught on the device
        run_sgmm(apr, x, As, Bs, idx, gate, ybs, BF16, kernel=apr.SGMM_BANK, max_rank=16)
    assert ei.value.status == apr.APR_ERR_DEVICE_INDEX
    ok = run_sgmm(apr, x, As, Bs, idx, gate, ybs, BF16, kernel=apr.SGMM_BANK)
    close(ok[0], oracle_group(x, As, Bs, idx, gate.astype(np.float64), ybs)[0], "bank after fault")
    x2, As2, Bs2, idx2, gate2, ybs2 = _case(rng, 100, 256, (128,), (16,) * 17, 2)   # E * 16 > 256
    x2, As2, Bs2, ybs2 = _rounded(x2, As2, Bs2, ybs2)
    with pytest.raises(apr.AprError) as ei:
        run_sgmm(apr, x2, As2, Bs2, idx2, gate2, ybs2, BF16, kernel=apr.SGMM_BANK)
    assert ei.value.status == apr.APR_ERR_UNSUPPORTED


def test_kernels_on_a_second_device(apr):
    """Kernel attributes are per device: every SGMM kernel class and the merge run on device 1
    after device 0 has set them up (skipped with fewer than two visible GPUs)."""
    if torch.cuda.device_count() < 2:
        pytest.skip("needs two visible GPUs")
    rng = np.random.default_rng(64)
    x, As, Bs, idx, gate, ybs = _case(rng, 300, 512, (256,), (16,) * 6, 2)
    x, As, Bs, ybs = _rounded(x, As, Bs, ybs)
    ref = oracle_group(x, As, Bs, idx, gate.astype(np.float64), ybs)
    for dev_i in (0, 1):
        with torch.cuda.device(dev_i):
            for kern in (apr.SGMM_SKINNY, apr.SGMM_TENSOR, apr.SGMM_BANK):
                close(run_sgmm(apr, x, As, Bs, idx, gate, ybs, BF16, kernel=kern)[0], ref[0], f"device {dev_i}")
            xs, As_d, Bs_d = x[:40], As, Bs
            close(run_sgmm(apr, xs, As_d, Bs_d, idx[:40], gate[:40], [ybs[0][:40]], BF16, kernel=apr.SGMM_DENSE)[0],
                  oracle_group(xs, As_d, Bs_d, idx[:40], gate[:40].astype(np.float64), [ybs[0][:40]])[0], "dense")


def test_sgmm_bank_every_row_and_rerun_bits(apr):
    """A prefill-shaped q/k/v group (8192 tokens, 16 adapters of rank 16, Zipf top-2) on the bank
    kernel: every output row against the oracle, and three runs equal bit for bit.  Each CTA's
    range of units crosses column blocks here, so a column block's Bcat is reloaded in the middle
    of a CTA's work and the first unit after it reads it at once (a reload that is not complete
    when the MMAs read it shows as wrong rows of the first row tile, differing from run to run)."""
    rng = np.random.default_rng(95)
    T, d_in, d_outs, ranks, k = 8192, 4096, (4096, 4096, 4096), (16,) * 16, 2
    idx = _zipf_idx(rng, T, len(ranks), k)
    x, As, Bs, idx, gate, ybs = _case(rng, T, d_in, d_outs, ranks, k, dist=idx)
    x, As, Bs, ybs = _rounded(x, As, Bs, ybs)
    runs = [run_sgmm(apr, x, As, Bs, idx, gate, ybs, BF16, kernel=apr.SGMM_BANK) for _ in range(3)]
    for r in runs[1:]:
        for p in range(3):
            assert np.array_equal(r[p], runs[0][p]), f"proj {p}: runs differ"
    ref = oracle_group(x, As, Bs, idx, gate.astype(np.float64), ybs)
    for p in range(3):
        close(runs[0][p], ref[p], f"bank proj {p} all rows")
