"""Base projection and adapters in one contraction (``apr_linear_lora``) against the fp64
oracle: y = x W^T + sum_j g B_e (A_e x), through the C ABI."""
import numpy as np
import pytest
import torch

from oracle import apr_oracle as O
from apr_testlib import bf16_exact, check_guards, close, dev, guarded, to_np

pytestmark = pytest.mark.gpu
BF16 = torch.bfloat16


@pytest.fixture(scope="module")
def apr():
    from adapter_pregate_router_b200 import build
    build.build()
    from adapter_pregate_router_b200 import apr as mod
    assert torch.cuda.is_available()
    return mod


def _zipf_idx(rng, T, E, k, s=1.1):
    p = 1.0 / np.arange(1, E + 1) ** s
    p /= p.sum()
    return np.stack([rng.choice(E, size=k, replace=False, p=p) for _ in range(T)]).astype(np.int32)


def _case(rng, T, d_in, d_outs, ranks, k, zipf=False, ints=False):
    E = len(ranks)
    idx = _zipf_idx(rng, T, E, k) if zipf else \
        np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    if ints:
        x = rng.integers(-1, 2, size=(T, d_in)).astype(np.float32)
        Ws = [rng.integers(-1, 2, size=(d, d_in)).astype(np.float32) for d in d_outs]
        As = [[rng.integers(-1, 2, size=(r, d_in)).astype(np.float32) for r in ranks] for _ in d_outs]
        Bs = [[rng.integers(-1, 2, size=(d, r)).astype(np.float32) for r in ranks] for d in d_outs]
        gate = np.full((T, k), 1.0 / k, np.float32)
        return x, Ws, As, Bs, idx, gate
    x = bf16_exact(rng.normal(size=(T, d_in)))
    Ws = [bf16_exact(0.02 * rng.normal(size=(d, d_in))) for d in d_outs]
    As = [[bf16_exact(0.02 * rng.normal(size=(r, d_in))) for r in ranks] for _ in d_outs]
    Bs = [[bf16_exact(0.02 * rng.normal(size=(d, r))) for r in ranks] for d in d_outs]
    gate = rng.dirichlet(np.ones(k), size=T).astype(np.float32)
    return x, Ws, As, Bs, idx, gate


def run_linear(apr, x, Ws, As, Bs, idx_np, gate_np, ranks=None, max_rank=None, ws_bytes=None):
    """One shared-input group through apr_linear_lora; outputs inside guard bands, W and x
    checked unchanged afterwards.  Returns the outputs (fp64)."""
    T, d_in = x.shape
    k = idx_np.shape[1]
    E = len(As[0])
    if ranks is None:
        ranks = np.array([a.shape[0] for a in As[0]], dtype=np.int32)
    if max_rank is None:
        max_rank = int(max(ranks.max(), 8) + 7) // 8 * 8
    sum_d_out = sum(w.shape[0] for w in Ws)
    ws = apr.linear_workspace(max(T, 1), k, E, max_rank, d_in, len(Ws), sum_d_out)
    if ws_bytes is not None:
        ws = ws[:ws_bytes]
    idx = torch.from_numpy(np.ascontiguousarray(idx_np, dtype=np.int32)).cuda()
    gate = torch.from_numpy(np.ascontiguousarray(gate_np, dtype=np.float32)).cuda()
    seg_off = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(max(T * k, 1), dtype=torch.int32, device="cuda")
    apr.segment_tokens(idx, E, seg_off, perm, ws)
    xd = dev(x, BF16)
    x_before = xd.clone()
    keep, projs, ys, bands, weights = [], [], [], [], []
    for p in range(len(Ws)):
        Wd = dev(Ws[p], BF16)
        A = [dev(a, BF16) for a in As[p]]
        B = [dev(b, BF16) for b in Bs[p]]
        At, Bt = apr.ptr_array(A), apr.ptr_array(B)
        ybuf, y = guarded(np.full((T, Ws[p].shape[0]), np.nan, np.float32), BF16)
        bands.append((ybuf, f"y {p}"))
        weights.append((Wd, Wd.clone(), p))
        keep += [A, B, At, Bt]
        projs.append(apr.make_linear_proj(Wd, y, At, Bt))
        ys.append(y)
    rk = torch.from_numpy(np.ascontiguousarray(ranks, dtype=np.int32)).cuda()
    apr.linear_lora(xd, projs, k, E, rk, max_rank, idx, gate, seg_off, perm, ws)
    apr.stream_status(ws)
    for buf, what in bands:
        check_guards(buf, what)
    for Wd, before, p in weights:
        assert torch.equal(Wd, before), f"W {p} written"
    assert torch.equal(xd, x_before), "x written"
    return [to_np(y) for y in ys]


def oracle_linear(x, Ws, As, Bs, idx, gate):
    return [O.linear_lora(x, Ws[p], As[p], Bs[p], idx, gate.astype(np.float64)) for p in range(len(Ws))]


@pytest.mark.parametrize("T,d_in,d_outs,ranks,k,zipf", [
    (300, 512, (256,), (16,) * 4, 2, False),                # partial row tile, one column tile
    (1000, 1024, (512, 1008), (16,) * 6, 2, True),          # two projections, last column tile 240 wide
    (700, 256, (128,), (8, 16, 32, 64), 1, False),          # top-1, rank slots of 64, ranks below the slot
    (517, 4096, (4096,), (16,) * 16, 2, True),              # prefill-shaped projection, 256 bank rows
    (129, 192, (64, 64, 64, 64), (32,) * 3, 2, False),      # four projections, bank of 96 rows (a partial K block)
    (1, 128, (16,), (16, 16), 2, False),                    # one token, one narrow column tile
    (65, 512, (264,), (16,) * 8, 4, False),                 # k = 4, a column tile 8 wide
    (8192, 512, (264,), (16,) * 16, 2, True),               # 64 full row tiles
])
def test_linear_lora_parity(apr, T, d_in, d_outs, ranks, k, zipf):
    rng = np.random.default_rng(T + d_in + k + 71)
    x, Ws, As, Bs, idx, gate = _case(rng, T, d_in, d_outs, ranks, k, zipf)
    got = run_linear(apr, x, Ws, As, Bs, idx, gate)
    ref = oracle_linear(x, Ws, As, Bs, idx, gate)
    for p in range(len(d_outs)):
        close(got[p], ref[p], f"fused proj {p}")
    # the adapter term alone (W = 0) and the base alone (B = 0): neither part may be dropped
    Wz = [np.zeros_like(w) for w in Ws]
    got = run_linear(apr, x, Wz, As, Bs, idx, gate)
    ref = oracle_linear(x, Wz, As, Bs, idx, gate)
    for p in range(len(d_outs)):
        close(got[p], ref[p], f"adapter term of proj {p}")
    Bz = [[np.zeros_like(b) for b in P] for P in Bs]
    got = run_linear(apr, x, Ws, As, Bz, idx, gate)
    for p in range(len(d_outs)):
        close(got[p], x.astype(np.float64) @ Ws[p].astype(np.float64).T, f"base of proj {p}")


def test_linear_lora_integer_inputs_exact(apr):
    """Small integers, gates of 1/2: both terms are exact in fp32, so the result is the exact
    value rounded once to bf16 (pins the K order of x/W and V/Bcat blocks, the bank slots and
    the tile edges)."""
    rng = np.random.default_rng(81)
    x, Ws, As, Bs, idx, gate = _case(rng, 400, 512, (128, 264), (16, 8, 16, 16, 8), 2, ints=True)
    got = run_linear(apr, x, Ws, As, Bs, idx, gate)
    ref = oracle_linear(x, Ws, As, Bs, idx, gate)
    for p in range(2):
        want = bf16_exact(ref[p]).astype(np.float64)
        assert np.array_equal(got[p], want), f"proj {p}: max diff {np.abs(got[p] - want).max()}"


def test_linear_lora_properties(apr):
    """Two runs agree bit for bit; a token permutation permutes the output bits; gates scaled by
    zero give the base product bit for bit."""
    rng = np.random.default_rng(82)
    x, Ws, As, Bs, idx, gate = _case(rng, 900, 512, (1008, 80), (16,) * 6, 2, zipf=True)
    a = run_linear(apr, x, Ws, As, Bs, idx, gate)
    b = run_linear(apr, x, Ws, As, Bs, idx, gate)
    for p in range(2):
        assert np.array_equal(a[p], b[p])
    perm = rng.permutation(900)
    c = run_linear(apr, x[perm], Ws, As, Bs, idx[perm], gate[perm])
    for p in range(2):
        assert np.array_equal(c[p], a[p][perm])
    Bz = [[np.zeros_like(bb) for bb in P] for P in Bs]
    z = run_linear(apr, x, Ws, As, Bz, idx, gate)
    g0 = run_linear(apr, x, Ws, As, Bs, idx, np.zeros_like(gate))
    for p in range(2):
        assert np.array_equal(z[p], g0[p])


def test_linear_lora_limits_and_faults(apr):
    rng = np.random.default_rng(83)
    x, Ws, As, Bs, idx, gate = _case(rng, 200, 256, (128,), (16, 16, 32), 2)
    with pytest.raises(apr.AprError) as ei:                   # a rank above max_rank, caught on the device
        run_linear(apr, x, Ws, As, Bs, idx, gate, max_rank=16)
    assert ei.value.status == apr.APR_ERR_DEVICE_INDEX
    ok = run_linear(apr, x, Ws, As, Bs, idx, gate)
    close(ok[0], oracle_linear(x, Ws, As, Bs, idx, gate)[0], "fused after fault")
    x2, Ws2, As2, Bs2, idx2, gate2 = _case(rng, 100, 256, (128,), (16,) * 17, 2)   # E * 16 > 256
    with pytest.raises(apr.AprError) as ei:
        run_linear(apr, x2, Ws2, As2, Bs2, idx2, gate2)
    assert ei.value.status == apr.APR_ERR_UNSUPPORTED
    x3, Ws3, As3, Bs3, idx3, gate3 = _case(rng, 100, 200, (128,), (16,) * 4, 2)     # d_in % 64 != 0
    with pytest.raises(apr.AprError) as ei:
        run_linear(apr, x3, Ws3, As3, Bs3, idx3, gate3)
    assert ei.value.status == apr.APR_ERR_UNSUPPORTED
    with pytest.raises(apr.AprError) as ei:                   # workspace too small
        run_linear(apr, x, Ws, As, Bs, idx, gate, ws_bytes=4096)
    assert ei.value.status == apr.APR_ERR_WORKSPACE


def test_linear_lora_full_size_sampled_rows(apr):
    """A prefill gate/up group at full size (8192 tokens, 4096 -> 2 x 11008, 16 adapters of
    rank 16, top-2 Zipf routing), checked on sampled token rows in fp64 (rows are independent)."""
    rng = np.random.default_rng(84)
    T, d_in, d_outs, E, k = 8192, 4096, (11008, 11008), 16, 2
    idx = _zipf_idx(rng, T, E, k)
    gate = rng.dirichlet(np.ones(k), size=T).astype(np.float32)
    x = bf16_exact(rng.normal(size=(T, d_in)))
    Ws = [bf16_exact(0.02 * rng.standard_normal(size=(d, d_in), dtype=np.float32)) for d in d_outs]
    As = [[bf16_exact(0.02 * rng.normal(size=(16, d_in))) for _ in range(E)] for _ in d_outs]
    Bs = [[bf16_exact(0.02 * rng.normal(size=(d, 16))) for _ in range(E)] for d in d_outs]
    got = run_linear(apr, x, Ws, As, Bs, idx, gate)
    rows = np.concatenate([[0, 127, 128, T - 1], rng.choice(T, size=12, replace=False)])
    for p in range(2):
        ref = O.linear_lora(x[rows], Ws[p], As[p], Bs[p], idx[rows], gate[rows].astype(np.float64))
        close(got[p][rows], ref, f"full-size proj {p}")
