"""The shared input generator: determinism, exact bf16 values, host/device agreement (CPU)."""
import numpy as np
import torch

from adapter_pregate_router_b200 import workloads as W


def test_round_to_bf16_matches_torch():
    rng = np.random.default_rng(0)
    a = np.concatenate([rng.normal(size=10000).astype(np.float32) * 10,
                        np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -(1.0 + 2 ** -8), 0.0, -0.0], np.float32)])
    ours = W.round_to_bf16(a)
    ref = torch.from_numpy(a).to(torch.bfloat16).to(torch.float32).numpy()
    assert np.array_equal(ours.view(np.uint32), ref.view(np.uint32))


def test_windows_are_deterministic_and_rows_agree():
    cfg = W.CONFIGS["decode"]
    a = W.host_tensor(cfg, "x/3/qkv", (32, 4096))
    b = W.host_tensor(cfg, "x/3/qkv", (32, 4096))
    assert np.array_equal(a, b)
    rows = [0, 5, 31]
    assert np.array_equal(W.host_rows(cfg, "x/3/qkv", (32, 4096), rows), a[rows])
    assert not np.array_equal(a, W.host_tensor(cfg, "x/4/qkv", (32, 4096)))
    # exact bf16 values
    assert np.array_equal(W.round_to_bf16(a), a)


def test_device_tensor_matches_host_on_cpu():
    cfg = W.scaled(W.CONFIGS["decode"], seed=3)
    n = W.POOL_LEN + 12345          # wraps around the pool
    host = W.host_tensor(cfg, "B/0/o/o/1", (n,))
    dev = W.device_tensor(cfg, "B/0/o/o/1", (n,), device="cpu")
    assert dev.dtype == torch.bfloat16
    assert np.array_equal(dev.to(torch.float32).numpy(), host)
    W.clear_device_pools()


def test_pool_statistics():
    cfg = W.CONFIGS["decode"]
    x = W.host_tensor(cfg, "x/0/qkv", (1 << 20,))
    a = W.host_tensor(cfg, "A/0/qkv/q/0", (1 << 20,))
    assert abs(x.std() - 1.0) < 0.01 and abs(a.std() - 0.02) < 0.001


def test_ranks_and_popularity():
    r = W.ranks(W.CONFIGS["multitenant"])
    assert r.shape == (256,) and set(r.tolist()) <= {8, 16, 32, 64} and len(set(r.tolist())) == 4
    assert np.array_equal(r, W.ranks(W.CONFIGS["multitenant"]))
    p = W.popularity(W.CONFIGS["prefill"])
    assert np.all(np.diff(p) < 0) and abs(p.sum() - 1) < 1e-12
    t = W.forced_adapter_tuples(W.CONFIGS["prefill"])
    assert t.shape == (8192, 2) and np.all(t[:, 0] != t[:, 1])
    counts = np.bincount(t.ravel(), minlength=16)
    assert counts[0] > counts[5] > counts[15] > 0


def test_algorithmic_bytes_match_the_workload_budgets():
    """The bench's roofline numerator against the per-step budgets derived separately from the
    workload shapes (router excluded there): decode 861.4 MB, prefill 58.05 GB, merge 39.0 GB
    (26.06 merge + 12.96 GEMV); many tenants ~13.4 GB at the expected mean rank of 30, which the
    drawn ranks only approach (hence the looser bound)."""
    from adapter_pregate_router_b200 import pipeline as P

    def step_bytes(name):
        c = W.CONFIGS[name]
        b = P.algorithmic_bytes(c, range(c.layers), W.ranks(c), W.forced_adapter_tuples(c))
        el = 2 if c.dtype == "bf16" else 4
        return b - (c.T + c.E) * c.d_router * el

    assert abs(step_bytes("decode") - 861.4e6) < 0.05e6
    assert abs(step_bytes("prefill") - 58.05e9) < 0.005e9
    assert abs(step_bytes("merge") - 39.0e9) < 0.05e9
    assert abs(step_bytes("multitenant") / 13.42e9 - 1) < 0.03
    # an adapter nobody selected moves no bytes
    c = W.CONFIGS["decode"]
    idx_all = W.forced_adapter_tuples(c)
    idx_one = np.zeros_like(idx_all)
    full = P.algorithmic_bytes(c, [0], W.ranks(c), idx_all)
    one = P.algorithmic_bytes(c, [0], W.ranks(c), idx_one)
    per_adapter = sum(16 * (g.d_in + d) * 2 for g in c.groups for d in g.d_outs)
    assert full - one == 7 * per_adapter
