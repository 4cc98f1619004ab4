"""Seeded synthetic inputs for the pre-gated mixture-of-LoRA path.

This module only draws inputs: it holds none of the method's arithmetic (no
router product, no top-k, no sort, no low-rank product).  Both the fp64 CPU
oracle and the CUDA library are fed from here, so the two sides see the same
bits.  It imports numpy only; ``device_tensor`` imports torch lazily to copy a
window of a pool to the GPU.

Workload shapes follow the AdaFuse summary (gist.science, "Resumen técnico"
§4: Llama2-7B / Mistral-7B backbones) and the five named configurations:

* ``tiny``        4 layers x one 256->256 projection, 8 adapters of rank 8,
                  top-2, 64 tokens, fp32, free (unforced) routing.
* ``decode``      Llama-2-7B layer set (q,k,v,o 4096->4096; gate,up
                  4096->11008; down 11008->4096) x 32 layers, 8 adapters of
                  rank 16, top-2, 32 tokens, uniform adapter choice, bf16.
* ``prefill``     same layers, 16 adapters of rank 16, top-2, 8192 tokens,
                  Zipf(s=1.1) adapter popularity, bf16.
* ``multitenant`` 32 layers x {q, v} 4096->4096, 256 adapters with ranks drawn
                  from {8,16,32,64}, top-1, 4096 tokens uniform, bf16.
* ``merge``       batch-1: the decode layer set, one token, its top-2
                  adapters merged into the base weights, then one GEMV per
                  projection, bf16 W ~ N(0, 0.02).

Value recipe
------------
Activations and adapter weights are windows of a few large seeded pools
(``numpy.random.Generator(PCG64)``): a tensor named ``key`` of ``n`` elements is
``pool[(off(key) + arange(n)) mod P]`` with ``off`` a hash of the key.  The
pools are N(0,1) (x, y_base) and N(0,0.02) (A, B, W), rounded once to bf16 with
round-to-nearest-even for the bf16 configurations, plain fp32 for ``tiny``.
Windows keep full-size workloads (tens of GB) cheap to build on the device
while the oracle can rebuild any row on the host bit for bit.

Router inputs are small integers scaled by powers of two so that every router
logit is exact in fp32.  For the forced configurations each token's ordered
adapter tuple is drawn first (uniform or Zipf, without replacement) and the
router weight ``Wr`` and hidden ``h`` are built so that this tuple is the
unique top-k with a strict margin (no ties); ``tiny`` draws free random
integers, so ties do occur there.
"""
from __future__ import annotations

import hashlib
from dataclasses import dataclass, field

import numpy as np

# --------------------------------------------------------------------------
# configurations
# --------------------------------------------------------------------------


@dataclass(frozen=True)
class Group:
    """Projections that read the same input activation x (one SGMM call)."""

    name: str
    d_in: int
    proj_names: tuple
    d_outs: tuple


LLAMA7B_GROUPS = (
    Group("qkv", 4096, ("q", "k", "v"), (4096, 4096, 4096)),
    Group("o", 4096, ("o",), (4096,)),
    Group("gate_up", 4096, ("gate", "up"), (11008, 11008)),
    Group("down", 11008, ("down",), (4096,)),
)


@dataclass(frozen=True)
class Config:
    name: str
    T: int                      # tokens per step
    E: int                      # adapters
    k: int                      # adapters per token
    d_router: int               # router input width
    layers: int
    groups: tuple
    rank_choices: tuple         # one rank for all, or the set ranks are drawn from
    popularity: str             # "free" | "uniform" | "zipf"
    zipf_s: float = 1.1
    dtype: str = "bf16"         # "bf16" | "f32"
    merge: bool = False
    seed: int = 0
    notes: str = field(default="", compare=False)

    @property
    def nproj(self) -> int:
        return self.layers * sum(len(g.proj_names) for g in self.groups)


CONFIGS = {
    "tiny": Config(
        "tiny", T=64, E=8, k=2, d_router=256, layers=4,
        groups=(Group("p", 256, ("p",), (256,)),),
        rank_choices=(8,), popularity="free", dtype="f32"),
    "decode": Config(
        "decode", T=32, E=8, k=2, d_router=4096, layers=32,
        groups=LLAMA7B_GROUPS, rank_choices=(16,), popularity="uniform"),
    "prefill": Config(
        "prefill", T=8192, E=16, k=2, d_router=4096, layers=32,
        groups=LLAMA7B_GROUPS, rank_choices=(16,), popularity="zipf", zipf_s=1.1),
    "multitenant": Config(
        "multitenant", T=4096, E=256, k=1, d_router=4096, layers=32,
        groups=(Group("qv", 4096, ("q", "v"), (4096, 4096)),),
        rank_choices=(8, 16, 32, 64), popularity="uniform"),
    "merge": Config(
        "merge", T=1, E=8, k=2, d_router=4096, layers=32,
        groups=LLAMA7B_GROUPS, rank_choices=(16,), popularity="uniform", merge=True),
}


def scaled(cfg: Config, **kw) -> Config:
    """A copy of ``cfg`` with fields replaced (smaller test cases)."""
    d = dict(cfg.__dict__)
    d.update(kw)
    return Config(**d)


def ranks(cfg: Config) -> np.ndarray:
    """Per-adapter LoRA rank (int32 [E]); drawn per adapter when several are allowed."""
    if len(cfg.rank_choices) == 1:
        return np.full(cfg.E, cfg.rank_choices[0], dtype=np.int32)
    rng = np.random.Generator(np.random.PCG64([cfg.seed, 0x52414E4B]))
    return rng.choice(np.asarray(cfg.rank_choices, dtype=np.int32), size=cfg.E).astype(np.int32)


# --------------------------------------------------------------------------
# bf16 helpers (input preparation only)
# --------------------------------------------------------------------------


def round_to_bf16(a: np.ndarray) -> np.ndarray:
    """fp32 -> nearest bf16 value (ties to even), returned as fp32.  Inputs are finite."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    r = (u + np.uint32(0x7FFF) + lsb) & np.uint32(0xFFFF0000)
    return r.view(np.float32)


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """Bit pattern (uint16) of fp32 values that are already exact bf16 values."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    return (a.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


# --------------------------------------------------------------------------
# value pools and windows
# --------------------------------------------------------------------------

POOL_LEN = (1 << 25) + 43      # ~33.5M values; odd so windows do not align to rows
POOL_LEN_F32 = (1 << 20) + 7   # fp32 pools serve only the small fp32 configuration
_POOL_SIGMA = {"unit": 1.0, "small": 0.02}
_pool_cache: dict = {}


def _pool(kind: str, dtype: str, seed: int) -> np.ndarray:
    key = (kind, dtype, seed)
    if key not in _pool_cache:
        n = POOL_LEN if dtype == "bf16" else POOL_LEN_F32
        tag = 0x504F4F4C + (0 if kind == "unit" else 1) + (0 if dtype == "bf16" else 2)
        rng = np.random.Generator(np.random.PCG64([seed, tag]))
        v = rng.standard_normal(n, dtype=np.float32) * np.float32(_POOL_SIGMA[kind])
        if dtype == "bf16":
            v = round_to_bf16(v)
        _pool_cache[key] = v
    return _pool_cache[key]


def _offset(key: str, seed: int, plen: int) -> int:
    h = hashlib.blake2b(f"{seed}/{key}".encode(), digest_size=8).digest()
    return int.from_bytes(h, "little") % plen


def kind_of(key: str) -> str:
    """Pool a named tensor is drawn from: weights are N(0,0.02), activations N(0,1)."""
    return "small" if key.split("/")[0] in ("A", "B", "W") else "unit"


def host_tensor(cfg: Config, key: str, shape) -> np.ndarray:
    """The named tensor as fp32 numpy (values exact in the config's dtype)."""
    shape = tuple(int(s) for s in shape)
    n = int(np.prod(shape)) if shape else 1
    pool = _pool(kind_of(key), cfg.dtype, cfg.seed)
    off = _offset(key, cfg.seed, pool.size)
    idx = (off + np.arange(n, dtype=np.int64)) % pool.size
    return pool[idx].reshape(shape)


def host_rows(cfg: Config, key: str, shape, rows) -> np.ndarray:
    """Selected rows of a 2-D named tensor (same values as ``host_tensor``)."""
    R, C = (int(shape[0]), int(shape[1]))
    rows = np.asarray(rows, dtype=np.int64)
    pool = _pool(kind_of(key), cfg.dtype, cfg.seed)
    off = _offset(key, cfg.seed, pool.size)
    idx = (off + rows[:, None] * C + np.arange(C, dtype=np.int64)[None, :]) % pool.size
    return pool[idx]


_dev_pool_cache: dict = {}


def device_tensor(cfg: Config, key: str, shape, device="cuda"):
    """The named tensor materialised on ``device`` as a torch tensor of the config dtype.

    Built by copying slices of the pool already resident on the device, so it
    holds exactly the values of ``host_tensor``.
    """
    import torch

    shape = tuple(int(s) for s in shape)
    n = int(np.prod(shape)) if shape else 1
    tdt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    pk = (kind_of(key), cfg.dtype, cfg.seed, str(device))
    if pk not in _dev_pool_cache:
        host = _pool(kind_of(key), cfg.dtype, cfg.seed)
        _dev_pool_cache[pk] = torch.from_numpy(host).to(device=device).to(tdt)
    pool = _dev_pool_cache[pk]
    P = pool.numel()
    off = _offset(key, cfg.seed, P)
    out = torch.empty(n, dtype=tdt, device=device)
    pos = 0
    src = off
    while pos < n:
        take = min(n - pos, P - src)
        out[pos:pos + take].copy_(pool[src:src + take])
        pos += take
        src = 0
    return out.view(shape)


def clear_device_pools():
    _dev_pool_cache.clear()


# --------------------------------------------------------------------------
# router inputs
# --------------------------------------------------------------------------

# Real values are integers times these powers of two; logits are integers * 2^-(H+W).
H_SHIFT = 2
W_SHIFT = 3
FREE_SHIFT = 2


def popularity(cfg: Config) -> np.ndarray:
    if cfg.popularity == "zipf":
        p = 1.0 / np.arange(1, cfg.E + 1, dtype=np.float64) ** cfg.zipf_s
    else:
        p = np.ones(cfg.E, dtype=np.float64)
    return p / p.sum()


def forced_adapter_tuples(cfg: Config, T: int | None = None, seed_offset: int = 0) -> np.ndarray:
    """Each token's ordered adapter tuple [T, k], drawn without replacement.

    Successive draws without replacement from the popularity distribution
    (Gumbel keys: ``log p + Gumbel`` ranked, which is the sequential draw).
    """
    T = cfg.T if T is None else T
    rng = np.random.Generator(np.random.PCG64([cfg.seed, 0x53455453, seed_offset]))
    keys = np.log(popularity(cfg))[None, :] + rng.gumbel(size=(T, cfg.E))
    order = np.argsort(-keys, axis=1, kind="stable")
    return order[:, :cfg.k].astype(np.int32)


def router_inputs(cfg: Config, T: int | None = None, seed_offset: int = 0):
    """(h [T, d], Wr [E, d], tuples or None) as fp32 arrays of exact values.

    Forced configurations: columns < E of ``Wr`` are 4*identity, the other
    columns share a common integer row ``c`` plus +-1 in four random columns
    per adapter; ``h`` carries the forced ranking in its first E columns with
    steps of >= 5 integer units between consecutive ranks and small integers
    elsewhere.  The adapter-specific part of a logit then moves it by at most
    8 units while the forced steps are >= 20 units, so the drawn tuple is the
    strict top-k.
    """
    T = cfg.T if T is None else T
    E, d, k = cfg.E, cfg.d_router, cfg.k
    rng = np.random.Generator(np.random.PCG64([cfg.seed, 0x524F5554, seed_offset]))
    if cfg.popularity == "free":
        h_int = rng.integers(-3, 4, size=(T, d))
        w_int = rng.integers(-3, 4, size=(E, d))
        s = np.float32(2.0 ** -FREE_SHIFT)
        return (h_int.astype(np.float32) * s, w_int.astype(np.float32) * s, None)
    assert E <= d, "forced routing needs E <= d_router"
    tuples = forced_adapter_tuples(cfg, T, seed_offset)
    w_int = np.zeros((E, d), dtype=np.int64)
    w_int[np.arange(E), np.arange(E)] = 4
    common = rng.integers(-2, 3, size=d - E)
    w_int[:, E:] = common[None, :]
    for e in range(E):
        cols = E + rng.choice(d - E, size=4, replace=False)
        w_int[e, cols] += rng.choice(np.array([-1, 1]), size=4)
    h_int = np.zeros((T, d), dtype=np.int64)
    h_int[:, E:] = rng.integers(-2, 3, size=(T, d - E))
    top = 50 + rng.integers(0, 11, size=T)
    level = top.copy()
    for j in range(k):
        h_int[np.arange(T), tuples[:, j]] = level
        if j + 1 < k:
            level = level - rng.integers(5, 11, size=T)
    # every adapter not in the tuple sits at least 5 units under the last one
    sel = np.zeros((T, E), dtype=bool)
    sel[np.arange(T)[:, None], tuples] = True
    low = rng.integers(0, 1 << 30, size=(T, E))
    span = np.maximum(level - 5, 0) + 1
    rest = low % span[:, None]
    h_first = h_int[:, :E]
    h_first[~sel] = rest[~sel]
    h_int[:, :E] = h_first
    h = h_int.astype(np.float32) * np.float32(2.0 ** -H_SHIFT)
    Wr = w_int.astype(np.float32) * np.float32(2.0 ** -W_SHIFT)
    return h, Wr, tuples


# --------------------------------------------------------------------------
# tensor names for one step
# --------------------------------------------------------------------------


def x_key(l, g):
    return f"x/{l}/{g}"


def ybase_key(l, g, p):
    return f"ybase/{l}/{g}/{p}"


def a_key(l, g, p, e):
    return f"A/{l}/{g}/{p}/{e}"


def b_key(l, g, p, e):
    return f"B/{l}/{g}/{p}/{e}"


def w_key(l, g, p):
    return f"W/{l}/{g}/{p}"


def xm_key(l, g, p):
    return f"xm/{l}/{g}/{p}"
