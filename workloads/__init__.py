"""Seeded synthetic inputs for the retention-scored KV eviction step.

This module only draws random numbers and lays them out; it holds none of the
method's arithmetic (no scores, ranking, attention or compaction).  The tests,
the bench and the smoke check feed the same tensors to the CUDA library and to
the CPU oracle.

Workloads follow the shapes the pages describe (8B-class models, 8K-128K
contexts, budgets of 256-2048 per head or 10 % retention, a VLM with vision and
text tokens).  No public benchmark items are used; these synthetic tensors
stand in for them:

* K, V ~ N(0, 1), rounded to bfloat16 (float32 for the tiny case).  In the
  "planted" workloads, 1 % of positions per head (Bernoulli(0.01)) get
  k += 3 * d, with d the unit direction of the sum of that head's step-0
  queries.
* queries ~ N(0, 1) float32, fresh for every step.
* log-retention lb = float32(log(u)), u drawn from a per-entry mixture of Beta
  distributions (plus a constant component), clamped to [1e-4, 1 - 1e-6].
* prefill state: head c = (b*L + l)*H + h owns pages [c*P0, (c+1)*P0),
  P0 = ceil(T0/16), slot k holds position k; the free stack lists the other
  pages so that pops return ascending ids.
"""
from __future__ import annotations

import math
import zlib
from dataclasses import dataclass, field, replace

import numpy as np
import torch

PAGE = 16
U_LO, U_HI = 1e-4, 1.0 - 1e-6

# A mixture component is ("beta", a, b) or ("const", u); weights sum to 1.
MIX_TINY = ((1.0, ("beta", 2.0, 2.0)),)
MIX_8B = ((0.70, ("beta", 2.0, 8.0)), (0.25, ("beta", 8.0, 2.0)), (0.05, ("const", 1.0 - 1e-4)))
MIX_LONG = ((0.80, ("beta", 2.0, 10.0)), (0.20, ("beta", 10.0, 1.5)))
MIX_VISION = ((1.0, ("beta", 1.5, 6.0)),)
MIX_TEXT = ((1.0, ("beta", 6.0, 2.0)),)


@dataclass(frozen=True)
class Config:
    name: str
    L: int
    H: int
    Hq: int
    D: int
    B: int
    T0: int
    M: int                      # global budget per sequence
    steps: int                  # decode steps of the workload
    evict_every: int = 1        # step s evicts iff s % evict_every == 0
    kv_dtype: str = "bf16"      # "bf16" | "f32"
    mix: tuple = MIX_8B         # retention mixture of prefill (and decode) tokens
    vision: int = 0             # positions [0, vision) draw from mix_vision
    mix_vision: tuple = ()
    mix_decode: tuple | None = None  # decode tokens (default: mix)
    planted: float = 0.0
    slack: int = 0              # entries a head may gain between evictions
    P: int = PAGE

    @property
    def G(self) -> int:
        return self.Hq // self.H

    @property
    def C(self) -> int:
        return self.B * self.L * self.H

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)

    def evicts(self, s: int) -> bool:
        return s % self.evict_every == 0


CONFIGS: dict[str, Config] = {
    "tiny": Config("tiny", L=2, H=4, Hq=4, D=64, B=1, T0=512, M=1024, steps=1,
                   kv_dtype="f32", mix=MIX_TINY),
    "llama32k": Config("llama32k", L=32, H=8, Hq=32, D=128, B=1, T0=32768, M=32 * 8 * 2048,
                       steps=256, planted=0.01),
    "qwen8k": Config("qwen8k", L=36, H=8, Hq=32, D=128, B=16, T0=8192, M=36 * 8 * 512,
                     steps=128, planted=0.01),
    "long128k": Config("long128k", L=32, H=8, Hq=32, D=128, B=1, T0=131072,
                       M=(32 * 8 * 131072) // 10, steps=64, mix=MIX_LONG, planted=0.01),
    "vlm16k": Config("vlm16k", L=28, H=4, Hq=28, D=128, B=8, T0=16384, M=28 * 4 * 512,
                     steps=1024, evict_every=16, mix=MIX_TEXT, vision=12288,
                     mix_vision=MIX_VISION, mix_decode=MIX_TEXT, slack=16),
}


def seed_for(seed: int, *keys) -> int:
    """Deterministic 63-bit seed for one named stream."""
    h = zlib.crc32(repr((seed,) + tuple(keys)).encode())
    h2 = zlib.crc32(repr(tuple(keys) + (seed, "x")).encode())
    return ((h << 31) ^ h2) & ((1 << 63) - 1)


def _gen(device, seed: int, *keys) -> torch.Generator:
    g = torch.Generator(device=torch.device(device))
    g.manual_seed(seed_for(seed, *keys))
    return g


def _gamma(alpha: float, n: int, gen: torch.Generator, device) -> torch.Tensor:
    """Gamma(alpha, 1) for alpha >= 1 by Marsaglia-Tsang rejection (float64)."""
    assert alpha >= 1.0
    d = alpha - 1.0 / 3.0
    c = 1.0 / math.sqrt(9.0 * d)
    out = torch.empty(n, dtype=torch.float64, device=device)
    todo = torch.arange(n, device=device)
    while todo.numel() > 0:
        m = todo.numel()
        x = torch.randn(m, generator=gen, dtype=torch.float64, device=device)
        u = torch.rand(m, generator=gen, dtype=torch.float64, device=device)
        v = (1.0 + c * x) ** 3
        ok = (v > 0) & (torch.log(u) < 0.5 * x * x + d - d * v + d * torch.log(v.clamp_min(1e-300)))
        out[todo[ok]] = d * v[ok]
        todo = todo[~ok]
    return out


def sample_u(mix: tuple, n: int, gen: torch.Generator, device) -> torch.Tensor:
    """n draws (float64) from a retention mixture, clamped to [1e-4, 1-1e-6]."""
    pick = torch.rand(n, generator=gen, dtype=torch.float64, device=device)
    u = torch.empty(n, dtype=torch.float64, device=device)
    edge = 0.0
    for k, (w, comp) in enumerate(mix):
        hi = 1.0 if k == len(mix) - 1 else edge + w
        sel = (pick >= edge) & (pick < hi) if k < len(mix) - 1 else (pick >= edge)
        m = int(sel.sum().item())
        if comp[0] == "const":
            u[sel] = comp[1]
        else:
            _, a, b = comp
            ga = _gamma(a, m, gen, device)
            gb = _gamma(b, m, gen, device)
            u[sel] = ga / (ga + gb)
        edge = hi
    return u.clamp(U_LO, U_HI)


def log_retention(mix: tuple, n: int, gen: torch.Generator, device) -> torch.Tensor:
    """float32 log(u) for n mixture draws (the gate output the pages learn)."""
    return torch.log(sample_u(mix, n, gen, device)).to(torch.float32)


def kv_torch_dtype(cfg: Config) -> torch.dtype:
    return torch.bfloat16 if cfg.kv_dtype == "bf16" else torch.float32


def queries(cfg: Config, seed: int, step: int, device="cpu") -> torch.Tensor:
    """q for decode step `step`: float32 [B, L, Hq, D] ~ N(0, 1)."""
    g = _gen(device, seed, "q", step)
    return torch.randn(cfg.B, cfg.L, cfg.Hq, cfg.D, generator=g, device=device, dtype=torch.float32)


def step_inputs(cfg: Config, seed: int, step: int, device="cpu") -> dict:
    """Inputs of decode step `step` (t = T0 + step for every sequence)."""
    q = queries(cfg, seed, step, device)
    gk = _gen(device, seed, "k_new", step)
    gv = _gen(device, seed, "v_new", step)
    gl = _gen(device, seed, "lb_new", step)
    dt = kv_torch_dtype(cfg)
    k_new = torch.randn(cfg.C, cfg.D, generator=gk, device=device).to(dt)
    v_new = torch.randn(cfg.C, cfg.D, generator=gv, device=device).to(dt)
    lb_new = log_retention(cfg.mix_decode or cfg.mix, cfg.C, gl, device)
    t = torch.full((cfg.B,), cfg.T0 + step, dtype=torch.int32, device=device)
    m = torch.full((cfg.B,), cfg.M, dtype=torch.int64, device=device)
    return dict(q=q, k_new=k_new, v_new=v_new, lb_new=lb_new, t=t, m_global=m, evict=cfg.evicts(step))


def memory_weights(cfg: Config, seed: int, device="cpu") -> dict:
    """Synthetic slow weights of the latent memory (no trained ones exist
    here): proj [L, D, D] ~ N(0, 1/D), gate_w [L, Hq, D] ~ N(0, 1/D),
    gate_b [L, Hq] ~ N(0, 1), float32."""
    g = _gen(device, seed, "memory")
    s = 1.0 / math.sqrt(cfg.D)
    return dict(proj=torch.randn(cfg.L, cfg.D, cfg.D, generator=g, device=device) * s,
                gate_w=torch.randn(cfg.L, cfg.Hq, cfg.D, generator=g, device=device) * s,
                gate_b=torch.randn(cfg.L, cfg.Hq, generator=g, device=device))


def pool_geometry(cfg: Config, n_steps: int) -> tuple[int, int, int]:
    """(P0, n_pages, max_pages) for a run of n_steps decode steps."""
    P0 = -(-cfg.T0 // cfg.P)
    grow = -(-max(n_steps, cfg.slack, 1) // cfg.P)
    n_pages = cfg.C * P0 + cfg.C * grow + cfg.C
    max_pages = -(-(cfg.T0 + n_steps) // cfg.P) + 1
    return P0, n_pages, max_pages


@dataclass
class DeviceCache:
    """Cache tensors (torch), in the layout both sides share."""
    cfg: Config
    k_pool: torch.Tensor      # [n_pages, P, D] bf16 / f32
    v_pool: torch.Tensor
    pos_pool: torch.Tensor    # [n_pages, P] int32
    lb_pool: torch.Tensor     # [n_pages, P] float32
    block_table: torch.Tensor # [C, max_pages] int32, -1 = none
    len: torch.Tensor         # [C] int32
    free_stack: torch.Tensor  # [n_pages] int32
    free_top: torch.Tensor    # [1] int32
    extra: dict = field(default_factory=dict)

    @property
    def n_pages(self) -> int:
        return self.k_pool.shape[0]

    @property
    def max_pages(self) -> int:
        return self.block_table.shape[1]

    def clone(self) -> "DeviceCache":
        return replace(self, **{f: getattr(self, f).clone() for f in (
            "k_pool", "v_pool", "pos_pool", "lb_pool", "block_table", "len", "free_stack", "free_top")},
            extra=dict(self.extra))

    def to(self, device) -> "DeviceCache":
        return replace(self, **{f: getattr(self, f).to(device) for f in (
            "k_pool", "v_pool", "pos_pool", "lb_pool", "block_table", "len", "free_stack", "free_top")},
            extra=dict(self.extra))


def _fill_kv(cfg: Config, seed: int, device, pool: torch.Tensor, name: str, P0: int,
             planted_dir: torch.Tensor | None, head_chunk: int) -> None:
    dt = kv_torch_dtype(cfg)
    view = pool[: cfg.C * P0].view(cfg.C, P0 * cfg.P, cfg.D)
    for c0 in range(0, cfg.C, head_chunk):
        c1 = min(cfg.C, c0 + head_chunk)
        g = _gen(device, seed, name, c0)
        x = torch.randn(c1 - c0, cfg.T0, cfg.D, generator=g, device=device, dtype=torch.float32)
        if planted_dir is not None and cfg.planted > 0:
            gp = _gen(device, seed, "planted", c0)
            hit = torch.rand(c1 - c0, cfg.T0, generator=gp, device=device) < cfg.planted
            x += 3.0 * hit.unsqueeze(-1).to(x.dtype) * planted_dir[c0:c1].unsqueeze(1)
        view[c0:c1, : cfg.T0] = x.to(dt)


def prefill_cache(cfg: Config, seed: int, device="cpu", n_steps: int | None = None,
                  head_chunk: int = 16) -> DeviceCache:
    """Cache after prefill of T0 tokens per sequence (nothing evicted yet)."""
    n_steps = cfg.steps if n_steps is None else n_steps
    P0, n_pages, max_pages = pool_geometry(cfg, n_steps)
    C, P, D = cfg.C, cfg.P, cfg.D
    dt = kv_torch_dtype(cfg)
    k_pool = torch.zeros(n_pages, P, D, dtype=dt, device=device)
    v_pool = torch.zeros(n_pages, P, D, dtype=dt, device=device)
    pos_pool = torch.zeros(n_pages, P, dtype=torch.int32, device=device)
    lb_pool = torch.zeros(n_pages, P, dtype=torch.float32, device=device)

    planted_dir = None
    if cfg.planted > 0:
        q0 = queries(cfg, seed, 0, device).reshape(C, cfg.G, D).sum(dim=1)
        planted_dir = q0 / q0.norm(dim=-1, keepdim=True).clamp_min(1e-30)
    _fill_kv(cfg, seed, device, k_pool, "k", P0, planted_dir, head_chunk)
    _fill_kv(cfg, seed, device, v_pool, "v", P0, None, head_chunk)

    pos = torch.arange(cfg.T0, dtype=torch.int32, device=device)
    pos_pool[: C * P0].view(C, P0 * P)[:, : cfg.T0] = pos
    lbv = lb_pool[: C * P0].view(C, P0 * P)
    g = _gen(device, seed, "lb")
    if cfg.vision > 0:
        lbv[:, : cfg.vision] = log_retention(cfg.mix_vision, C * cfg.vision, g, device).view(C, cfg.vision)
        nt = cfg.T0 - cfg.vision
        lbv[:, cfg.vision: cfg.T0] = log_retention(cfg.mix, C * nt, g, device).view(C, nt)
    else:
        lbv[:, : cfg.T0] = log_retention(cfg.mix, C * cfg.T0, g, device).view(C, cfg.T0)

    block_table = torch.full((C, max_pages), -1, dtype=torch.int32, device=device)
    block_table[:, :P0] = (torch.arange(C, device=device, dtype=torch.int32).unsqueeze(1) * P0
                           + torch.arange(P0, device=device, dtype=torch.int32).unsqueeze(0))
    length = torch.full((C,), cfg.T0, dtype=torch.int32, device=device)
    free_stack = torch.full((n_pages,), -1, dtype=torch.int32, device=device)
    n_free = n_pages - C * P0
    free_stack[:n_free] = torch.arange(n_pages - 1, C * P0 - 1, -1, dtype=torch.int32, device=device)
    free_top = torch.tensor([n_free], dtype=torch.int32, device=device)
    return DeviceCache(cfg, k_pool, v_pool, pos_pool, lb_pool, block_table, length, free_stack, free_top)


def ragged_cache(cfg: Config, seed: int, lengths, device="cpu", *, n_pages: int | None = None,
                 max_pages: int | None = None, shuffle_pages: bool = True,
                 shuffle_slots: bool = True, lb_override: torch.Tensor | None = None) -> DeviceCache:
    """A valid mid-decode cache with arbitrary per-head lengths.

    Head c holds lengths[c] distinct positions drawn from [0, T0) (slot order
    random when shuffle_slots), on pages drawn at random from the pool when
    shuffle_pages; the free stack holds the remaining pages in random order."""
    lengths = [int(x) for x in lengths]
    C, P, D = cfg.C, cfg.P, cfg.D
    assert len(lengths) == C
    pages_needed = [-(-n // P) for n in lengths]
    if max_pages is None:
        max_pages = max(pages_needed + [1]) + 2
    if n_pages is None:
        n_pages = sum(pages_needed) + C + 8
    dt = kv_torch_dtype(cfg)
    rng = np.random.default_rng(seed_for(seed, "ragged"))
    perm = rng.permutation(n_pages) if shuffle_pages else np.arange(n_pages)
    table = np.full((C, max_pages), -1, np.int32)
    pos_pool = np.zeros((n_pages, P), np.int32)
    used = 0
    for c in range(C):
        k = pages_needed[c]
        table[c, :k] = perm[used: used + k]
        used += k
        pos = rng.choice(cfg.T0, size=lengths[c], replace=False).astype(np.int32)
        if not shuffle_slots:
            pos.sort()
        for s, p in enumerate(pos):
            pos_pool[table[c, s // P], s % P] = p
    free = perm[used:].astype(np.int32)
    free_stack = np.full(n_pages, -1, np.int32)
    free_stack[: free.size] = free
    gk, gv, gl = (_gen(device, seed, name, "ragged") for name in ("k", "v", "lb"))
    k_pool = torch.randn(n_pages, P, D, generator=gk, device=device).to(dt)
    v_pool = torch.randn(n_pages, P, D, generator=gv, device=device).to(dt)
    if lb_override is not None:
        lb_pool = lb_override.to(device=device, dtype=torch.float32).reshape(n_pages, P).clone()
    else:
        lb_pool = log_retention(cfg.mix, n_pages * P, gl, device).view(n_pages, P)
    return DeviceCache(cfg, k_pool, v_pool, torch.from_numpy(pos_pool).to(device), lb_pool,
                       torch.from_numpy(table).to(device),
                       torch.tensor(lengths, dtype=torch.int32, device=device),
                       torch.from_numpy(free_stack).to(device),
                       torch.tensor([free.size], dtype=torch.int32, device=device))


def small_config(name="small", *, L=2, H=3, G=2, D=128, B=2, T0=200, M=300, kv_dtype="bf16",
                 mix=MIX_8B, steps=4, evict_every=1) -> Config:
    """A test-sized config (any shape the kernels support)."""
    return Config(name, L=L, H=H, Hq=H * G, D=D, B=B, T0=T0, M=M, steps=steps,
                  evict_every=evict_every, kv_dtype=kv_dtype, mix=mix)


def to_host(cache: DeviceCache):
    """numpy copy of a cache for the oracle (bf16 as uint16 bit patterns)."""
    from_t = lambda x: x.detach().cpu().contiguous()
    kp, vp = from_t(cache.k_pool), from_t(cache.v_pool)
    if kp.dtype == torch.bfloat16:
        kp = kp.view(torch.int16).numpy().view(np.uint16)
        vp = vp.view(torch.int16).numpy().view(np.uint16)
    else:
        kp, vp = kp.numpy(), vp.numpy()
    cfg = cache.cfg
    return dict(B=cfg.B, L=cfg.L, H=cfg.H, G=cfg.G, D=cfg.D, P=cfg.P, k_pool=kp, v_pool=vp,
                pos_pool=from_t(cache.pos_pool).numpy(), lb_pool=from_t(cache.lb_pool).numpy(),
                block_table=from_t(cache.block_table).numpy(), len=from_t(cache.len).numpy(),
                free_stack=from_t(cache.free_stack).numpy(), free_top=from_t(cache.free_top).numpy())


def rows_to_host(x: torch.Tensor) -> np.ndarray:
    """numpy copy of K/V rows (bf16 as uint16 bit patterns)."""
    x = x.detach().cpu().contiguous()
    if x.dtype == torch.bfloat16:
        return x.view(torch.int16).numpy().view(np.uint16)
    return x.numpy()
