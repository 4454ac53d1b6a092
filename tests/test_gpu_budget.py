"""GPU parity of the budget-allocation variants (rkv_score_select_budget)
against the oracle: per-head budgets (Cache What Lasts (TRIM-KV), core
mechanism 4) and the ContourKV allocation (Trust the Mass, Methodology 3:
recency floor in every head, a fixed budget for flat heads, the rest of the
global budget ranked globally).  Keep masks, kept counts, n_pre and the
free-page plan bit for bit; then compaction and append of the selection are
compared with the oracle's whole step state.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.gpu_helpers import compare_state, keep_flags, masked_keep, rkv_cache, sync, to_dev
from tests.oracle_helpers import host_cache

pytestmark = pytest.mark.gpu


def _plan(n_pre, kept):
    freed = (n_pre + 15) // 16 - (kept + 15) // 16
    return np.concatenate([[0], np.cumsum(freed)[:-1]]).astype(np.int64), int(freed.sum())


def _check(rkv, dc, hc, sel, ws, keep_o, kept_o, then_step=True):
    sync()
    assert ws.status() == 0, ws.counters()
    keep_g = masked_keep(keep_flags(sel, dc.max_pages), hc.len)
    assert np.array_equal(sel.n_pre.cpu().numpy(), hc.len), "n_pre"
    assert np.array_equal(sel.kept.cpu().numpy(), kept_o), "kept per head"
    assert np.array_equal(keep_g, keep_o), f"keep flags differ at {np.argwhere(keep_g != keep_o)[:5].tolist()}"
    pfx, total = _plan(hc.len.astype(np.int64), kept_o.astype(np.int64))
    plan = sel.plan.cpu().numpy()
    assert np.array_equal(plan[:-2], pfx) and plan[-2] == total and plan[-1] == int(hc.free_top[0]), "plan"
    if then_step:
        # the variants feed the unchanged compaction: same tables and pools
        cache = rkv_cache(rkv, dc)
        rkv.compact_pages(cache, sel, ws)
        sync()
        oracle.compact(hc, keep_o)
        compare_state(dc, hc)


@pytest.mark.parametrize("seed", range(4))
def test_per_head_budgets(rkv, seed):
    rng = np.random.default_rng(300 + seed)
    cfg = workloads.small_config(L=int(rng.integers(1, 4)), H=int(rng.integers(1, 5)), G=2, D=64,
                                 B=int(rng.integers(1, 3)), T0=5000, kv_dtype="bf16")
    lengths = rng.integers(0, 3000, size=cfg.C)
    if seed == 3:
        lengths[0] = 14000 - 1   # past the kernel's shared-memory key cache
        cfg = workloads.small_config(L=cfg.L, H=cfg.H, G=2, D=64, B=cfg.B, T0=15000, kv_dtype="bf16")
    dc = to_dev(workloads.ragged_cache(cfg, seed, lengths))
    hc = host_cache(dc)
    t = [cfg.T0] * cfg.B
    for trial in range(3):
        m_head = rng.integers(-5, 2500, size=cfg.C).astype(np.int32)
        m_head[rng.integers(0, cfg.C)] = 0
        cache = rkv_cache(rkv, dc)
        sel, ws = rkv.Selection.empty(cache), rkv.Workspace(cache)
        rkv.score_select_per_head(cache, torch.tensor(t, dtype=torch.int32, device="cuda"),
                                  torch.from_numpy(m_head).cuda(), sel, ws)
        keep_o, kept_o = oracle.select_per_head(hc, t, m_head)
        _check(rkv, dc, hc, sel, ws, keep_o, kept_o, then_step=(trial == 2))


@pytest.mark.parametrize("seed", range(5))
def test_contour_allocation(rkv, seed):
    rng = np.random.default_rng(400 + seed)
    cfg = workloads.small_config(L=int(rng.integers(1, 4)), H=int(rng.integers(2, 5)), G=4, D=128,
                                 B=int(rng.integers(1, 3)), T0=4000, kv_dtype="bf16")
    lengths = rng.integers(0, 2500, size=cfg.C)
    dc = to_dev(workloads.ragged_cache(cfg, seed, lengths))
    if seed == 4:  # exact score ties everywhere
        vals = torch.tensor([-0.5, -0.25, -1e-3, -2.0], dtype=torch.float32)
        g = torch.Generator().manual_seed(4)
        dc.lb_pool = vals[torch.randint(0, 4, dc.lb_pool.shape, generator=g)].cuda().contiguous()
    hc = host_cache(dc)
    t = [cfg.T0] * cfg.B
    for trial in range(3):
        dm = (rng.random((cfg.C, cfg.G)) * 0.6).astype(np.float32)
        tau = float(rng.choice([0.1, 0.3, 0.45]))
        F, r = int(rng.integers(0, 600)), int(rng.integers(0, 200))
        tot = [int(hc.len[b * cfg.L * cfg.H:(b + 1) * cfg.L * cfg.H].sum()) for b in range(cfg.B)]
        m = [int(x * rng.choice([0.0, 0.2, 0.6, 1.1])) for x in tot]
        cache = rkv_cache(rkv, dc)
        sel, ws = rkv.Selection.empty(cache), rkv.Workspace(cache)
        rkv.score_select_contour(cache, torch.tensor(t, dtype=torch.int32, device="cuda"),
                                 torch.tensor(m, dtype=torch.int64, device="cuda"),
                                 torch.from_numpy(dm).cuda().view(cfg.B, cfg.L, cfg.Hq), tau, F, r, sel, ws)
        keep_o, kept_o, flat = oracle.select_contour(hc, t, m, dm, tau, F, r)
        _check(rkv, dc, hc, sel, ws, keep_o, kept_o, then_step=(trial == 2))


def test_contour_edges(rkv):
    # every head flat; no head flat with a floor longer than the heads; a
    # mean exactly at the threshold (not flat); empty heads
    cfg = workloads.small_config(L=1, H=4, G=2, D=128, B=1, T0=3000, kv_dtype="bf16")
    lengths = [0, 700, 33, 2900]
    dc = to_dev(workloads.ragged_cache(cfg, 6, lengths))
    hc = host_cache(dc)
    for dm_val, tau, F, r, m in ((0.9, 0.5, 100, 0, 500), (0.0, 0.5, 10, 5000, 0), (0.3, 0.3, 50, 17, 1000),
                                 (0.31, 0.3, 0, 1, 3633)):
        dm = np.full((cfg.C, cfg.G), dm_val, np.float32)
        cache = rkv_cache(rkv, dc)
        sel, ws = rkv.Selection.empty(cache), rkv.Workspace(cache)
        rkv.score_select_contour(cache, torch.tensor([3000], dtype=torch.int32, device="cuda"),
                                 torch.tensor([m], dtype=torch.int64, device="cuda"),
                                 torch.from_numpy(dm).cuda().view(1, 1, cfg.Hq), tau, F, r, sel, ws)
        keep_o, kept_o, _ = oracle.select_contour(hc, [3000], [m], dm, tau, F, r)
        _check(rkv, dc, hc, sel, ws, keep_o, kept_o, then_step=False)
