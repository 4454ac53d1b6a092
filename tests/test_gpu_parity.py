"""GPU parity: each librkv entry point against the CPU oracle on the same
seeded inputs (small and ragged shapes, several CTAs per head, ragged page
tails, edge cases).  Selection, masks, lengths, tables, free stack and pools
must match bit for bit; attention outputs within 2e-3 of the row norm and
dropped mass within 1e-4.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.gpu_helpers import (assert_outputs_close, compare_state, keep_flags, masked_keep, rkv_cache, sync,
                               to_dev)
from tests.oracle_helpers import host_cache

pytestmark = pytest.mark.gpu


def _ragged(cfg, seed, lengths, **kw):
    return to_dev(workloads.ragged_cache(cfg, seed, lengths, **kw))


def _select(rkv, dc, t, m):
    cache = rkv_cache(rkv, dc)
    sel = rkv.Selection.empty(cache)
    ws = rkv.Workspace(cache)
    tt = torch.tensor(t, dtype=torch.int32, device="cuda")
    mm = torch.tensor(m, dtype=torch.int64, device="cuda")
    rkv.score_select(cache, tt, mm, sel, ws)
    sync()
    return cache, sel, ws


def _check_select(dc, sel, ws, t, m):
    hc = host_cache(dc)
    keep_o, kept_o = oracle.select(hc, t, m)
    keep_g = masked_keep(keep_flags(sel, dc.max_pages), hc.len)
    assert ws.status() == 0
    assert np.array_equal(sel.kept.cpu().numpy(), kept_o), "kept per head"
    assert np.array_equal(sel.n_pre.cpu().numpy(), hc.len), "n_pre"
    assert np.array_equal(keep_g, keep_o), f"keep flags differ at {np.argwhere(keep_g != keep_o)[:5].tolist()}"
    return hc, keep_o, kept_o


def test_select_tiny_config(rkv):
    cfg = workloads.CONFIGS["tiny"]
    dc = to_dev(workloads.prefill_cache(cfg, 0))
    _, sel, ws = _select(rkv, dc, [cfg.T0], [cfg.M])
    _check_select(dc, sel, ws, [cfg.T0], [cfg.M])
    assert int(sel.kept.sum()) == cfg.M


@pytest.mark.parametrize("seed", range(5))
def test_select_ragged_batches(rkv, seed):
    rng = np.random.default_rng(100 + seed)
    B = int(rng.integers(1, 4))
    cfg = workloads.small_config(L=int(rng.integers(1, 5)), H=int(rng.integers(1, 5)), G=1, D=64, B=B, T0=3000,
                                 kv_dtype="bf16")
    lengths = rng.integers(0, 900, size=cfg.C)
    lengths[rng.integers(0, cfg.C)] = 0
    dc = _ragged(cfg, seed, lengths)
    hc0 = host_cache(dc)
    totals = [int(hc0.len[b * cfg.L * cfg.H:(b + 1) * cfg.L * cfg.H].sum()) for b in range(B)]
    t = [3000] * B
    for frac in (0.0, 0.1, 0.5, 0.97, 1.0, 1.3):
        m = [int(x * frac) for x in totals]
        _, sel, ws = _select(rkv, dc, t, m)
        _check_select(dc, sel, ws, t, m)


@pytest.mark.parametrize("case", ["all_tie", "neg_inf", "one_head", "m_edges", "few_values"])
def test_select_edge_cases(rkv, case):
    cfg = workloads.small_config(L=2, H=4, G=1, D=64, B=1, T0=2000, kv_dtype="bf16")
    rng = np.random.default_rng(7)
    lengths = rng.integers(50, 700, size=cfg.C)
    if case == "one_head":
        lengths = np.zeros(cfg.C, int)
        lengths[5] = 1999
    base = workloads.ragged_cache(cfg, 3, lengths)
    lb = base.lb_pool.clone()
    if case == "all_tie":
        lb[:] = -0.01          # equal ages across heads tie exactly
    elif case == "neg_inf":
        lb[torch.rand(lb.shape, generator=torch.Generator().manual_seed(1)) < 0.6] = -float("inf")
    elif case == "few_values":
        vals = torch.tensor([-0.5, -0.25, -1e-3, -2.0], dtype=torch.float32)
        lb = vals[torch.randint(0, 4, lb.shape, generator=torch.Generator().manual_seed(2))]
    base.lb_pool = lb.contiguous()
    dc = to_dev(base)
    n = int(np.asarray(lengths).sum())
    ms = [0, 1, n - 1, n, n + 1, n // 3] if case in ("m_edges", "one_head") else [n // 7, n // 2, n - 3]
    for m in ms:
        _, sel, ws = _select(rkv, dc, [2000], [m])
        _check_select(dc, sel, ws, [2000], [m])


def _attn_case(rkv, cfg, seed, lengths, frac, *, use_sel=True):
    dc = _ragged(cfg, seed, lengths)
    hc = host_cache(dc)
    n = int(hc.len.sum())
    t = [cfg.T0] * cfg.B
    m = [int(n * frac / cfg.B)] * cfg.B
    cache, sel, ws = _select(rkv, dc, t, m)
    q = workloads.queries(cfg, seed, 0, "cuda")
    out = torch.empty(cfg.B, cfg.L, cfg.Hq, cfg.D, device="cuda")
    lse = torch.empty(cfg.B, cfg.L, cfg.Hq, device="cuda")
    dm = torch.empty(cfg.B, cfg.L, cfg.Hq, device="cuda")
    rkv.paged_decode_attn(cache, q, cfg.scale, sel if use_sel else None, out, lse, dm, ws)
    dm2 = torch.empty_like(dm)
    if use_sel:
        rkv.dropped_mass(cache, q, cfg.scale, sel, dm2, ws)
    sync()
    assert ws.status() == 0
    keep = oracle.select(hc, t, m)[0] if use_sel else None
    o_ref, lse_ref, dm_ref = oracle.attention(hc, q.cpu().numpy().reshape(cfg.C, cfg.G, cfg.D), cfg.scale, keep)
    kept_any = np.array([bool(keep[c, :hc.len[c]].any()) if keep is not None else bool(hc.len[c] > 0)
                         for c in range(cfg.C)])
    assert_outputs_close(out.cpu().numpy().reshape(cfg.C, cfg.G, cfg.D), lse.cpu().numpy().reshape(cfg.C, cfg.G),
                         dm.cpu().numpy().reshape(cfg.C, cfg.G), o_ref, lse_ref, dm_ref, kept_any)
    if use_sel:
        assert np.abs(dm2.cpu().numpy().reshape(cfg.C, cfg.G) - dm_ref).max() <= 1e-4


@pytest.mark.parametrize("kv,D,G", [("bf16", 128, 4), ("bf16", 128, 1), ("bf16", 128, 7), ("bf16", 128, 2),
                                    ("f32", 64, 1), ("bf16", 64, 4), ("f32", 128, 2)])
def test_attention_parity_shapes(rkv, kv, D, G):
    cfg = workloads.small_config(L=2, H=3, G=G, D=D, B=1, T0=4000, kv_dtype=kv)
    rng = np.random.default_rng(D + G)
    lengths = rng.integers(1, 2500, size=cfg.C)
    lengths[2] = 0
    lengths[3] = 17
    _attn_case(rkv, cfg, 11, lengths, 0.4)


@pytest.mark.parametrize("frac", [0.0, 0.02, 0.6, 1.0])
def test_attention_budget_fractions(rkv, frac):
    cfg = workloads.small_config(L=3, H=2, G=4, D=128, B=2, T0=3000, kv_dtype="bf16")
    rng = np.random.default_rng(5)
    _attn_case(rkv, cfg, 5, rng.integers(0, 2000, size=cfg.C), frac)


def test_attention_without_selection(rkv):
    cfg = workloads.small_config(L=2, H=2, G=4, D=128, B=1, T0=3000, kv_dtype="bf16")
    _attn_case(rkv, cfg, 6, [1500, 0, 33, 2900], 1.0, use_sel=False)


def test_attention_few_pages_many_ctas(rkv):
    # fewer pages than CTAs: empty CTA ranges, heads split into one-page pieces
    cfg = workloads.small_config(L=1, H=3, G=4, D=128, B=1, T0=200, kv_dtype="bf16")
    _attn_case(rkv, cfg, 8, [40, 1, 0], 0.5)


@pytest.mark.parametrize("seed", range(3))
def test_compaction_and_append_bit_exact(rkv, seed):
    rng = np.random.default_rng(200 + seed)
    cfg = workloads.small_config(L=2, H=3, G=2, D=128, B=2, T0=3000, kv_dtype="bf16")
    lengths = rng.integers(0, 1500, size=cfg.C)
    dc = _ragged(cfg, seed, lengths, n_pages=int(np.ceil(lengths / 16).sum()) + 80)
    hc = host_cache(dc)
    n = [int(hc.len[b * 6:(b + 1) * 6].sum()) for b in range(2)]
    t = [3000, 3000]
    m = [n[0] // 4, (n[1] * 3) // 4]
    cache, sel, ws = _select(rkv, dc, t, m)
    keep, _ = oracle.select(hc, t, m)
    rkv.compact_pages(cache, sel, ws)
    sync()
    oracle.compact(hc, keep)
    compare_state(dc, hc)
    for s in range(20):   # several appends cross page boundaries
        inp = workloads.step_inputs(cfg, seed, s, "cuda")
        rkv.append(cache, inp["t"], inp["k_new"], inp["v_new"], inp["lb_new"], ws)
        sync()
        rc = oracle.append(hc, inp["t"].cpu().numpy(), workloads.rows_to_host(inp["k_new"]),
                           workloads.rows_to_host(inp["v_new"]), inp["lb_new"].cpu().numpy())
        assert rc == oracle.OK
        compare_state(dc, hc)
    assert ws.status() == 0


@pytest.mark.parametrize("name", ["tiny"])
def test_full_step_config(rkv, name):
    cfg = workloads.CONFIGS[name]
    dc = to_dev(workloads.prefill_cache(cfg, 0, n_steps=4))
    hc = host_cache(dc)
    cache = rkv_cache(rkv, dc)
    sel = rkv.Selection.empty(cache)
    ws = rkv.Workspace(cache)
    outs = rkv.StepOutputs.empty(cache)
    for s in range(4):
        inp = workloads.step_inputs(cfg, 0, s, "cuda")
        len_before = hc.len.copy()
        rkv.step(cache, sel, ws, outs, q=inp["q"], t=inp["t"], m_global=inp["m_global"], k_new=inp["k_new"],
                 v_new=inp["v_new"], lb_new=inp["lb_new"], evict=inp["evict"], scale=cfg.scale)
        sync()
        ref = oracle.step(hc, inp["t"].cpu().numpy(), inp["m_global"].cpu().numpy(),
                          inp["q"].cpu().numpy().reshape(cfg.C, cfg.G, cfg.D), workloads.rows_to_host(inp["k_new"]),
                          workloads.rows_to_host(inp["v_new"]), inp["lb_new"].cpu().numpy(), evict=inp["evict"],
                          scale=cfg.scale)
        kept_any = (ref["kept"] > 0) if ref["kept"] is not None else (len_before > 0)
        assert_outputs_close(outs.out.cpu().numpy().reshape(cfg.C, cfg.G, cfg.D),
                             outs.lse.cpu().numpy().reshape(cfg.C, cfg.G),
                             outs.dropped.cpu().numpy().reshape(cfg.C, cfg.G), ref["out"], ref["lse"],
                             ref["dropped"], kept_any)
        compare_state(dc, hc)
    assert ws.status() == 0


def test_multi_step_small_evict_every_other(rkv):
    cfg = workloads.small_config(L=2, H=2, G=4, D=128, B=2, T0=1000, M=1500, kv_dtype="bf16", steps=12,
                                 evict_every=2)
    dc = to_dev(workloads.prefill_cache(cfg, 3, n_steps=12))
    hc = host_cache(dc)
    cache = rkv_cache(rkv, dc)
    sel = rkv.Selection.empty(cache)
    ws = rkv.Workspace(cache)
    outs = rkv.StepOutputs.empty(cache)
    for s in range(12):
        inp = workloads.step_inputs(cfg, 3, s, "cuda")
        len_before = hc.len.copy()
        rkv.step(cache, sel, ws, outs, q=inp["q"], t=inp["t"], m_global=inp["m_global"], k_new=inp["k_new"],
                 v_new=inp["v_new"], lb_new=inp["lb_new"], evict=inp["evict"], scale=cfg.scale)
        sync()
        ref = oracle.step(hc, inp["t"].cpu().numpy(), inp["m_global"].cpu().numpy(),
                          inp["q"].cpu().numpy().reshape(cfg.C, cfg.G, cfg.D), workloads.rows_to_host(inp["k_new"]),
                          workloads.rows_to_host(inp["v_new"]), inp["lb_new"].cpu().numpy(), evict=inp["evict"],
                          scale=cfg.scale)
        kept_any = (ref["kept"] > 0) if ref["kept"] is not None else (len_before > 0)
        assert_outputs_close(outs.out.cpu().numpy().reshape(cfg.C, cfg.G, cfg.D),
                             outs.lse.cpu().numpy().reshape(cfg.C, cfg.G),
                             outs.dropped.cpu().numpy().reshape(cfg.C, cfg.G), ref["out"], ref["lse"],
                             ref["dropped"], kept_any)
        compare_state(dc, hc)
    assert ws.status() == 0


def test_select_reuses_threshold_window_across_calls(rkv):
    # One workspace across many calls: the previous call's threshold window is
    # hit (similar budgets), missed (budget jumps) and overflows (dense ties);
    # every call must match the oracle exactly.
    cfg = workloads.small_config(L=3, H=4, G=1, D=64, B=1, T0=6000, kv_dtype="bf16")
    rng = np.random.default_rng(31)
    dc = _ragged(cfg, 31, rng.integers(200, 2500, size=cfg.C))
    cache = rkv_cache(rkv, dc)
    ws = rkv.Workspace(cache)
    n = int(dc.len.sum())
    budgets = [n // 2, n // 2 + 3, n // 2 - 40, n // 2 + 100, n // 5, n // 5 + 1, (9 * n) // 10, (9 * n) // 10 - 7,
               1, n - 1, n // 3]
    for i, m in enumerate(budgets):
        t = 6000 + (i % 3)
        sel = rkv.Selection.empty(cache)
        rkv.score_select(cache, torch.tensor([t], dtype=torch.int32, device="cuda"),
                         torch.tensor([m], dtype=torch.int64, device="cuda"), sel, ws)
        sync()
        _check_select(dc, sel, ws, [t], [m])
    few = torch.tensor([-0.5, -0.25], dtype=torch.float32, device="cuda")
    dc.lb_pool.copy_(few[torch.randint(0, 2, dc.lb_pool.shape, device="cuda")])   # many exact ties
    for m in (n // 2, n // 2 + 1, n // 4):
        sel = rkv.Selection.empty(cache)
        rkv.score_select(cache, torch.tensor([6000], dtype=torch.int32, device="cuda"),
                         torch.tensor([m], dtype=torch.int64, device="cuda"), sel, ws)
        sync()
        _check_select(dc, sel, ws, [6000], [m])
