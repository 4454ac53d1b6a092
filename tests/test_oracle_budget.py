"""Pins of the oracle's budget-allocation variants.

Per-head budget -- Cache What Lasts (TRIM-KV), core mechanism 4 and the
analogy's section 3: a head over its budget evicts its lowest retention
beta^(t-i); Make Each Token Count (DBTrimKV), Methodology 3 names this fixed
per-head allocation as what its global budget replaces.  Head c keeps its
top m_head[c] entries, equal scores by ascending position.

ContourKV allocation -- Trust the Mass (ContourKV), Methodology 3: flat
cells (high dropped mass) get a fixed budget, every cell keeps a recency
floor, the scores are reused.  Readings in oracle.c (orc_select_contour).
"""
import itertools
import math

import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.oracle_helpers import hand_cache, host_cache, kept_positions, load_golden


def _entries(hc, t):
    """[(score f32, l, h, i, c, slot)] of every entry (numpy binary32 multiply)."""
    out = []
    for c in range(hc.C):
        b, cl = divmod(c, hc.L * hc.H)
        l, h = divmod(cl, hc.H)
        for k in range(int(hc.len[c])):
            page = hc.block_table[c, k // hc.P]
            i = int(hc.pos_pool[page, k % hc.P])
            s = float(np.float32(np.float32(t[b] - i) * hc.lb_pool[page, k % hc.P]))
            out.append((s, l, h, i, c, k, b))
    return out


def _small(seed, ties, B=2, L=2, H=2, T0=60, G=2):
    rng = np.random.default_rng(seed)
    cfg = workloads.small_config(L=L, H=H, G=G, D=8, B=B, T0=T0, kv_dtype="f32")
    dc = workloads.ragged_cache(cfg, seed, rng.integers(0, 30, size=cfg.C))
    if ties:  # a few distinct log-retentions: exact score ties
        choices = torch.tensor([-0.5, -0.25, -1.0, -2.0 ** -7], dtype=torch.float32)
        idx = torch.from_numpy(rng.integers(0, 4, size=dc.lb_pool.numel()))
        dc.lb_pool = choices[idx].view_as(dc.lb_pool).clone()
    return cfg, host_cache(dc), rng


# ----------------------------------------------------------- per-head ---
@pytest.mark.parametrize("seed", range(4))
def test_per_head_brute_force(seed):
    cfg, hc, rng = _small(seed, ties=seed % 2 == 0)
    t = [cfg.T0] * cfg.B
    ents = _entries(hc, t)
    for trial in range(4):
        m_head = rng.integers(-2, 32, size=cfg.C)
        keep, kept = oracle.select_per_head(hc, t, m_head)
        want = np.zeros_like(keep)
        for e in ents:
            before = sum(1 for f in ents if f[4] == e[4] and (f[0] > e[0] or (f[0] == e[0] and f[3] < e[3])))
            if before < m_head[e[4]]:
                want[e[4], e[5]] = 1
        assert np.array_equal(keep, want), (seed, trial)
        assert kept.tolist() == [min(max(int(m), 0), int(n)) for m, n in zip(m_head, hc.len)]


def test_per_head_single_head_equals_global_select():
    cfg = workloads.small_config(L=1, H=1, G=1, D=8, B=1, T0=200, kv_dtype="f32")
    hc = host_cache(workloads.ragged_cache(cfg, 3, [150]))
    for m in (0, 1, 40, 149, 150, 170):
        assert np.array_equal(oracle.select_per_head(hc, [200], [m])[0], oracle.select(hc, [200], [m])[0])


def test_per_head_constant_beta_keeps_most_recent():
    cfg = workloads.Config("const", L=2, H=2, Hq=2, D=4, B=1, T0=40, M=0, steps=1, kv_dtype="f32",
                           mix=((1.0, ("const", 0.9)),))
    hc = host_cache(workloads.prefill_cache(cfg, 0))
    m_head = [0, 3, 17, 40]
    keep, _ = oracle.select_per_head(hc, [cfg.T0], m_head)
    got = kept_positions(hc, keep)
    for c, m in enumerate(m_head):
        assert got[c] == set(range(cfg.T0 - m, cfg.T0))


# ----------------------------------------------------------- ContourKV ---
def test_contour_golden_hand_worked():
    g = load_golden("contour_three_heads.json")
    P = g["P"]
    table = [[0], [1], [2]]
    hc = hand_cache(g["B"], g["L"], g["H"], g["G"], 4, P, 3, 1, table, [len(x) for x in g["slot_pos"]],
                    g["slot_pos"], g["slot_lb"])
    dm = np.array(g["dm_prev"], np.float32)
    for case in g["cases"]:
        keep, kept, flat = oracle.select_contour(hc, [g["t"]], [case["M"]], dm, g["tau"], g["flat_budget"],
                                                 g["floor"])
        assert flat.tolist() == g["expect_flat"]
        got = [keep[c, :len(g["slot_pos"][c])].tolist() for c in range(3)]
        assert got == case["keep"], case["M"]
        assert kept.tolist() == [sum(r) for r in case["keep"]]


def _contour_brute(hc, t, m_global, dm, tau, F, r):
    """The ContourKV rule by counting (no sort), straight from its readings."""
    ents = _entries(hc, t)
    keep = np.zeros((hc.C, hc.max_pages * hc.P), np.uint8)
    G = hc.G
    # float32 sum in ascending g order, then the binary32 division
    flat = []
    for c in range(hc.C):
        s = np.float32(0.0)
        for g in range(G):
            s = np.float32(s + np.float32(dm[c][g]))
        flat.append(bool(np.float32(s / np.float32(G)) > np.float32(tau)))
    floor = set()
    for e in ents:
        newer = sum(1 for f in ents if f[4] == e[4] and f[3] > e[3])
        if newer < r:
            floor.add((e[4], e[5]))
    forced = set(floor)
    for e in ents:
        if not flat[e[4]] or (e[4], e[5]) in floor:
            continue
        before = sum(1 for f in ents if f[4] == e[4] and (f[4], f[5]) not in floor
                     and (f[0] > e[0] or (f[0] == e[0] and f[3] < e[3])))
        if before < F:
            forced.add((e[4], e[5]))
    for b in range(hc.B):
        pool = [e for e in ents if e[6] == b and not flat[e[4]] and (e[4], e[5]) not in floor]
        n_forced = sum(1 for (c, k) in forced if c // (hc.L * hc.H) == b)
        m_rest = max(0, m_global[b] - n_forced)
        for e in pool:
            before = sum(1 for f in pool if f[0] > e[0] or (f[0] == e[0] and f[1:4] < e[1:4]))
            if before < m_rest:
                forced.add((e[4], e[5]))
    for (c, k) in forced:
        keep[c, k] = 1
    return keep, flat


@pytest.mark.parametrize("seed", range(4))
def test_contour_brute_force(seed):
    cfg, hc, rng = _small(10 + seed, ties=seed % 2 == 1)
    t = [cfg.T0] * cfg.B
    for trial in range(3):
        dm = rng.random((cfg.C, cfg.G)).astype(np.float32) * 0.5
        tau, F, r = float(rng.choice([0.1, 0.25, 0.4])), int(rng.integers(0, 8)), int(rng.integers(0, 6))
        n_b = [int(hc.len[b * 4:(b + 1) * 4].sum()) for b in range(cfg.B)]
        m = [int(rng.integers(0, x + 5)) for x in n_b]
        keep, kept, flat = oracle.select_contour(hc, t, m, dm, tau, F, r)
        want, want_flat = _contour_brute(hc, t, m, dm, tau, F, r)
        assert flat.astype(bool).tolist() == want_flat
        assert np.array_equal(keep, want), (seed, trial)


def test_contour_reduces_to_global_and_per_head_selection():
    cfg, hc, rng = _small(21, ties=False, B=1)
    t = [cfg.T0]
    n = int(hc.len.sum())
    dm = rng.random((cfg.C, cfg.G)).astype(np.float32)
    for m in (0, 5, n // 2, n):
        # no flat head and no floor: the global top-M
        k1, _, flat = oracle.select_contour(hc, t, [m], dm, math.inf, 7, 0)
        assert not flat.any()
        assert np.array_equal(k1, oracle.select(hc, t, [m])[0])
    # every head flat (dm >= 0 > -1) and no floor: each head's top-F
    for F in (0, 3, 29):
        k2, _, flat = oracle.select_contour(hc, t, [n], dm, -1.0, F, 0)
        assert flat.all()
        assert np.array_equal(k2, oracle.select_per_head(hc, t, [F] * cfg.C)[0])


def test_contour_floor_alone_keeps_most_recent():
    cfg, hc, rng = _small(22, ties=True, B=1)
    dm = np.zeros((cfg.C, cfg.G), np.float32)
    for r in (0, 1, 4, 100):
        keep, kept, _ = oracle.select_contour(hc, [cfg.T0], [0], dm, 1.0, 5, r)
        got = kept_positions(hc, keep)
        for c in range(cfg.C):
            pos = sorted((int(hc.pos_pool[hc.block_table[c, k // hc.P], k % hc.P]) for k in range(int(hc.len[c]))),
                         reverse=True)
            assert got[c] == set(pos[:r]), (r, c)
