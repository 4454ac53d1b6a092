"""Pins of the oracle's global top-M_global selection.

Make Each Token Count (DBTrimKV), Methodology 3: one global budget M_global,
every cached entry of all layers and heads ranked together, the top M_global
kept.  Cache What Lasts (TRIM-KV), core mechanism 4: the lowest beta^(t-i)
are evicted.  Tie rule: ascending (layer, kv head, position).
"""
import itertools

import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.oracle_helpers import hand_cache, host_cache, kept_positions, load_golden


def test_golden_hand_worked_ties():
    g = load_golden("select_ties.json")
    P = g["P"]
    table = [[0, -1], [1, -1]]
    hc = hand_cache(g["B"], g["L"], g["H"], 1, 4, P, 4, 2, table,
                    [len(x) for x in g["slot_pos"]], g["slot_pos"], g["slot_lb"])
    for c in range(2):
        s, ok = oracle.score([g["t"]] * 4, g["slot_pos"][c], g["slot_lb"][c])
        assert ok.all() and s.tolist() == g["expect_scores"][c]
    for case in g["cases"]:
        keep, kept = oracle.select(hc, [g["t"]], [case["M"]])
        got = [keep[c, :4].tolist() for c in range(2)]
        assert got == case["keep"], case["M"]
        assert kept.tolist() == [sum(r) for r in case["keep"]]


def _brute_force_keep(hc, t, m_global):
    """Entry e is kept iff fewer than M entries of its sequence rank before
    it: pairwise counting (no sort), scores by numpy binary32 multiply."""
    keep = np.zeros((hc.C, hc.max_pages * hc.P), np.uint8)
    for b in range(hc.B):
        ents = []
        for l, h in itertools.product(range(hc.L), range(hc.H)):
            c = (b * hc.L + l) * hc.H + h
            for k in range(int(hc.len[c])):
                page = hc.block_table[c, k // hc.P]
                i = int(hc.pos_pool[page, k % hc.P])
                s = np.float32(np.float32(t[b] - i) * hc.lb_pool[page, k % hc.P])
                ents.append((float(s), l, h, i, c, k))
        for e in ents:
            before = sum(1 for f in ents if f[0] > e[0] or (f[0] == e[0] and f[1:4] < e[1:4]))
            if before < m_global[b]:
                keep[e[4], e[5]] = 1
    return keep


@pytest.mark.parametrize("seed", range(6))
def test_brute_force_small_random(seed):
    rng = np.random.default_rng(seed)
    cfg = workloads.small_config(L=2, H=2, G=1, D=8, B=2, T0=60, kv_dtype="f32")
    lengths = rng.integers(0, 30, size=cfg.C)
    dc = workloads.ragged_cache(cfg, seed, lengths)
    if seed % 2 == 0:  # force exact ties: a few distinct log-retentions only
        choices = torch.tensor([-0.5, -0.25, -1.0, -2.0 ** -7], dtype=torch.float32)
        idx = torch.from_numpy(rng.integers(0, 4, size=dc.lb_pool.numel()))
        dc.lb_pool = choices[idx].view_as(dc.lb_pool).clone()
    hc = host_cache(dc)
    t = [60, 60]
    n_total = [int(hc.len[b * 4:(b + 1) * 4].sum()) for b in range(2)]
    for m in sorted({0, 1, 7, n_total[0] // 2, n_total[0] - 1, n_total[0], n_total[0] + 5}):
        mg = [m, max(0, n_total[1] - m)]
        keep, kept = oracle.select(hc, t, mg)
        want = _brute_force_keep(hc, t, mg)
        assert np.array_equal(keep, want), (seed, m)
        for b in range(2):
            assert kept[b * 4:(b + 1) * 4].sum() == min(max(mg[b], 0), n_total[b])


def test_constant_beta_closed_form():
    # Constant log beta = c < 0 and every head holding positions 0..T0-1:
    # distinct ages give distinct scores, so with M = k*L*H + r the k most
    # recent positions of every head are kept, plus position T0-k-1 in the
    # first r heads in ascending (l, h).
    cfg = workloads.Config("const", L=3, H=2, Hq=2, D=4, B=1, T0=40, M=0, steps=1, kv_dtype="f32",
                           mix=((1.0, ("const", 0.9)),))
    dc = workloads.prefill_cache(cfg, 0)
    hc = host_cache(dc)
    LH = cfg.L * cfg.H
    t = cfg.T0
    for M in (0, 1, 5, 6, 7, 13, 17, 60, LH * cfg.T0 - 1, LH * cfg.T0):
        keep, kept = oracle.select(hc, [t], [M])
        k, r = divmod(M, LH)
        got = kept_positions(hc, keep)
        for c in range(LH):
            want = set(range(cfg.T0 - k, cfg.T0))
            if c < r and k < cfg.T0:
                want.add(cfg.T0 - k - 1)
            assert got[c] == want, (M, c)


def test_budget_at_least_total_keeps_everything_and_nesting():
    cfg = workloads.small_config(L=2, H=3, G=1, D=8, B=1, T0=120, kv_dtype="f32")
    rng = np.random.default_rng(5)
    dc = workloads.ragged_cache(cfg, 5, rng.integers(0, 50, size=cfg.C))
    hc = host_cache(dc)
    n = int(hc.len.sum())
    keep_all, kept_all = oracle.select(hc, [120], [n])
    assert kept_all.tolist() == hc.len.tolist()
    keep_more, _ = oracle.select(hc, [120], [n + 1000])
    assert np.array_equal(keep_all, keep_more)
    prev = np.zeros_like(keep_all)
    for M in range(0, n + 1):
        keep, kept = oracle.select(hc, [120], [M])
        assert int(kept.sum()) == M
        assert np.all(keep >= prev), M          # kept(M-1) is a subset of kept(M)
        assert int((keep.astype(int) - prev).sum()) == (1 if M > 0 else 0)
        prev = keep


def test_sequences_are_independent():
    cfg = workloads.small_config(L=2, H=2, G=1, D=8, B=3, T0=80, kv_dtype="f32")
    rng = np.random.default_rng(9)
    dc = workloads.ragged_cache(cfg, 9, rng.integers(0, 40, size=cfg.C))
    hc = host_cache(dc)
    t = [80, 80, 80]
    keep, _ = oracle.select(hc, t, [10, 25, 3])
    for b, M in enumerate((10, 25, 3)):
        ms = [0, 0, 0]
        ms[b] = M
        kb, _ = oracle.select(hc, t, ms)
        sl = slice(b * 4, (b + 1) * 4)
        assert np.array_equal(keep[sl], kb[sl])


def test_invalid_entries_refused():
    cfg = workloads.small_config(L=1, H=2, G=1, D=8, B=1, T0=30, kv_dtype="f32")
    dc = workloads.ragged_cache(cfg, 1, [5, 5])
    dc.lb_pool[dc.block_table[0, 0], 0] = float("nan")
    with pytest.raises(ValueError):
        oracle.select(host_cache(dc), [30], [3])
    dc2 = workloads.ragged_cache(cfg, 1, [5, 5])
    with pytest.raises(ValueError):  # some position equals t -> age 0
        oracle.select(host_cache(dc2), [int(dc2.pos_pool.max())], [3])
