"""Pins of the oracle's physical compaction, free-page stack and append.

Trust the Mass (ContourKV), Methodology 2: the budget is enforced physically
(ragged storage), not by masking a full cache.  Make Each Token Count
(DBTrimKV), Methodology 4: paged layout with a variable length per head.  The
hole-fill pairing and free-stack order are this library's own rule and are
pinned by a hand-worked fixture.
"""
import numpy as np
import pytest

import oracle
import workloads
from tests.oracle_helpers import (all_positions, hand_cache, host_cache, kept_positions, load_golden,
                                  slot_values)


def _golden_cache(g):
    return hand_cache(g["B"], g["L"], g["H"], g["G"], g["D"], g["P"], g["n_pages"], g["max_pages"],
                      g["block_table"], g["len"], g["slot_pos"],
                      [[-0.01 * (p % 7 + 1) for p in row] for row in g["slot_pos"]],
                      free_stack=g["free_stack"][: g["free_top"]], free_top=g["free_top"],
                      kv_fn=lambda c, p: ([float(p), -float(p)], [p + 0.5, 1.0]))


def test_golden_compaction_then_appends():
    g = load_golden("compact_append_two_heads.json")
    hc = _golden_cache(g)
    keep = np.zeros((2, g["max_pages"] * g["P"]), np.uint8)
    for c in range(2):
        keep[c, : len(g["keep"][c])] = g["keep"][c]
    oracle.compact(hc, keep)
    a = g["after_compact"]
    assert hc.block_table.tolist() == a["block_table"]
    assert hc.len.tolist() == a["len"]
    assert int(hc.free_top[0]) == a["free_top"]
    assert hc.free_stack[: a["free_top"]].tolist() == a["free_stack_prefix"]
    for c in range(2):
        pos = [int(x) for x in slot_values(hc, c, hc.pos_pool)]
        assert pos == a["slot_pos"][c]
        ks = slot_values(hc, c, hc.k_pool)
        assert [list(map(float, r)) for r in ks] == [[float(p), -float(p)] for p in pos]   # rows moved whole
        lbs = [float(x) for x in slot_values(hc, c, hc.lb_pool)]
        assert lbs == [float(np.float32(-0.01 * (p % 7 + 1))) for p in pos]
    for ap in g["appends"]:
        k_new = np.array([[ap["t"], 0.0], [0.0, ap["t"]]], np.float32)
        rc = oracle.append(hc, [ap["t"]], k_new, k_new + 1, np.array(ap["lb_new"], np.float32))
        assert rc == oracle.OK
    z = g["after_appends"]
    assert hc.block_table.tolist() == z["block_table"]
    assert hc.len.tolist() == z["len"]
    assert int(hc.free_top[0]) == z["free_top"]
    assert hc.free_stack[: z["free_top"]].tolist() == z["free_stack_prefix"]
    for c in range(2):
        assert [int(x) for x in slot_values(hc, c, hc.pos_pool)] == z["slot_pos"][c]
        tail = [float(x) for x in slot_values(hc, c, hc.lb_pool)][-3:]
        assert tail == z["slot_lb_tail"][c]


@pytest.mark.parametrize("seed", range(4))
def test_compaction_invariants_random(seed):
    cfg = workloads.small_config(L=2, H=3, G=1, D=8, B=2, T0=150, kv_dtype="bf16")
    rng = np.random.default_rng(seed)
    dc = workloads.ragged_cache(cfg, seed, rng.integers(0, 100, size=cfg.C))
    hc = host_cache(dc)
    before = hc.copy()
    t = [150, 150]
    totals = [int(hc.len[b * 6:(b + 1) * 6].sum()) for b in range(2)]
    keep, kept = oracle.select(hc, t, [totals[0] // 3, totals[1] // 2])
    want_sets = kept_positions(hc, keep)
    # rows by position before compaction
    rows_before = []
    for c in range(cfg.C):
        d = {}
        for k in range(int(hc.len[c])):
            page, off = hc.block_table[c, k // hc.P], k % hc.P
            d[int(hc.pos_pool[page, off])] = (hc.k_pool[page, off].copy(), hc.v_pool[page, off].copy(),
                                              float(hc.lb_pool[page, off]))
        rows_before.append(d)
    oracle.compact(hc, keep)
    assert hc.len.tolist() == kept.tolist()
    assert all_positions(hc) == want_sets                     # decoding gives exactly the kept set
    for c in range(cfg.C):
        n_new, n_old = int(kept[c]), int(before.len[c])
        keep_pages = -(-n_new // hc.P)
        assert np.array_equal(hc.block_table[c, :keep_pages], before.block_table[c, :keep_pages])
        assert np.all(hc.block_table[c, keep_pages:] == -1)
        for k in range(n_new):
            page, off = hc.block_table[c, k // hc.P], k % hc.P
            kr, vr, lb = rows_before[c][int(hc.pos_pool[page, off])]
            assert np.array_equal(hc.k_pool[page, off], kr) and np.array_equal(hc.v_pool[page, off], vr)
            assert float(hc.lb_pool[page, off]) == lb
    # every page is in exactly one head table or on the free stack
    used = [p for c in range(cfg.C) for p in hc.block_table[c] if p >= 0]
    stack = hc.free_stack[: hc.free_top[0]].tolist()
    assert sorted(used + stack) == list(range(hc.n_pages))
    # pushes are appended on top of the old stack
    old_top = int(before.free_top[0])
    assert hc.free_stack[:old_top].tolist() == before.free_stack[:old_top].tolist()


def test_prefill_then_append_pops_ascending_pages():
    cfg = workloads.Config("p", L=1, H=3, Hq=3, D=4, B=1, T0=32, M=10, steps=20, kv_dtype="f32")
    hc = host_cache(workloads.prefill_cache(cfg, 0, n_steps=20))
    first_free = cfg.C * 2
    for s in range(3):
        t = cfg.T0 + s
        assert oracle.append(hc, [t], np.zeros((3, 4), np.float32), np.zeros((3, 4), np.float32),
                             np.full(3, -0.5, np.float32)) == oracle.OK
    # T0 = 32 is a page multiple: the first append of each head takes a page,
    # heads in ascending order, pages popped in ascending id
    assert hc.block_table[:, 2].tolist() == [first_free, first_free + 1, first_free + 2]
    for c in range(3):
        assert [int(x) for x in slot_values(hc, c, hc.pos_pool)][-3:] == [32, 33, 34]


def test_append_reports_pool_exhaustion():
    cfg = workloads.small_config(L=1, H=2, G=1, D=4, B=1, T0=40, kv_dtype="f32")
    dc = workloads.ragged_cache(cfg, 0, [16, 32], n_pages=3)   # 1 + 2 pages used, none free
    hc = host_cache(dc)
    z = np.zeros((2, 4), np.float32)
    assert oracle.append(hc, [40], z, z, np.zeros(2, np.float32)) == oracle.ERR_POOL


def test_golden_multi_page_free_order():
    g = load_golden("compact_append_two_heads.json")["multi_page_case"]
    hc = _golden_cache(g)
    keep = np.zeros((1, g["max_pages"] * g["P"]), np.uint8)
    keep[0, : len(g["keep"][0])] = g["keep"][0]
    oracle.compact(hc, keep)
    a = g["after_compact"]
    assert hc.block_table.tolist() == a["block_table"]
    assert hc.len.tolist() == a["len"]
    assert hc.free_stack[: a["free_top"]].tolist() == a["free_stack_prefix"]
    assert [int(x) for x in slot_values(hc, 0, hc.pos_pool)] == a["slot_pos"][0]
