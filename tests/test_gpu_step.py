"""GPU parity of the fused decode step (rkv_decode_step) against the oracle.

Every step is compared with oracle.step on the same seeded inputs: keep flags
and kept counts bit for bit, lengths / tables / free stack / pools bit for
bit, attention outputs within 2e-3 of the row norm and dropped mass within
1e-4.  The fused kernel decides most entries against a threshold window kept
from the previous call and falls back to an exact selection when the window
cannot decide; `WindowModel` follows the window from the oracle's thresholds
so the tests can also assert which path each step exercised (the results
must not depend on it).
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.gpu_helpers import assert_outputs_close, compare_state, keep_flags, masked_keep, rkv_cache, sync, to_dev
from tests.oracle_helpers import host_cache

pytestmark = pytest.mark.gpu

WIN_CAP = 1024
WIN_LO, WIN_HI = 16, 128   # a window that resolved its call doubles below WIN_LO candidates, halves above WIN_HI
WIN_OFF = 144   # byte offset of the threshold windows ([B][4] uint32) in the workspace


def score_keys(hc, t):
    """64-bit rank keys of every entry, per sequence: list of (keys[], head[], slot[])."""
    LH = hc.L * hc.H
    ib = 32 - int(np.ceil(np.log2(LH))) if LH > 1 else 32
    out = []
    for b in range(hc.B):
        ks, hs, ss = [], [], []
        for cl in range(LH):
            c = b * LH + cl
            n = int(hc.len[c])
            if n == 0:
                continue
            slots = np.arange(n)
            pages = hc.block_table[c, slots // 16]
            pos = hc.pos_pool[pages, slots % 16].astype(np.int64)
            lb = hc.lb_pool[pages, slots % 16].astype(np.float32)
            s = (np.float32(t[b]) - pos.astype(np.float32)).astype(np.float32) * lb   # exact age, one rounding
            s = np.where(s == 0, np.float32(0.0), s).astype(np.float32)
            u = s.view(np.uint32).astype(np.uint64)
            hi = np.where(u & 0x80000000, u, (~u) & 0x7FFFFFFF)
            lo = (np.uint64(cl) << np.uint64(ib)) | pos.astype(np.uint64) if ib < 32 else pos.astype(np.uint64)
            ks.append((hi << np.uint64(32)) | lo)
            hs.append(np.full(n, c))
            ss.append(slots)
        out.append((np.concatenate(ks) if ks else np.zeros(0, np.uint64),
                    np.concatenate(hs) if hs else np.zeros(0, int), np.concatenate(ss) if ss else np.zeros(0, int)))
    return out


class WindowModel:
    """The per-sequence threshold window of the fused kernel, replayed from
    the oracle's keys: predicts whether a call resolves in the window.

    Mirrors the kernel's rule: a resolved call halves the half width above
    WIN_HI candidates (not below the floor) and doubles it below WIN_LO; a
    miss quadruples it and sets the floor to twice the half width that
    missed; too many candidates quarter it and drop the floor.  After every
    call but an overflowing one the floor is also at least DRIFT_MARGIN times
    the threshold's move from the previous window's centre (power of two,
    capped at the half width where WIN_CAP/2 keys would fall inside at the
    density this call saw), and the half width is raised to the floor.  A
    first window is sized from the keys in the threshold's 1024-wide bucket
    of score keys (the exact selection's second radix pass) to hold about
    WIN_INIT keys, or 2^14 when the selection ended after one pass."""

    DRIFT_MARGIN, WIN_INIT = 4, 256

    def __init__(self, B):
        self.w = [None] * B        # (lo, hi) score-key range, or None
        self.hw = [0] * B
        self.floor = [0] * B       # half width the window does not shrink below

    @staticmethod
    def _h1(keys, thr, m):
        """Keys in the threshold's 1024-wide score-key bucket, or 0 when the
        radix selection ends after its first 11-bit digit (the threshold's
        bucket of that digit is kept whole)."""
        hi = (keys >> np.uint64(32)).astype(np.int64)
        t_hi = int(thr >> 32)
        d0 = hi >> 21
        h0 = int((d0 == (t_hi >> 21)).sum())
        below = int((d0 < (t_hi >> 21)).sum())
        if h0 == m - below:
            return 0
        return int(((hi >> 10) == (t_hi >> 10)).sum())

    def call(self, keys_by_seq, m):
        hits = []
        for b, (keys, _, _) in enumerate(keys_by_seq):
            n = len(keys)
            mb = max(0, min(int(m[b]), n))
            if mb == 0 or mb == n:
                hits.append(None)     # trivial: no window involved
                continue
            kap = int(np.sort(keys)[mb - 1]) + 1
            hi_words = (keys >> np.uint64(32)).astype(np.int64)
            wres = 0
            had = self.w[b] is not None
            if had:
                lo, hi = self.w[b]
                above = int((hi_words < lo).sum())
                nc = int(((hi_words >= lo) & (hi_words < hi)).sum())
                hit = nc <= WIN_CAP and above < mb <= above + nc
                wres = 1 if hit else (3 if nc > WIN_CAP else 2)
                hits.append(hit)
            else:
                hits.append(False)
                nc = 0
            center = (kap - 1) >> 32
            hw = self.hw[b]
            if hw == 0:
                hw = 1 << 14
                h1 = self._h1(keys, kap - 1, mb)
                if h1:
                    hw = 1
                    while hw < (1 << 20) and hw * h1 < self.WIN_INIT * 512:
                        hw <<= 1
            fl = self.floor[b]
            if had and wres != 3:
                lo, hi = self.w[b]
                old = lo + self.hw[b] if lo > 0 else hi - self.hw[b]
                d = abs(center - old)
                lim = 1 << 26
                if wres == 1 and nc > 0:
                    lim = min(lim, self.hw[b] * (WIN_CAP // 2) // nc)
                fd = 1
                while fd * 2 <= lim and fd < self.DRIFT_MARGIN * d:
                    fd <<= 1
                fl = max(fl, fd)
                hw = max(hw, fl)
            if wres == 1:
                if nc > WIN_HI:
                    if hw > 1 and (hw >> 1) >= fl:
                        hw >>= 1
                elif nc < WIN_LO and hw < (1 << 28):
                    hw <<= 1
            elif wres == 2:
                fl = hw << 1 if hw < (1 << 27) else (1 << 28)
                hw = hw << 2 if hw < (1 << 26) else (1 << 28)
            elif wres == 3:
                fl = 0
                hw = hw >> 2 if hw > 4 else 1
            self.floor[b] = fl
            self.w[b] = (center - hw if center > hw else 0, center + hw if center < 0xFFFFFFFF - hw else 0xFFFFFFFF)
            self.hw[b] = hw
        return hits

    def words(self, b):
        """The four window words the kernel keeps for sequence b."""
        lo, hi = self.w[b]
        fl = self.floor[b]
        return [1 | ((fl.bit_length() << 8) if fl else 0), lo, hi, self.hw[b]]


def run_fused(rkv, cfg, seed, steps, *, budgets=None, model=True, mutate=None):
    """Fused steps against oracle.step; returns the window model's hit list per step."""
    dc = to_dev(workloads.prefill_cache(cfg, seed, n_steps=steps + 1))
    hc = host_cache(dc)
    cache = rkv_cache(rkv, dc)
    sel = rkv.Selection.empty(cache)
    ws = rkv.Workspace(cache)
    outs = rkv.StepOutputs.empty(cache)
    wm = WindowModel(cfg.B)
    trace = []
    for s in range(steps):
        inp = workloads.step_inputs(cfg, seed, s, "cuda")
        if budgets is not None:
            inp["m_global"] = torch.tensor(budgets[s], dtype=torch.int64, device="cuda")
        if mutate is not None:
            mutate(s, dc, hc)
        t = inp["t"].cpu().numpy()
        mg = inp["m_global"].cpu().numpy()
        len_before = hc.len.copy()
        hc_prev = oracle.HostCache(**{f: (getattr(hc, f).copy() if isinstance(getattr(hc, f), np.ndarray) else getattr(hc, f))
                                      for f in hc.__dataclass_fields__})
        wm_prev = list(wm.w)
        if inp["evict"] and model:
            trace.append(wm.call(score_keys(hc, t), mg))
        c0 = ws.counters()
        win_before = ws.buf[WIN_OFF:WIN_OFF + 16 * cfg.B].view(torch.int32).cpu().numpy().view(np.uint32).reshape(cfg.B, 4)
        rkv.decode_step(cache, inp["t"], inp["m_global"] if inp["evict"] else None, inp["q"], cfg.scale,
                        inp["k_new"], inp["v_new"], inp["lb_new"], sel if inp["evict"] else None, outs.out, outs.lse,
                        outs.dropped, ws)
        sync()
        c1 = ws.counters()
        assert c1["status"] == 0, f"step {s}: device status {c1}"
        if inp["evict"] and model:
            # the path the kernel took is the one the window model predicts
            window = all(h is not False for h in trace[-1])
            took = (c1["window_steps"] - c0["window_steps"], c1["exact_steps"] - c0["exact_steps"])
            if took != ((1, 0) if window else (0, 1)):
                info = []
                for b, (keys, _, _) in enumerate(score_keys(hc_prev, t)):
                    hw_ = (keys >> np.uint64(32)).astype(np.int64)
                    lo, hi = int(win_before[b, 1]), int(win_before[b, 2])
                    info.append(dict(kernel_win=win_before[b].tolist(), model_win=wm_prev[b], n=len(keys), m=int(mg[b]),
                                     above=int((hw_ < lo).sum()), nc=int(((hw_ >= lo) & (hw_ < hi)).sum())))
                raise AssertionError(f"step {s}: took {took}, model {trace[-1]}: {info}")
            win_after = ws.buf[WIN_OFF:WIN_OFF + 16 * cfg.B].view(torch.int32).cpu().numpy().view(np.uint32).reshape(cfg.B, 4)
            for b in range(cfg.B):
                if wm.w[b] is not None:
                    assert win_after[b].tolist() == wm.words(b), f"step {s}: window of sequence {b}"
        ref = oracle.step(hc, t, mg, inp["q"].cpu().numpy().reshape(cfg.C, cfg.G, cfg.D),
                          workloads.rows_to_host(inp["k_new"]), workloads.rows_to_host(inp["v_new"]),
                          inp["lb_new"].cpu().numpy(), evict=inp["evict"], scale=cfg.scale)
        if inp["evict"]:
            keep_g = masked_keep(keep_flags(sel, dc.max_pages), len_before)
            assert np.array_equal(sel.kept.cpu().numpy(), ref["kept"]), f"step {s}: kept"
            assert np.array_equal(sel.n_pre.cpu().numpy(), len_before), f"step {s}: n_pre"
            assert np.array_equal(keep_g, ref["keep"]), f"step {s}: keep flags at {np.argwhere(keep_g != ref['keep'])[:5].tolist()}"
            kept_any = ref["kept"] > 0
        else:
            kept_any = len_before > 0
        assert_outputs_close(outs.out.cpu().numpy().reshape(cfg.C, cfg.G, cfg.D),
                             outs.lse.cpu().numpy().reshape(cfg.C, cfg.G),
                             outs.dropped.cpu().numpy().reshape(cfg.C, cfg.G), ref["out"], ref["lse"],
                             ref["dropped"], kept_any)
        compare_state(dc, hc)
    return trace


def _hits(trace):
    return sum(1 for step in trace for h in step if h)


def test_fused_tiny_config(rkv):
    run_fused(rkv, workloads.CONFIGS["tiny"], 0, 4)


def test_fused_steady_steps_resolve_in_the_window(rkv):
    cfg = workloads.small_config(L=2, H=4, G=4, D=128, B=1, T0=3000, M=4000, kv_dtype="bf16", steps=10)
    trace = run_fused(rkv, cfg, 1, 10)
    assert trace[0] == [False]          # first call: no window yet, exact path
    assert _hits(trace) >= 6, trace     # then the window decides


@pytest.mark.parametrize("G,D", [(1, 64), (2, 64), (4, 64), (1, 128), (2, 128), (7, 128), (8, 128)])
def test_fused_shapes(rkv, G, D):
    cfg = workloads.small_config(L=2, H=2, G=G, D=D, B=1, T0=1500, M=1400, kv_dtype="bf16", steps=5)
    run_fused(rkv, cfg, 10 + G, 5)


@pytest.mark.parametrize("G,D", [(1, 64), (4, 64), (2, 128), (4, 128)])
def test_fused_fp32_pools(rkv, G, D):
    cfg = workloads.small_config(L=2, H=2, G=G, D=D, B=1, T0=700, M=900, kv_dtype="f32", steps=4)
    run_fused(rkv, cfg, 20 + G, 4)


def test_fused_batched_sequences(rkv):
    cfg = workloads.small_config(L=2, H=2, G=4, D=128, B=5, T0=1200, M=1500, kv_dtype="bf16", steps=6)
    trace = run_fused(rkv, cfg, 4, 6)
    assert _hits(trace) >= 10, trace


@pytest.mark.parametrize("dtype,G,D", [("bf16", 4, 128), ("f32", 2, 64)])
def test_fused_head_per_warp(rkv, dtype, G, D):
    # enough short heads that every CTA's range holds at least eight of them:
    # each consumer warp takes whole heads (prefill eviction, evicting and
    # non-evicting steps, heads split across CTAs)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    L, H = 12, 8
    B = min(16, -(-10 * sms // (L * H)))
    cfg = workloads.small_config(L=L, H=H, G=G, D=D, B=B, T0=300, M=L * H * 220, kv_dtype=dtype, steps=6,
                                 evict_every=2)
    run_fused(rkv, cfg, 31 + G, 6)


def test_fused_non_evicting_steps_between_evictions(rkv):
    cfg = workloads.small_config(L=2, H=2, G=4, D=128, B=2, T0=1000, M=1500, kv_dtype="bf16", steps=12,
                                 evict_every=3)
    run_fused(rkv, cfg, 3, 12)


def test_fused_budget_jumps_miss_the_window(rkv):
    # budgets far from the previous threshold: the window misses and the exact
    # path runs inside the same launch; trivial budgets (0, all) in between
    cfg = workloads.small_config(L=2, H=3, G=2, D=128, B=2, T0=2500, M=3000, kv_dtype="bf16", steps=9)
    n = 2 * 3 * 2500
    budgets = [[3000, 3000], [3001, 2990], [9000, 500], [9001, 510], [0, n + 9], [4000, 4000], [4002, n + 20],
               [1, 2], [4100, 4100]]
    trace = run_fused(rkv, cfg, 5, 9, budgets=budgets)
    flat = [h for step in trace for h in step]
    assert False in flat and True in flat, trace


def test_fused_window_overflow_with_ties(rkv):
    # log-retentions from a two-value set: thousands of exact score ties
    # crowd the window (more than it can rank), forcing the exact path
    cfg = workloads.small_config(L=2, H=4, G=1, D=64, B=1, T0=4000, M=9000, kv_dtype="bf16", steps=4)

    def ties(s, dc, hc):
        if s == 1:
            few = torch.tensor([-0.5, -0.25], dtype=torch.float32, device="cuda")
            g = torch.Generator(device="cuda").manual_seed(5)
            dc.lb_pool.copy_(few[torch.randint(0, 2, dc.lb_pool.shape, device="cuda", generator=g)])
            hc.lb_pool[...] = dc.lb_pool.cpu().numpy()

    run_fused(rkv, cfg, 6, 4, mutate=ties)


def test_fused_matches_separate_calls(rkv):
    # the same steps through the separate entry points and through the fused
    # launch: every integer output and the whole cache state are identical
    cfg = workloads.small_config(L=3, H=2, G=4, D=128, B=2, T0=2000, M=2500, kv_dtype="bf16", steps=6)
    a = to_dev(workloads.prefill_cache(cfg, 8, n_steps=7))
    b = to_dev(workloads.prefill_cache(cfg, 8, n_steps=7))
    ca, cb = rkv_cache(rkv, a), rkv_cache(rkv, b)
    sa, sb = rkv.Selection.empty(ca), rkv.Selection.empty(cb)
    wa, wb = rkv.Workspace(ca), rkv.Workspace(cb)
    oa, ob = rkv.StepOutputs.empty(ca), rkv.StepOutputs.empty(cb)
    for s in range(6):
        inp = workloads.step_inputs(cfg, 8, s, "cuda")
        kw = dict(q=inp["q"], t=inp["t"], m_global=inp["m_global"], k_new=inp["k_new"], v_new=inp["v_new"],
                  lb_new=inp["lb_new"], evict=inp["evict"], scale=cfg.scale)
        rkv.step(ca, sa, wa, oa, fused=False, **kw)
        rkv.step(cb, sb, wb, ob, fused=True, **kw)
        sync()
        for name in ("kappa", "kept", "n_pre", "plan"):
            assert torch.equal(getattr(sa, name), getattr(sb, name)), f"step {s}: {name}"
        assert np.array_equal(masked_keep(keep_flags(sa, a.max_pages), sa.n_pre.cpu().numpy()),
                              masked_keep(keep_flags(sb, b.max_pages), sb.n_pre.cpu().numpy()))
        for name in ("len", "block_table", "pos_pool", "k_pool", "v_pool"):
            assert torch.equal(getattr(a, name), getattr(b, name)), f"step {s}: {name}"
        assert torch.equal(a.lb_pool.view(torch.int32), b.lb_pool.view(torch.int32))
        top = int(a.free_top.item())
        assert top == int(b.free_top.item())
        assert torch.equal(a.free_stack[:top], b.free_stack[:top])
        assert torch.allclose(oa.out, ob.out, rtol=0, atol=1e-4)
        assert torch.allclose(oa.dropped, ob.dropped, rtol=0, atol=1e-5)
    assert wa.status() == 0 and wb.status() == 0


def test_fused_empty_and_ragged_heads(rkv):
    cfg = workloads.small_config(L=1, H=5, G=4, D=128, B=1, T0=900, kv_dtype="bf16")
    lengths = [0, 1, 17, 899, 160]
    dc = to_dev(workloads.ragged_cache(cfg, 12, lengths, n_pages=200))
    hc = host_cache(dc)
    cache = rkv_cache(rkv, dc)
    sel = rkv.Selection.empty(cache)
    ws = rkv.Workspace(cache)
    outs = rkv.StepOutputs.empty(cache)
    for s, m in enumerate([700, 650, 651, 1077, 0, 300]):
        inp = workloads.step_inputs(cfg, 12, s, "cuda")
        t = np.array([900 + s], np.int32)
        tt = torch.tensor(t, device="cuda")
        mm = torch.tensor([m], dtype=torch.int64, device="cuda")
        len_before = hc.len.copy()
        rkv.decode_step(cache, tt, mm, inp["q"], cfg.scale, inp["k_new"], inp["v_new"], inp["lb_new"], sel,
                        outs.out, outs.lse, outs.dropped, ws)
        sync()
        assert ws.status() == 0
        ref = oracle.step(hc, t, np.array([m]), inp["q"].cpu().numpy().reshape(cfg.C, cfg.G, cfg.D),
                          workloads.rows_to_host(inp["k_new"]), workloads.rows_to_host(inp["v_new"]),
                          inp["lb_new"].cpu().numpy(), evict=True, scale=cfg.scale)
        assert np.array_equal(sel.kept.cpu().numpy(), ref["kept"])
        assert np.array_equal(masked_keep(keep_flags(sel, dc.max_pages), len_before), ref["keep"])
        assert_outputs_close(outs.out.cpu().numpy().reshape(cfg.C, cfg.G, cfg.D),
                             outs.lse.cpu().numpy().reshape(cfg.C, cfg.G),
                             outs.dropped.cpu().numpy().reshape(cfg.C, cfg.G), ref["out"], ref["lse"],
                             ref["dropped"], ref["kept"] > 0)
        compare_state(dc, hc)


def _edge_cache(rkv, seed):
    """L=1, H=3 (position field 30 bits wide), heads of 40, 150 and 300
    entries; the 300-entry head holds every position in [0, 300)."""
    cfg = workloads.small_config(L=1, H=3, G=2, D=64, B=1, T0=300, kv_dtype="bf16")
    dc = to_dev(workloads.ragged_cache(cfg, seed, [40, 150, 300], n_pages=64))
    return cfg, dc


def _set_pos(dc, c, k, pos):
    dc.pos_pool[int(dc.block_table[c, k // 16]), k % 16] = pos


@pytest.mark.parametrize("case", ["ages", "positions"])
def test_fused_exact_path_key_edges(rkv, case):
    # entries exactly at the edges of the scorable range are scored, on the
    # first call (the exact selection): ages 1 and 2^24 - 1 with position 0,
    # or positions up to 2^30 - 1, the widest that fits beside the head
    # index when L*H = 3
    cfg, dc = _edge_cache(rkv, 21)
    if case == "ages":
        t = (1 << 24) - 1            # the entry at position 0 has age 2^24 - 1
        _set_pos(dc, 0, 0, t - 1)    # age 1
    else:
        dc.pos_pool += (1 << 30) - 300   # the 300-entry head now ends at 2^30 - 1
        t = (1 << 30) + 5
    hc = host_cache(dc)
    cache = rkv_cache(rkv, dc)
    sel, ws, outs = rkv.Selection.empty(cache), rkv.Workspace(cache), rkv.StepOutputs.empty(cache)
    inp = workloads.step_inputs(cfg, 21, 0, "cuda")
    tt = np.array([t], np.int32)
    len_before = hc.len.copy()
    rkv.decode_step(cache, torch.tensor(tt, device="cuda"), torch.tensor([200], dtype=torch.int64, device="cuda"),
                    inp["q"], cfg.scale, inp["k_new"], inp["v_new"], inp["lb_new"], sel, outs.out, outs.lse,
                    outs.dropped, ws)
    sync()
    c = ws.counters()
    assert c["status"] == 0 and c["exact_steps"] == 1, c
    ref = oracle.step(hc, tt, np.array([200]), inp["q"].cpu().numpy().reshape(cfg.C, cfg.G, cfg.D),
                      workloads.rows_to_host(inp["k_new"]), workloads.rows_to_host(inp["v_new"]),
                      inp["lb_new"].cpu().numpy(), evict=True, scale=cfg.scale)
    assert np.array_equal(sel.kept.cpu().numpy(), ref["kept"])
    assert np.array_equal(masked_keep(keep_flags(sel, dc.max_pages), len_before), ref["keep"])
    assert_outputs_close(outs.out.cpu().numpy().reshape(cfg.C, cfg.G, cfg.D),
                         outs.lse.cpu().numpy().reshape(cfg.C, cfg.G),
                         outs.dropped.cpu().numpy().reshape(cfg.C, cfg.G), ref["out"], ref["lse"],
                         ref["dropped"], ref["kept"] > 0)
    compare_state(dc, hc)


@pytest.mark.parametrize("kind", ["nan", "age0", "age2^24", "negative", "past_field"])
def test_fused_exact_path_flags_unscorable_entry(rkv, kind):
    # one entry the method cannot score (head 1, slot 5), every other entry
    # valid: the first call's exact selection flags RKV_DEV_BAD_INPUT,
    # finishes, and keeps nothing of that entry
    cfg, dc = _edge_cache(rkv, 22)
    t = cfg.T0 + 5
    if kind == "nan":
        dc.lb_pool[int(dc.block_table[1, 0]), 5] = float("nan")
    elif kind == "age0":
        _set_pos(dc, 1, 5, t)
    elif kind == "age2^24":
        dc.pos_pool += 1000
        t = (1 << 24) + 999
        _set_pos(dc, 1, 5, 999)
    elif kind == "negative":
        _set_pos(dc, 1, 5, -5)
    else:
        dc.pos_pool += (1 << 30) - 300
        t = (1 << 30) + 5
        _set_pos(dc, 1, 5, 1 << 30)      # age 5, but past the 30-bit position field
    cache = rkv_cache(rkv, dc)
    sel, ws, outs = rkv.Selection.empty(cache), rkv.Workspace(cache), rkv.StepOutputs.empty(cache)
    inp = workloads.step_inputs(cfg, 22, 0, "cuda")
    rkv.decode_step(cache, torch.tensor([t], dtype=torch.int32, device="cuda"),
                    torch.tensor([200], dtype=torch.int64, device="cuda"), inp["q"], cfg.scale, inp["k_new"],
                    inp["v_new"], inp["lb_new"], sel, outs.out, outs.lse, outs.dropped, ws)
    sync()
    assert ws.status() & rkv.DEV_BAD_INPUT
    assert keep_flags(sel, dc.max_pages)[1, 5] == 0
    rkv.workspace_init(ws)
    sync()
    assert ws.status() == 0


def test_fused_graph_replay(rkv):
    # the fused step captured once in a CUDA graph and replayed on new inputs
    cfg = workloads.small_config(L=2, H=2, G=4, D=128, B=1, T0=1500, M=2000, kv_dtype="bf16", steps=6)
    dc = to_dev(workloads.prefill_cache(cfg, 9, n_steps=7))
    hc = host_cache(dc)
    runner = rkv.StepRunner(rkv_cache(rkv, dc), scale=cfg.scale, fused=True, stream=torch.cuda.Stream())
    for s in range(6):
        inp = workloads.step_inputs(cfg, 9, s, "cuda")
        for k in ("q", "k_new", "v_new", "lb_new", "t", "m_global"):
            runner.inp[k].copy_(inp[k].reshape(runner.inp[k].shape))
        sync()   # inputs written on the default stream, the step runs on the runner's
        if s == 0:
            runner.run(True)         # first (exact) call eagerly, then capture
            sync()
            assert runner.capture(), runner.capture_error
        else:
            runner.run(True)
        sync()
        ref = oracle.step(hc, inp["t"].cpu().numpy(), inp["m_global"].cpu().numpy(),
                          inp["q"].cpu().numpy().reshape(cfg.C, cfg.G, cfg.D), workloads.rows_to_host(inp["k_new"]),
                          workloads.rows_to_host(inp["v_new"]), inp["lb_new"].cpu().numpy(), evict=True,
                          scale=cfg.scale)
        assert np.array_equal(runner.sel.kept.cpu().numpy(), ref["kept"])
        assert_outputs_close(runner.outs.out.cpu().numpy().reshape(cfg.C, cfg.G, cfg.D),
                             runner.outs.lse.cpu().numpy().reshape(cfg.C, cfg.G),
                             runner.outs.dropped.cpu().numpy().reshape(cfg.C, cfg.G), ref["out"], ref["lse"],
                             ref["dropped"], ref["kept"] > 0)
        compare_state(dc, hc)
    assert runner.ws.status() == 0


def test_runner_two_buffer_slots_match_one(rkv):
    # run_host with two buffer slots (copies overlapped with the neighbouring
    # steps on a second stream) gives the same outputs and cache as one slot
    cfg = workloads.small_config(L=2, H=2, G=4, D=128, B=2, T0=1500, M=2500, kv_dtype="bf16", steps=8,
                                 evict_every=2)
    dcs = [to_dev(workloads.prefill_cache(cfg, 12, n_steps=9)) for _ in range(2)]
    runners = [rkv.StepRunner(rkv_cache(rkv, dc), scale=cfg.scale, fused=True, stream=torch.cuda.Stream(),
                              buffers=nb) for dc, nb in zip(dcs, (1, 2))]
    steps = [workloads.step_inputs(cfg, 12, s, "cuda") for s in range(8)]
    outs = [[], []]
    for r, runner in enumerate(runners):
        host_in = [torch.empty(runner.in_bytes, dtype=torch.uint8, pin_memory=True) for _ in steps]
        host_out = [torch.zeros(runner.out_bytes, dtype=torch.uint8, pin_memory=True) for _ in steps]
        for s, inp in enumerate(steps):
            runner.pack(host_in[s], q=inp["q"].cpu(), k_new=inp["k_new"].cpu(), v_new=inp["v_new"].cpu(),
                        lb_new=inp["lb_new"].cpu(), t=inp["t"].cpu(), m_global=inp["m_global"].cpu())
        runner.run_host(host_in[0], host_out[0], bool(steps[0]["evict"]))   # exact first call, eager
        runner.finish()
        sync()
        assert runner.capture(), runner.capture_error
        for s in range(1, len(steps)):
            runner.run_host(host_in[s], host_out[s], bool(steps[s]["evict"]))
        runner.finish()
        sync()
        assert runner.ws.status() == 0
        outs[r] = [runner.unpack(h) for h in host_out]
    for s in range(len(steps)):
        for k in ("out", "lse", "dropped"):
            # (the order in which candidates enter a merge can differ between
            # runs, so the sums may differ in the last bits)
            np.testing.assert_allclose(outs[1][s][k].numpy(), outs[0][s][k].numpy(), rtol=1e-5, atol=1e-6,
                                       err_msg=f"step {s}: {k}")
    for name in ("len", "block_table", "k_pool", "v_pool", "pos_pool", "free_top"):
        assert torch.equal(getattr(dcs[0], name), getattr(dcs[1], name)), name
