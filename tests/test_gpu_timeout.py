"""The device-timeout path, run on purpose without any hang.

With a wait limit of 1 microsecond on the workspace, the CTAs of a launch
give up at their first grid-wide barrier (the others have not arrived
yet), record RKV_DEV_TIMEOUT and the wait's site code, and leave the kernel;
nothing waits for ever.  After rkv_workspace_init (which also restores the
default limit) a normal call on a restored cache gives the oracle's results
bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.gpu_helpers import compare_state, keep_flags, masked_keep, rkv_cache, sync, to_dev
from tests.oracle_helpers import host_cache

pytestmark = pytest.mark.gpu


def _fresh(cfg, seed):
    dc = to_dev(workloads.prefill_cache(cfg, seed, n_steps=4))
    return dc, dc.clone()


def _timed_out(ws, rkv):
    c = ws.counters()
    return (c["status"] & rkv.DEV_TIMEOUT) != 0 and c["timeout_site"] != 0


def test_select_times_out_then_recovers(rkv):
    cfg = workloads.small_config(L=32, H=8, G=4, D=128, B=1, T0=4000, M=200000, kv_dtype="bf16")
    dc, backup = _fresh(cfg, 3)
    cache = rkv_cache(rkv, dc)
    sel, ws = rkv.Selection.empty(cache), rkv.Workspace(cache)
    inp = workloads.step_inputs(cfg, 3, 0, "cuda")
    rkv.workspace_set_wait_limit(ws, 1)
    rkv.score_select(cache, inp["t"], inp["m_global"], sel, ws)
    sync()
    assert _timed_out(ws, rkv), ws.counters()
    # re-initialise the workspace (default limit again) and select on the intact cache
    rkv.workspace_init(ws)
    rkv.score_select(cache, inp["t"], inp["m_global"], sel, ws)
    sync()
    assert ws.status() == 0
    hc = host_cache(backup)
    keep, kept = oracle.select(hc, inp["t"].cpu().numpy(), inp["m_global"].cpu().numpy())
    assert np.array_equal(sel.kept.cpu().numpy(), kept)
    assert np.array_equal(masked_keep(keep_flags(sel, dc.max_pages), hc.len), keep)


@pytest.mark.parametrize("steps_before", [0, 2])
def test_decode_step_times_out_then_recovers(rkv, steps_before):
    # steps_before = 0: the first call takes the exact path (its first grid
    # barrier is in the radix select); 2: the window path (first barrier after
    # the speculative attention pass)
    cfg = workloads.small_config(L=4, H=8, G=4, D=128, B=1, T0=3000, M=30000, kv_dtype="bf16", steps=4)
    dc, _ = _fresh(cfg, 5)
    cache = rkv_cache(rkv, dc)
    sel, ws, outs = rkv.Selection.empty(cache), rkv.Workspace(cache), rkv.StepOutputs.empty(cache)
    for s in range(steps_before):
        inp = workloads.step_inputs(cfg, 5, s, "cuda")
        rkv.decode_step(cache, inp["t"], inp["m_global"], inp["q"], cfg.scale, inp["k_new"], inp["v_new"],
                        inp["lb_new"], sel, outs.out, outs.lse, outs.dropped, ws)
    sync()
    assert ws.status() == 0
    backup = dc.clone()
    inp = workloads.step_inputs(cfg, 5, steps_before, "cuda")
    rkv.workspace_set_wait_limit(ws, 1)
    rkv.decode_step(cache, inp["t"], inp["m_global"], inp["q"], cfg.scale, inp["k_new"], inp["v_new"],
                    inp["lb_new"], sel, outs.out, outs.lse, outs.dropped, ws)
    sync()
    assert _timed_out(ws, rkv), ws.counters()
    # restore the cache, re-initialise the workspace, run the step normally
    for f in ("k_pool", "v_pool", "pos_pool", "lb_pool", "block_table", "len", "free_stack", "free_top"):
        getattr(dc, f).copy_(getattr(backup, f))
    rkv.workspace_init(ws)
    hc = host_cache(dc)
    rkv.decode_step(cache, inp["t"], inp["m_global"], inp["q"], cfg.scale, inp["k_new"], inp["v_new"],
                    inp["lb_new"], sel, outs.out, outs.lse, outs.dropped, ws)
    sync()
    assert ws.status() == 0, ws.counters()
    ref = oracle.step(hc, inp["t"].cpu().numpy(), inp["m_global"].cpu().numpy(),
                      inp["q"].cpu().numpy().reshape(cfg.C, cfg.G, cfg.D), workloads.rows_to_host(inp["k_new"]),
                      workloads.rows_to_host(inp["v_new"]), inp["lb_new"].cpu().numpy(), evict=True, scale=cfg.scale)
    assert np.array_equal(sel.kept.cpu().numpy(), ref["kept"])
    compare_state(dc, hc)
