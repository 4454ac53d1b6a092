"""Device-side error reporting without faulting the GPU: bad inputs and
exhausted pools set sticky RKV_DEV_* bits in the workspace status word, the
kernels finish, and rkv_workspace_init clears the word."""
import numpy as np
import pytest
import torch

import workloads
from tests.gpu_helpers import rkv_cache, sync, to_dev

pytestmark = pytest.mark.gpu


def _setup(rkv, lengths, **kw):
    cfg = workloads.small_config(L=1, H=len(lengths), G=1, D=64, B=1, T0=500, kv_dtype="bf16")
    dc = to_dev(workloads.ragged_cache(cfg, 4, lengths, **kw))
    cache = rkv_cache(rkv, dc)
    return cfg, dc, cache, rkv.Selection.empty(cache), rkv.Workspace(cache)


def test_nan_log_retention_sets_bad_input(rkv):
    cfg, dc, cache, sel, ws = _setup(rkv, [40, 50])
    dc.lb_pool[dc.block_table[1, 1], 3] = float("nan")
    t = torch.tensor([cfg.T0], dtype=torch.int32, device="cuda")
    rkv.score_select(cache, t, torch.tensor([30], dtype=torch.int64, device="cuda"), sel, ws)
    sync()
    assert ws.status() & rkv.DEV_BAD_INPUT
    rkv.workspace_init(ws)
    sync()
    assert ws.status() == 0


def test_age_out_of_range_sets_bad_input(rkv):
    cfg, dc, cache, sel, ws = _setup(rkv, [40, 50])
    t = torch.tensor([int(dc.pos_pool.max())], dtype=torch.int32, device="cuda")  # some entry has age 0
    rkv.score_select(cache, t, torch.tensor([30], dtype=torch.int64, device="cuda"), sel, ws)
    sync()
    assert ws.status() & rkv.DEV_BAD_INPUT


def _append(rkv, cfg, cache, ws, fused):
    """The append alone: rkv_append, or a non-evicting rkv_decode_step
    (attention over every entry, then the append)."""
    inp = workloads.step_inputs(cfg, 0, 0, "cuda")
    if fused:
        outs = rkv.StepOutputs.empty(cache)
        rkv.decode_step(cache, inp["t"], None, inp["q"], cfg.scale, inp["k_new"], inp["v_new"], inp["lb_new"],
                        None, outs.out, outs.lse, outs.dropped, ws)
    else:
        rkv.append(cache, inp["t"], inp["k_new"], inp["v_new"], inp["lb_new"], ws)
    sync()


@pytest.mark.parametrize("fused", [False, True])
def test_append_with_empty_free_stack_sets_pool_exhausted(rkv, fused):
    # both heads sit at a page boundary and the pool has no free page: both
    # are skipped, their lengths and the stack top stay as they were
    cfg, dc, cache, sel, ws = _setup(rkv, [32, 16], n_pages=3)
    assert int(dc.free_top.item()) == 0
    table = dc.block_table.clone()
    _append(rkv, cfg, cache, ws, fused)
    assert ws.status() & rkv.DEV_POOL_EXHAUSTED
    assert dc.len.tolist() == [32, 16]
    assert int(dc.free_top.item()) == 0
    assert torch.equal(dc.block_table, table)


@pytest.mark.parametrize("fused", [False, True])
def test_append_past_max_pages_sets_table_overflow(rkv, fused):
    # head 0's table is full (skipped, length kept); head 1 appends in its page
    cfg, dc, cache, sel, ws = _setup(rkv, [32, 5], max_pages=2, n_pages=8)
    top = int(dc.free_top.item())
    _append(rkv, cfg, cache, ws, fused)
    assert ws.status() & rkv.DEV_TABLE_OVERFLOW
    assert dc.len.tolist() == [32, 6]
    assert int(dc.free_top.item()) == top


@pytest.mark.parametrize("fused", [False, True])
def test_full_table_takes_no_page(rkv, fused):
    # head 0 is full and would pop; head 1 pops the one free page: the full
    # head takes no pop rank, so head 1 still gets the top page
    cfg, dc, cache, sel, ws = _setup(rkv, [32, 16], max_pages=2, n_pages=4)
    assert int(dc.free_top.item()) == 1
    page = int(dc.free_stack[0].item())
    _append(rkv, cfg, cache, ws, fused)
    assert ws.status() == rkv.DEV_TABLE_OVERFLOW
    assert dc.len.tolist() == [32, 17]
    assert int(dc.free_top.item()) == 0
    assert int(dc.block_table[1, 1].item()) == page
    assert int(dc.pos_pool[page, 0].item()) == cfg.T0


def test_length_past_the_table_is_clamped_and_reported(rkv):
    # a length beyond max_pages*16 is read as the table's capacity: the
    # selection sees 32 entries in head 0 and flags bad input
    cfg, dc, cache, sel, ws = _setup(rkv, [32, 20], max_pages=2, n_pages=8)
    dc.len[0] = 40
    t = torch.tensor([cfg.T0], dtype=torch.int32, device="cuda")
    rkv.score_select(cache, t, torch.tensor([10], dtype=torch.int64, device="cuda"), sel, ws)
    sync()
    assert ws.status() & rkv.DEV_BAD_INPUT
    assert sel.n_pre.tolist() == [32, 20]
