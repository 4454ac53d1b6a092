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


def test_append_with_empty_free_stack_sets_pool_exhausted(rkv):
    # both heads sit at a page boundary and the pool has no free page
    cfg, dc, cache, sel, ws = _setup(rkv, [32, 16], n_pages=3)
    assert int(dc.free_top.item()) == 0
    inp = workloads.step_inputs(cfg, 0, 0, "cuda")
    rkv.append(cache, inp["t"], inp["k_new"], inp["v_new"], inp["lb_new"], ws)
    sync()
    assert ws.status() & rkv.DEV_POOL_EXHAUSTED


def test_append_past_max_pages_sets_table_overflow(rkv):
    cfg, dc, cache, sel, ws = _setup(rkv, [32, 5], max_pages=2, n_pages=8)
    inp = workloads.step_inputs(cfg, 0, 0, "cuda")
    rkv.append(cache, inp["t"], inp["k_new"], inp["v_new"], inp["lb_new"], ws)
    sync()
    assert ws.status() & rkv.DEV_TABLE_OVERFLOW
