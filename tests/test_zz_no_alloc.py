"""The allocation-free selection entry point, rkv_score_select_noalloc.

Some callers cannot allocate device memory for a workspace -- code that runs
where cudaMalloc is not allowed (inside a host callback or a captured region
of someone else's stream), or under a memory manager that hands out only
fixed buffers.  rkv_score_select_noalloc serves them: it takes the same cache,
inputs and output buffers as rkv_score_select but keeps its scratch in a fixed
array inside the library.  This test calls it through the C ABI and checks,
on two calls in a row (so the second call starts from the scratch the first
one left behind), that every output matches rkv_score_select bit for bit.
Selection outputs are integers, so the comparison is exact.
"""
import ctypes

import numpy as np
import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu


def _noalloc(rkv):
    lib = rkv.load()
    fn = lib.rkv_score_select_noalloc
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.POINTER(rkv.CacheStruct), ctypes.c_void_p, ctypes.c_void_p,
                   ctypes.POINTER(rkv.SelectStruct), ctypes.c_void_p]
    return fn


def _outputs(sel):
    torch.cuda.synchronize()
    return {k: getattr(sel, k).cpu().numpy().copy() for k in ("kappa", "kept", "n_pre", "keep_mask", "plan")}


def test_noalloc_select_matches_workspace_select_twice(rkv):
    fn = _noalloc(rkv)
    cfg = workloads.small_config(L=3, H=4, G=2, D=128, B=2, T0=4000, kv_dtype="bf16")
    rng = np.random.default_rng(77)
    lengths = rng.integers(0, 2500, size=cfg.C)
    dc = workloads.ragged_cache(cfg, 77, lengths, device="cuda")
    cache = rkv.Cache.from_tensors(dc, cfg.B, cfg.L, cfg.H, cfg.Hq)
    ws = rkv.Workspace(cache)
    t = torch.full((cfg.B,), cfg.T0, dtype=torch.int32, device="cuda")
    per_seq = [int(dc.len[b * cfg.L * cfg.H:(b + 1) * cfg.L * cfg.H].sum()) for b in range(cfg.B)]
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for frac in (0.3, 0.75):  # two calls in a row on the shared scratch
        m = torch.tensor([int(n * frac) for n in per_seq], dtype=torch.int64, device="cuda")
        ref = rkv.Selection.empty(cache)
        rkv.score_select(cache, t, m, ref, ws)
        want = _outputs(ref)
        got_sel = rkv.Selection.empty(cache)
        cs, ss = cache.struct(), got_sel.struct()
        rc = fn(ctypes.byref(cs), ctypes.c_void_p(t.data_ptr()), ctypes.c_void_p(m.data_ptr()), ctypes.byref(ss),
                stream)
        assert rc == 0, rkv.last_error()
        got = _outputs(got_sel)
        for k in want:
            assert np.array_equal(got[k], want[k]), f"{k} differs (budget fraction {frac})"
        assert int(got_sel.kept.sum()) == int(m.sum())
    assert ws.status() == 0


def test_noalloc_select_rejects_oversized_batch(rkv):
    fn = _noalloc(rkv)
    cfg = workloads.small_config(L=1, H=1, G=1, D=64, B=17, T0=100, kv_dtype="bf16")
    dc = workloads.ragged_cache(cfg, 1, [10] * cfg.C, device="cuda")
    cache = rkv.Cache.from_tensors(dc, cfg.B, cfg.L, cfg.H, cfg.Hq)
    sel = rkv.Selection.empty(cache)
    t = torch.full((cfg.B,), cfg.T0, dtype=torch.int32, device="cuda")
    m = torch.full((cfg.B,), 5, dtype=torch.int64, device="cuda")
    cs, ss = cache.struct(), sel.struct()
    rc = fn(ctypes.byref(cs), ctypes.c_void_p(t.data_ptr()), ctypes.c_void_p(m.data_ptr()), ctypes.byref(ss),
            ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == rkv.ERR_UNSUPPORTED
    assert "16" in rkv.last_error()
