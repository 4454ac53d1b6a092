"""GPU parity of the eviction error (rkv_eviction_error) against the oracle.

Trust the Mass (ContourKV), Methodology 1: err = ||mu - m_A||, the distance
between the dense attention output and the forced-weight output over the
kept set, per query head.  The library reads the evicted rows' K and V and
combines their forced-weight output with the attention call's out and
dropped mass; the oracle computes mu and m_A from their definitions in
fp64.  Tolerance: the attention tolerances carried through the
combination (tests/gpu_helpers.assert_error_close).
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.gpu_helpers import assert_error_close, rkv_cache, sync, to_dev
from tests.oracle_helpers import host_cache

pytestmark = pytest.mark.gpu


def _run(rkv, cfg, seed, lengths, m):
    dc = to_dev(workloads.ragged_cache(cfg, seed, lengths))
    hc = host_cache(dc)
    cache = rkv_cache(rkv, dc)
    sel, ws = rkv.Selection.empty(cache), rkv.Workspace(cache)
    t = torch.full((cfg.B,), cfg.T0, dtype=torch.int32, device="cuda")
    mm = torch.tensor(m, dtype=torch.int64, device="cuda")
    q = workloads.queries(cfg, seed, 0, "cuda")
    out = torch.empty(cfg.B, cfg.L, cfg.Hq, cfg.D, device="cuda")
    lse = torch.empty(cfg.B, cfg.L, cfg.Hq, device="cuda")
    dm = torch.empty(cfg.B, cfg.L, cfg.Hq, device="cuda")
    err = torch.full((cfg.B, cfg.L, cfg.Hq), float("nan"), device="cuda")
    rkv.score_select(cache, t, mm, sel, ws)
    rkv.paged_decode_attn(cache, q, cfg.scale, sel, out, lse, dm, ws)
    rkv.eviction_error(cache, q, cfg.scale, sel, out, dm, err, ws)
    sync()
    assert ws.status() == 0
    qn = q.cpu().numpy().reshape(cfg.C, cfg.G, cfg.D)
    keep, _ = oracle.select(hc, t.cpu().numpy(), m)
    err_ref = oracle.eviction_error(hc, qn, cfg.scale, keep)
    m_k, _, dm_ref = oracle.attention(hc, qn, cfg.scale, keep)
    evicted = np.zeros_like(keep)
    for c in range(cfg.C):
        evicted[c, : hc.len[c]] = 1 - keep[c, : hc.len[c]]
    m_e, _, _ = oracle.attention(hc, qn, cfg.scale, evicted)
    assert_error_close(err.cpu().numpy().reshape(cfg.C, cfg.G), err_ref, dm_ref, m_k, m_e)
    return err.cpu().numpy().reshape(cfg.C, cfg.G), err_ref, hc, keep


@pytest.mark.parametrize("G,D,kv", [(4, 128, "bf16"), (1, 64, "bf16"), (7, 128, "bf16"), (2, 64, "f32"),
                                    (4, 128, "f32")])
def test_error_ragged(rkv, G, D, kv):
    cfg = workloads.small_config(L=2, H=3, G=G, D=D, B=2, T0=1500, kv_dtype=kv)
    rng = np.random.default_rng(G * 10 + D)
    lengths = rng.integers(1, 1400, size=cfg.C)
    n = int(lengths.sum())
    for frac in (0.1, 0.6, 0.97):
        _run(rkv, cfg, G + D, lengths, [int(n * frac / cfg.B)] * cfg.B)


def test_error_edges(rkv):
    # an empty head, a one-entry head, a head with nothing kept (budget 0 in
    # sequence 1), and a sequence that keeps everything
    cfg = workloads.small_config(L=1, H=4, G=4, D=128, B=2, T0=900, kv_dtype="bf16")
    lengths = [0, 1, 530, 77, 300, 16, 17, 899]
    err, ref, hc, keep = _run(rkv, cfg, 3, lengths, [200, 0])
    assert np.all(err[0] == 0)                                  # no entries
    assert np.all(err[4:] > 0)                                  # nothing kept: ||mu||
    err, ref, hc, keep = _run(rkv, cfg, 3, lengths, [10 ** 6, 10 ** 6])
    assert np.all(err == 0)                                     # nothing evicted


def test_error_steady_state_sparse_evictions(rkv):
    # a steady decoding shape: a few evictions per step among many kept rows
    # (most pages hold no evicted row and pass through without a copy)
    cfg = workloads.small_config(L=4, H=4, G=4, D=128, B=1, T0=4000, kv_dtype="bf16")
    lengths = [1001] * cfg.C
    _run(rkv, cfg, 9, lengths, [1000 * cfg.C])
