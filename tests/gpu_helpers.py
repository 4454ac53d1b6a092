"""GPU-side helpers for the parity tests (test code only)."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import workloads
from tests.oracle_helpers import host_cache

OUT_RTOL = 2e-3   # max-abs error per (head, query) row relative to the oracle row's L2 norm
DM_ATOL = 1e-4    # dropped mass, absolute
LSE_ATOL = 5e-5   # log-sum-exp of kept logits (natural log), plus LSE_RTOL * |lse|
LSE_RTOL = 1e-5


def rkv_cache(rkv, dc: workloads.DeviceCache):
    cfg = dc.cfg
    return rkv.Cache.from_tensors(dc, cfg.B, cfg.L, cfg.H, cfg.Hq)


def keep_flags(sel, max_pages: int) -> np.ndarray:
    """Per-slot keep flags [C, max_pages*16] from the device keep masks."""
    m = sel.keep_mask.cpu().numpy().view(np.uint16).astype(np.uint32)
    bits = (m[:, :, None] >> np.arange(16, dtype=np.uint32)[None, None, :]) & 1
    return bits.reshape(m.shape[0], max_pages * 16).astype(np.uint8)


def masked_keep(keep: np.ndarray, lengths) -> np.ndarray:
    out = np.zeros_like(keep)
    for c, n in enumerate(lengths):
        out[c, :n] = keep[c, :n]
    return out


def assert_outputs_close(out, lse, dm, o_ref, lse_ref, dm_ref, kept_any):
    """out [C, G, D]; lse, dm [C, G]; kept_any [C] bool (oracle)."""
    out = np.asarray(out, np.float64)
    o_ref = np.asarray(o_ref, np.float64)
    C, G, D = o_ref.shape
    norm = np.linalg.norm(o_ref, axis=-1)
    err = np.abs(out - o_ref).max(axis=-1)
    for c in range(C):
        if not kept_any[c]:
            assert np.all(out[c] == 0.0), f"head {c}: nothing kept but output nonzero"
            if lse is not None:
                assert np.all(np.isneginf(lse[c])), f"head {c}: lse must be -inf"
    ok = err <= OUT_RTOL * np.maximum(norm, 1e-30)
    bad = np.argwhere(~ok & kept_any[:, None])
    assert bad.size == 0, f"{len(bad)} rows out of tolerance, worst rel {float((err / np.maximum(norm, 1e-30)).max()):.3e} at {bad[:5].tolist()}"
    if lse is not None:
        fin = np.isfinite(lse_ref)
        assert np.array_equal(np.isfinite(lse), fin)
        d = np.abs(np.asarray(lse, np.float64)[fin] - lse_ref[fin].astype(np.float64))
        assert np.all(d <= LSE_ATOL + LSE_RTOL * np.abs(lse_ref[fin])), float(d.max())
    if dm is not None:
        assert np.abs(np.asarray(dm, np.float64) - dm_ref.astype(np.float64)).max() <= DM_ATOL


def assert_error_close(err, err_ref, dm_ref, m_kept_ref, m_ev_ref):
    """Eviction error err = ||mu - m_A|| = dm * ||m_ev - m_A|| [C, G] against
    the oracle.  The library forms it from its own m_ev, m_A (each within
    OUT_RTOL of its row norm) and dm (within DM_ATOL), so the bound is
    OUT_RTOL * dm * (||m_ev|| + ||m_A||) + DM_ATOL * ||m_ev - m_A|| (+1e-6)."""
    err = np.asarray(err, np.float64)
    ref = np.asarray(err_ref, np.float64)
    m_k = np.asarray(m_kept_ref, np.float64)
    m_e = np.asarray(m_ev_ref, np.float64)
    dm = np.asarray(dm_ref, np.float64)
    tol = (OUT_RTOL * dm * (np.linalg.norm(m_e, axis=-1) + np.linalg.norm(m_k, axis=-1))
           + DM_ATOL * np.linalg.norm(m_e - m_k, axis=-1) + 1e-6)
    bad = np.argwhere(np.abs(err - ref) > tol)
    assert bad.size == 0, f"{len(bad)} rows out of tolerance, first {bad[:5].tolist()}: " \
                          f"{[(float(err[tuple(i)]), float(ref[tuple(i)])) for i in bad[:3]]}"


def compare_state(dc: workloads.DeviceCache, hc: oracle.HostCache, pools: bool = True):
    """Bit-exact comparison of a device cache with an oracle cache."""
    g = host_cache(dc) if pools else None
    assert np.array_equal(dc.len.cpu().numpy(), hc.len), "len"
    assert np.array_equal(dc.block_table.cpu().numpy(), hc.block_table), "block_table"
    top = int(dc.free_top.cpu()[0])
    assert top == int(hc.free_top[0]), f"free_top {top} vs {int(hc.free_top[0])}"
    assert np.array_equal(dc.free_stack.cpu().numpy()[:top], hc.free_stack[:top]), "free_stack"
    if pools:
        assert np.array_equal(g.pos_pool, hc.pos_pool), "pos_pool"
        assert np.array_equal(g.lb_pool.view(np.uint32), hc.lb_pool.view(np.uint32)), "lb_pool"
        assert np.array_equal(g.k_pool, hc.k_pool), "k_pool"
        assert np.array_equal(g.v_pool, hc.v_pool), "v_pool"


def to_dev(dc: workloads.DeviceCache) -> workloads.DeviceCache:
    return dc.to("cuda")


def sync():
    torch.cuda.synchronize()
