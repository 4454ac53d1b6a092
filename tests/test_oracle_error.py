"""Pins of the oracle's eviction error.

Trust the Mass (ContourKV), Methodology 1 (theoretical analysis and
enumeration): a kept subset A is scored by e(A) = ||mu - m_A||, the distance
between the dense attention output mu and the forced-weight output m_A over
A.  Readings: Euclidean norm over the head dimension, per query head; a head
with no entries has e = 0; with nothing kept m_A = 0, so e = ||mu||.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
import workloads
from tests.oracle_helpers import hand_cache, head_rows, host_cache


def _cache(seed, kv="f32", lengths=None, G=2, D=16):
    cfg = workloads.small_config(L=2, H=2, G=G, D=D, B=1, T0=90, kv_dtype=kv)
    rng = np.random.default_rng(seed)
    if lengths is None:
        lengths = rng.integers(1, 60, size=cfg.C)
    return cfg, host_cache(workloads.ragged_cache(cfg, seed, lengths))


def _q(cfg, seed):
    return workloads.queries(cfg, seed, 0).numpy().reshape(cfg.C, cfg.G, cfg.D)


def _random_keep(hc, seed, frac):
    rng = np.random.default_rng(seed)
    keep = np.zeros((hc.C, hc.max_pages * hc.P), np.uint8)
    for c in range(hc.C):
        n = int(hc.len[c])
        keep[c, :n] = rng.random(n) < frac
    return keep


def _sdpa(q, K, V, scale, mask=None):
    """Library attention in float64: q [G, D], K/V [n, D], mask [n] bool."""
    qt = torch.from_numpy(q.astype(np.float64)).unsqueeze(1)           # [G, 1, D]
    kt = torch.from_numpy(K).unsqueeze(0).expand(q.shape[0], -1, -1)     # [G, n, D]
    vt = torch.from_numpy(V).unsqueeze(0).expand(q.shape[0], -1, -1)
    am = None if mask is None else torch.from_numpy(mask).view(1, 1, -1).expand(q.shape[0], 1, -1)
    return F.scaled_dot_product_attention(qt, kt, vt, attn_mask=am, scale=scale)[:, 0].numpy()


@pytest.mark.parametrize("kv,frac", [("f32", 0.5), ("bf16", 0.3), ("bf16", 0.9)])
def test_error_is_distance_of_library_outputs(kv, frac):
    cfg, hc = _cache(7, kv)
    q = _q(cfg, 7)
    keep = _random_keep(hc, 7, frac)
    err, mu = oracle.eviction_error(hc, q, cfg.scale, keep, with_dense=True)
    for c in range(cfg.C):
        _, _, K, V = head_rows(hc, c)
        n = K.shape[0]
        k = keep[c, :n].astype(bool)
        dense = _sdpa(q[c], K, V, cfg.scale)
        kept = _sdpa(q[c], K, V, cfg.scale, k) if k.any() else np.zeros_like(dense)
        ref = np.linalg.norm(dense - kept, axis=-1)
        assert np.allclose(mu[c], dense, atol=1e-6)
        assert np.allclose(err[c], ref, rtol=1e-5, atol=1e-7), (c, err[c], ref)


def test_error_mixture_identity():
    # mu - m_A = dm * (m_evicted - m_A): the error is the dropped mass times
    # the distance between the evicted set's and the kept set's outputs
    cfg, hc = _cache(8, "bf16")
    q = _q(cfg, 8)
    keep = _random_keep(hc, 8, 0.4)
    evicted = np.zeros_like(keep)
    for c in range(cfg.C):
        evicted[c, : hc.len[c]] = 1 - keep[c, : hc.len[c]]
    err = oracle.eviction_error(hc, q, cfg.scale, keep)
    out_k, _, dm = oracle.attention(hc, q, cfg.scale, keep)
    out_e, _, _ = oracle.attention(hc, q, cfg.scale, evicted)
    d = np.linalg.norm(out_e.astype(np.float64) - out_k.astype(np.float64), axis=-1)
    assert np.allclose(err, dm.astype(np.float64) * d, rtol=1e-5, atol=1e-6)


def test_error_zero_when_everything_kept():
    cfg, hc = _cache(9, "f32")
    q = _q(cfg, 9)
    assert np.all(oracle.eviction_error(hc, q, cfg.scale, None) == 0)
    keep = np.ones((hc.C, hc.max_pages * hc.P), np.uint8)
    assert np.all(oracle.eviction_error(hc, q, cfg.scale, keep) == 0)


def test_error_with_nothing_kept_is_dense_norm_and_empty_head_is_zero():
    cfg, hc = _cache(10, "f32", lengths=[0, 6, 11, 3], G=2, D=8)
    q = _q(cfg, 10)
    keep = np.zeros((hc.C, hc.max_pages * hc.P), np.uint8)
    keep[3, 1] = 1
    err = oracle.eviction_error(hc, q, cfg.scale, keep)
    assert np.all(err[0] == 0)                                   # no entries
    for c in (1, 2):                                             # nothing kept: ||mu||
        _, _, K, V = head_rows(hc, c)
        assert np.allclose(err[c], np.linalg.norm(_sdpa(q[c], K, V, cfg.scale), axis=-1), rtol=1e-6)
    assert np.all(err[3] > 0)


def test_hand_worked_two_keys():
    # One head, G = 1, D = 2: keys k0 = (1, 0), k1 = (0, 1), values v0 = (2, 0),
    # v1 = (0, 4), q = (ln 3, 0), scale 1: dense weights 3/4 and 1/4, so
    # mu = (1.5, 1).  Keeping only k0 gives m_A = v0 and e = |(-0.5, 1)| =
    # sqrt(5)/2 = (1/4) * |v1 - v0|.
    hc = hand_cache(1, 1, 1, 1, 2, 16, 1, 1, [[0]], [2], [[5, 6]], [[-1.0, -1.0]],
                    kv_fn=lambda c, p: ([1.0, 0.0], [2.0, 0.0]) if p == 5 else ([0.0, 1.0], [0.0, 4.0]))
    q = np.array([[[math.log(3.0), 0.0]]], np.float32)
    keep = np.zeros((1, 16), np.uint8)
    keep[0, 0] = 1
    err, mu = oracle.eviction_error(hc, q, 1.0, keep, with_dense=True)
    assert np.allclose(mu[0, 0], [1.5, 1.0], atol=1e-6)
    assert math.isclose(float(err[0, 0]), math.sqrt(5.0) / 2.0, rel_tol=1e-6)
    keep[0, 0], keep[0, 1] = 0, 1                # keep k1 instead: m_A = v1, e = (3/4) |v0 - v1|
    err = oracle.eviction_error(hc, q, 1.0, keep)
    assert math.isclose(float(err[0, 0]), 0.75 * math.sqrt(20.0), rel_tol=1e-6)
