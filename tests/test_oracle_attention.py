"""Pins of the oracle's forced-weight attention and dropped mass.

Trust the Mass (ContourKV), Problem definition: after selection the softmax
is renormalised over the kept set (forced weights).  Methodology 3 and main
contributions: the dropped mass is the dense attention weight held by the
discarded keys.  Grouped-query attention: query head h*G+g reads KV head h.
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


@pytest.mark.parametrize("kv", ["f32", "bf16"])
def test_all_kept_equals_library_sdpa(kv):
    cfg, hc = _cache(3, kv)
    q = _q(cfg, 3)
    out, lse, dm = oracle.attention(hc, q, cfg.scale, None)
    assert np.all(dm == 0)
    for c in range(cfg.C):
        _, _, K, V = head_rows(hc, c)
        qt = torch.from_numpy(q[c].astype(np.float64)).unsqueeze(0)          # [1, G, D]
        kt = torch.from_numpy(K).unsqueeze(0).expand(cfg.G, -1, -1)           # [G, n, D]
        vt = torch.from_numpy(V).unsqueeze(0).expand(cfg.G, -1, -1)
        ref = F.scaled_dot_product_attention(qt.transpose(0, 1), kt, vt, scale=cfg.scale)
        assert np.allclose(out[c], ref[:, 0].numpy(), atol=1e-6, rtol=1e-6)
        logits = cfg.scale * (torch.from_numpy(q[c].astype(np.float64)) @ torch.from_numpy(K).T)
        assert np.allclose(lse[c], torch.logsumexp(logits, dim=-1).numpy(), atol=1e-5)


def test_dropped_mass_is_dense_weight_of_evicted_and_mixture_identity():
    cfg, hc = _cache(4, "bf16")
    q = _q(cfg, 4)
    rng = np.random.default_rng(4)
    keep = np.zeros((cfg.C, hc.max_pages * hc.P), np.uint8)
    for c in range(cfg.C):
        n = int(hc.len[c])
        keep[c, :n] = rng.random(n) < 0.4
    out_k, _, dm = oracle.attention(hc, q, cfg.scale, keep)
    evicted = np.zeros_like(keep)
    for c in range(cfg.C):
        evicted[c, : hc.len[c]] = 1 - keep[c, : hc.len[c]]
    out_e, _, _ = oracle.attention(hc, q, cfg.scale, evicted)
    out_d, _, _ = oracle.attention(hc, q, cfg.scale, None)
    for c in range(cfg.C):
        _, _, K, _ = head_rows(hc, c)
        n = int(hc.len[c])
        logits = cfg.scale * (torch.from_numpy(q[c].astype(np.float64)) @ torch.from_numpy(K).T)
        p = torch.softmax(logits, dim=-1).numpy()                       # dense weights
        kept_w = p[:, keep[c, :n].astype(bool)].sum(axis=1)
        assert np.allclose(dm[c], 1.0 - kept_w, atol=2e-7)
        # dense output = (1 - dm) * kept output + dm * evicted output
        mix = (1 - dm[c].astype(np.float64))[:, None] * out_k[c] + dm[c].astype(np.float64)[:, None] * out_e[c]
        assert np.allclose(out_d[c], mix, atol=2e-6)


def test_single_kept_key_returns_its_value_and_zero_query_gives_mean():
    cfg, hc = _cache(5, "f32", lengths=[7, 9, 1, 12], G=3, D=8)
    q = _q(cfg, 5)
    keep = np.zeros((cfg.C, hc.max_pages * hc.P), np.uint8)
    keep[0, 3] = 1
    keep[1, :9] = 1
    keep[2, 0] = 1
    keep[3, [0, 5, 11]] = 1
    out, lse, dm = oracle.attention(hc, q, cfg.scale, keep)
    _, _, K0, V0 = head_rows(hc, 0)
    assert np.allclose(out[0], np.broadcast_to(V0[3], (cfg.G, cfg.D)), atol=1e-7)
    assert np.allclose(lse[0], cfg.scale * q[0].astype(np.float64) @ K0[3], atol=1e-6)
    out0, _, _ = oracle.attention(hc, np.zeros_like(q), cfg.scale, keep)
    _, _, _, V3 = head_rows(hc, 3)
    assert np.allclose(out0[3], np.broadcast_to(V3[[0, 5, 11]].mean(axis=0), (cfg.G, cfg.D)), atol=1e-7)
    _, _, _, V1 = head_rows(hc, 1)
    assert np.allclose(out0[1], np.broadcast_to(V1.mean(axis=0), (cfg.G, cfg.D)), atol=1e-7)
    assert np.all(dm[1] == 0)        # nothing of head 1 evicted
    assert np.all(dm[2] == 0)        # head 2's only entry kept


def test_empty_and_fully_evicted_heads():
    cfg, hc = _cache(6, "f32", lengths=[0, 5, 3, 4], G=2, D=8)
    q = _q(cfg, 6)
    keep = np.zeros((cfg.C, hc.max_pages * hc.P), np.uint8)
    keep[2, :3] = 1
    keep[3, 1] = 1
    out, lse, dm = oracle.attention(hc, q, cfg.scale, keep)
    assert np.all(out[0] == 0) and np.all(np.isneginf(lse[0])) and np.all(dm[0] == 0)  # no entries
    assert np.all(out[1] == 0) and np.all(np.isneginf(lse[1])) and np.all(dm[1] == 1)  # all evicted
    assert np.all(dm[2] == 0)
    assert np.all((dm[3] > 0) & (dm[3] < 1))


def test_hand_worked_two_keys():
    # One head, G = 1, D = 2, keys k0 = (1, 0), k1 = (0, 1), values v0 = (2, 0),
    # v1 = (0, 4), q = (ln 3, 0) with scale 1: logits ln 3 and 0, dense
    # weights 3/4 and 1/4.  Keeping only k0 drops mass 1/4 and returns v0.
    hc = hand_cache(1, 1, 1, 1, 2, 16, 1, 1, [[0]], [2], [[5, 6]], [[-1.0, -1.0]],
                    kv_fn=lambda c, p: ([1.0, 0.0], [2.0, 0.0]) if p == 5 else ([0.0, 1.0], [0.0, 4.0]))
    q = np.array([[[math.log(3.0), 0.0]]], np.float32)
    out, lse, dm = oracle.attention(hc, q, 1.0, None)
    assert np.allclose(out[0, 0], [1.5, 1.0], atol=1e-6)           # 3/4*(2,0) + 1/4*(0,4)
    assert np.isclose(lse[0, 0], math.log(4.0), atol=1e-6)
    keep = np.zeros((1, 16), np.uint8)
    keep[0, 0] = 1
    out, lse, dm = oracle.attention(hc, q, 1.0, keep)
    assert np.allclose(out[0, 0], [2.0, 0.0]) and np.isclose(dm[0, 0], 0.25, atol=1e-7)
    assert np.isclose(lse[0, 0], math.log(3.0), atol=1e-6)
