"""Pins of the oracle's latent memory for evicted tokens.

IndexMem (learned KV eviction with latent memory), Methodology B: evicted
tokens update a fixed-size state M and a stabilising vector b online by
outer-product accumulation with decay (fast weights); a learned projection
and a gate g(q) read it (slow weights); o = o_attn + g(q) * m(q).  Readings
(in oracle.c): phi(x) = elu(P_l x) + 1, M_c = decay*M_c + sum phi(k) v^T,
b_c = decay*b_c + sum phi(k), m = phi(q)^T M_c / phi(q)^T b_c (0 when the
denominator is 0), g = sigmoid(w . q + beta).
"""
import math

import numpy as np
import pytest

import oracle
import workloads
from tests.oracle_helpers import hand_cache, head_rows, host_cache, load_golden


def _one_head(keys, values, pos0=0):
    D = len(keys[0])
    n = len(keys)
    kv = {pos0 + i: (keys[i], values[i]) for i in range(n)}
    return hand_cache(1, 1, 1, 1, D, 16, 1, 1, [[0]], [n], [[pos0 + i for i in range(n)]], [[-1.0] * n],
                      kv_fn=lambda c, p: kv[p])


def _state(hc):
    return np.zeros((hc.C, hc.D, hc.D)), np.zeros((hc.C, hc.D))


def test_golden_three_tokens():
    g = load_golden("memory_three_tokens.json")
    D = g["D"]
    P = np.eye(D, dtype=np.float32)[None]
    q = np.array(g["q"], np.float32).reshape(1, 1, D)
    gw = np.array(g["gate_w"], np.float32).reshape(1, 1, D)
    gb = np.array([[g["gate_b"]]], np.float32)
    o = np.array(g["o_attn"], np.float32).reshape(1, 1, D)
    gate = 1.0 / (1.0 + math.exp(-1.0))
    hc = _one_head(g["keys"], g["values"])
    # all three evicted in one step
    M, b = _state(hc)
    oracle.memory_update(hc, np.zeros((1, 16), np.uint8), P, 0.5, M, b)
    out = oracle.memory_read(hc, q, P, gw, gb, M, b, o)
    assert np.allclose(out[0, 0], np.array(g["o_attn"]) + gate * np.array(g["one_step"]["m"]), atol=1e-6)
    # k1 at the first step, k2 and k3 at the second, decay 1/2
    M, b = _state(hc)
    first = np.ones((1, 16), np.uint8)
    first[0, 0] = 0
    oracle.memory_update(hc, first, P, 0.5, M, b)
    second = np.zeros((1, 16), np.uint8)
    second[0, 0] = 1
    oracle.memory_update(hc, second, P, 0.5, M, b)
    out = oracle.memory_read(hc, q, P, gw, gb, M, b, o)
    assert np.allclose(out[0, 0], np.array(g["o_attn"]) + gate * np.array(g["two_steps_decay_half"]["m"]),
                       atol=1e-6)


def test_single_evicted_token_reads_back_its_value():
    # one evicted token: m(q) = phi^T phi(k) v / phi^T phi(k) = v for any q
    rng = np.random.default_rng(1)
    D = 16
    k, v = rng.normal(size=(1, D)), rng.normal(size=(1, D))
    hc = _one_head(k.tolist(), v.tolist())
    P = (rng.normal(size=(1, D, D)) / math.sqrt(D)).astype(np.float32)
    M, b = _state(hc)
    oracle.memory_update(hc, np.zeros((1, 16), np.uint8), P, 0.9, M, b)
    for s in range(3):
        q = rng.normal(size=(1, 1, D)).astype(np.float32)
        out = oracle.memory_read(hc, q, P, np.zeros((1, 1, D), np.float32), np.full((1, 1), 30.0, np.float32),
                                 M, b, np.zeros((1, 1, D), np.float32))
        assert np.allclose(out[0, 0], v.astype(np.float32)[0], atol=1e-5)   # gate sigmoid(30) ~ 1


def test_zero_projection_reads_the_plain_mean_and_kept_rows_do_not_count():
    # P = 0: phi = 1 everywhere, every evicted token weighs the same
    cfg = workloads.small_config(L=2, H=2, G=2, D=16, B=1, T0=90, kv_dtype="f32")
    hc = host_cache(workloads.ragged_cache(cfg, 3, [20, 0, 35, 7]))
    rng = np.random.default_rng(3)
    keep = np.zeros((hc.C, hc.max_pages * hc.P), np.uint8)
    for c in range(hc.C):
        keep[c, : hc.len[c]] = rng.random(int(hc.len[c])) < 0.5
    P = np.zeros((cfg.L, cfg.D, cfg.D), np.float32)
    M, b = _state(hc)
    oracle.memory_update(hc, keep, P, 1.0, M, b)
    q = workloads.queries(cfg, 3, 0).numpy().reshape(cfg.C, cfg.G, cfg.D)
    zero = np.zeros((cfg.C, cfg.G, cfg.D), np.float32)
    out = oracle.memory_read(hc, q, P, np.zeros((cfg.L, cfg.Hq, cfg.D), np.float32),
                             np.zeros((cfg.L, cfg.Hq), np.float32), M, b, zero)
    for c in range(hc.C):
        _, _, _, V = head_rows(hc, c)
        ev = ~keep[c, : hc.len[c]].astype(bool)
        want = 0.5 * V[ev].mean(axis=0) if ev.any() else np.zeros(cfg.D)   # gate sigmoid(0) = 1/2
        assert np.allclose(out[c], np.broadcast_to(want, (cfg.G, cfg.D)), atol=1e-6), c


def test_nothing_evicted_leaves_the_output_and_decay_scales_the_state():
    cfg = workloads.small_config(L=1, H=2, G=1, D=8, B=1, T0=40, kv_dtype="f32")
    hc = host_cache(workloads.ragged_cache(cfg, 4, [10, 12]))
    P = np.ones((1, 8, 8), np.float32) * 0.1
    M, b = _state(hc)
    ev = np.zeros((hc.C, hc.max_pages * hc.P), np.uint8)
    oracle.memory_update(hc, ev, P, 1.0, M, b)               # everything evicted once
    M1, b1 = M.copy(), b.copy()
    allkeep = np.ones_like(ev)
    oracle.memory_update(hc, allkeep, P, 0.25, M, b)         # nothing evicted: only the decay
    assert np.allclose(M, 0.25 * M1) and np.allclose(b, 0.25 * b1)
    q = workloads.queries(cfg, 4, 0).numpy().reshape(cfg.C, cfg.G, cfg.D)
    o = np.arange(cfg.C * cfg.D, dtype=np.float32).reshape(cfg.C, 1, cfg.D)
    Z, z = _state(hc)
    out = oracle.memory_read(hc, q, P, np.ones((1, 2, 8), np.float32), np.zeros((1, 2), np.float32), Z, z, o)
    assert np.array_equal(out, o)                            # empty memory: m = 0
