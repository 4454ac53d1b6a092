"""Helpers shared by the oracle pins and the GPU parity tests (test code only)."""
from __future__ import annotations

import json
import os

import numpy as np

import oracle
import workloads

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def load_golden(name: str) -> dict:
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def host_cache(dc: workloads.DeviceCache) -> oracle.HostCache:
    return oracle.HostCache(**workloads.to_host(dc))


def hand_cache(B, L, H, G, D, P, n_pages, max_pages, block_table, lengths, slot_pos, slot_lb=None,
               free_stack=None, free_top=0, kv_fn=None) -> oracle.HostCache:
    """Build a float32 HostCache by hand: slot k of head c on page
    block_table[c][k//P] at offset k%P holds position slot_pos[c][k]."""
    C = B * L * H
    k_pool = np.zeros((n_pages, P, D), np.float32)
    v_pool = np.zeros((n_pages, P, D), np.float32)
    pos_pool = np.zeros((n_pages, P), np.int32)
    lb_pool = np.zeros((n_pages, P), np.float32)
    for c in range(C):
        for k, p in enumerate(slot_pos[c]):
            page = block_table[c][k // P]
            pos_pool[page, k % P] = p
            if slot_lb is not None:
                lb_pool[page, k % P] = slot_lb[c][k]
            if kv_fn is not None:
                kr, vr = kv_fn(c, p)
                k_pool[page, k % P] = kr
                v_pool[page, k % P] = vr
    fs = np.full(n_pages, -1, np.int32)
    if free_stack is not None:
        fs[: len(free_stack)] = free_stack
    return oracle.HostCache(B, L, H, G, D, P, k_pool, v_pool, pos_pool, lb_pool,
                            np.array(block_table, np.int32), np.array(lengths, np.int32), fs,
                            np.array([free_top], np.int32))


def slot_values(hc: oracle.HostCache, c: int, arr: np.ndarray) -> list:
    """Per-slot values of a [n_pages, P(, ...)] pool for head c, slots < len."""
    out = []
    for k in range(int(hc.len[c])):
        page = hc.block_table[c, k // hc.P]
        out.append(arr[page, k % hc.P])
    return out


def kept_positions(hc: oracle.HostCache, keep: np.ndarray) -> list[set]:
    """For each head, the set of positions whose slot is flagged kept."""
    res = []
    for c in range(hc.C):
        s = set()
        for k in range(int(hc.len[c])):
            if keep[c, k]:
                page = hc.block_table[c, k // hc.P]
                s.add(int(hc.pos_pool[page, k % hc.P]))
        res.append(s)
    return res


def all_positions(hc: oracle.HostCache) -> list[set]:
    return [set(int(x) for x in slot_values(hc, c, hc.pos_pool)) for c in range(hc.C)]


def bf16_to_f32(x: np.ndarray) -> np.ndarray:
    if x.dtype == np.uint16:
        return (x.astype(np.uint32) << 16).view(np.float32)
    return x.astype(np.float32)


def head_rows(hc: oracle.HostCache, c: int):
    """(pos [n], lb [n], K [n, D] f64, V [n, D] f64) of head c in slot order."""
    n = int(hc.len[c])
    pages = hc.block_table[c, (np.arange(n) // hc.P)]
    offs = np.arange(n) % hc.P
    K = bf16_to_f32(hc.k_pool[pages, offs]).astype(np.float64)
    V = bf16_to_f32(hc.v_pool[pages, offs]).astype(np.float64)
    return hc.pos_pool[pages, offs].copy(), hc.lb_pool[pages, offs].copy(), K, V
