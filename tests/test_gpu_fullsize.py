"""Parity at the full workload sizes, in the launch configuration bench.py times.

Selection, compaction and append are compared with the oracle bit for bit
(the oracle runs on the metadata pools -- positions, log-retentions, tables,
lengths, free stack -- with one-element stand-in K/V rows, since none of those
steps reads K or V values); for batched workloads the oracle runs on a subset
of the independent sequences and the shared free stack is checked by its
invariants.  Attention and dropped mass are compared on sampled heads, whose
rows are gathered into a small oracle cache, and on every head of one steady
step of llama32k and of two qwen8k sequences.  K/V row moves are checked on
sampled heads against the pre-compaction rows of the same positions.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.gpu_helpers import assert_outputs_close, keep_flags, masked_keep, rkv_cache, sync

pytestmark = pytest.mark.gpu


def meta_host(dc, seqs=None):
    """Oracle cache of the metadata of `seqs` (all sequences if None)."""
    cfg = dc.cfg
    LH = cfg.L * cfg.H
    seqs = list(range(cfg.B)) if seqs is None else list(seqs)
    heads = np.concatenate([np.arange(b * LH, (b + 1) * LH) for b in seqs])
    n_pages = dc.n_pages
    dummy = np.zeros((n_pages, cfg.P, 1), np.uint16)
    return oracle.HostCache(len(seqs), cfg.L, cfg.H, cfg.G, 1, cfg.P, dummy, dummy.copy(),
                            dc.pos_pool.cpu().numpy(), dc.lb_pool.cpu().numpy(),
                            np.ascontiguousarray(dc.block_table.cpu().numpy()[heads]),
                            np.ascontiguousarray(dc.len.cpu().numpy()[heads]),
                            dc.free_stack.cpu().numpy(), dc.free_top.cpu().numpy()), heads


def head_rows(dc, c):
    """(K [n,D], V [n,D], pos [n], lb [n]) of head c in slot order, from the device."""
    n = int(dc.len[c])
    pages = dc.block_table[c, torch.arange(n, device="cuda") // 16].long()
    offs = torch.arange(n, device="cuda") % 16
    return dc.k_pool[pages, offs], dc.v_pool[pages, offs], dc.pos_pool[pages, offs], dc.lb_pool[pages, offs]


def mini_cache(dc, heads):
    """Oracle cache holding only `heads` (each as its own KV head, fresh pages)."""
    cfg = dc.cfg
    rows = [head_rows(dc, c) for c in heads]
    lens = [int(r[0].shape[0]) for r in rows]
    maxp = max(1, max(-(-n // 16) for n in lens))
    n_pages = len(heads) * maxp
    kp = np.zeros((n_pages, 16, cfg.D), np.uint16 if cfg.kv_dtype == "bf16" else np.float32)
    vp = np.zeros_like(kp)
    pp = np.zeros((n_pages, 16), np.int32)
    lp = np.zeros((n_pages, 16), np.float32)
    table = np.full((len(heads), maxp), -1, np.int32)
    for j, (K, V, pos, lb) in enumerate(rows):
        n = lens[j]
        npg = -(-n // 16)
        table[j, :npg] = np.arange(npg) + j * maxp
        pad = npg * 16 - n
        kh = np.concatenate([workloads.rows_to_host(K), np.zeros((pad, cfg.D), kp.dtype)]).reshape(npg, 16, cfg.D)
        vh = np.concatenate([workloads.rows_to_host(V), np.zeros((pad, cfg.D), vp.dtype)]).reshape(npg, 16, cfg.D)
        kp[j * maxp: j * maxp + npg] = kh
        vp[j * maxp: j * maxp + npg] = vh
        pp[j * maxp: j * maxp + npg] = np.concatenate([pos.cpu().numpy(), np.zeros(pad, np.int32)]).reshape(npg, 16)
        lp[j * maxp: j * maxp + npg] = np.concatenate([lb.cpu().numpy(), np.zeros(pad, np.float32)]).reshape(npg, 16)
    return oracle.HostCache(1, 1, len(heads), cfg.G, cfg.D, 16, kp, vp, pp, lp, table, np.array(lens, np.int32),
                            np.zeros(1, np.int32), np.zeros(1, np.int32)), maxp


def check_attention(dc, heads, q, keep, out, lse, dm, scale):
    cfg = dc.cfg
    hc, maxp = mini_cache(dc, heads)
    kk = None
    if keep is not None:
        kk = np.zeros((len(heads), maxp * 16), np.uint8)
        for j, c in enumerate(heads):
            n = int(dc.len[c])
            kk[j, :n] = keep[j][:n]
    qs = q.reshape(cfg.C, cfg.G, cfg.D)[heads].cpu().numpy()
    o_ref, lse_ref, dm_ref = oracle.attention(hc, qs, scale, kk)
    kept_any = np.array([bool(kk[j, : hc.len[j]].any()) if kk is not None else hc.len[j] > 0
                         for j in range(len(heads))])
    assert_outputs_close(out.reshape(cfg.C, cfg.G, cfg.D)[heads].cpu().numpy(),
                         lse.reshape(cfg.C, cfg.G)[heads].cpu().numpy(),
                         dm.reshape(cfg.C, cfg.G)[heads].cpu().numpy(), o_ref, lse_ref, dm_ref, kept_any)


def run_workload(rkv, name, steps, seqs=None, sample=6, seed=0):
    cfg = workloads.CONFIGS[name]
    dc = workloads.prefill_cache(cfg, seed, device="cuda", n_steps=steps + 1)
    cache = rkv_cache(rkv, dc)
    sel = rkv.Selection.empty(cache)
    ws = rkv.Workspace(cache)
    outs = rkv.StepOutputs.empty(cache)
    LH = cfg.L * cfg.H
    rng = np.random.default_rng(seed)
    check_seqs = list(range(cfg.B)) if seqs is None else seqs
    full = len(check_seqs) == cfg.B
    for s in range(steps):
        inp = workloads.step_inputs(cfg, seed, s, "cuda")
        host, heads = meta_host(dc, check_seqs)
        sampled = sorted(int(x) for x in rng.choice(heads, size=min(sample, len(heads)), replace=False))
        before = {c: head_rows(dc, c) for c in sampled}
        top_before = int(dc.free_top.item())
        if inp["evict"]:
            rkv.score_select(cache, inp["t"], inp["m_global"], sel, ws)
            rkv.paged_decode_attn(cache, inp["q"], cfg.scale, sel, outs.out, outs.lse, outs.dropped, ws)
            sync()
            t_sub = inp["t"].cpu().numpy()[check_seqs]
            m_sub = inp["m_global"].cpu().numpy()[check_seqs]
            keep_o, kept_o = oracle.select(host, t_sub, m_sub)
            keep_g = masked_keep(keep_flags(sel, dc.max_pages)[heads], host.len)
            assert np.array_equal(sel.kept.cpu().numpy()[heads], kept_o), f"{name} step {s}: kept"
            assert np.array_equal(keep_g, keep_o), f"{name} step {s}: keep flags"
            pos_idx = {c: j for j, c in enumerate(heads)}
            check_attention(dc, sampled, inp["q"], [keep_o[pos_idx[c]] for c in sampled], outs.out, outs.lse,
                            outs.dropped, cfg.scale)
            rkv.compact_pages(cache, sel, ws)
            sync()
            oracle.compact(host, keep_o)
            assert np.array_equal(dc.len.cpu().numpy()[heads], host.len), f"{name} step {s}: len"
            assert np.array_equal(dc.block_table.cpu().numpy()[heads], host.block_table), f"{name} step {s}: tables"
            plan = sel.plan.cpu().numpy()
            assert int(dc.free_top.item()) == top_before + int(plan[cfg.C])
            if full:
                top = int(host.free_top[0])
                assert np.array_equal(dc.free_stack.cpu().numpy()[:top], host.free_stack[:top])
                assert np.array_equal(dc.pos_pool.cpu().numpy(), host.pos_pool)
                assert np.array_equal(dc.lb_pool.cpu().numpy().view(np.uint32), host.lb_pool.view(np.uint32))
            for c in sampled:  # rows moved whole: slot k now holds the row of the position it reports
                K0, V0, P0, _ = before[c]
                K1, V1, P1, _ = head_rows(dc, c)
                where = {int(p): i for i, p in enumerate(P0.cpu().numpy())}
                idx = torch.tensor([where[int(p)] for p in P1.cpu().numpy()], device="cuda", dtype=torch.long)
                assert torch.equal(K1, K0[idx]) and torch.equal(V1, V0[idx])
        else:
            rkv.paged_decode_attn(cache, inp["q"], cfg.scale, None, outs.out, outs.lse, outs.dropped, ws)
            sync()
            check_attention(dc, sampled, inp["q"], None, outs.out, outs.lse, outs.dropped, cfg.scale)
            assert float(outs.dropped.abs().max()) == 0.0
        rkv.append(cache, inp["t"], inp["k_new"], inp["v_new"], inp["lb_new"], ws)
        sync()
        rc = oracle.append(host, inp["t"].cpu().numpy()[check_seqs],
                           np.zeros((len(heads), 1), np.uint16), np.zeros((len(heads), 1), np.uint16),
                           inp["lb_new"].cpu().numpy()[heads])
        if full:
            assert rc == oracle.OK
            assert np.array_equal(dc.block_table.cpu().numpy(), host.block_table), f"{name} step {s}: append"
            assert np.array_equal(dc.len.cpu().numpy(), host.len)
            assert int(dc.free_top.item()) == int(host.free_top[0])
        assert ws.status() == 0
    return dc


def run_workload_fused(rkv, name, steps, seqs=None, sample=6, seed=0, all_heads_at=()):
    """As run_workload, through the single-launch rkv_decode_step: the oracle
    state, the sampled heads' rows and their attention inputs are taken before
    the call (the launch compacts and appends in place).  At the steps in
    all_heads_at every head of the checked sequences is compared, not a
    sample (heads split across CTAs, merged by warps or block-wide)."""
    cfg = workloads.CONFIGS[name]
    dc = workloads.prefill_cache(cfg, seed, device="cuda", n_steps=steps + 1)
    cache = rkv_cache(rkv, dc)
    sel = rkv.Selection.empty(cache)
    ws = rkv.Workspace(cache)
    outs = rkv.StepOutputs.empty(cache)
    rng = np.random.default_rng(seed)
    check_seqs = list(range(cfg.B)) if seqs is None else seqs
    full = len(check_seqs) == cfg.B
    for s in range(steps):
        inp = workloads.step_inputs(cfg, seed, s, "cuda")
        host, heads = meta_host(dc, check_seqs)
        sampled = sorted(int(x) for x in rng.choice(heads, size=min(sample, len(heads)), replace=False))
        if s in all_heads_at:
            sampled = [int(c) for c in heads]
        before = {c: head_rows(dc, c) for c in sampled}
        mini, maxp = mini_cache(dc, sampled)
        len_pre = host.len.copy()
        rkv.decode_step(cache, inp["t"], inp["m_global"] if inp["evict"] else None, inp["q"], cfg.scale,
                        inp["k_new"], inp["v_new"], inp["lb_new"], sel if inp["evict"] else None, outs.out, outs.lse,
                        outs.dropped, ws)
        sync()
        assert ws.status() == 0, f"{name} step {s}: {ws.counters()}"
        qs = inp["q"].reshape(cfg.C, cfg.G, cfg.D)[sampled].cpu().numpy()
        if inp["evict"]:
            t_sub = inp["t"].cpu().numpy()[check_seqs]
            m_sub = inp["m_global"].cpu().numpy()[check_seqs]
            keep_o, kept_o = oracle.select(host, t_sub, m_sub)
            keep_g = masked_keep(keep_flags(sel, dc.max_pages)[heads], len_pre)
            assert np.array_equal(sel.kept.cpu().numpy()[heads], kept_o), f"{name} step {s}: kept"
            assert np.array_equal(keep_g, keep_o), f"{name} step {s}: keep flags"
            pos_idx = {c: j for j, c in enumerate(heads)}
            kk = np.zeros((len(sampled), maxp * 16), np.uint8)
            for j, c in enumerate(sampled):
                kk[j, :len_pre[pos_idx[c]]] = keep_o[pos_idx[c]][:len_pre[pos_idx[c]]]
        else:
            kk = None
        o_ref, lse_ref, dm_ref = oracle.attention(mini, qs, cfg.scale, kk)
        kept_any = np.array([bool(kk[j, : mini.len[j]].any()) if kk is not None else mini.len[j] > 0
                             for j in range(len(sampled))])
        assert_outputs_close(outs.out.reshape(cfg.C, cfg.G, cfg.D)[sampled].cpu().numpy(),
                             outs.lse.reshape(cfg.C, cfg.G)[sampled].cpu().numpy(),
                             outs.dropped.reshape(cfg.C, cfg.G)[sampled].cpu().numpy(), o_ref, lse_ref, dm_ref,
                             kept_any)
        if inp["evict"]:
            oracle.compact(host, keep_o)
        rc = oracle.append(host, inp["t"].cpu().numpy()[check_seqs],
                           np.zeros((len(heads), 1), np.uint16), np.zeros((len(heads), 1), np.uint16),
                           inp["lb_new"].cpu().numpy()[heads])
        assert np.array_equal(dc.len.cpu().numpy()[heads], host.len), f"{name} step {s}: len"
        tb = dc.block_table.cpu().numpy()[heads]
        if not full:
            # a page popped by the append comes from the stack shared by every
            # head (pops in ascending head order): only full runs can check it
            for j in range(len(heads)):
                k = int(host.len[j]) - 1
                if k % 16 == 0:
                    tb[j, k // 16] = host.block_table[j, k // 16]
        assert np.array_equal(tb, host.block_table), f"{name} step {s}: tables"
        if full:
            assert rc == oracle.OK
            top = int(host.free_top[0])
            assert int(dc.free_top.item()) == top
            assert np.array_equal(dc.free_stack.cpu().numpy()[:top], host.free_stack[:top])
            assert np.array_equal(dc.pos_pool.cpu().numpy(), host.pos_pool)
            assert np.array_equal(dc.lb_pool.cpu().numpy().view(np.uint32), host.lb_pool.view(np.uint32))
        for c in sampled:  # kept rows moved whole, the new row appended last
            K0, V0, P0, _ = before[c]
            K1, V1, P1, _ = head_rows(dc, c)
            where = {int(p): i for i, p in enumerate(P0.cpu().numpy())}
            old_pos = P1.cpu().numpy()[:-1]
            idx = torch.tensor([where[int(p)] for p in old_pos], device="cuda", dtype=torch.long)
            assert torch.equal(K1[:-1], K0[idx]) and torch.equal(V1[:-1], V0[idx])
            assert torch.equal(K1[-1], inp["k_new"][c]) and torch.equal(V1[-1], inp["v_new"][c])
    return ws.counters()


def test_llama32k_prefill_eviction_and_steady_steps(rkv):
    run_workload(rkv, "llama32k", steps=3)


def test_long128k_prefill_eviction_and_steady_step(rkv):
    run_workload(rkv, "long128k", steps=2, sample=4)


def test_qwen8k_batched_subset(rkv):
    run_workload(rkv, "qwen8k", steps=2, seqs=[0, 15], sample=4)


def test_vlm16k_evicting_and_non_evicting_steps(rkv):
    run_workload(rkv, "vlm16k", steps=3, seqs=[0, 7], sample=4)


def test_fused_llama32k_prefill_eviction_and_steady_steps(rkv):
    ctr = run_workload_fused(rkv, "llama32k", steps=4)
    assert ctr["exact_steps"] >= 1 and ctr["window_steps"] >= 2, ctr   # prefill eviction exact, then mostly the window


def test_fused_llama32k_every_head_on_a_steady_step(rkv):
    # all 256 KV heads (1,024 query rows) of a steady evicting step, in the
    # launch configuration the benchmark times
    run_workload_fused(rkv, "llama32k", steps=3, sample=4, all_heads_at={2})


def test_fused_qwen8k_every_head_of_two_sequences_on_a_steady_step(rkv):
    run_workload_fused(rkv, "qwen8k", steps=3, seqs=[0, 15], sample=4, all_heads_at={2})


def test_fused_long128k_prefill_eviction_and_steady_steps(rkv):
    run_workload_fused(rkv, "long128k", steps=3, sample=4)


def test_fused_qwen8k_batched_subset(rkv):
    run_workload_fused(rkv, "qwen8k", steps=3, seqs=[0, 15], sample=4)


def test_fused_vlm16k_evicting_and_non_evicting_steps(rkv):
    run_workload_fused(rkv, "vlm16k", steps=3, seqs=[0, 7], sample=4)
