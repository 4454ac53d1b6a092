"""GPU parity of the latent memory for evicted tokens (rkv_memory_update,
rkv_memory_read) against the oracle.

IndexMem, Methodology B: evicted tokens folded into a decayed outer-product
state M, b; a gated read adds g(q) * m(q) to the attention output.  The state
is compared after every step (fp32 sums of products against fp64:
max |M - M_ref| <= 1e-4 * max |M_ref|, the accumulated rounding of a few
thousand fp32 terms) and the outputs at the attention tolerance (2e-3 of the
row norm), over several decode steps through the separate calls.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.gpu_helpers import assert_outputs_close, compare_state, keep_flags, masked_keep, rkv_cache, sync, to_dev
from tests.oracle_helpers import host_cache

pytestmark = pytest.mark.gpu

STATE_RTOL = 1e-4


def _run(rkv, cfg, seed, steps, decay):
    dc = to_dev(workloads.prefill_cache(cfg, seed, n_steps=steps + 1))
    hc = host_cache(dc)
    cache = rkv_cache(rkv, dc)
    sel, ws, outs = rkv.Selection.empty(cache), rkv.Workspace(cache), rkv.StepOutputs.empty(cache)
    w = workloads.memory_weights(cfg, seed, "cuda")
    mem = rkv.Memory.zeros(cache, w["proj"], w["gate_w"], w["gate_b"], decay)
    M_ref, b_ref = np.zeros((cfg.C, cfg.D, cfg.D)), np.zeros((cfg.C, cfg.D))
    wn = {k: v.cpu().numpy() for k, v in w.items()}
    for s in range(steps):
        inp = workloads.step_inputs(cfg, seed, s, "cuda")
        t, m = inp["t"].cpu().numpy(), inp["m_global"].cpu().numpy()
        q = inp["q"].cpu().numpy().reshape(cfg.C, cfg.G, cfg.D)
        len_before = hc.len.copy()
        rkv.step(cache, sel, ws, outs, q=inp["q"], t=inp["t"], m_global=inp["m_global"], k_new=inp["k_new"],
                 v_new=inp["v_new"], lb_new=inp["lb_new"], evict=inp["evict"], scale=cfg.scale, mem=mem)
        sync()
        assert ws.status() == 0
        keep = None
        if inp["evict"]:
            keep, kept = oracle.select(hc, t, m)
            assert np.array_equal(masked_keep(keep_flags(sel, dc.max_pages), len_before), keep)
            oracle.memory_update(hc, keep, wn["proj"], decay, M_ref, b_ref)
        o_ref, lse_ref, dm_ref = oracle.attention(hc, q, cfg.scale, keep)
        o_ref = oracle.memory_read(hc, q, wn["proj"], wn["gate_w"], wn["gate_b"], M_ref, b_ref, o_ref)
        Mg, bg = mem.M.cpu().numpy(), mem.b.cpu().numpy()
        assert np.abs(Mg - M_ref).max() <= STATE_RTOL * max(np.abs(M_ref).max(), 1e-30), f"step {s}: M"
        assert np.abs(bg - b_ref).max() <= STATE_RTOL * max(np.abs(b_ref).max(), 1e-30), f"step {s}: b"
        kept_any = (kept > 0) if keep is not None else (len_before > 0)
        assert_outputs_close(outs.out.cpu().numpy().reshape(cfg.C, cfg.G, cfg.D), None, None, o_ref, lse_ref,
                             dm_ref, kept_any | (np.abs(b_ref).sum(axis=1) > 0))
        if keep is not None:
            oracle.compact(hc, keep)
        assert oracle.append(hc, t, workloads.rows_to_host(inp["k_new"]), workloads.rows_to_host(inp["v_new"]),
                             inp["lb_new"].cpu().numpy()) == oracle.OK
        compare_state(dc, hc, pools=False)


@pytest.mark.parametrize("G,D,kv", [(4, 128, "bf16"), (2, 64, "bf16"), (7, 128, "bf16"), (1, 64, "f32")])
def test_memory_steps(rkv, G, D, kv):
    cfg = workloads.small_config(L=2, H=2, G=G, D=D, B=2, T0=900, M=1200, kv_dtype=kv, steps=4)
    _run(rkv, cfg, 31 + G, 4, 0.9)


def test_memory_with_steps_between_evictions(rkv):
    cfg = workloads.small_config(L=2, H=3, G=4, D=128, B=1, T0=1500, M=2000, kv_dtype="bf16", steps=6,
                                 evict_every=3)
    _run(rkv, cfg, 5, 6, 0.5)
