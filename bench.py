#!/usr/bin/env python
"""Benchmark: one decode step of retention-scored global KV eviction + paged
decode attention over the kept entries (select -> attention + dropped mass
-> compaction -> append), on synthetic 8B-class workloads.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl rkv|reference] [--config NAME]
                    [--per-config A,B,...] [--path fused|separate]

The printed line is for the headline workload (--config, default
"long128k": 32 layers x 8 KV heads, 32 query heads, head dim 128, bf16 K/V,
batch 1, 128K-token prefill, global budget M = 10% of the entries, evicting
every step).  The same process also measures the workloads of --per-config
(default llama32k, qwen8k, vlm16k) with the same K and W and reports them
under "per_config".

Every workload: step 0 (the prefill eviction) is run and timed alone
(step0_ms, with its own algorithmic bytes); W warm-up steps and K timed
steps follow the workload's schedule (vlm16k evicts every 16th step, the
others every step; a non-evicting step attends over every entry and
appends).  The per-step working set (hundreds of MB of K/V) is larger than
the 126 MB L2, so no L2 flush is inserted between steps.

Timing: the K timed steps are one CUDA graph replay bracketed by a barrier
and synchronize on both sides, timed with CUDA events on the launching
stream; multi-GPU runs are independent replicas (one copy of the workload
per rank, "scaling": "weak") and report the maximum over ranks.  On the
fused path (default: one rkv_decode_step launch per step) the graph holds
only the K launches, and the step kernel's average duration is the timed
region / K, launch gaps included.  For a workload that mixes evicting and
non-evicting steps, a second graph over 32 further steps records a CUDA
event after every launch and splits the time by step kind (the events add a
fixed cost per launch, reported and subtracted).  On the separate path
per-kernel CUDA events inside the graph split each step into its kernels.
The dominant kernel's algorithmic bytes over its duration is the roofline
entry.  e2e repeats the headline measurement through the public API with
packed pinned host inputs and outputs (one H2D + graph replay + one D2H per
step).  "variants" times the eviction error, the latent memory and the
per-head / ContourKV selections on steady llama32k steps through the
separate calls.  cpu_baseline times the CPU oracle on whole steady-state steps of the
headline workload on the host cores (one step single-threaded, two on every
core).  ``--impl reference`` times the oracle alone on whole steps, every
core.
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

import workloads  # noqa: E402

METRIC = "evict+paged-decode steps/s"
UNIT = "steps/s"
HEADLINE = "long128k"
PER_CONFIG = "llama32k,qwen8k,vlm16k"
SPLIT_STEPS = 32  # event-timed steps for the evicting / non-evicting split

# DRAM traffic (ncu dram__bytes_read.sum + dram__bytes_write.sum) of one
# launch of the fused step kernel on a steady long128k step: the 4-layer
# capture (read 218.88 MB + write 8.74 MB) x8 to the full 32-layer launch
# (pages, hence traffic, grow with the layer count).  Reported only while the
# kernel's sources hash to the captured version.
STEP_TRAFFIC = {"sources_sha256": "84b76a0cbdb33dbf", "workload": "long128k", "bytes_per_launch": 8 * 227.614208e6}
# The same for the separate path's attention kernel on a steady llama32k
# step: the 16-layer capture (read 135.23 MB + write 3.43 MB) x2.
ATTN_TRAFFIC = {"sources_sha256": "e28da1e460e372cf", "workload": "llama32k", "bytes_per_launch": 2 * 138.661632e6}


# ------------------------------------------------------------------ ranks ---
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    return world, rank, local


def dist_init(world: int, backend: str):
    if world > 1 and not torch.distributed.is_initialized():
        import datetime
        torch.distributed.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))


def barrier(world: int):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(x: float, world: int, device=None) -> float:
    """Maximum of a per-rank scalar (all ranks call this, in the same order)."""
    if world <= 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


# ----------------------------------------------------------------- clocks ---
class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
        0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
        0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
    }

    def __init__(self, index: int, period_s: float = 0.005):
        self.index, self.period = index, period_s
        self.samples: list[tuple[int, int]] = []
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self._nv = None

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                clk = nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                self.samples.append((clk, rs))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self._stop.clear()
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *exc):
        if self._t is not None:
            self._stop.set()
            self._t.join()
            self._t = None

    def summary(self) -> dict:
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        clks = [c for c, _ in self.samples]
        rs = 0
        for _, r in self.samples:
            rs |= r
        names = [n for bit, n in self.REASONS.items() if rs & bit and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(clks), "sm_max_mhz": self.max_mhz, "reasons": names,
                "samples": len(clks)}


def merge_clocks(parts: list[dict]) -> dict:
    """One clocks record over several sampled regions: median of the
    medians, every reason seen, the sample count."""
    got = [p for p in parts if p and p.get("samples")]
    if not got:
        return parts[0] if parts else {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
    return {"sm_mhz": statistics.median(p["sm_mhz"] for p in got), "sm_max_mhz": got[0]["sm_max_mhz"],
            "reasons": sorted(set(r for p in got for r in p["reasons"])), "samples": sum(p["samples"] for p in got)}


# ------------------------------------------------------------- CPU oracle ---
def host_cpu() -> dict:
    """The host the oracle runs on: logical CPUs and the CPU model name."""
    model = None
    try:
        with open("/proc/cpuinfo") as fh:
            for line in fh:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"nproc": os.cpu_count(), "model": model}


def one_sequence(cfg: workloads.Config) -> workloads.Config:
    return dataclasses.replace(cfg, name=cfg.name, B=1, M=cfg.M)


def oracle_steady_state(cfg: workloads.Config, n_steps: int, seed: int):
    """Host cache of one sequence in the steady-state shape of an evicting
    step: every head holds M/(L*H) + 1 entries (the kept set plus the token
    appended after the last eviction)."""
    import oracle
    per_head = cfg.M // (cfg.L * cfg.H) + 1
    pages = -(-per_head // 16)
    dc = workloads.ragged_cache(cfg, seed, [per_head] * cfg.C, n_pages=cfg.C * (pages + 2 + n_steps // 16 + 2),
                                max_pages=pages + n_steps // 16 + 4)
    return oracle.HostCache(**workloads.to_host(dc))


def time_oracle(cfg: workloads.Config, steps: int, warmup: int, seed: int, threads: int) -> dict:
    """Whole steady-state evicting steps of one sequence of the workload
    through the CPU oracle (select, fp64 attention + dropped mass,
    compaction, append): seconds per step, measured step by step."""
    import oracle
    cs = one_sequence(cfg)
    hc = oracle_steady_state(cs, steps + warmup + 2, seed)
    used = oracle.use_threads(threads)
    per = []
    for s in range(steps + warmup):
        inp = workloads.step_inputs(cs, seed, s)
        t0 = time.perf_counter()
        oracle.step(hc, inp["t"].numpy(), inp["m_global"].numpy(), inp["q"].numpy().reshape(cs.C, cs.G, cs.D),
                    workloads.rows_to_host(inp["k_new"]), workloads.rows_to_host(inp["v_new"]),
                    inp["lb_new"].numpy(), evict=True, scale=cs.scale)
        if s >= warmup:
            per.append(time.perf_counter() - t0)
    oracle.use_threads(1)
    sec = sum(per) / max(len(per), 1)
    # the sequences of a batch are independent: a batch step is B of these
    return {"sec_per_seq_step": sec, "value": 1.0 / (sec * cfg.B), "timed": len(per), "cores": used,
            "sample": (f"{len(per)} whole steady-state evicting step(s) of {cfg.name} "
                       f"(N_pre {cs.M + cs.C}, M {cs.M}, {cs.L} layers x {cs.H} KV heads)"
                       + (f" of one of the {cfg.B} independent sequences, time x{cfg.B}" if cfg.B > 1 else ""))}


# ------------------------------------------------------------------ bytes ---
def elt(cfg: workloads.Config) -> int:
    return 2 if cfg.kv_dtype == "bf16" else 4


def attn_bytes(cfg: workloads.Config, n_pre: int, kept: int, pages: int) -> int:
    """Algorithmic HBM bytes of one attention pass: K of every pre-eviction
    entry (dense logits for the dropped mass), V of the kept entries, q, out,
    lse + dropped, block-table entries and keep-mask words."""
    e = elt(cfg)
    return (e * cfg.D * n_pre + e * cfg.D * kept + 2 * 4 * cfg.C * cfg.G * cfg.D + 2 * 4 * cfg.C * cfg.G
            + 4 * pages + 2 * pages)


def step_bytes(cfg: workloads.Config, n_pre: int, kept: int, pages: int, evict: bool = True, moves: int = 0) -> int:
    """Algorithmic bytes of the whole step: attention + (evicting steps) the
    position and log-retention of every entry (selection) + rows moved by
    compaction (read and written) + the appended rows (K, V, position, lb)."""
    row = 2 * elt(cfg) * cfg.D + 8
    sel = 8 * n_pre if evict else 0
    return attn_bytes(cfg, n_pre, kept, pages) + sel + 2 * row * moves + cfg.C * row


# -------------------------------------------------------------- rkv arm ---
def run_config(name: str, args, world: int, rank: int, local: int, *, e2e: bool) -> dict:
    """Prefill, step 0, warm-up and K timed steps of one workload on this rank."""
    import retention_scored_kv_b200 as rkv
    cfg = workload_config(name, args.layers)
    dev = torch.device("cuda", local)
    seed = args.seed + 1000 * rank
    K, W = args.steps, args.warmup
    fused = args.path == "fused"
    split = cfg.evict_every > 1 and fused
    total = 1 + W + K + (SPLIT_STEPS if split else 0) + (W + K if e2e else 0) + 2
    dc = workloads.prefill_cache(cfg, seed, device=dev, n_steps=total)
    cache = rkv.Cache.from_tensors(dc, cfg.B, cfg.L, cfg.H, cfg.Hq)
    stream = torch.cuda.Stream(device=dev)
    runner = rkv.StepRunner(cache, scale=cfg.scale, stream=stream, fused=fused, buffers=2)
    sel, ws, outs = runner.sel, runner.ws, runner.outs
    per_step = [workloads.step_inputs(cfg, seed, s, dev) for s in range(total)]
    kernel_names = ["step"] if fused else ["select", "attn", "compact", "append"]

    def enqueue(s, ev=None):
        inp = per_step[s]
        ev_ = ev if ev is not None else [None] * 4
        if fused:
            rkv.decode_step(cache, inp["t"], inp["m_global"] if inp["evict"] else None, inp["q"], cfg.scale,
                            inp["k_new"], inp["v_new"], inp["lb_new"], sel if inp["evict"] else None, outs.out,
                            outs.lse, outs.dropped, ws, stream)
            if ev_[0] is not None:
                ev_[0].record(stream)
            return
        if inp["evict"]:
            rkv.score_select(cache, inp["t"], inp["m_global"], sel, ws, stream)
        if ev_[0] is not None:
            ev_[0].record(stream)
        rkv.paged_decode_attn(cache, inp["q"], cfg.scale, sel if inp["evict"] else None, outs.out, outs.lse,
                              outs.dropped, ws, stream)
        if ev_[1] is not None:
            ev_[1].record(stream)
        if inp["evict"]:
            rkv.compact_pages(cache, sel, ws, stream)
        if ev_[2] is not None:
            ev_[2].record(stream)
        rkv.append(cache, inp["t"], inp["k_new"], inp["v_new"], inp["lb_new"], ws, stream)
        if ev_[3] is not None:
            ev_[3].record(stream)

    # load the kernels of this shape once on a throwaway cache, so that the
    # first-launch cost (module loading) stays out of step 0's time
    wcfg = workloads.small_config(L=1, H=1, G=cfg.G, D=cfg.D, B=1, T0=64, M=32, kv_dtype=cfg.kv_dtype, steps=1)
    wdc = workloads.prefill_cache(wcfg, 0, device=dev, n_steps=2)
    wcache = rkv.Cache.from_tensors(wdc, wcfg.B, wcfg.L, wcfg.H, wcfg.Hq)
    winp = workloads.step_inputs(wcfg, 0, 0, dev)
    wsel, wws, wouts = rkv.Selection.empty(wcache), rkv.Workspace(wcache, stream), rkv.StepOutputs.empty(wcache)
    rkv.step(wcache, wsel, wws, wouts, q=winp["q"], t=winp["t"], m_global=winp["m_global"], k_new=winp["k_new"],
             v_new=winp["v_new"], lb_new=winp["lb_new"], scale=wcfg.scale, fused=fused, stream=stream)
    torch.cuda.synchronize()
    del wdc, wcache, wsel, wws, wouts

    # step 0: the prefill eviction, timed alone
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        enqueue(0)
        e1.record(stream)
    torch.cuda.synchronize()
    step0_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    step0 = step0_record(cfg, sel, step0_ms, _peaks())
    s_next = 1

    with torch.cuda.stream(stream):
        for _ in range(W):
            enqueue(s_next)
            s_next += 1
    torch.cuda.synchronize()

    # timed: K steps captured in one graph (separate path: per-kernel events
    # inside; the fused path's graph holds the launches alone)
    evs = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(5)] for _ in range(K)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    first = s_next

    def timed_body():
        for i in range(K):
            if fused:
                enqueue(first + i)
            else:
                evs[i][4].record(stream)
                enqueue(first + i, evs[i][:4])

    graph = capture(timed_body, stream, args.no_graph)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    sel0 = ws.counters()
    with ClockSampler(local) as clk:
        with torch.cuda.stream(stream):
            t_start.record(stream)
            if graph is not None:
                graph.replay()
            else:
                timed_body()
            t_end.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    s_next = first + K
    ms_max = max_over_ranks(t_start.elapsed_time(t_end), world, dev)
    if ws.status() != 0:
        raise RuntimeError(f"{cfg.name}: device status {ws.counters()} after the timed steps")
    sel1 = ws.counters()
    # how the timed steps selected: inside the threshold window kept from the
    # previous step, or by the exact radix fallback
    selection = {k: sel1[k] - sel0[k] for k in ("window_steps", "exact_steps")}
    evicting = [per_step[first + i]["evict"] for i in range(K)]
    if fused:
        # one launch per step and nothing else in the timed region: the step
        # kernel's average duration is at most the region / K
        kern_us = {"step": 1000.0 * ms_max / K}
    else:
        kern = {k: [] for k in kernel_names}
        for i in range(K):
            marks = [evs[i][4]] + evs[i][:4]
            for j, k in enumerate(kernel_names):
                kern[k].append(marks[j].elapsed_time(marks[j + 1]))
        kern_us = {k: 1000.0 * statistics.mean(v) for k, v in kern.items()}
    del graph

    # sizes of the timed steps.  An evicting step sees N_pre = M + C(j)
    # entries per sequence (M kept at the last eviction, one appended per
    # head and step since); head c of a step j steps after the last eviction
    # holds kept_c + j entries (kept_c from the last evicting step).
    kept_c = sel.kept.to(torch.int64)
    n_pre_ev = int(sel.n_pre.sum().item())
    kept_ev = int(sel.kept.sum().item())
    pages_ev = int(((sel.n_pre + 15) // 16).sum().item())
    moves_ev = count_moves(sel)
    bytes_of = []
    for i in range(K):
        s = first + i
        if per_step[s]["evict"]:
            bytes_of.append(step_bytes(cfg, n_pre_ev, kept_ev, pages_ev, True, moves=moves_ev))
        else:
            j = s % cfg.evict_every
            n = kept_ev + j * cfg.C
            pages = int(((kept_c + j + 15) // 16).sum().item())
            bytes_of.append(step_bytes(cfg, n, n, pages, False))
    clocks = clk.summary()

    split_rec = None
    if split:
        split_rec, s_next = evict_split(cfg, enqueue, per_step, s_next, stream, world, dev, kept_ev, kept_c,
                                        n_pre_ev, pages_ev, moves_ev, 1000.0 * ms_max / K)

    e2e_rec = None
    if e2e and not args.skip_e2e:
        e2e_rec, s_next, c2 = run_e2e(runner, per_step, s_next, W, K, stream, world, local, dev)
        clocks = merge_clocks([clocks, c2])

    peaks = _peaks()
    step_s = ms_max / K / 1000.0
    s_bytes = sum(bytes_of) / K
    if fused:
        a_bytes, dom_s = s_bytes, kern_us["step"] * 1e-6
        kernel_desc = "step_kernel (selection + paged decode attention + dropped mass + compaction + append)"
        traffic = kernel_traffic(cfg, args.traffic, STEP_TRAFFIC, TRAFFIC_SOURCES)
    else:
        a_bytes = attn_bytes(cfg, n_pre_ev, kept_ev, pages_ev)
        dom_s = kern_us["attn"] * 1e-6
        kernel_desc = "attn_kernel (paged decode attention + dropped mass)"
        traffic = kernel_traffic(cfg, args.traffic, ATTN_TRAFFIC, ATTN_TRAFFIC_SOURCES)
    achieved = a_bytes / dom_s / 1e9
    retained = elt(cfg) * 2 * cfg.D * kept_ev
    return {
        "cfg": cfg, "ms_max": ms_max, "value": world * K / (ms_max / 1000.0), "us_per_step": 1000.0 * ms_max / K,
        "kernels_us": kern_us, "selection": selection, "clocks": clocks, "step0": step0,
        "n_pre_per_evicting_step": n_pre_ev, "kept_per_evicting_step": kept_ev,
        "evicting_steps": sum(evicting), "non_evicting_steps": K - sum(evicting),
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / peaks["hbm_gbs"], "traffic": traffic, "kernel": kernel_desc,
                     "bytes_per_launch": a_bytes, "peak_source": peaks["source"],
                     "duration": ("timed region / K (one launch per step, launch gaps included)" if fused
                                  else "per-kernel CUDA events inside the timed graph")},
        "step_hbm": {"bytes_per_step": s_bytes, "achieved_gbs": s_bytes / step_s / 1e9,
                     "frac": s_bytes / step_s / 1e9 / peaks["hbm_gbs"]},
        "retained_kv": {"gbs": retained / step_s / 1e9, "frac_of_peak": retained / step_s / 1e9 / peaks["hbm_gbs"]},
        "split": split_rec, "e2e": e2e_rec, "gpu_launches": len(kernel_names) * K,
        "head_lengths": head_length_stats(sel), "dropped_mass": dropped_stats(outs, evicting[-1] if K else True),
    }


def capture(body, stream, no_graph: bool):
    """body() captured into one CUDA graph on `stream` (None: eager timing)."""
    if no_graph:
        return None
    try:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream, capture_error_mode="thread_local"):
            body()
        _graph_upload(graph, stream)
        return graph
    except Exception as ex:  # capture refused: time eager launches instead
        print(f"[bench] graph capture failed ({ex}); timing eager launches", file=sys.stderr)
        return None


def step0_record(cfg: workloads.Config, sel, ms: float, peaks: dict) -> dict:
    """Step 0 (the prefill eviction): its time and algorithmic bytes -- the
    position, log-retention and K of every prefill entry, V of the kept
    ones, q/out, rows moved by the hole-fill compaction (read and written),
    the appended rows -- against the HBM peak."""
    n_pre = int(sel.n_pre.sum().item())
    kept = int(sel.kept.sum().item())
    pages = int(((sel.n_pre + 15) // 16).sum().item())
    moves = count_moves(sel)
    b = step_bytes(cfg, n_pre, kept, pages, True, moves=moves)
    gbs = b / (ms * 1e-3) / 1e9
    return {"ms": ms, "n_pre": n_pre, "kept": kept, "moves": moves, "bytes": b, "achieved_gbs": gbs,
            "frac": gbs / peaks["hbm_gbs"]}


def count_moves(sel) -> int:
    """Rows the hole-fill compaction of the last evicting step moved: kept
    slots at or above each head's new length (one per hole filled)."""
    moves = 0
    for c0 in range(0, sel.kept.shape[0], 64):
        m = sel.keep_mask[c0:c0 + 64].view(torch.int16).to(torch.int32) & 0xFFFF
        bits = (m.unsqueeze(-1) >> torch.arange(16, device=m.device, dtype=torch.int32)) & 1
        slot = torch.arange(m.shape[1] * 16, device=m.device, dtype=torch.int32).view(1, -1)
        flags = bits.view(m.shape[0], -1).bool()
        valid = slot < sel.n_pre[c0:c0 + 64].view(-1, 1)
        moves += int((flags & valid & (slot >= sel.kept[c0:c0 + 64].view(-1, 1))).sum().item())
    return moves


def head_length_stats(sel) -> dict:
    """Kept entries per head after the last evicting step: min / median / max."""
    k = sel.kept.to(torch.float64)
    return {"min": int(k.min().item()), "median": float(k.median().item()), "max": int(k.max().item())}


def dropped_stats(outs, evicting: bool) -> dict | None:
    """Dropped mass of the last timed step over every (sequence, layer, query
    head): mean, median, max (None after a non-evicting step, where it is 0)."""
    if not evicting:
        return None
    d = outs.dropped.to(torch.float64).flatten()
    return {"mean": float(d.mean().item()), "median": float(d.median().item()), "max": float(d.max().item())}


def evict_split(cfg, enqueue, per_step, s_next, stream, world, dev, kept_ev, kept_c, n_pre_ev, pages_ev, moves_ev,
                mean_free_us):
    """Per-kind step times of a mixed schedule: SPLIT_STEPS further steps in
    one graph with a CUDA event after every launch.  The events add a fixed
    cost per launch; it is estimated as the event-timed mean minus the
    event-free mean of the main timing (same schedule) and subtracted."""
    n = SPLIT_STEPS
    evs = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(n + 1)]
    first = s_next

    def body():
        evs[0].record(stream)
        for i in range(n):
            enqueue(first + i)
            evs[i + 1].record(stream)

    graph = capture(body, stream, False)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        if graph is not None:
            graph.replay()
        else:
            body()
    torch.cuda.synchronize()
    ms = [evs[i].elapsed_time(evs[i + 1]) for i in range(n)]
    ms = [max_over_ranks(x, world, dev) for x in ms]
    del graph
    kinds = [per_step[first + i]["evict"] for i in range(n)]
    ev_us = [1000.0 * x for x, e in zip(ms, kinds) if e]
    ne_us = [1000.0 * x for x, e in zip(ms, kinds) if not e]
    # event cost per launch: event-timed mean over whole cycles vs event-free mean
    cyc = (n // cfg.evict_every) * cfg.evict_every
    over = max(0.0, 1000.0 * sum(ms[:cyc]) / max(cyc, 1) - mean_free_us) if cyc else 0.0
    peaks = _peaks()
    b_ev = step_bytes(cfg, n_pre_ev, kept_ev, pages_ev, True, moves=moves_ev)
    j_mean = (cfg.evict_every) / 2.0
    n_ne = kept_ev + int(round(j_mean * cfg.C))
    pages_ne = int(((kept_c + int(round(j_mean)) + 15) // 16).sum().item())
    b_ne = step_bytes(cfg, n_ne, n_ne, pages_ne, False)

    def rec(us, b):
        if not us:
            return None
        raw = statistics.mean(us)
        adj = max(raw - over, 1e-3)
        return {"us_events": raw, "us": adj, "steps": len(us), "bytes": b,
                "frac": b / (adj * 1e-6) / 1e9 / peaks["hbm_gbs"]}

    return {"evicting": rec(ev_us, b_ev), "non_evicting": rec(ne_us, b_ne), "event_cost_us": over,
            "note": (f"{n} steps, CUDA event after every launch; the per-launch event cost (event-timed mean "
                     f"minus the event-free mean over whole {cfg.evict_every}-step cycles) is subtracted")}, \
        first + n


def run_e2e(runner, per_step, s_next, W, K, stream, world, local, dev):
    """The headline metric through the public API from pinned host memory:
    every step one H2D copy of the packed inputs, the step, one D2H copy of
    the packed outputs."""
    runner.capture()
    host_in = [torch.empty(runner.in_bytes, dtype=torch.uint8, pin_memory=True) for _ in range(W + K)]
    host_out = [torch.empty(runner.out_bytes, dtype=torch.uint8, pin_memory=True) for _ in range(W + K)]
    evict = []
    for i in range(W + K):
        inp = per_step[s_next + i]
        runner.pack(host_in[i], q=inp["q"].cpu(), k_new=inp["k_new"].cpu(), v_new=inp["v_new"].cpu(),
                    lb_new=inp["lb_new"].cpu(), t=inp["t"].cpu(), m_global=inp["m_global"].cpu())
        evict.append(bool(inp["evict"]))
    for i in range(W):
        runner.run_host(host_in[i], host_out[i], evict[i])
    runner.finish()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk2:
        a.record(stream)
        for i in range(W, W + K):
            runner.run_host(host_in[i], host_out[i], evict[i])
        runner.finish()
        b.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    e2e_ms = max_over_ranks(a.elapsed_time(b), world, dev)
    if runner.ws.status() != 0:
        raise RuntimeError(f"device status {runner.ws.counters()} after the e2e steps")
    rec = {"value": world * K / (e2e_ms / 1000.0), "unit": UNIT, "h2d_bytes_per_step": runner.in_bytes,
           "d2h_bytes_per_step": runner.out_bytes, "graph": bool(runner.graphs),
           "copies": "two buffer slots: step s+1's inputs and step s-1's outputs copied on a second stream while step s runs"}
    return rec, s_next + W + K, clk2.summary()


def run_variants(args, world: int, rank: int, local: int) -> dict:
    """The rows beyond the default step, measured on steady llama32k decode
    steps through the separate calls (one CUDA graph of K steps with an
    event after every launch): the eviction error, the latent-memory update
    and read, and the per-head and ContourKV selections (run on the same
    pre-step cache into their own selection buffers).  Each reports its
    device time and its algorithmic bytes against the HBM peak."""
    import retention_scored_kv_b200 as rkv
    cfg = workload_config("llama32k", args.layers)
    dev = torch.device("cuda", local)
    seed = args.seed + 1000 * rank + 7
    K, W = args.steps, args.warmup
    total = 1 + W + K + 2
    dc = workloads.prefill_cache(cfg, seed, device=dev, n_steps=total)
    cache = rkv.Cache.from_tensors(dc, cfg.B, cfg.L, cfg.H, cfg.Hq)
    stream = torch.cuda.Stream(device=dev)
    sel, ws, outs = rkv.Selection.empty(cache), rkv.Workspace(cache, stream), rkv.StepOutputs.empty(cache)
    sel_h, sel_c = rkv.Selection.empty(cache), rkv.Selection.empty(cache)
    wts = workloads.memory_weights(cfg, seed, dev)
    mem = rkv.Memory.zeros(cache, wts["proj"], wts["gate_w"], wts["gate_b"], 0.99)
    err = torch.empty(cfg.B, cfg.L, cfg.Hq, device=dev)
    per_step = [workloads.step_inputs(cfg, seed, s, dev) for s in range(total)]
    m_head = torch.full((cfg.C,), cfg.M // cfg.C, dtype=torch.int32, device=dev)
    dm_prev = torch.zeros(cfg.B, cfg.L, cfg.Hq, device=dev)
    tau, flat_budget, floor = 2e-4, 2048, 64
    names = ["per_head_select", "contour_select", "select", "memory_update", "attn", "eviction_error",
             "memory_read", "compact", "append"]

    def enqueue(s, ev=None):
        i = per_step[s]
        calls = [
            lambda: rkv.score_select_per_head(cache, i["t"], m_head, sel_h, ws, stream),
            lambda: rkv.score_select_contour(cache, i["t"], i["m_global"], dm_prev, tau, flat_budget, floor, sel_c,
                                             ws, stream),
            lambda: rkv.score_select(cache, i["t"], i["m_global"], sel, ws, stream),
            lambda: rkv.memory_update(cache, sel, mem, stream),
            lambda: rkv.paged_decode_attn(cache, i["q"], cfg.scale, sel, outs.out, outs.lse, outs.dropped, ws,
                                          stream),
            lambda: rkv.eviction_error(cache, i["q"], cfg.scale, sel, outs.out, outs.dropped, err, ws, stream),
            lambda: rkv.memory_read(cache, i["q"], mem, outs.out, stream),
            lambda: rkv.compact_pages(cache, sel, ws, stream),
            lambda: rkv.append(cache, i["t"], i["k_new"], i["v_new"], i["lb_new"], ws, stream),
        ]
        if ev is not None:
            ev[0].record(stream)
        for j, f in enumerate(calls):
            f()
            if ev is not None:
                ev[j + 1].record(stream)
        dm_prev.copy_(outs.dropped)  # the next step's ContourKV statistic

    with torch.cuda.stream(stream):
        # step 0 (prefill eviction) and warm-up through the fused launch
        for s in range(1 + W):
            i = per_step[s]
            rkv.decode_step(cache, i["t"], i["m_global"], i["q"], cfg.scale, i["k_new"], i["v_new"], i["lb_new"],
                            sel, outs.out, outs.lse, outs.dropped, ws, stream)
        for s in range(1 + W, 1 + W + 2):
            enqueue(s)   # loads the variants' kernels
    torch.cuda.synchronize()
    first = 1 + W + 2
    Kv = min(K, total - first)
    evs = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(len(names) + 1)] for _ in range(Kv)]
    graph = capture(lambda: [enqueue(first + i, evs[i]) for i in range(Kv)], stream, args.no_graph)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        if graph is not None:
            graph.replay()
        else:
            for i in range(Kv):
                enqueue(first + i, evs[i])
    torch.cuda.synchronize()
    if ws.status() != 0:
        raise RuntimeError(f"variants: device status {ws.counters()}")
    us = {n: 1000.0 * statistics.mean(evs[i][j].elapsed_time(evs[i][j + 1]) for i in range(Kv))
          for j, n in enumerate(names)}
    us = {n: max_over_ranks(v, world, dev) for n, v in us.items()}
    del graph
    # algorithmic bytes of the last step (steady state)
    e = elt(cfg)
    n_pre = int(sel.n_pre.sum().item())
    kept = int(sel.kept.sum().item())
    pages = int(((sel.n_pre + 15) // 16).sum().item())
    evicted = n_pre - kept
    rows_q = cfg.C * cfg.G
    state = cfg.C * (cfg.D * cfg.D + cfg.D) * 4
    proj = cfg.L * cfg.D * cfg.D * 4
    sel_bytes = 8 * n_pre + 6 * pages + 12 * cfg.C
    byts = {
        "per_head_select": sel_bytes,
        "contour_select": sel_bytes + 4 * rows_q,
        "eviction_error": 2 * e * cfg.D * evicted + 6 * pages + 2 * 4 * rows_q * cfg.D + 3 * 4 * rows_q,
        "memory_update": 2 * e * cfg.D * evicted + 6 * pages + 2 * state + proj,
        "memory_read": state + proj + 3 * 4 * rows_q * cfg.D + 4 * cfg.L * cfg.Hq * (cfg.D + 1),
    }
    peak = _peaks()["hbm_gbs"]
    out = {}
    for n, b in byts.items():
        gbs = b / (us[n] * 1e-6) / 1e9
        out[n] = {"us": us[n], "bytes": b, "achieved_gbs": gbs, "frac": gbs / peak}
    out["context"] = {"workload": describe(cfg), "evicted_per_step": evicted, "steps": Kv,
                      "timing": "CUDA events after every launch inside one graph of K separate-call steps",
                      "other_kernels_us": {n: us[n] for n in ("select", "attn", "compact", "append")},
                      "contour": {"flat_threshold": tau, "flat_budget": flat_budget, "recency_floor": floor,
                                  "flat_heads": int((dm_prev.view(cfg.C, cfg.G).mean(dim=1) > tau).sum().item())},
                      "per_head_budget": cfg.M // cfg.C}
    return out


def describe(cfg: workloads.Config) -> str:
    sched = "every step evicts" if cfg.evict_every == 1 else f"evicts every {cfg.evict_every} steps"
    return (f"{cfg.name}: L{cfg.L} H{cfg.H} Hq{cfg.Hq} D{cfg.D} B{cfg.B} T0 {cfg.T0} M {cfg.M} per sequence, "
            f"{cfg.kv_dtype} K/V, steady-state decode steps ({sched})")


def summary(r: dict) -> dict:
    """The per-workload record reported under per_config."""
    cfg = r["cfg"]
    out = {"workload": describe(cfg), "us_per_step": r["us_per_step"], "value": r["value"], "unit": UNIT,
           "roofline": {k: r["roofline"][k] for k in ("achieved", "peak", "frac", "bytes_per_launch", "traffic")},
           "selection": r["selection"], "step0": r["step0"], "clocks": r["clocks"],
           "evicting_steps": r["evicting_steps"], "non_evicting_steps": r["non_evicting_steps"],
           "head_lengths": r["head_lengths"], "dropped_mass": r["dropped_mass"]}
    if r["split"] is not None:
        out["split"] = r["split"]
    return out


def run_rkv(args, world, rank, local):
    import retention_scored_kv_b200 as rkv
    torch.cuda.set_device(local)
    dist_init(world, "nccl")
    rkv.load()
    head = run_config(args.config, args, world, rank, local, e2e=True)
    per = {}
    for name in [n for n in args.per_config.split(",") if n and n != args.config]:
        r = run_config(name, args, world, rank, local, e2e=False)
        per[name] = summary(r)
        del r
        torch.cuda.empty_cache()
    variants = None
    if not args.skip_variants:
        variants = run_variants(args, world, rank, local)
        torch.cuda.empty_cache()
    cfg = head["cfg"]

    cpu = None
    if rank == 0 and world == 1 and not args.skip_cpu_baseline:
        one = time_oracle(cfg, steps=1, warmup=0, seed=args.seed, threads=1)
        allc = time_oracle(cfg, steps=2, warmup=0, seed=args.seed, threads=0)
        cpu = {"value": allc["value"], "unit": UNIT, "cores": allc["cores"], "kind": "oracle",
               "sample": allc["sample"] + ", every core (OpenMP over heads)",
               "single_core": {"value": one["value"], "cores": 1, "sample": one["sample"]},
               "host": host_cpu()}

    line = {
        "metric": METRIC, "value": head["value"], "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": head["ms_max"] / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": cfg.kv_dtype, "data": "synthetic",
        "config": {"workload": describe(cfg), "kv_dtype": cfg.kv_dtype, "accumulate": "f32",
                   "batch": cfg.B, "context": cfg.T0, "budget": cfg.M,
                   "n_pre_per_step": head["n_pre_per_evicting_step"], "kept_per_step": head["kept_per_evicting_step"],
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "l2": "no flush: per-step K/V working set > 126 MB L2", "graph": not args.no_graph},
        "roofline": head["roofline"], "step_hbm": head["step_hbm"], "retained_kv": head["retained_kv"],
        "kernels_us": head["kernels_us"], "us_per_step": head["us_per_step"], "step0_ms": head["step0"]["ms"],
        "step0": head["step0"], "cpu_baseline": cpu, "e2e": head["e2e"], "gpu_launches": head["gpu_launches"],
        "clocks": merge_clocks([head["clocks"]] + [p["clocks"] for p in per.values()]),
        "path": args.path, "selection": head["selection"], "head_lengths": head["head_lengths"],
        "dropped_mass": head["dropped_mass"], "per_config": per, "variants": variants,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


def workload_config(name: str, layers: int = 0) -> workloads.Config:
    """The named workload, optionally cut to fewer layers (budget scaled alike)
    -- a smaller case of the same kernels for profiler captures."""
    cfg = workloads.CONFIGS[name]
    if layers and layers != cfg.L:
        cfg = dataclasses.replace(cfg, name=f"{cfg.name}-{layers}L", L=layers, M=cfg.M * layers // cfg.L)
    return cfg


def _graph_upload(graph, stream):
    """Upload an instantiated graph ahead of its first replay (cudaGraphUpload)."""
    try:
        import ctypes
        lib = ctypes.CDLL("libcudart.so.12")
        lib.cudaGraphUpload.restype = ctypes.c_int
        lib.cudaGraphUpload.argtypes = [ctypes.c_void_p, ctypes.c_void_p]
        lib.cudaGraphUpload(ctypes.c_void_p(graph.raw_cuda_graph_exec()), ctypes.c_void_p(stream.cuda_stream))
    except Exception:
        pass


TRAFFIC_SOURCES = ("retention_scored_kv_b200/csrc/step.cu", "retention_scored_kv_b200/csrc/attn_core.cuh",
                   "retention_scored_kv_b200/csrc/common.cuh")
ATTN_TRAFFIC_SOURCES = ("retention_scored_kv_b200/csrc/attn.cu", "retention_scored_kv_b200/csrc/attn_core.cuh",
                        "retention_scored_kv_b200/csrc/common.cuh")


def sources_sha(files=TRAFFIC_SOURCES) -> str:
    import hashlib
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def kernel_traffic(cfg: workloads.Config, override, rec: dict, files) -> float | None:
    """ncu DRAM bytes per launch of the kernel `rec` records on this workload,
    or None if not measured for these sources and this workload."""
    if override is not None:
        return override
    if rec and cfg.name == rec["workload"] and sources_sha(files) == rec["sources_sha256"]:
        return rec["bytes_per_launch"]
    return None


def _peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "source": "measured (MEASURED_PEAKS.json)"}
    except Exception:
        return {"hbm_gbs": 6650.0, "source": "fallback 6.65 TB/s"}


# -------------------------------------------------------- reference arm ---
def run_reference(args, world, rank):
    """The CPU oracle alone, on whole steady-state steps of the workload,
    every host core; rank 0 only."""
    if rank != 0:
        return
    cfg = workload_config(args.config, args.layers)
    o = time_oracle(cfg, steps=args.steps, warmup=args.warmup, seed=args.seed, threads=0)
    value = o["value"]
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "impl": "reference", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1000.0 / value, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": describe(cfg), "kv_dtype": cfg.kv_dtype, "batch": cfg.B, "context": cfg.T0,
                   "budget": cfg.M},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": o["cores"], "kind": "oracle",
                         "sample": o["sample"] + ", every core (OpenMP over heads)", "host": host_cpu()},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["rkv", "reference"], default="rkv")
    ap.add_argument("--config", default=HEADLINE, choices=sorted(workloads.CONFIGS))
    ap.add_argument("--per-config", default=PER_CONFIG,
                    help="comma-separated workloads measured after the headline ('' for none)")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--layers", type=int, default=0, help="cut the workloads to this many layers (profiling)")
    ap.add_argument("--path", choices=["fused", "separate"], default="fused",
                    help="fused: one rkv_decode_step launch per step; separate: the four entry points")
    ap.add_argument("--no-graph", action="store_true")
    ap.add_argument("--skip-e2e", action="store_true")
    ap.add_argument("--skip-cpu-baseline", action="store_true")
    ap.add_argument("--skip-variants", action="store_true",
                    help="skip the eviction-error, latent-memory and budget-variant timings")
    ap.add_argument("--traffic", type=float, default=None,
                    help="ncu dram bytes per launch of the timed kernel for this workload (null if not measured)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    for n in args.per_config.split(","):
        if n and n not in workloads.CONFIGS:
            ap.error(f"unknown workload {n!r} in --per-config")
    world, rank, local = dist_env()
    if args.impl == "reference":
        run_reference(args, world, rank)
    else:
        run_rkv(args, world, rank, local)


if __name__ == "__main__":
    main()
