#!/usr/bin/env python
"""Benchmark: one decode step of retention-scored global KV eviction + paged
decode attention over the kept entries (select -> attention + dropped mass
-> compaction -> append), on synthetic Llama-3.1-8B-shaped data.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl rkv|reference] [--config NAME]
                    [--path fused|separate]

--path fused (default) runs each step as one rkv_decode_step launch; separate
runs the four entry points (select, attention, compaction, append).

Default workload "llama32k": 32 layers x 8 KV heads (32 query heads, GQA 4),
head dim 128, bf16 K/V, batch 1, 32K-token prefill, global budget
M = 32*8*2048 = 524,288 entries, evicting every step.  Step 0 (the prefill
eviction 8.4M -> 524K entries) is run and reported separately (step0_ms); the
W warm-up and K timed steps are steady-state evicting steps (N_pre = M + 256
entries each).  The per-step working set (268 MB of retained K/V) is larger
than the 126 MB L2, so no L2 flush is inserted between steps.

Timing: the K timed steps are one CUDA graph replay bracketed by a barrier
and synchronize on both sides, timed with CUDA events on the launching
stream; multi-GPU runs are independent replicas (one sequence per rank,
"scaling": "weak") and report the maximum over ranks.  On the fused path the
graph holds only the K step launches (event records between launches cost
~8 us per step on a B200), and the step kernel's average duration is taken as
the timed region / K, launch gaps included; on the separate path per-kernel
CUDA events inside the graph split each step into its four kernels.  The
dominant kernel's algorithmic bytes over its duration is the roofline entry
(the fused step kernel: the whole step's bytes; separate path: the attention
kernel's).  e2e repeats the
measurement through the public API with packed pinned host inputs and
outputs (one H2D + graph replay + one D2H per step).  cpu_baseline times the
CPU oracle on a bounded sample of the same step (2 of 32 layers) on the host
cores, scaled to the full step.  ``--impl reference`` times that oracle alone.
"""
from __future__ import annotations

import argparse
import json
import math
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

# DRAM traffic (ncu dram__bytes_read.sum + dram__bytes_write.sum) of one
# attention launch of the llama32k steady step, from the 16-layer capture in
# profiles/attn_kernel_llama32k_16L.md scaled x2 to the full launch.  Reported
# only while the attention kernel's sources are the ones that were captured.
ATTN_TRAFFIC = {"sources_sha256": "6e67ee544df2f78e", "workload": "llama32k", "bytes_per_launch": 2 * 139.574528e6}
# The same for the fused step kernel: the 16-layer capture in
# profiles/step_kernel_llama32k_16L.md (read 137.71 MB + write 4.15 MB) x2.
STEP_TRAFFIC = {"sources_sha256": "f4c114055eede79d", "workload": "llama32k", "bytes_per_launch": 2 * 141.859584e6}
UNIT = "steps/s"
SAMPLE_LAYERS = 2  # CPU oracle sample: 2 of the workload's layers, time scaled by L / 2


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


# ------------------------------------------------------------- CPU oracle ---
def sample_config(cfg: workloads.Config) -> workloads.Config:
    Ls = min(SAMPLE_LAYERS, cfg.L)
    return workloads.Config(cfg.name + f"-{Ls}L", L=Ls, H=cfg.H, Hq=cfg.Hq, D=cfg.D, B=1, T0=cfg.T0,
                            M=cfg.M // cfg.B * Ls // cfg.L, steps=cfg.steps, kv_dtype=cfg.kv_dtype, mix=cfg.mix,
                            mix_decode=cfg.mix_decode)


def oracle_steady_state(cfg_s: workloads.Config, n_steps: int, seed: int):
    """Host cache in the steady-state shape: every head holds M/(L*H) + 1 entries."""
    import oracle
    per_head = cfg_s.M // (cfg_s.L * cfg_s.H) + 1
    pages = -(-per_head // 16)
    dc = workloads.ragged_cache(cfg_s, seed, [per_head] * cfg_s.C, n_pages=cfg_s.C * (pages + 2 + n_steps // 16 + 2),
                                max_pages=pages + n_steps // 16 + 4)
    return oracle.HostCache(**workloads.to_host(dc))


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


def time_oracle(cfg: workloads.Config, steps: int, warmup: int, seed: int) -> dict:
    """Seconds per oracle step on the sample, and the full-step throughput it implies."""
    import oracle
    cfg_s = sample_config(cfg)
    hc = oracle_steady_state(cfg_s, steps + warmup + 2, seed)
    inputs = [workloads.step_inputs(cfg_s, seed, s) for s in range(steps + warmup)]
    per = []
    for s, inp in enumerate(inputs):
        t0 = time.perf_counter()
        oracle.step(hc, inp["t"].numpy(), inp["m_global"].numpy(), inp["q"].numpy().reshape(cfg_s.C, cfg_s.G, cfg_s.D),
                    workloads.rows_to_host(inp["k_new"]), workloads.rows_to_host(inp["v_new"]),
                    inp["lb_new"].numpy(), evict=True, scale=cfg_s.scale)
        if s >= warmup:
            per.append(time.perf_counter() - t0)
    sec_sample = sum(per) / max(len(per), 1)
    scale = cfg.L * cfg.B / cfg_s.L
    return {"sec_per_sample_step": sec_sample, "value": 1.0 / (sec_sample * scale), "timed": len(per),
            "sample": (f"{len(per)} steady-state evicting steps of {cfg_s.L} of {cfg.L} layers "
                       f"(N_pre {cfg_s.M + cfg_s.C}, M {cfg_s.M}, same heads/dims/retention mix), "
                       f"time x{scale:g} to the full step"),
            "cores": 1}


# ------------------------------------------------------------------ bytes ---
def attn_bytes(cfg: workloads.Config, n_pre: int, kept: int, pages: int) -> int:
    """Algorithmic HBM bytes of one attention launch: K of every pre-eviction
    entry (dense logits for the dropped mass), V of the kept entries, q, out,
    lse + dropped, block-table entries and keep-mask words."""
    elt = 2 if cfg.kv_dtype == "bf16" else 4
    return (elt * cfg.D * n_pre + elt * cfg.D * kept + 2 * 4 * cfg.C * cfg.G * cfg.D + 2 * 4 * cfg.C * cfg.G
            + 4 * pages + 2 * pages)


def step_bytes(cfg: workloads.Config, n_pre: int, kept: int, pages: int) -> int:
    """Algorithmic bytes of the whole step: attention + position/log-retention
    of every entry (selection) + the appended rows (K, V, position, lb)."""
    elt = 2 if cfg.kv_dtype == "bf16" else 4
    return attn_bytes(cfg, n_pre, kept, pages) + 8 * n_pre + cfg.C * (2 * elt * cfg.D + 8)


# -------------------------------------------------------------- rkv arm ---
def run_rkv(args, world, rank, local):
    import retention_scored_kv_b200 as rkv
    torch.cuda.set_device(local)
    dist_init(world, "nccl")
    rkv.load()
    cfg = workload_config(args)
    dev = torch.device("cuda", local)
    seed = args.seed + 1000 * rank
    K, W = args.steps, args.warmup
    total = 1 + W + K + W + K + 2
    dc = workloads.prefill_cache(cfg, seed, device=dev, n_steps=total)
    cache = rkv.Cache.from_tensors(dc, cfg.B, cfg.L, cfg.H, cfg.Hq)
    stream = torch.cuda.Stream(device=dev)
    fused = args.path == "fused"
    runner = rkv.StepRunner(cache, scale=cfg.scale, stream=stream, fused=fused)
    sel, ws, outs = runner.sel, runner.ws, runner.outs

    # inputs of every step, resident on the device
    per_step = [workloads.step_inputs(cfg, seed, s, dev) for s in range(total)]
    kernel_names = ["step"] if fused else ["select", "attn", "compact", "append"]

    def enqueue(s, ev=None):
        inp = per_step[s]
        if not inp["evict"]:
            raise RuntimeError("bench workloads evict every step")
        if fused:
            rkv.decode_step(cache, inp["t"], inp["m_global"], inp["q"], cfg.scale, inp["k_new"], inp["v_new"],
                            inp["lb_new"], sel, outs.out, outs.lse, outs.dropped, ws, stream)
            if ev is not None:
                ev[0].record(stream)
            return
        rkv.score_select(cache, inp["t"], inp["m_global"], sel, ws, stream)
        if ev is not None:
            ev[0].record(stream)
        rkv.paged_decode_attn(cache, inp["q"], cfg.scale, sel, outs.out, outs.lse, outs.dropped, ws, stream)
        if ev is not None:
            ev[1].record(stream)
        rkv.compact_pages(cache, sel, ws, stream)
        if ev is not None:
            ev[2].record(stream)
        rkv.append(cache, inp["t"], inp["k_new"], inp["v_new"], inp["lb_new"], ws, stream)
        if ev is not None:
            ev[3].record(stream)

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
    # step 0: prefill eviction (timed alone)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        enqueue(0)
        e1.record(stream)
    torch.cuda.synchronize()
    step0_ms = e0.elapsed_time(e1)
    s_next = 1

    # warm-up: W steps
    with torch.cuda.stream(stream):
        for _ in range(W):
            enqueue(s_next)
            s_next += 1
    torch.cuda.synchronize()

    # timed: K steps captured in one graph (separate path: with per-kernel
    # events inside; the fused path's graph holds the launches alone)
    evs = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(5)] for _ in range(K)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    use_graph = not args.no_graph
    graph = None
    first = s_next
    if use_graph:
        try:
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph, stream=stream, capture_error_mode="thread_local"):
                for i in range(K):
                    if fused:
                        enqueue(first + i)
                    else:
                        evs[i][4].record(stream)
                        enqueue(first + i, evs[i][:4])
            _graph_upload(graph, stream)
        except Exception as ex:  # capture refused: time eager launches instead
            print(f"[bench] graph capture failed ({ex}); timing eager launches", file=sys.stderr)
            graph, use_graph = None, False
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
                for i in range(K):
                    if fused:
                        enqueue(first + i)
                    else:
                        evs[i][4].record(stream)
                        enqueue(first + i, evs[i][:4])
            t_end.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    s_next = first + K
    ms = t_start.elapsed_time(t_end)
    ms_max = max_over_ranks(ms, world, dev)
    status = ws.status()
    if status != 0:
        raise RuntimeError(f"device status {status} after the timed steps")
    sel1 = ws.counters()
    # how the timed steps selected: inside the threshold window kept from the
    # previous step, or by the exact radix fallback
    selection = {k: sel1[k] - sel0[k] for k in ("window_steps", "exact_steps")}
    if fused:
        # one launch per step and nothing else in the timed region: the step
        # kernel's average duration is at most the region / K
        kern_us = {"step": 1000.0 * ms_max / K}
    else:
        kern = {k: [] for k in kernel_names}
        for i in range(K):
            e = evs[i]
            marks = [e[4]] + e[:len(kernel_names)]
            for j, k in enumerate(kernel_names):
                kern[k].append(marks[j].elapsed_time(marks[j + 1]))
        kern_us = {k: 1000.0 * statistics.mean(v) for k, v in kern.items()}
    clocks = clk.summary()

    # steady-state sizes of the timed steps (N_pre = kept + C after each append)
    n_pre = int(sel.n_pre.sum().item())
    kept = int(sel.kept.sum().item())
    pages = int(((sel.n_pre + 15) // 16).sum().item())

    # ------------------------------------------------------------- e2e ---
    e2e = None
    if not args.skip_e2e:
        runner.capture()
        host_in = [torch.empty(runner.in_bytes, dtype=torch.uint8, pin_memory=True) for _ in range(W + K)]
        host_out = [torch.empty(runner.out_bytes, dtype=torch.uint8, pin_memory=True) for _ in range(W + K)]
        for i in range(W + K):
            inp = per_step[s_next + i]
            runner.pack(host_in[i], q=inp["q"].cpu(), k_new=inp["k_new"].cpu(), v_new=inp["v_new"].cpu(),
                        lb_new=inp["lb_new"].cpu(), t=inp["t"].cpu(), m_global=inp["m_global"].cpu())
        for i in range(W):
            runner.run_host(host_in[i], host_out[i], True)
        torch.cuda.synchronize()
        barrier(world)
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with ClockSampler(local) as clk2:
            a.record(stream)
            for i in range(W, W + K):
                runner.run_host(host_in[i], host_out[i], True)
            b.record(stream)
            torch.cuda.synchronize()
        barrier(world)
        e2e_ms = max_over_ranks(a.elapsed_time(b), world, dev)
        if runner.ws.status() != 0:
            raise RuntimeError(f"device status {runner.ws.status()} after the e2e steps")
        s2 = clk2.summary()
        if s2["samples"]:
            clocks["e2e_sm_mhz"] = s2["sm_mhz"]
            clocks["reasons"] = sorted(set(clocks["reasons"]) | set(s2["reasons"]))
        e2e = {"value": world * K / (e2e_ms / 1000.0), "unit": UNIT, "h2d_bytes_per_step": runner.in_bytes,
               "d2h_bytes_per_step": runner.out_bytes, "graph": bool(runner.graphs)}

    # ----------------------------------------------------- CPU baseline ---
    cpu = None
    if rank == 0 and world == 1 and not args.skip_cpu_baseline:
        o = time_oracle(cfg, steps=args.cpu_steps, warmup=1, seed=seed)
        cpu = {"value": o["value"], "unit": UNIT, "cores": o["cores"], "kind": "oracle", "sample": o["sample"],
               "host": host_cpu()}

    peaks = _peaks()
    s_bytes = step_bytes(cfg, n_pre, kept, pages)
    if fused:
        # one launch does the whole step: its algorithmic bytes are the step's
        a_bytes, dom_s = s_bytes, kern_us["step"] * 1e-6
        kernel_desc = "step_kernel (selection + paged decode attention + dropped mass + compaction + append)"
        traffic = attn_traffic(cfg, args.traffic, STEP_TRAFFIC, "step")
    else:
        a_bytes, dom_s = attn_bytes(cfg, n_pre, kept, pages), kern_us["attn"] * 1e-6
        kernel_desc = "attn_kernel (paged decode attention + dropped mass)"
        traffic = attn_traffic(cfg, args.traffic, ATTN_TRAFFIC, "attn")
    achieved = a_bytes / dom_s / 1e9
    step_s = ms_max / K / 1000.0
    retained = (2 if cfg.kv_dtype == "bf16" else 4) * 2 * cfg.D * kept
    line = {
        "metric": METRIC, "value": world * K / (ms_max / 1000.0), "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": W, "ms_per_step": ms_max / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32", "data": "synthetic",
        "config": {"workload": f"{cfg.name}: L{cfg.L} H{cfg.H} Hq{cfg.Hq} D{cfg.D} B{cfg.B} T0 {cfg.T0} "
                               f"M {cfg.M} bf16 K/V, steady-state evicting steps",
                   "kv_dtype": cfg.kv_dtype, "batch": cfg.B, "context": cfg.T0, "budget": cfg.M,
                   "n_pre_per_step": n_pre, "kept_per_step": kept,
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "l2": "no flush: per-step K/V working set > 126 MB L2", "graph": use_graph},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / peaks["hbm_gbs"], "traffic": traffic, "kernel": kernel_desc,
                     "bytes_per_launch": a_bytes, "peak_source": peaks["source"],
                     "duration": ("timed region / K (one launch per step, launch gaps included)" if fused
                                  else "per-kernel CUDA events inside the timed graph")},
        "step_hbm": {"bytes_per_step": s_bytes, "achieved_gbs": s_bytes / step_s / 1e9,
                     "frac": s_bytes / step_s / 1e9 / peaks["hbm_gbs"]},
        "retained_kv": {"gbs": retained / step_s / 1e9, "frac_of_peak": retained / step_s / 1e9 / peaks["hbm_gbs"]},
        "kernels_us": kern_us, "us_per_step": 1000.0 * ms_max / K, "step0_ms": step0_ms,
        "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": len(kernel_names) * K, "clocks": clocks, "path": args.path,
        "selection": selection,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    del graph
    if world > 1:
        torch.distributed.destroy_process_group()


def workload_config(args) -> workloads.Config:
    """The named workload, optionally cut to fewer layers (budget scaled alike)
    -- a smaller case of the same kernels for profiler captures."""
    import dataclasses
    cfg = workloads.CONFIGS[args.config]
    if args.layers and args.layers != cfg.L:
        cfg = dataclasses.replace(cfg, name=f"{cfg.name}-{args.layers}L", L=args.layers,
                                  M=cfg.M * args.layers // cfg.L)
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


TRAFFIC_SOURCES = {
    "attn": ("retention_scored_kv_b200/csrc/attn.cu", "retention_scored_kv_b200/csrc/attn_core.cuh",
             "retention_scored_kv_b200/csrc/common.cuh"),
    "step": ("retention_scored_kv_b200/csrc/step.cu", "retention_scored_kv_b200/csrc/attn_core.cuh",
             "retention_scored_kv_b200/csrc/common.cuh"),
}


def sources_sha(kind: str) -> str:
    import hashlib
    h = hashlib.sha256()
    for f in TRAFFIC_SOURCES[kind]:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def attn_traffic(cfg: workloads.Config, override, record: dict | None, kind: str):
    """ncu DRAM bytes per launch of the dominant kernel, or None if not
    measured for these sources and this workload."""
    if override is not None:
        return override
    if record and cfg.name == record["workload"] and sources_sha(kind) == record["sources_sha256"]:
        return record["bytes_per_launch"]
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
    if rank != 0:
        return
    cfg = workload_config(args)
    o = time_oracle(cfg, steps=args.steps, warmup=args.warmup, seed=args.seed)
    value = o["value"]
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "impl": "reference", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1000.0 / value, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"{cfg.name}: L{cfg.L} H{cfg.H} Hq{cfg.Hq} D{cfg.D} B{cfg.B} T0 {cfg.T0} "
                               f"M {cfg.M} bf16 K/V, steady-state evicting steps",
                   "kv_dtype": cfg.kv_dtype, "batch": cfg.B, "context": cfg.T0, "budget": cfg.M},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": o["cores"], "kind": "oracle", "sample": o["sample"],
                         "host": host_cpu()},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["rkv", "reference"], default="rkv")
    ap.add_argument("--config", default="llama32k", choices=sorted(workloads.CONFIGS))
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--layers", type=int, default=0, help="cut the workload to this many layers (profiling)")
    ap.add_argument("--cpu-steps", type=int, default=250)
    ap.add_argument("--path", choices=["fused", "separate"], default="fused",
                    help="fused: one rkv_decode_step launch per step; separate: the four entry points")
    ap.add_argument("--no-graph", action="store_true")
    ap.add_argument("--skip-e2e", action="store_true")
    ap.add_argument("--skip-cpu-baseline", action="store_true")
    ap.add_argument("--traffic", type=float, default=None,
                    help="ncu dram bytes per attention launch for this workload (null if not measured)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world, rank, local = dist_env()
    if args.impl == "reference":
        run_reference(args, world, rank)
    else:
        run_rkv(args, world, rank, local)


if __name__ == "__main__":
    main()
