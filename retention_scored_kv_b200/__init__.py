"""Thin Python binding of librkv (include/rkv.h) for B200 (sm_100a).

Argument marshalling only: every step of the hot path runs in the CUDA
kernels of librkv.so.  PyTorch supplies device memory and streams.  There is
no CPU fallback: if the library is missing or fails to load, every call
raises.

Entry points (same names as the C ABI, without the ``rkv_`` prefix):
``score_select``, ``score_select_budget`` (as ``score_select_per_head`` and
``score_select_contour``), ``paged_decode_attn``, ``dropped_mass``, ``eviction_error``,
``memory_update``, ``memory_read``, ``compact_pages``,
``append``, ``decode_step``, ``workspace_size``, ``workspace_init``,
``device_status``, ``version``, ``last_error``.  ``Cache``/``Selection``/
``Workspace`` hold the tensors and build the C structs; ``step`` runs one
decode step, either as the separate calls select -> attention (+ dropped
mass) -> compaction -> append or as the single fused ``decode_step`` launch.
"""
from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "librkv.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_WORKSPACE_TOO_SMALL, ERR_CUDA, ERR_NOT_IMPLEMENTED = 0, -1, -2, -3, -4, -5
DEV_BAD_INPUT, DEV_POOL_EXHAUSTED, DEV_TABLE_OVERFLOW, DEV_TIMEOUT = 1, 2, 4, 8
BF16, F32 = 0, 1
PAGE = 16

EXPORTS = ("rkv_version", "rkv_last_error", "rkv_workspace_size", "rkv_workspace_init", "rkv_device_status",
           "rkv_workspace_set_wait_limit",
           "rkv_score_select", "rkv_score_select_budget", "rkv_paged_decode_attn", "rkv_dropped_mass",
           "rkv_eviction_error", "rkv_memory_update", "rkv_memory_read", "rkv_compact_pages", "rkv_append",
           "rkv_decode_step")
BUDGET_PER_HEAD, BUDGET_CONTOUR = 0, 1


class RkvError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"librkv error {code}: {msg}")
        self.code = code


class CacheStruct(ctypes.Structure):
    _fields_ = [("k_pool", ctypes.c_void_p), ("v_pool", ctypes.c_void_p), ("pos_pool", ctypes.c_void_p),
                ("lb_pool", ctypes.c_void_p), ("block_table", ctypes.c_void_p), ("len", ctypes.c_void_p),
                ("free_stack", ctypes.c_void_p), ("free_top", ctypes.c_void_p)] + [
        (n, ctypes.c_int32) for n in ("B", "L", "H", "Hq", "D", "P", "n_pages", "max_pages", "dtype")]


class SelectStruct(ctypes.Structure):
    _fields_ = [("kappa", ctypes.c_void_p), ("kept", ctypes.c_void_p), ("n_pre", ctypes.c_void_p),
                ("keep_mask", ctypes.c_void_p), ("plan", ctypes.c_void_p)]


class BudgetStruct(ctypes.Structure):
    _fields_ = [("mode", ctypes.c_int32), ("m_head", ctypes.c_void_p), ("m_global", ctypes.c_void_p),
                ("dm_prev", ctypes.c_void_p), ("flat_threshold", ctypes.c_float), ("flat_budget", ctypes.c_int32),
                ("recency_floor", ctypes.c_int32)]


class MemoryStruct(ctypes.Structure):
    _fields_ = [("proj", ctypes.c_void_p), ("gate_w", ctypes.c_void_p), ("gate_b", ctypes.c_void_p),
                ("decay", ctypes.c_float), ("M", ctypes.c_void_p), ("b", ctypes.c_void_p)]


_lib = None


def load(path: str | None = None):
    """Load librkv.so (built in-tree by __graft_entry__.build()); raises if absent."""
    global _lib
    if _lib is not None:
        return _lib
    path = path or LIB_PATH
    if not os.path.exists(path):
        raise RuntimeError(f"librkv.so not found at {path}: build it with "
                           "`python -m retention_scored_kv_b200.build`")
    lib = ctypes.CDLL(path)
    P, I, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    CP, SP = ctypes.POINTER(CacheStruct), ctypes.POINTER(SelectStruct)
    sig = {
        "rkv_version": (ctypes.c_char_p, []),
        "rkv_last_error": (ctypes.c_char_p, []),
        "rkv_workspace_size": (SZ, [CP]),
        "rkv_workspace_init": (I, [P, SZ, P]),
        "rkv_device_status": (P, [P]),
        "rkv_workspace_set_wait_limit": (I, [P, SZ, ctypes.c_uint32, P]),
        "rkv_score_select": (I, [CP, P, P, SP, P, SZ, P]),
        "rkv_score_select_budget": (I, [CP, P, ctypes.POINTER(BudgetStruct), SP, P, SZ, P]),
        "rkv_paged_decode_attn": (I, [CP, P, ctypes.c_float, SP, P, P, P, P, SZ, P]),
        "rkv_dropped_mass": (I, [CP, P, ctypes.c_float, SP, P, P, SZ, P]),
        "rkv_eviction_error": (I, [CP, P, ctypes.c_float, SP, P, P, P, P, SZ, P]),
        "rkv_memory_update": (I, [CP, SP, ctypes.POINTER(MemoryStruct), P]),
        "rkv_memory_read": (I, [CP, P, ctypes.POINTER(MemoryStruct), P, P]),
        "rkv_compact_pages": (I, [CP, SP, P, SZ, P]),
        "rkv_append": (I, [CP, P, P, P, P, P, SZ, P]),
        "rkv_decode_step": (I, [CP, P, P, P, ctypes.c_float, P, P, P, SP, P, P, P, P, SZ, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _check(rc: int):
    if rc != OK:
        raise RkvError(rc, load().rkv_last_error().decode())


def _ptr(t: torch.Tensor | None):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("librkv needs contiguous tensors")
    return t.data_ptr()


def _stream(stream: torch.cuda.Stream | None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


@dataclass
class Cache:
    """The paged cache (device tensors, caller-owned); layout as in rkv.h."""
    k_pool: torch.Tensor      # [n_pages, 16, D] bf16 / f32
    v_pool: torch.Tensor
    pos_pool: torch.Tensor    # [n_pages, 16] int32
    lb_pool: torch.Tensor     # [n_pages, 16] float32
    block_table: torch.Tensor # [C, max_pages] int32
    len: torch.Tensor         # [C] int32
    free_stack: torch.Tensor  # [n_pages] int32
    free_top: torch.Tensor    # [1] int32
    B: int
    L: int
    H: int
    Hq: int

    @property
    def D(self) -> int:
        return self.k_pool.shape[-1]

    @property
    def G(self) -> int:
        return self.Hq // self.H

    @property
    def C(self) -> int:
        return self.B * self.L * self.H

    @property
    def n_pages(self) -> int:
        return self.k_pool.shape[0]

    @property
    def max_pages(self) -> int:
        return self.block_table.shape[1]

    @property
    def dtype_code(self) -> int:
        return BF16 if self.k_pool.dtype == torch.bfloat16 else F32

    @classmethod
    def from_tensors(cls, t, B: int, L: int, H: int, Hq: int) -> "Cache":
        return cls(t.k_pool, t.v_pool, t.pos_pool, t.lb_pool, t.block_table, t.len, t.free_stack, t.free_top,
                   B, L, H, Hq)

    def struct(self) -> CacheStruct:
        return CacheStruct(_ptr(self.k_pool), _ptr(self.v_pool), _ptr(self.pos_pool), _ptr(self.lb_pool),
                           _ptr(self.block_table), _ptr(self.len), _ptr(self.free_stack), _ptr(self.free_top),
                           self.B, self.L, self.H, self.Hq, self.D, PAGE, self.n_pages, self.max_pages,
                           self.dtype_code)


@dataclass
class Selection:
    """Device outputs of score_select, consumed by the rest of the step."""
    kappa: torch.Tensor      # [B] uint64 (stored as int64)
    kept: torch.Tensor       # [C] int32
    n_pre: torch.Tensor      # [C] int32
    keep_mask: torch.Tensor  # [C, max_pages] uint16 (stored as int16)
    plan: torch.Tensor       # [C + 2] int32

    @classmethod
    def empty(cls, cache: Cache) -> "Selection":
        dev = cache.len.device
        return cls(torch.zeros(cache.B, dtype=torch.int64, device=dev),
                   torch.zeros(cache.C, dtype=torch.int32, device=dev),
                   torch.zeros(cache.C, dtype=torch.int32, device=dev),
                   torch.zeros(cache.C, cache.max_pages, dtype=torch.int16, device=dev),
                   torch.zeros(cache.C + 2, dtype=torch.int32, device=dev))

    def struct(self) -> SelectStruct:
        return SelectStruct(_ptr(self.kappa), _ptr(self.kept), _ptr(self.n_pre), _ptr(self.keep_mask),
                            _ptr(self.plan))


class Workspace:
    """Caller-owned scratch of librkv, sized by rkv_workspace_size."""

    def __init__(self, cache: Cache, stream: torch.cuda.Stream | None = None):
        self.nbytes = workspace_size(cache)
        self.buf = torch.empty(self.nbytes, dtype=torch.uint8, device=cache.len.device)
        workspace_init(self, stream)

    @property
    def ptr(self) -> int:
        return self.buf.data_ptr()

    def status(self) -> int:
        """RKV_DEV_* bits recorded on the device (reads one int32)."""
        return int(self.buf[:4].view(torch.int32).item())

    def counters(self) -> dict:
        """The device status block: bits, first timeout site, and the fused
        steps resolved in the threshold window / by the exact selection."""
        v = self.buf[:16].view(torch.int32).tolist()
        return {"status": v[0], "timeout_site": v[1], "window_steps": v[2], "exact_steps": v[3]}


def version() -> str:
    return load().rkv_version().decode()


def last_error() -> str:
    return load().rkv_last_error().decode()


def workspace_size(cache: Cache) -> int:
    st = cache.struct()
    n = load().rkv_workspace_size(ctypes.byref(st))
    if n == 0:
        raise RkvError(ERR_INVALID_ARG, last_error())
    return n


def workspace_init(ws: Workspace, stream=None):
    _check(load().rkv_workspace_init(ctypes.c_void_p(ws.ptr), ws.nbytes, _stream(stream)))


def workspace_set_wait_limit(ws: Workspace, microseconds: int, stream=None):
    """Limit of the waits on other CTAs for calls on this workspace (0: 2 s)."""
    _check(load().rkv_workspace_set_wait_limit(ctypes.c_void_p(ws.ptr), ws.nbytes, int(microseconds),
                                               _stream(stream)))


def device_status(ws: Workspace) -> int:
    return load().rkv_device_status(ctypes.c_void_p(ws.ptr))


def score_select(cache: Cache, t: torch.Tensor, m_global: torch.Tensor, sel: Selection, ws: Workspace,
                 stream=None):
    cs, ss = cache.struct(), sel.struct()
    _check(load().rkv_score_select(ctypes.byref(cs), _ptr(t), _ptr(m_global), ctypes.byref(ss),
                                   ctypes.c_void_p(ws.ptr), ws.nbytes, _stream(stream)))


def score_select_per_head(cache: Cache, t: torch.Tensor, m_head: torch.Tensor, sel: Selection, ws: Workspace,
                          stream=None):
    """Each head keeps its top m_head[c] entries (int32 [C])."""
    cs, ss = cache.struct(), sel.struct()
    bs = BudgetStruct(BUDGET_PER_HEAD, _ptr(m_head), None, None, 0.0, 0, 0)
    _check(load().rkv_score_select_budget(ctypes.byref(cs), _ptr(t), ctypes.byref(bs), ctypes.byref(ss),
                                          ctypes.c_void_p(ws.ptr), ws.nbytes, _stream(stream)))


def score_select_contour(cache: Cache, t: torch.Tensor, m_global: torch.Tensor, dm_prev: torch.Tensor,
                         flat_threshold: float, flat_budget: int, recency_floor: int, sel: Selection,
                         ws: Workspace, stream=None):
    """ContourKV allocation: dm_prev float32 [B, L, Hq] (the previous
    evicting step's dropped mass), recency floor, flat heads' budget, the
    rest of m_global ranked globally (see rkv.h)."""
    cs, ss = cache.struct(), sel.struct()
    bs = BudgetStruct(BUDGET_CONTOUR, None, _ptr(m_global), _ptr(dm_prev), float(flat_threshold), int(flat_budget),
                      int(recency_floor))
    _check(load().rkv_score_select_budget(ctypes.byref(cs), _ptr(t), ctypes.byref(bs), ctypes.byref(ss),
                                          ctypes.c_void_p(ws.ptr), ws.nbytes, _stream(stream)))


def paged_decode_attn(cache: Cache, q: torch.Tensor, scale: float, sel: Selection | None, out: torch.Tensor,
                      lse: torch.Tensor | None, dropped: torch.Tensor | None, ws: Workspace, stream=None):
    cs = cache.struct()
    ss = ctypes.byref(sel.struct()) if sel is not None else None
    _check(load().rkv_paged_decode_attn(ctypes.byref(cs), _ptr(q), ctypes.c_float(scale), ss, _ptr(out),
                                        _ptr(lse), _ptr(dropped), ctypes.c_void_p(ws.ptr), ws.nbytes,
                                        _stream(stream)))


def dropped_mass(cache: Cache, q: torch.Tensor, scale: float, sel: Selection, dropped: torch.Tensor,
                 ws: Workspace, stream=None):
    cs, ss = cache.struct(), sel.struct()
    _check(load().rkv_dropped_mass(ctypes.byref(cs), _ptr(q), ctypes.c_float(scale), ctypes.byref(ss),
                                   _ptr(dropped), ctypes.c_void_p(ws.ptr), ws.nbytes, _stream(stream)))


def eviction_error(cache: Cache, q: torch.Tensor, scale: float, sel: Selection, out_kept: torch.Tensor,
                   dropped: torch.Tensor, err: torch.Tensor, ws: Workspace, stream=None):
    cs, ss = cache.struct(), sel.struct()
    _check(load().rkv_eviction_error(ctypes.byref(cs), _ptr(q), ctypes.c_float(scale), ctypes.byref(ss),
                                     _ptr(out_kept), _ptr(dropped), _ptr(err), ctypes.c_void_p(ws.ptr), ws.nbytes,
                                     _stream(stream)))


@dataclass
class Memory:
    """Latent memory of the evicted tokens (rkv.h, rkv_memory_update/read):
    slow weights (proj [L, D, D], gate_w [L, Hq, D], gate_b [L, Hq]) and the
    state (M [C, D, D], b [C, D], zero for a fresh sequence), all float32."""
    proj: torch.Tensor
    gate_w: torch.Tensor
    gate_b: torch.Tensor
    M: torch.Tensor
    b: torch.Tensor
    decay: float = 0.99

    @classmethod
    def zeros(cls, cache: Cache, proj, gate_w, gate_b, decay: float = 0.99) -> "Memory":
        dev = cache.len.device
        return cls(proj, gate_w, gate_b, torch.zeros(cache.C, cache.D, cache.D, device=dev),
                   torch.zeros(cache.C, cache.D, device=dev), decay)

    def struct(self) -> MemoryStruct:
        return MemoryStruct(_ptr(self.proj), _ptr(self.gate_w), _ptr(self.gate_b), float(self.decay), _ptr(self.M),
                            _ptr(self.b))


def memory_update(cache: Cache, sel: Selection, mem: Memory, stream=None):
    cs, ss, ms = cache.struct(), sel.struct(), mem.struct()
    _check(load().rkv_memory_update(ctypes.byref(cs), ctypes.byref(ss), ctypes.byref(ms), _stream(stream)))


def memory_read(cache: Cache, q: torch.Tensor, mem: Memory, out: torch.Tensor, stream=None):
    cs, ms = cache.struct(), mem.struct()
    _check(load().rkv_memory_read(ctypes.byref(cs), _ptr(q), ctypes.byref(ms), _ptr(out), _stream(stream)))


def compact_pages(cache: Cache, sel: Selection, ws: Workspace, stream=None):
    cs, ss = cache.struct(), sel.struct()
    _check(load().rkv_compact_pages(ctypes.byref(cs), ctypes.byref(ss), ctypes.c_void_p(ws.ptr), ws.nbytes,
                                    _stream(stream)))


def append(cache: Cache, t: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor, lb_new: torch.Tensor,
           ws: Workspace, stream=None):
    cs = cache.struct()
    _check(load().rkv_append(ctypes.byref(cs), _ptr(t), _ptr(k_new), _ptr(v_new), _ptr(lb_new),
                             ctypes.c_void_p(ws.ptr), ws.nbytes, _stream(stream)))


def decode_step(cache: Cache, t: torch.Tensor, m_global: torch.Tensor | None, q: torch.Tensor, scale: float,
                k_new: torch.Tensor, v_new: torch.Tensor, lb_new: torch.Tensor, sel: Selection | None,
                out: torch.Tensor, lse: torch.Tensor | None, dropped: torch.Tensor | None, ws: Workspace,
                stream=None):
    cs = cache.struct()
    ss = ctypes.byref(sel.struct()) if sel is not None else None
    _check(load().rkv_decode_step(ctypes.byref(cs), _ptr(t), _ptr(m_global), _ptr(q), ctypes.c_float(scale),
                                  _ptr(k_new), _ptr(v_new), _ptr(lb_new), ss, _ptr(out), _ptr(lse), _ptr(dropped),
                                  ctypes.c_void_p(ws.ptr), ws.nbytes, _stream(stream)))


@dataclass
class StepOutputs:
    out: torch.Tensor      # [B, L, Hq, D] float32
    lse: torch.Tensor      # [B, L, Hq] float32
    dropped: torch.Tensor  # [B, L, Hq] float32

    @classmethod
    def empty(cls, cache: Cache) -> "StepOutputs":
        dev = cache.len.device
        return cls(torch.empty(cache.B, cache.L, cache.Hq, cache.D, dtype=torch.float32, device=dev),
                   torch.empty(cache.B, cache.L, cache.Hq, dtype=torch.float32, device=dev),
                   torch.empty(cache.B, cache.L, cache.Hq, dtype=torch.float32, device=dev))


def step(cache: Cache, sel: Selection, ws: Workspace, outs: StepOutputs, *, q, t, m_global, k_new, v_new,
         lb_new, evict: bool = True, scale: float | None = None, fused: bool = False, stream=None,
         err: torch.Tensor | None = None, mem: Memory | None = None):
    """One decode step: [select] -> attention + dropped mass -> [eviction
    error] -> [compaction] -> append.

    On a non-evicting step every entry is kept and the dropped mass is 0.
    ``fused`` runs the whole step as one ``decode_step`` launch; ``err``
    ([B, L, Hq] float32) asks for the eviction error of an evicting step,
    which the separate calls provide (not the fused launch); ``mem`` folds
    the evicted tokens into the latent memory and adds its gated read to
    the output (separate calls as well)."""
    if scale is None:
        scale = 1.0 / math.sqrt(cache.D)
    if (err is not None or mem is not None) and fused:
        raise ValueError("the eviction error and the latent memory come from the separate calls (fused=False)")
    if fused:
        decode_step(cache, t, m_global if evict else None, q, scale, k_new, v_new, lb_new, sel if evict else None,
                    outs.out, outs.lse, outs.dropped, ws, stream)
        return
    if evict:
        score_select(cache, t, m_global, sel, ws, stream)
        if mem is not None:
            memory_update(cache, sel, mem, stream)
        paged_decode_attn(cache, q, scale, sel, outs.out, outs.lse, outs.dropped, ws, stream)
        if err is not None:
            eviction_error(cache, q, scale, sel, outs.out, outs.dropped, err, ws, stream)
        if mem is not None:
            memory_read(cache, q, mem, outs.out, stream)
        compact_pages(cache, sel, ws, stream)
    else:
        paged_decode_attn(cache, q, scale, None, outs.out, outs.lse, outs.dropped, ws, stream)
        if mem is not None:
            memory_read(cache, q, mem, outs.out, stream)
    append(cache, t, k_new, v_new, lb_new, ws, stream)


def _align(n: int, a: int = 256) -> int:
    return (n + a - 1) // a * a


class StepRunner:
    """One decode step on static device buffers, optionally captured in CUDA graphs.

    Inputs live in one device buffer (q, k_new, v_new, lb_new, t, m_global) and
    outputs in another (out, lse, dropped), so a step driven from host memory
    costs one host-to-device copy, one graph replay (or the eager calls) and one
    device-to-host copy.  ``in_layout`` / ``out_layout`` give each field's byte
    offset, shape and dtype so callers can pack pinned host buffers."""

    def __init__(self, cache: Cache, *, scale: float | None = None, use_graph: bool = True, fused: bool = True,
                 stream=None, buffers: int = 1):
        if buffers not in (1, 2):
            raise ValueError("buffers must be 1 or 2")
        self.cache = cache
        self.fused = fused
        self.scale = 1.0 / math.sqrt(cache.D) if scale is None else scale
        self.stream = stream if stream is not None else torch.cuda.current_stream()
        dev = cache.len.device
        kvdt = cache.k_pool.dtype
        C, G, D, B = cache.C, cache.G, cache.D, cache.B
        self.in_layout, off = {}, 0
        for name, shape, dt in (("q", (B, cache.L, cache.Hq, D), torch.float32), ("k_new", (C, D), kvdt),
                                ("v_new", (C, D), kvdt), ("lb_new", (C,), torch.float32),
                                ("t", (B,), torch.int32), ("m_global", (B,), torch.int64)):
            n = math.prod(shape) * torch.empty((), dtype=dt).element_size()
            self.in_layout[name] = (off, shape, dt)
            off = _align(off + n)
        self.in_bytes = off
        self.out_layout, off = {}, 0
        for name, shape in (("out", (B, cache.L, cache.Hq, D)), ("lse", (B, cache.L, cache.Hq)),
                            ("dropped", (B, cache.L, cache.Hq))):
            self.out_layout[name] = (off, shape, torch.float32)
            off = _align(off + math.prod(shape) * 4)
        self.out_bytes = off
        # one set of device buffers per slot; with two, run_host overlaps a
        # step's copies with its neighbours' compute (copies on their own stream)
        self.inbufs = [torch.zeros(self.in_bytes, dtype=torch.uint8, device=dev) for _ in range(buffers)]
        self.outbufs = [torch.zeros(self.out_bytes, dtype=torch.uint8, device=dev) for _ in range(buffers)]
        self.inps = [{k: self._view(b, *v) for k, v in self.in_layout.items()} for b in self.inbufs]
        self.outss = []
        for b in self.outbufs:
            o = {k: self._view(b, *v) for k, v in self.out_layout.items()}
            self.outss.append(StepOutputs(o["out"], o["lse"], o["dropped"]))
        self.inbuf, self.outbuf, self.inp, self.outs = self.inbufs[0], self.outbufs[0], self.inps[0], self.outss[0]
        self.sel = Selection.empty(cache)
        self.ws = Workspace(cache, self.stream)
        self.use_graph = use_graph
        self.capture_error: str | None = None
        self.graphs: dict[tuple[int, bool], torch.cuda.CUDAGraph] = {}
        self.buffers = buffers
        self.copy_stream = torch.cuda.Stream(device=dev) if buffers > 1 else None
        self._ev = [{k: torch.cuda.Event() for k in ("in", "done", "out")} for _ in range(buffers)]
        self._n = 0                # steps submitted through run_host
        self._pending = None       # (host_out, slot) whose copy-out is not enqueued yet
        self._restart = True       # the next copy follows the runner's stream

    @staticmethod
    def _view(buf: torch.Tensor, off: int, shape, dt) -> torch.Tensor:
        n = math.prod(shape) * torch.empty((), dtype=dt).element_size()
        return buf[off: off + n].view(dt).view(shape)

    def pack(self, host: torch.Tensor, **fields) -> None:
        """Write input fields into a host (pinned) uint8 buffer of in_bytes."""
        for k, v in fields.items():
            self._view(host, *self.in_layout[k]).copy_(v)

    def unpack(self, host: torch.Tensor) -> dict:
        return {k: self._view(host, *v) for k, v in self.out_layout.items()}

    def _enqueue(self, evict: bool, slot: int = 0) -> None:
        i = self.inps[slot]
        step(self.cache, self.sel, self.ws, self.outss[slot], q=i["q"], t=i["t"], m_global=i["m_global"],
             k_new=i["k_new"], v_new=i["v_new"], lb_new=i["lb_new"], evict=evict, scale=self.scale,
             fused=self.fused, stream=self.stream)

    def capture(self) -> bool:
        """Capture the evicting and non-evicting step; False if capture is refused."""
        if not self.use_graph:
            return False
        if self.stream == torch.cuda.default_stream(self.stream.device):
            self.capture_error = "CUDA graphs need a non-default stream: pass stream=torch.cuda.Stream()"
            self.use_graph = False
            return False
        try:
            for slot in range(self.buffers):
                for evict in (True, False):
                    g = torch.cuda.CUDAGraph()
                    with torch.cuda.graph(g, stream=self.stream, capture_error_mode="thread_local"):
                        self._enqueue(evict, slot)
                    self.graphs[(slot, evict)] = g
            return True
        except Exception as ex:
            self.capture_error = f"{type(ex).__name__}: {ex}"
            self.graphs.clear()
            self.use_graph = False
            return False

    def run(self, evict: bool = True, slot: int = 0) -> None:
        """Run one step on the inputs already in a slot's static device buffer."""
        g = self.graphs.get((slot, evict))
        if g is not None:
            with torch.cuda.stream(self.stream):
                g.replay()
        else:
            self._enqueue(evict, slot)

    def run_host(self, host_in: torch.Tensor, host_out: torch.Tensor, evict: bool = True) -> None:
        """Copy packed host inputs in, run the step, copy packed outputs out (async).

        With two buffer slots the copies go on a copy stream: step n's inputs
        are copied while step n - 1 runs, and step n - 1's outputs are copied
        out after step n's inputs (so they overlap step n).  ``finish()``
        enqueues the last copy-out and orders it before later work on the
        runner's stream."""
        if self.buffers == 1:
            with torch.cuda.stream(self.stream):
                self.inbuf.copy_(host_in, non_blocking=True)
            self.run(evict)
            with torch.cuda.stream(self.stream):
                host_out.copy_(self.outbuf, non_blocking=True)
            return
        p = self._n % 2
        cs, ev = self.copy_stream, self._ev[p]
        if self._restart:
            cs.wait_stream(self.stream)
            self._restart = False
        with torch.cuda.stream(cs):
            if self._n >= 2:
                cs.wait_event(ev["done"])      # the slot's previous step has read its inputs
            self.inbufs[p].copy_(host_in, non_blocking=True)
            ev["in"].record(cs)
        self._flush_out()
        self.stream.wait_event(ev["in"])
        if self._n >= 2:
            self.stream.wait_event(ev["out"])  # the slot's previous outputs are copied out
        self.run(evict, p)
        ev["done"].record(self.stream)
        self._pending = (host_out, p)
        self._n += 1

    def _flush_out(self) -> None:
        if self._pending is None:
            return
        host_out, p = self._pending
        cs, ev = self.copy_stream, self._ev[p]
        with torch.cuda.stream(cs):
            cs.wait_event(ev["done"])
            host_out.copy_(self.outbufs[p], non_blocking=True)
            ev["out"].record(cs)
        self._pending = None

    def finish(self) -> None:
        """Enqueue the last step's copy-out; later work on the runner's stream follows it."""
        if self.buffers == 1:
            return
        self._flush_out()
        self.stream.wait_stream(self.copy_stream)
        self._restart = True
