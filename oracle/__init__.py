"""Plain CPU oracle for one decode step of retention-scored global KV eviction.

TEST INFRASTRUCTURE ONLY: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  The product path (``retention_scored_kv_b200``) never does, and the
two share no code.

The arithmetic lives in ``oracle.c`` (plain C99, binary64 attention, one
binary32 multiply per score, no FMA contraction); this module only builds it
with gcc, marshals numpy arrays through ctypes and composes one step in the
order select -> attention + dropped mass -> compaction -> append.

Functions whose result has no independent pin say so in their docstring;
every other function is pinned by ``tests/test_oracle_*.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_LIB_OMP_PATH = os.path.join(_HERE, "liboracle_omp.so")

GCC_FLAGS = ["-O2", "-std=c99", "-ffp-contract=off", "-fexcess-precision=standard",
             "-fno-fast-math", "-shared", "-fPIC"]

OK, ERR_INPUT, ERR_POOL, ERR_TABLE = 0, -1, -2, -3


def build(force: bool = False, openmp: bool = False) -> str:
    """Compile oracle.c next to it (gcc, no FMA contraction): liboracle.so,
    or with ``openmp`` liboracle_omp.so, whose attention spreads independent
    heads over threads (same per-head arithmetic, same results)."""
    path = _LIB_OMP_PATH if openmp else _LIB_PATH
    if force or not os.path.exists(path) or os.path.getmtime(path) < os.path.getmtime(_SRC):
        tmp = path + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *GCC_FLAGS, *(["-fopenmp"] if openmp else []), _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, path)
    return path


class _Cache(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("B", "L", "H", "G", "D", "P", "n_pages", "max_pages", "kv_f32")] + [
        ("k_pool", ctypes.c_void_p), ("v_pool", ctypes.c_void_p),
        ("pos_pool", ctypes.c_void_p), ("lb_pool", ctypes.c_void_p),
        ("block_table", ctypes.c_void_p), ("len", ctypes.c_void_p),
        ("free_stack", ctypes.c_void_p), ("free_top", ctypes.c_void_p),
    ]


_libs: dict = {}
_use_openmp = False


def use_threads(n: int) -> int:
    """Run the following oracle calls on the OpenMP build with n threads
    (n <= 0: every core; n == 1 or no call: the plain single-threaded build).
    Returns the number of threads in effect."""
    global _use_openmp
    _use_openmp = n != 1
    lib = _load()
    return int(lib.orc_threads(n if n > 1 else 0)) if _use_openmp else 1


def _load():
    key = "omp" if _use_openmp else "plain"
    if key not in _libs:
        # RKV_ORACLE_LIB: another build of oracle.c (the pin tests' planted-
        # mistake check runs them against altered copies)
        path = os.environ.get("RKV_ORACLE_LIB") or build(openmp=_use_openmp)
        lib = ctypes.CDLL(path)
        P = ctypes.c_void_p
        lib.orc_threads.restype = ctypes.c_int
        lib.orc_threads.argtypes = [ctypes.c_int]
        lib.orc_score.restype = ctypes.c_float
        lib.orc_score.argtypes = [ctypes.c_int32, ctypes.c_int32, ctypes.c_float]
        lib.orc_entry_ok.restype = ctypes.c_int
        lib.orc_entry_ok.argtypes = [ctypes.c_int32, ctypes.c_int32, ctypes.c_float]
        lib.orc_score_many.restype = None
        lib.orc_score_many.argtypes = [ctypes.c_int64, P, P, P, P, P]
        lib.orc_select.restype = ctypes.c_int
        lib.orc_select.argtypes = [ctypes.POINTER(_Cache), P, P, P, P]
        lib.orc_attention.restype = ctypes.c_int
        lib.orc_attention.argtypes = [ctypes.POINTER(_Cache), P, ctypes.c_float, P, P, P, P]
        lib.orc_select_per_head.restype = ctypes.c_int
        lib.orc_select_per_head.argtypes = [ctypes.POINTER(_Cache), P, P, P, P]
        lib.orc_select_contour.restype = ctypes.c_int
        lib.orc_select_contour.argtypes = [ctypes.POINTER(_Cache), P, P, P, ctypes.c_float, ctypes.c_int32,
                                           ctypes.c_int32, P, P, P]
        lib.orc_memory_update.restype = ctypes.c_int
        lib.orc_memory_update.argtypes = [ctypes.POINTER(_Cache), P, P, ctypes.c_double, P, P]
        lib.orc_memory_read.restype = ctypes.c_int
        lib.orc_memory_read.argtypes = [ctypes.POINTER(_Cache), P, P, P, P, P, P, P]
        lib.orc_eviction_error.restype = ctypes.c_int
        lib.orc_eviction_error.argtypes = [ctypes.POINTER(_Cache), P, ctypes.c_float, P, P, P]
        lib.orc_compact.restype = ctypes.c_int
        lib.orc_compact.argtypes = [ctypes.POINTER(_Cache), P]
        lib.orc_append.restype = ctypes.c_int
        lib.orc_append.argtypes = [ctypes.POINTER(_Cache), P, P, P, P]
        _libs[key] = lib
    return _libs[key]


def _ptr(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data


@dataclass
class HostCache:
    """Cache state as numpy arrays, in the layout both sides share.

    k_pool / v_pool: [n_pages, P, D] float32, or uint16 holding bfloat16 bits.
    pos_pool int32 / lb_pool float32: [n_pages, P].  block_table int32
    [C, max_pages] (-1 = no page).  len int32 [C].  free_stack int32 [n_pages],
    free_top int32 [1].  Heads c = (b*L + l)*H + h; G query heads per KV head.
    """
    B: int
    L: int
    H: int
    G: int
    D: int
    P: int
    k_pool: np.ndarray
    v_pool: np.ndarray
    pos_pool: np.ndarray
    lb_pool: np.ndarray
    block_table: np.ndarray
    len: np.ndarray
    free_stack: np.ndarray
    free_top: np.ndarray

    @property
    def C(self) -> int:
        return self.B * self.L * self.H

    @property
    def n_pages(self) -> int:
        return self.k_pool.shape[0]

    @property
    def max_pages(self) -> int:
        return self.block_table.shape[1]

    def copy(self) -> "HostCache":
        return HostCache(self.B, self.L, self.H, self.G, self.D, self.P,
                         *(np.array(getattr(self, f), copy=True) for f in (
                             "k_pool", "v_pool", "pos_pool", "lb_pool", "block_table",
                             "len", "free_stack", "free_top")))

    def _struct(self) -> _Cache:
        kv_f32 = 1 if self.k_pool.dtype == np.float32 else 0
        if not kv_f32:
            assert self.k_pool.dtype == np.uint16 and self.v_pool.dtype == np.uint16
        for name, dt in (("pos_pool", np.int32), ("lb_pool", np.float32), ("block_table", np.int32),
                         ("len", np.int32), ("free_stack", np.int32), ("free_top", np.int32)):
            assert getattr(self, name).dtype == dt, name
        return _Cache(self.B, self.L, self.H, self.G, self.D, self.P, self.n_pages, self.max_pages, kv_f32,
                      _ptr(self.k_pool), _ptr(self.v_pool), _ptr(self.pos_pool), _ptr(self.lb_pool),
                      _ptr(self.block_table), _ptr(self.len), _ptr(self.free_stack), _ptr(self.free_top))


def score(t, pos, lb):
    """Element-wise score fl32((t - i) * log beta) and validity flags.

    Returns (s float32, ok bool).  Invalid entries (NaN log-retention, age
    outside [1, 2^24)) have ok = False and s = 0."""
    t = np.ascontiguousarray(np.broadcast_to(np.asarray(t, np.int32), np.shape(pos)), np.int32)
    pos = np.ascontiguousarray(pos, np.int32)
    lb = np.ascontiguousarray(lb, np.float32)
    s = np.empty(pos.shape, np.float32)
    ok = np.empty(pos.shape, np.uint8)
    _load().orc_score_many(pos.size, _ptr(t), _ptr(pos), _ptr(lb), _ptr(s), _ptr(ok))
    return s, ok.astype(bool)


def select(cache: HostCache, t, m_global):
    """Global top-M_global per sequence.  Returns (keep uint8 [C, max_pages*P], kept int32 [C])."""
    t = np.ascontiguousarray(t, np.int32).reshape(cache.B)
    m = np.ascontiguousarray(m_global, np.int64).reshape(cache.B)
    keep = np.zeros((cache.C, cache.max_pages * cache.P), np.uint8)
    kept = np.zeros(cache.C, np.int32)
    st = cache._struct()
    rc = _load().orc_select(ctypes.byref(st), _ptr(t), _ptr(m), _ptr(keep), _ptr(kept))
    if rc != OK:
        raise ValueError(f"oracle select refused its input (code {rc})")
    return keep, kept


def select_per_head(cache: HostCache, t, m_head):
    """Top-m_head[c] entries of every head c by score (equal scores by
    ascending position).  Returns (keep uint8 [C, max_pages*P], kept int32 [C])."""
    t = np.ascontiguousarray(t, np.int32).reshape(cache.B)
    m = np.ascontiguousarray(m_head, np.int32).reshape(cache.C)
    keep = np.zeros((cache.C, cache.max_pages * cache.P), np.uint8)
    kept = np.zeros(cache.C, np.int32)
    st = cache._struct()
    rc = _load().orc_select_per_head(ctypes.byref(st), _ptr(t), _ptr(m), _ptr(keep), _ptr(kept))
    if rc != OK:
        raise ValueError(f"oracle per-head select refused its input (code {rc})")
    return keep, kept


def select_contour(cache: HostCache, t, m_global, dm_prev, tau: float, flat_budget: int, floor: int):
    """ContourKV allocation: recency floor in every head, a fixed budget for
    heads whose mean previous dropped mass exceeds tau, the rest of M_global
    by the global order over the other heads.  dm_prev float32 [C, G].
    Returns (keep, kept, flat uint8 [C])."""
    t = np.ascontiguousarray(t, np.int32).reshape(cache.B)
    m = np.ascontiguousarray(m_global, np.int64).reshape(cache.B)
    dm = np.ascontiguousarray(dm_prev, np.float32).reshape(cache.C, cache.G)
    keep = np.zeros((cache.C, cache.max_pages * cache.P), np.uint8)
    kept = np.zeros(cache.C, np.int32)
    flat = np.zeros(cache.C, np.uint8)
    st = cache._struct()
    rc = _load().orc_select_contour(ctypes.byref(st), _ptr(t), _ptr(m), _ptr(dm), ctypes.c_float(tau),
                                    int(flat_budget), int(floor), _ptr(keep), _ptr(kept), _ptr(flat))
    if rc != OK:
        raise ValueError(f"oracle ContourKV select refused its input (code {rc})")
    return keep, kept, flat


def attention(cache: HostCache, q: np.ndarray, scale: float, keep: np.ndarray | None):
    """Forced-weight attention over the kept set plus dropped mass.

    q float32 [C, G, D] (== [B, L, Hq, D]).  Returns (out [C, G, D], lse_kept
    [C, G], dropped [C, G]) as float32."""
    q = np.ascontiguousarray(q, np.float32).reshape(cache.C, cache.G, cache.D)
    out = np.zeros((cache.C, cache.G, cache.D), np.float32)
    lse = np.zeros((cache.C, cache.G), np.float32)
    dm = np.zeros((cache.C, cache.G), np.float32)
    if keep is not None:
        keep = np.ascontiguousarray(keep, np.uint8)
    st = cache._struct()
    rc = _load().orc_attention(ctypes.byref(st), _ptr(q), ctypes.c_float(scale), _ptr(keep),
                               _ptr(out), _ptr(lse), _ptr(dm))
    if rc != OK:
        raise ValueError(f"oracle attention failed (code {rc})")
    return out, lse, dm


def eviction_error(cache: HostCache, q: np.ndarray, scale: float, keep: np.ndarray | None,
                   with_dense: bool = False):
    """Per query head, the distance ||mu - m_A|| between the dense output mu
    (softmax over every entry present) and the forced-weight output m_A over
    the kept set.  Returns err float32 [C, G], and with ``with_dense`` also mu
    [C, G, D]."""
    q = np.ascontiguousarray(q, np.float32).reshape(cache.C, cache.G, cache.D)
    err = np.zeros((cache.C, cache.G), np.float32)
    mu = np.zeros((cache.C, cache.G, cache.D), np.float32) if with_dense else None
    if keep is not None:
        keep = np.ascontiguousarray(keep, np.uint8)
    st = cache._struct()
    rc = _load().orc_eviction_error(ctypes.byref(st), _ptr(q), ctypes.c_float(scale), _ptr(keep), _ptr(err),
                                    _ptr(mu))
    if rc != OK:
        raise ValueError(f"oracle eviction error failed (code {rc})")
    return (err, mu) if with_dense else err


def memory_update(cache: HostCache, keep: np.ndarray, proj: np.ndarray, decay: float, M: np.ndarray,
                  b: np.ndarray) -> None:
    """Latent memory update with this step's evicted entries, in place:
    M [C, D, D], b [C, D] float64; proj [L, D, D] float32."""
    assert M.dtype == np.float64 and b.dtype == np.float64 and M.flags["C_CONTIGUOUS"] and b.flags["C_CONTIGUOUS"]
    keep = np.ascontiguousarray(keep, np.uint8)
    proj = np.ascontiguousarray(proj, np.float32)
    st = cache._struct()
    rc = _load().orc_memory_update(ctypes.byref(st), _ptr(keep), _ptr(proj), float(decay), _ptr(M), _ptr(b))
    if rc != OK:
        raise ValueError(f"oracle memory update failed (code {rc})")


def memory_read(cache: HostCache, q: np.ndarray, proj: np.ndarray, gate_w: np.ndarray, gate_b: np.ndarray,
                M: np.ndarray, b: np.ndarray, out: np.ndarray) -> np.ndarray:
    """out + g(q) * m(q) per query head (a new float32 [C, G, D] array);
    gate_w [L, Hq, D], gate_b [L, Hq] float32."""
    q = np.ascontiguousarray(q, np.float32).reshape(cache.C, cache.G, cache.D)
    res = np.array(np.asarray(out, np.float32).reshape(cache.C, cache.G, cache.D), copy=True)
    st = cache._struct()
    rc = _load().orc_memory_read(ctypes.byref(st), _ptr(q), _ptr(np.ascontiguousarray(proj, np.float32)),
                                 _ptr(np.ascontiguousarray(gate_w, np.float32)),
                                 _ptr(np.ascontiguousarray(gate_b, np.float32)), _ptr(M), _ptr(b), _ptr(res))
    if rc != OK:
        raise ValueError(f"oracle memory read failed (code {rc})")
    return res


def compact(cache: HostCache, keep: np.ndarray) -> None:
    """Hole-fill compaction and free-page pushes, in place."""
    keep = np.ascontiguousarray(keep, np.uint8)
    st = cache._struct()
    rc = _load().orc_compact(ctypes.byref(st), _ptr(keep))
    if rc != OK:
        raise ValueError(f"oracle compaction failed (code {rc})")


def append(cache: HostCache, t, k_new: np.ndarray, v_new: np.ndarray, lb_new: np.ndarray) -> int:
    """Append token t's row to every head, in place.  Returns the status code
    (OK, ERR_POOL when the free stack runs out, ERR_TABLE past max_pages)."""
    t = np.ascontiguousarray(t, np.int32).reshape(cache.B)
    k_new = np.ascontiguousarray(k_new).reshape(cache.C, cache.D)
    v_new = np.ascontiguousarray(v_new).reshape(cache.C, cache.D)
    assert k_new.dtype == cache.k_pool.dtype and v_new.dtype == cache.v_pool.dtype
    lb_new = np.ascontiguousarray(lb_new, np.float32).reshape(cache.C)
    st = cache._struct()
    return _load().orc_append(ctypes.byref(st), _ptr(t), _ptr(k_new), _ptr(v_new), _ptr(lb_new))


def step(cache: HostCache, t, m_global, q, k_new, v_new, lb_new, *, evict: bool = True,
         scale: float | None = None):
    """One decode step, in place on ``cache``: select -> attention + dropped
    mass over the pre-compaction cache -> compaction -> append.

    Returns dict(keep, kept, out, lse, dropped).  On a non-evicting step every
    entry is kept and dropped mass is 0."""
    if scale is None:
        scale = 1.0 / float(np.sqrt(cache.D))
    keep = kept = None
    if evict:
        keep, kept = select(cache, t, m_global)
    out, lse, dm = attention(cache, q, scale, keep)
    if evict:
        compact(cache, keep)
    rc = append(cache, t, k_new, v_new, lb_new)
    if rc != OK:
        raise ValueError(f"oracle append failed (code {rc})")
    return dict(keep=keep, kept=kept, out=out, lse=lse, dropped=dm)
