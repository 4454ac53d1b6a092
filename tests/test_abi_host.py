"""Host-side checks of the C ABI that need no GPU: every symbol declared in
include/rkv.h is exported by librkv.so, and argument validation returns its
error codes (with a message) before any CUDA call is made."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from retention_scored_kv_b200 import build
    path = build.build()
    import retention_scored_kv_b200 as rkv
    return rkv, rkv.load(path)


def _declared_symbols():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            names += re.findall(r"RKV_API[^;(]*?\b(rkv_\w+)\s*\(", text)
    return names


def test_header_declares_the_boundary():
    names = set(_declared_symbols())
    for want in ("rkv_score_select", "rkv_compact_pages", "rkv_paged_decode_attn", "rkv_dropped_mass",
                 "rkv_eviction_error",
                 "rkv_append", "rkv_decode_step", "rkv_workspace_size", "rkv_workspace_init", "rkv_device_status",
                 "rkv_version", "rkv_last_error"):
        assert want in names


def test_every_declared_symbol_is_exported(lib):
    rkv, so = lib
    for name in _declared_symbols():
        assert hasattr(so, name), name
    assert set(rkv.EXPORTS) <= set(_declared_symbols())


def _cache(rkv, **kw):
    f = dict(k_pool=16, v_pool=16, pos_pool=16, lb_pool=16, block_table=16, len=16, free_stack=16, free_top=16,
             B=1, L=2, H=4, Hq=8, D=128, P=16, n_pages=64, max_pages=8, dtype=rkv.BF16)
    f.update(kw)
    return rkv.CacheStruct(*(f[n] for n, _ in rkv.CacheStruct._fields_))


def test_version_and_workspace_size(lib):
    rkv, so = lib
    assert so.rkv_version().decode().startswith("librkv")
    good = so.rkv_workspace_size(ctypes.byref(_cache(rkv)))
    assert good > 0
    bigger = so.rkv_workspace_size(ctypes.byref(_cache(rkv, B=4)))
    assert bigger > good
    assert so.rkv_workspace_size(ctypes.byref(_cache(rkv, B=0))) == 0
    assert so.rkv_workspace_size(ctypes.byref(_cache(rkv, P=8))) == 0
    assert so.rkv_workspace_size(ctypes.byref(_cache(rkv, Hq=6))) == 0


@pytest.mark.parametrize("kw,code,needle", [
    (dict(B=0), -1, "positive"),
    (dict(Hq=6), -1, "multiple"),
    (dict(P=8), -2, "page size"),
    (dict(dtype=7), -1, "dtype"),
    (dict(D=4, dtype=0), -2, "16"),
    (dict(k_pool=None), -1, "NULL"),
    (dict(k_pool=8), -1, "aligned"),
])
def test_invalid_cache_rejected_before_cuda(lib, kw, code, needle):
    rkv, so = lib
    cs = _cache(rkv, **kw)
    sel = rkv.SelectStruct(16, 16, 16, 16, 16)
    rc = so.rkv_score_select(ctypes.byref(cs), ctypes.c_void_p(16), ctypes.c_void_p(16), ctypes.byref(sel),
                             ctypes.c_void_p(16), 1 << 30, None)
    assert rc == code
    assert needle in so.rkv_last_error().decode()


def test_small_workspace_and_null_arguments(lib):
    rkv, so = lib
    cs = _cache(rkv)
    sel = rkv.SelectStruct(16, 16, 16, 16, 16)
    need = so.rkv_workspace_size(ctypes.byref(cs))
    rc = so.rkv_score_select(ctypes.byref(cs), ctypes.c_void_p(16), ctypes.c_void_p(16), ctypes.byref(sel),
                             ctypes.c_void_p(16), need - 1, None)
    assert rc == rkv.ERR_WORKSPACE_TOO_SMALL
    bad_sel = rkv.SelectStruct(16, 16, None, 16, 16)
    rc = so.rkv_score_select(ctypes.byref(cs), ctypes.c_void_p(16), ctypes.c_void_p(16), ctypes.byref(bad_sel),
                             ctypes.c_void_p(16), need, None)
    assert rc == rkv.ERR_INVALID_ARG
    rc = so.rkv_paged_decode_attn(ctypes.byref(cs), ctypes.c_void_p(16), ctypes.c_float(0.1), None, None, None,
                                  None, ctypes.c_void_p(16), need, None)
    assert rc == rkv.ERR_INVALID_ARG and "out" in so.rkv_last_error().decode()
    rc = so.rkv_dropped_mass(ctypes.byref(cs), ctypes.c_void_p(16), ctypes.c_float(0.1), None,
                             ctypes.c_void_p(16), ctypes.c_void_p(16), need, None)
    assert rc == rkv.ERR_INVALID_ARG and "sel" in so.rkv_last_error().decode()
    rc = so.rkv_eviction_error(ctypes.byref(cs), ctypes.c_void_p(16), ctypes.c_float(0.1), None, ctypes.c_void_p(16),
                               ctypes.c_void_p(16), ctypes.c_void_p(16), ctypes.c_void_p(16), need, None)
    assert rc == rkv.ERR_INVALID_ARG and "sel" in so.rkv_last_error().decode()
    rc = so.rkv_eviction_error(ctypes.byref(cs), ctypes.c_void_p(16), ctypes.c_float(0.1), ctypes.byref(sel), None,
                               ctypes.c_void_p(16), ctypes.c_void_p(16), ctypes.c_void_p(16), need, None)
    assert rc == rkv.ERR_INVALID_ARG and "out_kept" in so.rkv_last_error().decode()
    rc = so.rkv_append(ctypes.byref(cs), None, ctypes.c_void_p(16), ctypes.c_void_p(16), ctypes.c_void_p(16),
                       ctypes.c_void_p(16), need, None)
    assert rc == rkv.ERR_INVALID_ARG
    rc = so.rkv_compact_pages(ctypes.byref(cs), ctypes.byref(sel), None, need, None)
    assert rc == rkv.ERR_INVALID_ARG and "workspace" in so.rkv_last_error().decode()
    assert so.rkv_device_status(None) is None
    assert so.rkv_device_status(ctypes.c_void_p(4096)) == 4096


def test_unsupported_attention_shape(lib):
    rkv, so = lib
    cs = _cache(rkv, H=2, Hq=24)  # G = 12 is not built
    need = so.rkv_workspace_size(ctypes.byref(cs))
    rc = so.rkv_paged_decode_attn(ctypes.byref(cs), ctypes.c_void_p(16), ctypes.c_float(0.1), None,
                                  ctypes.c_void_p(16), None, None, ctypes.c_void_p(16), need, None)
    assert rc == rkv.ERR_UNSUPPORTED


def _decode_step(rkv, so, cs, *, q=16, m_global=16, sel=None, ws_bytes=None):
    """One rkv_decode_step call with placeholder device pointers.  Every case
    below must be rejected before the first CUDA call: a call that passed
    validation would launch on those pointers."""
    sel = rkv.SelectStruct(16, 16, 16, 16, 16) if sel is None else sel
    need = so.rkv_workspace_size(ctypes.byref(cs))
    return so.rkv_decode_step(ctypes.byref(cs), 16, m_global, q, 0.1, 16, 16, 16, ctypes.byref(sel), 16, 16, 16,
                              16, need if ws_bytes is None else ws_bytes, None)


def test_decode_step_rejects_bad_arguments_before_cuda(lib):
    rkv, so = lib
    cs = _cache(rkv)
    assert _decode_step(rkv, so, cs, q=None) == rkv.ERR_INVALID_ARG
    assert "non-NULL" in so.rkv_last_error().decode()
    assert _decode_step(rkv, so, cs, q=8) == rkv.ERR_INVALID_ARG
    assert "aligned" in so.rkv_last_error().decode()
    # a budget needs every selection buffer; without one (no eviction) the
    # selection is not read, and the call proceeds to the workspace check
    bad_sel = rkv.SelectStruct(16, 16, 16, None, 16)
    assert _decode_step(rkv, so, cs, sel=bad_sel) == rkv.ERR_INVALID_ARG
    assert "selection" in so.rkv_last_error().decode()
    assert _decode_step(rkv, so, cs, m_global=None, sel=bad_sel, ws_bytes=1) == rkv.ERR_WORKSPACE_TOO_SMALL
    assert _decode_step(rkv, so, cs, ws_bytes=1) == rkv.ERR_WORKSPACE_TOO_SMALL


@pytest.mark.parametrize("kw,needle", [
    (dict(B=65), "at most 64"),          # one launch holds at most 64 sequences
    (dict(H=2, Hq=6), "not built"),      # GQA group 3
    (dict(D=96), "not built"),
    (dict(dtype="F32", H=2, Hq=16), "not built"),  # fp32 pools with G = 8
])
def test_decode_step_unsupported_shapes(lib, kw, needle):
    rkv, so = lib
    if kw.get("dtype") == "F32":
        kw = dict(kw, dtype=rkv.F32)
    cs = _cache(rkv, **kw)
    assert _decode_step(rkv, so, cs) == rkv.ERR_UNSUPPORTED
    assert needle in so.rkv_last_error().decode()
