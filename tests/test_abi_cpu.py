"""The C-ABI library on a machine without a GPU: it loads, exports every entry
point include/spade.h declares, and rejects bad arguments on the host before
any CUDA call."""
import ctypes
import os
import re

import pytest

from input_adaptive_block_b200 import _lib
from input_adaptive_block_b200._lib import SpadeGeom, SpadeHeadScheme
from spade_workloads import CONFIGS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared(*headers):
    names = set()
    for h in headers or (os.path.join(ROOT, "include", "spade.h"),):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names |= set(re.findall(r"\b(spade_[a-z0-9_]+)\s*\(", text))
    return sorted(names)


def test_library_exports_its_selftest_entry_points():
    """The test-only entry points (declared in an internal header, not in
    include/spade.h) are exported too, and nothing else is exported under the
    spade_ prefix."""
    lib = _lib.load()
    internal = os.path.join(ROOT, "input_adaptive_block_b200", "csrc", "spade_selftest.h")
    names = _declared(internal)
    assert names == ["spade_selftest_bounded_wait"]
    for n in names:
        assert hasattr(lib, n) and n in _lib.SIGNATURES, n
    public = _declared()
    assert not set(names) & set(public)
    assert set(_lib.SIGNATURES) == set(public) | set(names)


def test_library_exports_every_declared_symbol():
    lib = _lib.load()
    names = _declared()
    assert len(names) >= 14
    for n in names:
        assert hasattr(lib, n), n
        assert n in _lib.SIGNATURES, n
    assert lib.spade_version() == 1


def test_status_strings():
    lib = _lib.load()
    for s in range(6):
        assert lib.spade_status_string(s)
    assert lib.spade_status_string(99) == b"unknown status"


def _mixed_tables():
    wl = CONFIGS["mixed"]
    gs = (SpadeGeom * len(wl.schemes))(*[SpadeGeom(*s.as_tuple()) for s in wl.schemes])
    rows = (SpadeHeadScheme * wl.heads)(*[SpadeHeadScheme(sc, t, int(dn)) for sc, t, dn in
                                          zip(wl.head_scheme, wl.head_tau, wl.head_dense)])
    return wl, gs, rows


def test_grouped_workspace_layout_host_only():
    lib = _lib.load()
    wl, gs, rows = _mixed_tables()
    total = lib.spade_grouped_workspace_bytes(gs, 3, rows, wl.heads, wl.d, 0)
    # lower bound: the per-scheme arrays of the sparse heads plus the work list
    lower = 0
    for s_id, sc in enumerate(wl.schemes):
        hs = sum(1 for h in range(wl.heads) if wl.head_scheme[h] == s_id and not wl.head_dense[h])
        lower += hs * sc.nb * (2 * wl.d * 4 + 2 * sc.nb * 4 + 4)
    n_items = sum(wl.schemes[wl.head_scheme[h]].nb for h in range(wl.heads))
    lower += 4 * n_items
    assert lower <= total <= lower + 64 * 256
    # head lists: dense heads have none; sparse heads get distinct, ordered regions
    co, io = ctypes.c_int64(), ctypes.c_int64()
    assert lib.spade_grouped_head_lists(gs, 3, rows, wl.heads, wl.d, 0, 0, ctypes.byref(co), ctypes.byref(io)) == 0
    assert co.value == -1 and io.value == -1
    prev = -1
    for h in range(13, 27):
        assert lib.spade_grouped_head_lists(gs, 3, rows, wl.heads, wl.d, 0, h,
                                            ctypes.byref(co), ctypes.byref(io)) == 0
        assert co.value > prev and io.value % 4 == 0 and io.value + 630 * 630 * 4 <= total
        prev = co.value


def test_host_validation_errors():
    lib = _lib.load()
    wl, gs, rows = _mixed_tables()
    # bad scheme index, bad tau, too many schemes, bad d
    bad = (SpadeHeadScheme * 2)(SpadeHeadScheme(5, 0.9, 0), SpadeHeadScheme(0, 0.9, 0))
    assert lib.spade_grouped_workspace_bytes(gs, 3, bad, 2, 128, 0) == 0
    bad = (SpadeHeadScheme * 1)(SpadeHeadScheme(1, -0.5, 0))
    assert lib.spade_grouped_workspace_bytes(gs, 3, bad, 1, 128, 0) == 0
    assert lib.spade_grouped_workspace_bytes(gs, 5, rows, wl.heads, 128, 0) == 0
    assert lib.spade_grouped_workspace_bytes(gs, 3, rows, wl.heads, 96, 0) == 0
    g = SpadeGeom(21, 45, 80, 2, 8, 8)
    fake = ctypes.c_void_p(1 << 20)                 # never dereferenced: validation fails first
    taus = (ctypes.c_float * 1)(0.9)
    assert lib.spade_select(fake, taus, fake, fake, 1, 2000, None) == _lib.SPADE_ERR_UNSUPPORTED
    assert lib.spade_select(None, taus, fake, fake, 1, 10, None) == _lib.SPADE_ERR_INVALID
    bad_tau = (ctypes.c_float * 1)(0.0)
    assert lib.spade_select(fake, bad_tau, fake, fake, 1, 10, None) == _lib.SPADE_ERR_INVALID
    assert lib.spade_estimate(fake, fake, fake, 1, 4096, 128, None) == _lib.SPADE_ERR_UNSUPPORTED
    assert lib.spade_block_sparse_attn(fake, fake, fake, fake, None, None, g, 40, 96, 0, 1, fake, 1 << 20,
                                       None) == _lib.SPADE_ERR_UNSUPPORTED
    assert lib.spade_block_sparse_attn(fake, fake, fake, fake, None, None, g, 40, 128, 0, 1, fake, 16,
                                       None) == _lib.SPADE_ERR_WORKSPACE
    odd = ctypes.c_void_p((1 << 20) + 8)
    assert lib.spade_block_sparse_attn(odd, fake, fake, fake, None, None, g, 40, 128, 0, 1, fake, 1 << 20,
                                       None) == _lib.SPADE_ERR_INVALID
    assert lib.spade_block_sparse_attn(fake, fake, fake, fake, fake, None, g, 40, 128, 0, 1, fake, 1 << 20,
                                       None) == _lib.SPADE_ERR_INVALID
    assert lib.spade_tile3d(fake, fake, SpadeGeom(0, 1, 1, 1, 1, 1), 1, 128, 1, None) == _lib.SPADE_ERR_INVALID
    assert b"extent" in lib.spade_last_error_message()


def test_attn_workspace_bytes():
    lib = _lib.load()
    g = SpadeGeom(21, 45, 80, 2, 8, 8)
    assert lib.spade_attn_workspace_bytes(g, 40, 128, 0) >= 40 * 660 * 4
    assert lib.spade_attn_workspace_bytes(g, 40, 128, 256) >= 40 * 662 * 4
    assert lib.spade_attn_workspace_bytes(SpadeGeom(0, 1, 1, 1, 1, 1), 1, 128, 0) == 0


def test_sics_host_validation():
    lib = _lib.load()
    g1 = SpadeGeom(21, 45, 80, 2, 8, 8)
    cands = (SpadeGeom * 3)(g1, SpadeGeom(21, 45, 80, 1, 8, 16), SpadeGeom(21, 45, 80, 8, 4, 4))
    need = lib.spade_sics_workspace_bytes(cands, 3, 40)
    assert need == 4 * 40 * (660 + 630 + 720)
    assert lib.spade_sics_workspace_bytes(cands, 0, 40) == 0
    fake = ctypes.c_void_p(1 << 20)                 # never dereferenced: validation fails first
    args = lambda **kw: dict(dict(q=fake, k=fake, c=cands, n=3, h=40, d=128, dt=1, s=fake, ch=fake, ws=fake,
                                  wsb=need), **kw)
    call = lambda a: lib.spade_sics(a["q"], a["k"], a["c"], a["n"], a["h"], a["d"], a["dt"], a["s"], a["ch"],
                                    a["ws"], a["wsb"], None)
    assert call(args(q=None)) == _lib.SPADE_ERR_INVALID
    assert call(args(n=0)) == _lib.SPADE_ERR_INVALID
    assert call(args(d=96)) == _lib.SPADE_ERR_UNSUPPORTED
    assert call(args(wsb=16)) == _lib.SPADE_ERR_WORKSPACE
    other = (SpadeGeom * 2)(g1, SpadeGeom(21, 45, 81, 2, 8, 8))
    assert call(args(c=other, n=2)) == _lib.SPADE_ERR_INVALID
    assert b"different number of tokens" in lib.spade_last_error_message()


def test_select_window_host_validation():
    lib = _lib.load()
    g = SpadeGeom(21, 45, 80, 2, 8, 8)
    fake = ctypes.c_void_p(1 << 20)
    taus = (ctypes.c_float * 1)(0.9)
    rad = (ctypes.c_int * 3)(0, -1, 0)
    assert lib.spade_select_window(fake, taus, rad, g, fake, fake, 1, None) == _lib.SPADE_ERR_INVALID
    rad = (ctypes.c_int * 3)(0, 1, 0)
    assert lib.spade_select_window(None, taus, rad, g, fake, fake, 1, None) == _lib.SPADE_ERR_INVALID
    big = SpadeGeom(64, 64, 64, 2, 2, 2)            # 32768 blocks: above the selection limit
    assert lib.spade_select_window(fake, taus, rad, big, fake, fake, 1, None) == _lib.SPADE_ERR_UNSUPPORTED


def test_copy_head_slice_host_validation():
    lib = _lib.load()
    fake = ctypes.c_void_p(1 << 20)
    assert lib.spade_copy_head_slice(None, fake, 10, 4, 0, 2, 128, 1, 1, None) == _lib.SPADE_ERR_INVALID
    assert lib.spade_copy_head_slice(fake, fake, 10, 4, 3, 2, 128, 1, 1, None) == _lib.SPADE_ERR_INVALID
    assert lib.spade_copy_head_slice(fake, fake, 0, 4, 0, 2, 128, 1, 1, None) == _lib.SPADE_ERR_INVALID


def test_fused_form_entry_points_host_validation():
    """spade_summarize_qk, spade_estimate_scores and spade_select_scores reject
    bad arguments on the host, before anything is enqueued."""
    lib = _lib.load()
    fake = ctypes.c_void_p(1 << 20)                 # never dereferenced: validation fails first
    odd = ctypes.c_void_p((1 << 20) + 8)
    g = SpadeGeom(21, 45, 80, 2, 8, 8)
    # summarize_qk: null / misaligned pointers, bad d, bad geometry, no heads
    assert lib.spade_summarize_qk(None, fake, fake, fake, g, 4, 128, 1, None) == _lib.SPADE_ERR_INVALID
    assert lib.spade_summarize_qk(fake, fake, odd, fake, g, 4, 128, 1, None) == _lib.SPADE_ERR_INVALID
    assert lib.spade_summarize_qk(fake, fake, fake, fake, g, 4, 96, 1, None) == _lib.SPADE_ERR_UNSUPPORTED
    assert lib.spade_summarize_qk(fake, fake, fake, fake, SpadeGeom(0, 1, 1, 1, 1, 1), 4, 128, 1,
                                  None) == _lib.SPADE_ERR_INVALID
    assert lib.spade_summarize_qk(fake, fake, fake, fake, g, 0, 128, 1, None) == _lib.SPADE_ERR_INVALID
    # estimate_scores: the same limits as spade_estimate
    assert lib.spade_estimate_scores(None, fake, fake, 1, 10, 128, None) == _lib.SPADE_ERR_INVALID
    assert lib.spade_estimate_scores(fake, fake, odd, 1, 10, 128, None) == _lib.SPADE_ERR_INVALID
    assert lib.spade_estimate_scores(fake, fake, fake, 1, 4096, 128, None) == _lib.SPADE_ERR_UNSUPPORTED
    assert lib.spade_estimate_scores(fake, fake, fake, 1, 10, 96, None) == _lib.SPADE_ERR_UNSUPPORTED
    assert lib.spade_estimate_scores(fake, fake, fake, 0, 10, 128, None) == _lib.SPADE_ERR_INVALID
    # select_scores: the same limits as spade_select
    taus = (ctypes.c_float * 2)(0.9, 0.9)
    bad_tau = (ctypes.c_float * 2)(0.9, float("nan"))
    assert lib.spade_select_scores(None, taus, fake, fake, 2, 10, None) == _lib.SPADE_ERR_INVALID
    assert lib.spade_select_scores(fake, taus, fake, fake, 2, 2000, None) == _lib.SPADE_ERR_UNSUPPORTED
    assert lib.spade_select_scores(fake, taus, fake, fake, 2, 0, None) == _lib.SPADE_ERR_INVALID
    assert lib.spade_select_scores(fake, bad_tau, fake, fake, 2, 10, None) == _lib.SPADE_ERR_INVALID
    assert lib.spade_select_scores(fake, taus, fake, fake, 2000, 10, None) == _lib.SPADE_ERR_UNSUPPORTED


def test_noalloc_host_validation():
    """spade_block_sparse_attn_noalloc refuses, on the host and before it
    touches the device or its fixed scratch: calls with more work items than
    the fixed scratch holds, and the same bad arguments the workspace entry
    point refuses."""
    lib = _lib.load()
    fake = ctypes.c_void_p(1 << 20)                 # never dereferenced: validation fails first
    odd = ctypes.c_void_p((1 << 20) + 8)
    g = SpadeGeom(21, 45, 80, 2, 8, 8)
    call = lambda q=fake, cnt=None, idx=None, geom=g, heads=40, d=128, text=0, dt=1: \
        lib.spade_block_sparse_attn_noalloc(q, fake, fake, fake, cnt, idx, geom, heads, d, text, dt, None)
    big = SpadeGeom(64, 64, 512, 2, 8, 8)           # 16384 blocks x 8 heads > 65536 work items
    assert call(geom=big, heads=8) == _lib.SPADE_ERR_UNSUPPORTED
    assert b"fixed scratch" in lib.spade_last_error_message()
    assert call(q=None) == _lib.SPADE_ERR_INVALID
    assert call(q=odd) == _lib.SPADE_ERR_INVALID
    assert call(cnt=fake) == _lib.SPADE_ERR_INVALID       # cnt without idx
    assert call(d=96) == _lib.SPADE_ERR_UNSUPPORTED
    assert call(heads=0) == _lib.SPADE_ERR_UNSUPPORTED
    assert call(heads=200) == _lib.SPADE_ERR_UNSUPPORTED
    assert call(text=-1) == _lib.SPADE_ERR_INVALID
    assert call(dt=7) == _lib.SPADE_ERR_INVALID
    assert call(geom=SpadeGeom(0, 1, 1, 1, 1, 1)) == _lib.SPADE_ERR_INVALID
    # blocks above 128 slots take the CUDA-core kernel, which cannot hold them
    assert call(geom=SpadeGeom(16, 16, 16, 2, 8, 16), heads=1, dt=0) == _lib.SPADE_ERR_UNSUPPORTED
    assert b"128 slots" in lib.spade_last_error_message()


def test_attention_refusals_before_any_launch():
    """Shapes the attention launch cannot run are refused by every entry point
    before anything is enqueued (no CUDA call is made, so this runs without a
    GPU): a head with more than 65536 query blocks (video + text; a work item
    packs the query block in 16 bits), and blocks above 128 slots on the
    CUDA-core path."""
    lib = _lib.load()
    fake = ctypes.c_void_p(1 << 20)
    huge = ctypes.c_size_t(1 << 40)
    flat = SpadeGeom(1, 1, 65535 * 128, 1, 1, 128)   # 65535 blocks of 128 tokens
    assert lib.spade_block_sparse_attn(fake, fake, fake, fake, None, None, flat, 1, 128, 256, 1, fake, huge,
                                       None) == _lib.SPADE_ERR_UNSUPPORTED
    assert b"65536 query blocks" in lib.spade_last_error_message()
    wide = SpadeGeom(16, 16, 16, 2, 8, 16)          # 256-slot blocks
    assert lib.spade_block_sparse_attn(fake, fake, fake, fake, None, None, wide, 1, 128, 0, 0, fake, huge,
                                       None) == _lib.SPADE_ERR_UNSUPPORTED
    assert b"128 slots" in lib.spade_last_error_message()
    # the grouped call refuses the same shape before its selection steps
    gs = (SpadeGeom * 1)(wide)
    rows = (SpadeHeadScheme * 1)(SpadeHeadScheme(0, 0.9, 0))
    need = lib.spade_grouped_workspace_bytes(gs, 1, rows, 1, 128, 0)
    assert need > 0
    assert lib.spade_grouped_attn(fake, fake, fake, fake, gs, 1, rows, 1, 128, 0, 0, fake, need,
                                  None) == _lib.SPADE_ERR_UNSUPPORTED
    assert b"128 slots" in lib.spade_last_error_message()


def test_host_layer_and_lists_host_validation():
    """spade_grouped_attn_host and spade_grouped_attn_lists check their
    arguments and workspace on the host before any CUDA call."""
    lib = _lib.load()
    wl, gs, rows = _mixed_tables()
    fake = ctypes.c_void_p(1 << 20)                 # never dereferenced: validation fails first
    need = lib.spade_grouped_host_workspace_bytes(gs, 3, rows, wl.heads, wl.d, 0, 1, 4)
    assert need >= 3 * 4 * wl.N * 4 * wl.d * 2       # three slots of Q, K, V, O for four heads
    assert lib.spade_grouped_host_workspace_bytes(gs, 3, rows, wl.heads, wl.d, 0, 1, 0) == 0
    assert lib.spade_grouped_host_workspace_bytes(gs, 3, rows, wl.heads, wl.d, 0, 1, wl.heads + 1) == 0
    assert lib.spade_grouped_host_workspace_bytes(gs, 3, rows, wl.heads, wl.d, 0, 1, 8) > need
    call = lambda q=fake, ws=fake, wsb=need, chunk=4: lib.spade_grouped_attn_host(
        q, fake, fake, fake, gs, 3, rows, wl.heads, wl.d, 0, 1, chunk, ws, wsb, None)
    assert call(q=None) == _lib.SPADE_ERR_INVALID
    assert call(wsb=16) == _lib.SPADE_ERR_WORKSPACE
    assert call(ws=None) == _lib.SPADE_ERR_WORKSPACE
    assert call(chunk=0) == _lib.SPADE_ERR_INVALID
    assert call(ws=ctypes.c_void_p((1 << 20) + 8)) == _lib.SPADE_ERR_INVALID
    gneed = lib.spade_grouped_workspace_bytes(gs, 3, rows, wl.heads, wl.d, 0)
    lists = lambda q=fake, ws=fake, wsb=gneed: lib.spade_grouped_attn_lists(
        q, fake, fake, fake, gs, 3, rows, wl.heads, wl.d, 0, 1, ws, wsb, None)
    assert lists(q=None) == _lib.SPADE_ERR_INVALID
    assert lists(wsb=gneed - 1) == _lib.SPADE_ERR_WORKSPACE
    assert lists(q=ctypes.c_void_p((1 << 20) + 4)) == _lib.SPADE_ERR_INVALID

