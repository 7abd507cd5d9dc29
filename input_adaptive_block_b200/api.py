"""PyTorch-facing binding of the C ABI (argument marshalling only).

Every function here hands device pointers of caller tensors and the current
CUDA stream to the matching `spade_*` entry point of libspade.so; all
arithmetic happens in its CUDA kernels.  PyTorch provides memory and streams.
"""
from __future__ import annotations

import ctypes
from typing import Optional, Sequence, Tuple

import torch

from . import _lib
from ._lib import SpadeGeom, SpadeHeadScheme, check

__all__ = [
    "geom", "dtype_code", "tile3d", "summarize", "summarize_qk", "estimate", "estimate_scores", "select", "select_scores",
    "attn_workspace_bytes",
    "block_sparse_attn", "block_sparse_attn_noalloc", "grouped_workspace_bytes", "grouped_attn", "grouped_head_lists",
    "last_device_status", "selftest_bounded_wait", "num_blocks", "sics_workspace_bytes", "sics", "select_window",
    "grouped_attn_from_host", "grouped_host_workspace_bytes", "grouped_attn_lists",
]


def geom(g) -> SpadeGeom:
    """(T, H, W, bt, bh, bw) tuple, Scheme, or SpadeGeom -> SpadeGeom."""
    if isinstance(g, SpadeGeom):
        return g
    t = g.as_tuple() if hasattr(g, "as_tuple") else tuple(g)
    return SpadeGeom(*[int(v) for v in t])


def num_blocks(g) -> int:
    gg = geom(g)
    return -(-gg.T // gg.bt) * -(-gg.H // gg.bh) * -(-gg.W // gg.bw)


def dtype_code(dt: torch.dtype) -> int:
    if dt == torch.float32:
        return _lib.SPADE_F32
    if dt == torch.bfloat16:
        return _lib.SPADE_BF16
    raise TypeError(f"unsupported dtype {dt}")


def _stream(stream: Optional[torch.cuda.Stream]) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _dev(t: torch.Tensor, name: str) -> int:
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA tensor")
    return t.data_ptr()


def tile3d(x: torch.Tensor, g, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    gg = geom(g)
    heads, d = x.shape[1], x.shape[2]
    nb, bs = num_blocks(gg), gg.bt * gg.bh * gg.bw
    if out is None:
        out = torch.empty(heads, nb, bs, d, dtype=x.dtype, device=x.device)
    check(_lib.load().spade_tile3d(_dev(x, "x"), _dev(out, "xt"), gg, heads, d, dtype_code(x.dtype),
                                   _stream(stream)), "spade_tile3d")
    return out


SUMMARY = {"mean": 0, "max": 1, "min": 2}


def summarize(x: torch.Tensor, g, out: Optional[torch.Tensor] = None, stream=None,
              mode: str = "mean") -> torch.Tensor:
    """Block summaries [heads, nb, d] float32: mean (default), max or min
    over each block's valid tokens."""
    gg = geom(g)
    heads, d = x.shape[1], x.shape[2]
    if out is None:
        out = torch.empty(heads, num_blocks(gg), d, dtype=torch.float32, device=x.device)
    if mode == "mean":
        check(_lib.load().spade_summarize(_dev(x, "x"), _dev(out, "xmean"), gg, heads, d, dtype_code(x.dtype),
                                          _stream(stream)), "spade_summarize")
    else:
        check(_lib.load().spade_summarize_mode(_dev(x, "x"), _dev(out, "out"), gg, heads, d, dtype_code(x.dtype),
                                               SUMMARY[mode], _stream(stream)), "spade_summarize_mode")
    return out


def summarize_qk(q: torch.Tensor, k: torch.Tensor, g, qout: Optional[torch.Tensor] = None,
                 kout: Optional[torch.Tensor] = None, stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Block means of Q and of K in one launch."""
    gg = geom(g)
    heads, d = q.shape[1], q.shape[2]
    if k.shape[1:] != q.shape[1:] or k.dtype != q.dtype:
        raise ValueError("q and k must have the same heads, d and dtype")
    nb = num_blocks(gg)
    if qout is None:
        qout = torch.empty(heads, nb, d, dtype=torch.float32, device=q.device)
    if kout is None:
        kout = torch.empty(heads, nb, d, dtype=torch.float32, device=q.device)
    check(_lib.load().spade_summarize_qk(_dev(q, "q"), _dev(k, "k"), _dev(qout, "qmean"), _dev(kout, "kmean"),
                                         gg, heads, d, dtype_code(q.dtype), _stream(stream)), "spade_summarize_qk")
    return qout, kout


def estimate(qmean: torch.Tensor, kmean: torch.Tensor, out: Optional[torch.Tensor] = None,
             stream=None) -> torch.Tensor:
    heads, nb, d = qmean.shape
    if out is None:
        out = torch.empty(heads, nb, nb, dtype=torch.float32, device=qmean.device)
    check(_lib.load().spade_estimate(_dev(qmean, "qmean"), _dev(kmean, "kmean"), _dev(out, "prob"),
                                     heads, nb, d, _stream(stream)), "spade_estimate")
    return out


def estimate_scores(qmean: torch.Tensor, kmean: torch.Tensor, out: Optional[torch.Tensor] = None,
                    stream=None) -> torch.Tensor:
    """The Estimator's pooled scores Qbar . Kbar^T / sqrt(d) (no softmax)."""
    heads, nb, d = qmean.shape
    if out is None:
        out = torch.empty(heads, nb, nb, dtype=torch.float32, device=qmean.device)
    check(_lib.load().spade_estimate_scores(_dev(qmean, "qmean"), _dev(kmean, "kmean"), _dev(out, "scores"),
                                            heads, nb, d, _stream(stream)), "spade_estimate_scores")
    return out


def _select(fn_name: str, x: torch.Tensor, taus: Sequence[float], cnt, idx, stream):
    heads, nb, _ = x.shape
    if cnt is None:
        cnt = torch.empty(heads, nb, dtype=torch.int32, device=x.device)
    if idx is None:
        idx = torch.full((heads, nb, nb), -1, dtype=torch.int32, device=x.device)
    tau_arr = (ctypes.c_float * heads)(*[float(t) for t in taus])
    check(getattr(_lib.load(), fn_name)(_dev(x, "input"), tau_arr, _dev(cnt, "cnt"), _dev(idx, "idx"),
                                        heads, nb, _stream(stream)), fn_name)
    return cnt, idx


def select(prob: torch.Tensor, taus: Sequence[float], cnt: Optional[torch.Tensor] = None,
           idx: Optional[torch.Tensor] = None, stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    return _select("spade_select", prob, taus, cnt, idx, stream)


def select_scores(scores: torch.Tensor, taus: Sequence[float], cnt: Optional[torch.Tensor] = None,
                  idx: Optional[torch.Tensor] = None, stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Softmax of each score row fused with the index search."""
    return _select("spade_select_scores", scores, taus, cnt, idx, stream)


def select_window(prob: torch.Tensor, taus: Sequence[float], radius, g, cnt: Optional[torch.Tensor] = None,
                  idx: Optional[torch.Tensor] = None, stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Selection with a static window per head: radius = (rt, ry, rx) for
    every head, or one such triple per head."""
    heads, nb, _ = prob.shape
    if cnt is None:
        cnt = torch.empty(heads, nb, dtype=torch.int32, device=prob.device)
    if idx is None:
        idx = torch.full((heads, nb, nb), -1, dtype=torch.int32, device=prob.device)
    rad = list(radius) if len(radius) == heads and hasattr(radius[0], "__len__") else [tuple(radius)] * heads
    rad_arr = (ctypes.c_int * (3 * heads))(*[int(r) for t in rad for r in t])
    tau_arr = (ctypes.c_float * heads)(*[float(t) for t in taus])
    check(_lib.load().spade_select_window(_dev(prob, "prob"), tau_arr, rad_arr, geom(g), _dev(cnt, "cnt"),
                                          _dev(idx, "idx"), heads, _stream(stream)), "spade_select_window")
    return cnt, idx


def attn_workspace_bytes(g, heads: int, d: int, text_tokens: int = 0) -> int:
    return int(_lib.load().spade_attn_workspace_bytes(geom(g), heads, d, text_tokens))


def block_sparse_attn(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, cnt: Optional[torch.Tensor],
                      idx: Optional[torch.Tensor], g, text_tokens: int = 0, out: Optional[torch.Tensor] = None,
                      workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    gg = geom(g)
    heads, d = q.shape[1], q.shape[2]
    if out is None:
        out = torch.empty_like(q)
    need = attn_workspace_bytes(gg, heads, d, text_tokens)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    cp = _dev(cnt, "cnt") if cnt is not None else None
    ip = _dev(idx, "idx") if idx is not None else None
    check(_lib.load().spade_block_sparse_attn(
        _dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(out, "out"), cp, ip, gg, heads, d, text_tokens,
        dtype_code(q.dtype), _dev(workspace, "workspace"), workspace.numel(), _stream(stream)),
        "spade_block_sparse_attn")
    return out


def block_sparse_attn_noalloc(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, cnt: Optional[torch.Tensor],
                              idx: Optional[torch.Tensor], g, text_tokens: int = 0,
                              out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """spade_block_sparse_attn without a workspace argument: the library keeps
    the scratch in a fixed device array of its own (see include/spade.h for
    the size limit and the rule that overlapping calls must be ordered)."""
    gg = geom(g)
    heads, d = q.shape[1], q.shape[2]
    if out is None:
        out = torch.empty_like(q)
    cp = _dev(cnt, "cnt") if cnt is not None else None
    ip = _dev(idx, "idx") if idx is not None else None
    check(_lib.load().spade_block_sparse_attn_noalloc(
        _dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(out, "out"), cp, ip, gg, heads, d, text_tokens,
        dtype_code(q.dtype), _stream(stream)), "spade_block_sparse_attn_noalloc")
    return out


def _tables(schemes, table):
    gs = (SpadeGeom * len(schemes))(*[geom(s) for s in schemes])
    rows = (SpadeHeadScheme * len(table))(*[SpadeHeadScheme(int(sc), float(tau), int(bool(dn)))
                                            for sc, tau, dn in table])
    return gs, rows


def grouped_workspace_bytes(schemes, table, d: int, text_tokens: int = 0) -> int:
    gs, rows = _tables(schemes, table)
    return int(_lib.load().spade_grouped_workspace_bytes(gs, len(schemes), rows, len(table), d, text_tokens))


def grouped_attn(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, schemes, table, text_tokens: int = 0,
                 out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                 stream=None, summary=("mean", "mean"), window=None) -> torch.Tensor:
    """table: per head (scheme index, tau, dense); summary: the Q and K
    Summarizer reduces ("mean", "max" or "min"); window: optional static
    window block radii (rt, ry, rx) per head."""
    heads, d = q.shape[1], q.shape[2]
    gs, rows = _tables(schemes, table)
    if out is None:
        out = torch.empty_like(q)
    if workspace is None:
        need = int(_lib.load().spade_grouped_workspace_bytes(gs, len(schemes), rows, heads, d, text_tokens))
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    if tuple(summary) == ("mean", "mean") and window is None:
        check(_lib.load().spade_grouped_attn(
            _dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(out, "out"), gs, len(schemes), rows, heads, d,
            text_tokens, dtype_code(q.dtype), _dev(workspace, "workspace"), workspace.numel(), _stream(stream)),
            "spade_grouped_attn")
    else:
        check(_lib.load().spade_grouped_attn_ex(
            _dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(out, "out"), gs, len(schemes), rows, heads, d,
            text_tokens, dtype_code(q.dtype), SUMMARY[summary[0]], SUMMARY[summary[1]],
            (ctypes.c_int * (3 * heads))(*[int(r) for t in window for r in t]) if window is not None else None,
            _dev(workspace, "workspace"), workspace.numel(), _stream(stream)), "spade_grouped_attn_ex")
    return out


def grouped_attn_lists(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, schemes, table, workspace: torch.Tensor,
                       text_tokens: int = 0, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Step 5 of a grouped layer under the kept lists an earlier grouped_attn
    call left in `workspace` (same schemes, table, d, text_tokens)."""
    heads, d = q.shape[1], q.shape[2]
    gs, rows = _tables(schemes, table)
    if out is None:
        out = torch.empty_like(q)
    check(_lib.load().spade_grouped_attn_lists(
        _dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(out, "out"), gs, len(schemes), rows, heads, d, text_tokens,
        dtype_code(q.dtype), _dev(workspace, "workspace"), workspace.numel(), _stream(stream)),
        "spade_grouped_attn_lists")
    return out


def grouped_host_workspace_bytes(schemes, table, d: int, text_tokens: int = 0, dtype=torch.bfloat16,
                                 head_chunk: int = 2) -> int:
    gs, rows = _tables(schemes, table)
    return int(_lib.load().spade_grouped_host_workspace_bytes(gs, len(schemes), rows, len(table), d, text_tokens,
                                                              dtype_code(dtype), head_chunk))


def grouped_attn_from_host(qh: torch.Tensor, kh: torch.Tensor, vh: torch.Tensor, out_h: torch.Tensor, schemes,
                           table, text_tokens: int = 0, head_chunk: int = 2,
                           workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """One layer from host memory to host memory (spade_grouped_attn_host):
    qh, kh, vh, out_h are host tensors [N (+text), heads, d], pinned for the
    copies to overlap the compute; the library streams the layer through the
    GPU in groups of head_chunk heads.  workspace: a device uint8 tensor of
    grouped_host_workspace_bytes (allocated here when omitted).  Returns
    out_h once the work is enqueued; it is complete when the current stream
    (or `stream`) is."""
    for t, name in ((qh, "q"), (kh, "k"), (vh, "v"), (out_h, "out")):
        if t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous host tensor")
    heads, d = qh.shape[1], qh.shape[2]
    gs, rows = _tables(schemes, table)
    if workspace is None:
        need = grouped_host_workspace_bytes(schemes, table, d, text_tokens, qh.dtype, head_chunk)
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device="cuda")
    check(_lib.load().spade_grouped_attn_host(
        qh.data_ptr(), kh.data_ptr(), vh.data_ptr(), out_h.data_ptr(), gs, len(schemes), rows, heads, d,
        text_tokens, dtype_code(qh.dtype), head_chunk, _dev(workspace, "workspace"), workspace.numel(),
        _stream(stream)), "spade_grouped_attn_host")
    return out_h


def grouped_head_lists(schemes, table, d: int, text_tokens: int, head: int) -> Tuple[int, int]:
    """Byte offsets of head's (cnt, idx) inside a grouped workspace; (-1, -1) for dense heads."""
    gs, rows = _tables(schemes, table)
    co, io = ctypes.c_int64(), ctypes.c_int64()
    check(_lib.load().spade_grouped_head_lists(gs, len(schemes), rows, len(table), d, text_tokens, head,
                                               ctypes.byref(co), ctypes.byref(io)), "spade_grouped_head_lists")
    return co.value, io.value


def sics_workspace_bytes(candidates, heads: int) -> int:
    gs = (SpadeGeom * len(candidates))(*[geom(c) for c in candidates])
    return int(_lib.load().spade_sics_workspace_bytes(gs, len(candidates), heads))


def sics(q: torch.Tensor, k: torch.Tensor, candidates, workspace: Optional[torch.Tensor] = None,
         stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Scheme generation: per head, the SICS of every candidate blocking
    scheme (Q plus K) and the index of the best one.  Returns (scores
    [heads, n_candidates] float32, choice [heads] int32), both on the device."""
    heads, d = q.shape[1], q.shape[2]
    gs = (SpadeGeom * len(candidates))(*[geom(c) for c in candidates])
    scores = torch.empty(heads, len(candidates), dtype=torch.float32, device=q.device)
    choice = torch.empty(heads, dtype=torch.int32, device=q.device)
    if workspace is None:
        need = int(_lib.load().spade_sics_workspace_bytes(gs, len(candidates), heads))
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    check(_lib.load().spade_sics(_dev(q, "q"), _dev(k, "k"), gs, len(candidates), heads, d, dtype_code(q.dtype),
                                 _dev(scores, "scores"), _dev(choice, "choice"), _dev(workspace, "workspace"),
                                 workspace.numel(), _stream(stream)), "spade_sics")
    return scores, choice


def last_device_status(stream=None) -> int:
    return int(_lib.load().spade_last_device_status(_stream(stream)))


def selftest_bounded_wait(timeout_ns: int, stream=None) -> None:
    check(_lib.load().spade_selftest_bounded_wait(int(timeout_ns), _stream(stream)),
          "spade_selftest_bounded_wait")
