"""Shared helpers for the GPU parity tests: run the library, read back its
masks, and compare with the oracle under the tolerances of the method's
precision (bf16 inputs, fp32 accumulation)."""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle as O
from input_adaptive_block_b200 import api
from spade_workloads import Workload

# tolerances (attention: bf16 I/O, fp32 accumulation; selection: margin rule)
ATTN_MAX_ABS_BF16 = 2e-2
ATTN_MEAN_ABS_BF16 = 2e-3
ATTN_MAX_ABS_F32 = 1e-4
MEAN_REL = 1e-5
PROB_ABS = 1e-5
SCORE_REL = 2e-5      # pooled scores (split-precision TF32), relative to the largest |score|
MARGIN = 1e-3


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu").double().numpy()


def table_of(wl: Workload):
    return [(wl.head_scheme[h], wl.head_tau[h], wl.head_dense[h]) for h in range(wl.heads)]


def run_grouped(wl: Workload, q, k, v):
    """One grouped call; returns (out, workspace, kept(h) -> list of lists or None)."""
    schemes = [s.as_tuple() for s in wl.schemes]
    table = table_of(wl)
    need = api.grouped_workspace_bytes(schemes, table, wl.d, wl.text_tokens)
    ws = torch.zeros(need, dtype=torch.uint8, device=q.device)
    out = api.grouped_attn(q, k, v, schemes, table, wl.text_tokens, workspace=ws)
    torch.cuda.synchronize()
    assert api.last_device_status() == 0

    def kept(h):
        if wl.head_dense[h]:
            return None
        co, io = api.grouped_head_lists(schemes, table, wl.d, wl.text_tokens, h)
        nb = wl.schemes[wl.head_scheme[h]].nb
        cnt = ws[co: co + 4 * nb].view(torch.int32).cpu().numpy()
        idx = ws[io: io + 4 * nb * nb].view(torch.int32).view(nb, nb).cpu().numpy()
        return [list(map(int, idx[i, : cnt[i]])) for i in range(nb)]

    return out, ws, kept


def oracle_selection(wl: Workload, qh: np.ndarray, kh: np.ndarray, h: int):
    """Oracle P, kept lists and per-row margins for head h (fp64 chain);
    qh, kh are that head's [n, 1, d] arrays."""
    geom = wl.schemes[wl.head_scheme[h]].as_tuple()
    N = wl.N
    qm = O.summarize(qh[:N], geom)
    km = O.summarize(kh[:N], geom)
    P = O.estimate(qm, km)[0]
    tau = wl.head_tau[h]
    kept = [O.select_row(P[i], i, tau) for i in range(P.shape[0])]
    margins = np.array([O.selection_margin(P[i], i, tau) for i in range(P.shape[0])])
    return P, kept, margins


def valid_cut(p: np.ndarray, i: int, tau: float, kept, mass_tol: float = 1e-4,
              score_tol: float = 1e-3) -> bool:
    """Property every kept list must have, in the oracle's fp64 probabilities,
    whatever its margin: it contains i, reaches tau (up to mass_tol), is
    minimal (dropping its smallest non-diagonal block falls below tau), and no
    dropped block scores above a kept one by more than score_tol."""
    kept = list(kept)
    nb = len(p)
    if i not in kept:
        return False
    if tau >= 1.0 or len(kept) == nb:
        return len(kept) == nb or float(np.sum(p[kept])) >= tau - mass_tol
    mass = float(np.sum(p[kept]))
    if mass < tau - mass_tol:
        return False
    others = [j for j in kept if j != i]
    if not others:
        return True
    low = min(float(p[j]) for j in others)
    if mass - low >= tau + mass_tol:
        return False
    dropped = np.setdiff1d(np.arange(nb), kept)
    if len(dropped) and low > 0:
        if math.log(float(p[dropped].max()) / low) > score_tol:
            return False
    return True


def compare_kept(gpu_kept, ora_kept, margins, thr=MARGIN, P=None, tau=None):
    """Bit-exact on rows whose oracle margin (score units) exceeds thr; every
    row must be ascending, contain its diagonal and, when the oracle's
    probabilities P are given, pass valid_cut.  Returns
    (checked, mismatched_rows, skipped)."""
    checked, bad, skipped = 0, [], 0
    for i, (g, o) in enumerate(zip(gpu_kept, ora_kept)):
        assert g == sorted(set(g)) and i in g and all(0 <= j < len(gpu_kept) for j in g), (i, g)
        if P is not None:
            assert valid_cut(P[i], i, tau, g), (i, g, o)
        if margins[i] > thr:
            checked += 1
            if g != o:
                bad.append(i)
        else:
            skipped += 1
    return checked, bad, skipped


def attn_errors(gpu: np.ndarray, ref: np.ndarray):
    mask = ~np.isnan(ref)
    diff = np.abs(gpu[mask] - ref[mask])
    return float(diff.max()), float(diff.mean()), int(mask.sum())
