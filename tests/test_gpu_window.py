"""Static windows merged with dynamic selection on the GPU (spade_select_window
and the grouped launch's window radii) against the oracle."""
import numpy as np
import pytest
import torch

import oracle as O
from input_adaptive_block_b200 import api
from spade_workloads import Scheme, Workload, make_qkv

from helpers import ATTN_MAX_ABS_BF16, ATTN_MEAN_ABS_BF16, MARGIN, attn_errors, table_of, to_np

pytestmark = pytest.mark.gpu


def _wl(T, H, W, heads, tau, cid=41):
    return Workload("window", cid, T, H, W, heads, 128, "bf16", 0, (Scheme(T, H, W, 2, 8, 8),),
                    (0,) * heads, (tau,) * heads, (False,) * heads)


def _window_cut_ok(p, win, tau, kept, mass_tol=1e-4):
    """Window kept, tau reached, and minimal: dropping the smallest
    non-window kept block falls below tau (in the oracle's probabilities)."""
    kept = list(kept)
    if not set(win) <= set(kept) or kept != sorted(set(kept)):
        return False
    if tau >= 1.0 or len(kept) == len(p):
        return True
    mass = float(p[kept].sum())
    if mass < tau - mass_tol:
        return False
    extra = [j for j in kept if j not in set(win)]
    if not extra:
        return True
    smallest = min(extra, key=lambda j: p[j])
    return mass - float(p[smallest]) < tau + mass_tol


def _oracle_P(q, k, g, h):
    qm = O.summarize(to_np(q)[:, h: h + 1], g)
    km = O.summarize(to_np(k)[:, h: h + 1], g)
    return O.estimate(qm, km)[0]


def test_radius_zero_equals_select():
    wl = _wl(6, 20, 28, 3, 0.9)
    q, k, _ = make_qkv(wl, device="cuda")
    g = wl.schemes[0].as_tuple()
    P = api.estimate(api.summarize(q, g), api.summarize(k, g))
    c0, i0 = api.select(P, wl.head_tau)
    c1, i1 = api.select_window(P, wl.head_tau, (0, 0, 0), g)
    torch.cuda.synchronize()
    assert torch.equal(c0, c1)
    nb = wl.schemes[0].nb
    for h in range(wl.heads):
        for r in range(nb):
            n = int(c0[h, r])
            assert torch.equal(i0[h, r, :n], i1[h, r, :n])


@pytest.mark.parametrize("radius,tau", [((0, 1, 1), 0.9), ((1, 0, 0), 0.8), ((1, 1, 1), 0.95)])
def test_select_window_against_oracle(radius, tau):
    wl = _wl(6, 20, 28, 2, tau, cid=42)
    q, k, _ = make_qkv(wl, device="cuda")
    g = wl.schemes[0].as_tuple()
    nb = wl.schemes[0].nb
    P = api.estimate(api.summarize(q, g), api.summarize(k, g))
    cnt, idx = api.select_window(P, wl.head_tau, radius, g)
    torch.cuda.synchronize()
    checked = 0
    for h in range(wl.heads):
        Po = _oracle_P(q, k, g, h)
        for i in range(nb):
            win = O.window_blocks(g, i, radius)
            got = list(map(int, idx[h, i, : int(cnt[h, i])].cpu()))
            assert _window_cut_ok(Po[i], win, tau, got), (h, i, got)
            if O.selection_margin(Po[i], i, tau, win) > MARGIN:
                checked += 1
                assert got == O.select_row(Po[i], i, tau, win), (h, i)
    assert checked > 0


def test_grouped_layer_with_windows():
    wl = _wl(6, 20, 28, 3, 0.85, cid=43)
    q, k, v = make_qkv(wl, device="cuda")
    schemes = [s.as_tuple() for s in wl.schemes]
    table = table_of(wl)
    radii = [(0, 0, 0), (0, 1, 1), (1, 1, 1)]
    ws = torch.zeros(api.grouped_workspace_bytes(schemes, table, wl.d, 0), dtype=torch.uint8, device="cuda")
    out = api.grouped_attn(q, k, v, schemes, table, 0, workspace=ws, window=radii)
    torch.cuda.synchronize()
    assert api.last_device_status() == 0
    g = schemes[0]
    nb = wl.schemes[0].nb
    kept = []
    for h in range(wl.heads):
        co, io = api.grouped_head_lists(schemes, table, wl.d, 0, h)
        cnt = ws[co: co + 4 * nb].view(torch.int32).cpu().numpy()
        idx = ws[io: io + 4 * nb * nb].view(torch.int32).view(nb, nb).cpu().numpy()
        kh = [list(map(int, idx[i, : cnt[i]])) for i in range(nb)]
        kept.append(kh)
        Po = _oracle_P(q, k, g, h)
        for i in range(nb):
            win = O.window_blocks(g, i, radii[h])
            assert _window_cut_ok(Po[i], win, wl.head_tau[h], kh[i]), (h, i)
            if O.selection_margin(Po[i], i, wl.head_tau[h], win) > MARGIN:
                assert kh[i] == O.select_row(Po[i], i, wl.head_tau[h], win), (h, i)
    ref = O.block_sparse_attention(to_np(q), to_np(k), to_np(v), [g] * wl.heads, kept, 0)
    mx, mean, n = attn_errors(to_np(out), ref)
    assert n == wl.N * wl.heads * wl.d
    assert mx <= ATTN_MAX_ABS_BF16 and mean <= ATTN_MEAN_ABS_BF16, (mx, mean)
