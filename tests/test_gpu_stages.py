"""GPU parity, stage by stage, through the C ABI: tiling (bit-exact), block
means (rel 1e-5), estimator probabilities (abs 1e-5), index search (bit-exact
on rows whose oracle margin exceeds 1e-3), plus the bounded-wait error path."""
import math

import numpy as np
import pytest
import torch

import oracle as O
from input_adaptive_block_b200 import api
from spade_workloads import Scheme, Workload, get_config, make_qkv

from helpers import MARGIN, MEAN_REL, PROB_ABS, SCORE_REL, compare_kept, to_np

pytestmark = pytest.mark.gpu


def _wl(name, T, H, W, heads, d, dtype, block, tau=0.9, text=0):
    return Workload(name, 7, T, H, W, heads, d, dtype, text, (Scheme(T, H, W, *block),),
                    (0,) * heads, (tau,) * heads, (False,) * heads)


RAGGED = [
    _wl("ragged-bf16", 5, 19, 23, 3, 128, "bf16", (2, 8, 8)),
    _wl("ragged-bf16-d64", 3, 9, 30, 2, 64, "bf16", (8, 4, 4)),
    _wl("one-block", 1, 4, 4, 2, 128, "bf16", (2, 8, 8)),
    get_config("tiny"),
]


@pytest.mark.parametrize("wl", RAGGED, ids=lambda w: w.name)
def test_tile3d_bitexact(wl):
    q, _, _ = make_qkv(wl, device="cuda")
    geom = wl.schemes[0].as_tuple()
    xt = api.tile3d(q, geom)
    ref = O.tile3d(to_np(q[: wl.N]), geom)
    assert np.array_equal(to_np(xt), ref)


@pytest.mark.parametrize("wl", RAGGED + [get_config("wan1.3b")], ids=lambda w: w.name)
def test_summarize(wl):
    q, k, _ = make_qkv(wl, device="cuda")
    geom = wl.schemes[0].as_tuple()
    for x in (q, k):
        got = to_np(api.summarize(x, geom))
        ref = O.summarize(to_np(x[: wl.N]), geom)
        err = np.abs(got - ref) / np.maximum(np.abs(ref), 1.0)
        assert err.max() <= MEAN_REL, err.max()


@pytest.mark.parametrize("wl", RAGGED + [get_config("wan1.3b")], ids=lambda w: w.name)
def test_summarize_qk(wl):
    """Q and K in one launch: against the oracle, and bit-identical to the
    one-tensor call (same per-unit arithmetic)."""
    q, k, _ = make_qkv(wl, device="cuda")
    geom = wl.schemes[0].as_tuple()
    qm, km = api.summarize_qk(q, k, geom)
    for x, got in ((q, qm), (k, km)):
        ref = O.summarize(to_np(x[: wl.N]), geom)
        err = np.abs(to_np(got) - ref) / np.maximum(np.abs(ref), 1.0)
        assert err.max() <= MEAN_REL, err.max()
        assert torch.equal(got, api.summarize(x, geom))


@pytest.mark.parametrize("wl", RAGGED + [get_config("wan1.3b")], ids=lambda w: w.name)
def test_estimate(wl):
    q, k, _ = make_qkv(wl, device="cuda")
    geom = wl.schemes[0].as_tuple()
    qm, km = api.summarize(q, geom), api.summarize(k, geom)
    P = api.estimate(qm, km)
    ref = O.estimate(to_np(qm), to_np(km))          # same means: isolates the estimator
    assert np.abs(to_np(P) - ref).max() <= PROB_ABS
    assert np.abs(to_np(P).sum(-1) - 1).max() <= 1e-5


def test_estimate_random_many_blocks():
    """nb spanning several column tiles and a ragged tail, large score range."""
    g = torch.Generator(device="cpu").manual_seed(11)
    qm = (torch.randn(3, 1001, 128, generator=g) * 0.6).cuda()
    km = (torch.randn(3, 1001, 128, generator=g) * 0.6).cuda()
    P = api.estimate(qm, km)
    ref = O.estimate(to_np(qm), to_np(km))
    assert np.abs(to_np(P) - ref).max() <= PROB_ABS


@pytest.mark.parametrize("wl", RAGGED + [get_config("wan1.3b")], ids=lambda w: w.name)
def test_estimate_scores(wl):
    """The scores the grouped path hands to the fused softmax + index search."""
    q, k, _ = make_qkv(wl, device="cuda")
    geom = wl.schemes[0].as_tuple()
    qm, km = api.summarize(q, geom), api.summarize(k, geom)
    S = to_np(api.estimate_scores(qm, km))
    ref = O.pooled_scores(to_np(qm), to_np(km))
    assert S.shape == ref.shape
    assert np.abs(S - ref).max() <= SCORE_REL * max(1.0, np.abs(ref).max())


def test_estimate_scores_random_many_blocks():
    """nb spanning several 128-block tiles with a ragged tail (1001 = 7 x 128 + 105,
    so the last key tile runs a short MMA), d = 64 and 128."""
    g = torch.Generator(device="cpu").manual_seed(12)
    for d in (64, 128):
        qm = (torch.randn(3, 1001, d, generator=g) * 0.6).cuda()
        km = (torch.randn(3, 1001, d, generator=g) * 0.6).cuda()
        S = to_np(api.estimate_scores(qm, km))
        ref = O.pooled_scores(to_np(qm), to_np(km))
        assert np.abs(S - ref).max() <= SCORE_REL * max(1.0, np.abs(ref).max()), d


@pytest.mark.parametrize("nb", [2047, 2048])
def test_estimate_at_the_block_limit(nb):
    """nb at the estimator's limit (2048: 16 key tiles per row, the widest
    row-softmax variant) and one below it (ragged last tile, rows not
    16-byte aligned)."""
    g = torch.Generator(device="cpu").manual_seed(nb)
    qm = (torch.randn(2, nb, 64, generator=g) * 0.6).cuda()
    km = (torch.randn(2, nb, 64, generator=g) * 0.6).cuda()
    S = to_np(api.estimate_scores(qm, km))
    ref = O.pooled_scores(to_np(qm), to_np(km))
    assert np.abs(S - ref).max() <= SCORE_REL * max(1.0, np.abs(ref).max())
    P = to_np(api.estimate(qm, km))
    assert np.abs(P - O.softmax_rows(ref)).max() <= PROB_ABS
    assert np.abs(P.sum(-1) - 1).max() <= 1e-5


@pytest.mark.parametrize("wl", RAGGED + [get_config("wan1.3b")], ids=lambda w: w.name)
def test_select_scores_against_oracle_chain(wl):
    """The grouped path's steps 3-4 (scores, then the softmax fused into the
    index search) against the oracle's fp64 chain."""
    q, k, _ = make_qkv(wl, device="cuda")
    geom = wl.schemes[0].as_tuple()
    S = api.estimate_scores(api.summarize(q, geom), api.summarize(k, geom))
    cnt, idx = api.select_scores(S, wl.head_tau)
    cnt, idx = cnt.cpu().numpy(), idx.cpu().numpy()
    Pref = O.estimate(O.summarize(to_np(q[: wl.N]), geom), O.summarize(to_np(k[: wl.N]), geom))
    total_checked = 0
    for h in range(wl.heads):
        nb = Pref.shape[1]
        gk = [list(idx[h, i, : cnt[h, i]]) for i in range(nb)]
        ok = [O.select_row(Pref[h, i], i, wl.head_tau[h]) for i in range(nb)]
        mg = [O.selection_margin(Pref[h, i], i, wl.head_tau[h]) for i in range(nb)]
        checked, bad, _ = compare_kept(gk, ok, mg, P=Pref[h], tau=wl.head_tau[h])
        assert not bad, (h, bad[:5])
        total_checked += checked
    assert total_checked >= 0.5 * wl.heads * Pref.shape[1]


@pytest.mark.parametrize("wl", RAGGED + [get_config("wan1.3b")], ids=lambda w: w.name)
def test_select_against_oracle_chain(wl):
    """GPU select on the GPU probabilities vs the oracle's fp64 chain."""
    q, k, _ = make_qkv(wl, device="cuda")
    geom = wl.schemes[0].as_tuple()
    P = api.estimate(api.summarize(q, geom), api.summarize(k, geom))
    cnt, idx = api.select(P, wl.head_tau)
    cnt, idx = cnt.cpu().numpy(), idx.cpu().numpy()
    qn, kn = to_np(q[: wl.N]), to_np(k[: wl.N])
    Pref = O.estimate(O.summarize(qn, geom), O.summarize(kn, geom))
    total_checked = 0
    for h in range(wl.heads):
        nb = Pref.shape[1]
        gk = [list(idx[h, i, : cnt[h, i]]) for i in range(nb)]
        ok = [O.select_row(Pref[h, i], i, wl.head_tau[h]) for i in range(nb)]
        mg = [O.selection_margin(Pref[h, i], i, wl.head_tau[h]) for i in range(nb)]
        checked, bad, _ = compare_kept(gk, ok, mg, P=Pref[h], tau=wl.head_tau[h])
        assert not bad, (h, bad[:5])
        total_checked += checked
    assert total_checked >= 0.5 * wl.heads * Pref.shape[1]


_ROWS = ([(nb, tau, "prob") for nb in (5, 33, 100, 630, 660, 1020, 1024) for tau in (0.3, 0.8, 0.9, 0.95, 0.999, 1.0)]
         + [(nb, tau, "scores") for nb in (5, 33, 630, 1024) for tau in (0.3, 0.9, 0.999, 1.0)])


@pytest.mark.parametrize("nb,tau,mode", _ROWS)
def test_select_random_rows(nb, tau, mode):
    """Synthetic rows with peaked and flat regions, exact ties (uniform rows)
    and tau = 1, given as probabilities (the oracle runs on the same fp32
    values) or as scores (the oracle runs on their fp64 softmax); nb = 630 is
    a row length that is not a multiple of 4 (unaligned rows)."""
    g = torch.Generator(device="cpu").manual_seed(nb * 7 + int(tau * 1000))
    heads = 3
    logits = torch.randn(heads, nb, nb, generator=g, dtype=torch.float64) * torch.tensor([0.5, 2.0, 0.0]).view(3, 1, 1).double()
    if mode == "prob":
        P = torch.softmax(logits, dim=-1).float()
        cnt, idx = api.select(P.cuda(), [tau] * heads)
        Pn = P.double().numpy()
    else:
        S = logits.float()
        cnt, idx = api.select_scores(S.cuda(), [tau] * heads)
        Pn = O.softmax_rows(S.double().numpy())
    cnt, idx = cnt.cpu().numpy(), idx.cpu().numpy()
    for h in range(heads):
        gk = [list(idx[h, i, : cnt[h, i]]) for i in range(nb)]
        ok = [O.select_row(Pn[h, i], i, tau) for i in range(nb)]
        mg = [O.selection_margin(Pn[h, i], i, tau) for i in range(nb)]
        if h == 2:   # uniform rows: every off-diagonal block ties, so the lowest ids must win;
            for i in range(nb):   # the count may differ by one where fp32 and fp64 sums straddle tau
                others = [j for j in range(nb) if j != i]
                assert gk[i] == sorted([i] + others[: int(cnt[h, i]) - 1]), i
                assert abs(int(cnt[h, i]) - len(ok[i])) <= 1, i
            continue
        _, bad, _ = compare_kept(gk, ok, mg, P=Pn[h], tau=tau)
        assert not bad, (h, bad[:5])


def test_bounded_wait_reports_timeout():
    assert api.last_device_status() == 0
    api.selftest_bounded_wait(50_000_000)            # 50 ms; nothing ever arrives
    assert api.last_device_status() == 4             # SPADE_ERR_TIMEOUT, read once
    assert api.last_device_status() == 0             # and cleared
    x = torch.ones(4, device="cuda")
    assert float((x + 1).sum()) == 8.0               # the context is still usable


def _geometric_row(rng, nb, n, total=1.0, skip=()):
    """n well-separated values total * 2^-(k+1) (k = 0..n-1, renormalised to
    `total`) at random positions outside `skip`; zeros elsewhere."""
    row = np.zeros(nb, np.float64)
    cols = [j for j in rng.permutation(nb) if j not in set(skip)][:n]
    vals = 0.5 ** (np.arange(n) + 1)
    row[cols] = vals / vals.sum() * total
    return row


@pytest.mark.parametrize("nb", [40, 660])
def test_select_degenerate_rows(nb):
    """Rows the index search must handle besides softmax output: exact zeros,
    a diagonal that alone reaches tau, a row summing to more than 1 (masses
    scaled per row), NaN / negative / above-1 entries (clamped to [0, 1], NaN
    counted as 0), an all-zero row (the mass never reaches tau: every block
    kept), and with a tiny tau a zero diagonal (one more block needed) and a
    non-zero one (the diagonal alone).  Values are powers of two far from the
    cut, so the oracle on the clamped row gives the one correct answer."""
    rng = np.random.default_rng(nb)
    P = np.stack([np.stack([_geometric_row(rng, nb, 30) for _ in range(nb)]) for _ in range(2)])
    special = {}
    # head 0, tau = 0.9
    special[(0, 0)] = _geometric_row(rng, nb, 20, skip=(0,))                  # zero diagonal, zeros elsewhere
    r = _geometric_row(rng, nb, 12, total=0.05, skip=(1,)); r[1] = 0.95
    special[(0, 1)] = r                                                        # the diagonal alone reaches tau
    special[(0, 2)] = _geometric_row(rng, nb, 16, total=1.7)                   # sums to 1.7
    r = _geometric_row(rng, nb, 16)
    others = [j for j in range(nb) if r[j] == 0 and j != 3]
    r[others[:3]] = np.nan
    r[others[3:6]] = -0.5
    special[(0, 3)] = r                                                        # NaN and negative entries
    r = _geometric_row(rng, nb, 16, total=0.3, skip=(4,))
    r[[j for j in range(nb) if r[j] == 0 and j != 4][0]] = 3.0
    special[(0, 4)] = r                                                        # an entry above 1
    special[(0, 5)] = np.zeros(nb)                                             # all zero
    # head 1, tau = 1e-6
    special[(1, 0)] = _geometric_row(rng, nb, 20, skip=(0,))                  # zero diagonal
    r = _geometric_row(rng, nb, 20, skip=(1,)); r[1] = 1e-3
    special[(1, 1)] = r                                                        # small non-zero diagonal
    for (h, i), row in special.items():
        P[h, i] = row
    taus = [0.9, 1e-6]
    cnt, idx = api.select(torch.tensor(P, dtype=torch.float32).cuda(), taus)
    cnt, idx = cnt.cpu().numpy(), idx.cpu().numpy()
    for (h, i), row in special.items():
        clamped = np.clip(np.nan_to_num(row.astype(np.float32).astype(np.float64), nan=0.0), 0.0, 1.0)
        want = O.select_row(clamped, i, taus[h])
        got = list(map(int, idx[h, i, : cnt[h, i]]))
        assert got == want, (h, i, got, want)
    assert cnt[0, 5] == nb and cnt[0, 1] == 1 and cnt[1, 1] == 1 and cnt[1, 0] == 2
    # every other row: ascending, diagonal present, ids in range
    for h in range(2):
        for i in range(nb):
            g = list(idx[h, i, : cnt[h, i]])
            assert g == sorted(set(g)) and i in g and all(0 <= j < nb for j in g)
