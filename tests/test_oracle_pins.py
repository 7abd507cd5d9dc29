"""Pins for the CPU oracle: hand-worked fixtures, closed forms, brute force and
library special cases.  None of these re-derive a value through the oracle's
own code path; each would fail on a plausible slip in it (a swapped raster
order, a mean over the padded size, a strict '>' at the cut, a missing
diagonal, a missing 1/sqrt(d), a transposed operand, an unmasked padded key).
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle as O
from spade_workloads import Scheme, get_config, make_qkv


def _load(golden_dir, name):
    with open(os.path.join(golden_dir, name)) as f:
        return json.load(f)


# ----------------------------------------------------------------- tiling ---

def test_tile_hand_fixture(golden_dir):
    g = _load(golden_dir, "tile_2x3x3_b1x2x2.json")
    geom = tuple(g["geom"])
    blocks = O.block_tokens(*geom)
    assert len(blocks) == g["nb"]
    for b, (toks, slots) in enumerate(blocks):
        expect = g["slots"][b]
        got = [-1] * len(expect)
        for t, s in zip(toks, slots):
            got[s] = int(t)
        assert got == expect, f"block {b}"
    assert list(O.valid_counts(geom)) == g["valid_counts"]
    # tile3d places token values at those slots and zero elsewhere
    x = np.arange(18, dtype=np.float64).reshape(18, 1, 1) + 1.0
    xt = O.tile3d(x, geom)
    for b, expect in enumerate(g["slots"]):
        assert list(xt[0, b, :, 0]) == [float(e + 1) if e >= 0 else 0.0 for e in expect]


@pytest.mark.parametrize("geom", [(4, 8, 8, 2, 4, 4), (3, 5, 7, 2, 4, 4), (21, 30, 52, 2, 8, 8),
                                  (5, 9, 11, 8, 4, 4), (1, 1, 300, 1, 1, 128)])
def test_tile_bijection_and_counts(geom):
    T, H, W, bt, bh, bw = geom
    blocks = O.block_tokens(*geom)
    allt = np.concatenate([t for t, _ in blocks])
    assert sorted(allt.tolist()) == list(range(T * H * W))           # each token exactly once
    # valid count = product of clipped extents, computed from integer division
    n = np.arange(T * H * W)
    t, y, x = n // (H * W), (n // W) % H, n % W
    bid = ((t // bt) * (-(-H // bh)) + (y // bh)) * (-(-W // bw)) + (x // bw)
    assert (np.bincount(bid, minlength=len(blocks)) == O.valid_counts(geom)).all()
    for b, (toks, _) in enumerate(blocks):
        assert (bid[toks] == b).all()
    rng = np.random.default_rng(1)
    xx = rng.standard_normal((T * H * W, 2, 3))
    assert np.array_equal(O.untile3d(O.tile3d(xx, geom), geom), xx)  # round trip


# -------------------------------------------------------------- summarize ---

@pytest.mark.parametrize("geom", [(3, 5, 7, 2, 4, 4), (21, 30, 52, 2, 8, 8), (5, 9, 11, 8, 4, 4)])
def test_summarize_closed_forms(geom):
    T, H, W, bt, bh, bw = geom
    N = T * H * W
    n = np.arange(N)
    t, y, x = n // (H * W), (n // W) % H, n % W
    # channels: constant 3.5, t, y, x  -> means: 3.5 and the midpoints of the clipped ranges
    xx = np.stack([np.full(N, 3.5), t, y, x], axis=1).reshape(N, 1, 4).astype(np.float64)
    m = O.summarize(xx, geom)
    nbh, nbw = -(-H // bh), -(-W // bw)
    for b in range(m.shape[1]):
        bi, bj, bk = b // (nbh * nbw), (b // nbw) % nbh, b % nbw
        mid = lambda i, s, E: (i * s + min(E, (i + 1) * s) - 1) / 2.0
        assert m[0, b, 0] == pytest.approx(3.5, abs=1e-14)
        assert m[0, b, 1] == pytest.approx(mid(bi, bt, T), abs=1e-12)
        assert m[0, b, 2] == pytest.approx(mid(bj, bh, H), abs=1e-12)
        assert m[0, b, 3] == pytest.approx(mid(bk, bw, W), abs=1e-12)


# --------------------------------------------------------------- estimate ---

def test_estimate_closed_forms():
    e = math.e
    # S = Qbar.Kbar/sqrt(4): row 0 -> [1, 0], row 1 -> [0, 0]
    qm = np.array([[[2, 0, 0, 0], [0, 0, 2, 0]]], dtype=np.float64)
    km = np.array([[[1, 0, 0, 0], [0, 0, 0, 0]]], dtype=np.float64)
    P = O.estimate(qm, km)
    assert P[0, 0, 0] == pytest.approx(e / (e + 1), abs=1e-15)      # sigmoid(1)
    assert P[0, 0, 1] == pytest.approx(1 / (e + 1), abs=1e-15)
    assert P[0, 1] == pytest.approx([0.5, 0.5], abs=1e-15)
    # three key blocks: S = [1, 1, 0]
    qm = np.array([[[1, 1, 1, 1]]], dtype=np.float64)
    km = np.array([[[2, 0, 0, 0], [0, 2, 0, 0], [0, 0, 0, 0]]], dtype=np.float64)
    P = O.estimate(qm, km)
    assert P[0, 0] == pytest.approx([e / (2 * e + 1), e / (2 * e + 1), 1 / (2 * e + 1)], abs=1e-15)
    # a non-symmetric case catches a transposed product: S[i,j] uses Q row i, K row j
    qm = np.array([[[2, 0], [0, 0]]], dtype=np.float64)
    km = np.array([[[0, 0], [math.sqrt(2) * math.log(3), 0]]], dtype=np.float64)
    P = O.estimate(qm, km)
    # row 0: S = [0, 2*sqrt2*ln3/sqrt2] = [0, 2 ln 3] -> [1/10, 9/10];  row 1: uniform
    assert P[0, 0] == pytest.approx([0.1, 0.9], abs=1e-14)
    assert P[0, 1] == pytest.approx([0.5, 0.5], abs=1e-15)


def test_pooled_scores_hand_worked():
    # d = 4, sqrt(d) = 2.  Q rows (1,2,0,0), (0,0,1,1); K rows (1,0,0,0), (0,1,1,0):
    # q0.k0 = 1, q0.k1 = 2, q1.k0 = 0, q1.k1 = 1  ->  S = [[0.5, 1.0], [0.0, 0.5]]
    qm = np.array([[[1, 2, 0, 0], [0, 0, 1, 1]]], dtype=np.float64)
    km = np.array([[[1, 0, 0, 0], [0, 1, 1, 0]]], dtype=np.float64)
    S = O.pooled_scores(qm, km)
    assert S.shape == (1, 2, 2)
    assert np.array_equal(S[0], np.array([[0.5, 1.0], [0.0, 0.5]]))
    # two heads are independent: the second head's scores do not mix with the first's
    qm2 = np.concatenate([qm, 3 * qm])
    km2 = np.concatenate([km, km])
    assert np.array_equal(O.pooled_scores(qm2, km2)[1], 3 * S[0])
    # the estimator is exactly the row softmax of these scores: S row 0 -> [e^0.5, e^1] / sum
    P = O.estimate(qm, km)
    e0, e1 = math.exp(0.5), math.exp(1.0)
    assert P[0, 0] == pytest.approx([e0 / (e0 + e1), e1 / (e0 + e1)], abs=1e-15)


def test_estimate_rows_sum_to_one_and_uniform_rank1():
    rng = np.random.default_rng(3)
    P = O.estimate(rng.standard_normal((3, 17, 64)) * 4, rng.standard_normal((3, 17, 64)) * 4)
    assert np.abs(P.sum(-1) - 1).max() <= 1e-12
    assert (P >= 0).all()
    c = rng.standard_normal(64)
    P = O.estimate(np.tile(c, (1, 9, 1)), np.tile(c, (1, 9, 1)))
    assert np.abs(P - 1 / 9).max() <= 1e-15


# ----------------------------------------------------------------- select ---

def test_select_hand_fixture(golden_dir):
    g = _load(golden_dir, "select_hand.json")
    for r in g["rows"]:
        p = np.array(r["p"])
        assert O.select_row(p, r["i"], r["tau"]) == r["kept"], r
        m = O.selection_margin(p, r["i"], r["tau"])
        if r["margin"] is None:
            assert m == math.inf
        else:
            assert m == pytest.approx(r["margin"], abs=1e-12), r


def _brute_force(p, i, tau):
    """Smallest set containing i with mass >= tau; ties -> larger mass, then
    lexicographically smaller ids.  Plain enumeration of every subset."""
    nb = len(p)
    if tau >= 1.0:
        return list(range(nb))
    others = [j for j in range(nb) if j != i]
    for size in range(0, nb):
        best = None
        for comb in itertools.combinations(others, size):
            s = sorted(comb + (i,))
            mass = math.fsum(p[j] for j in s)
            if mass >= tau:
                key = (-mass, s)
                if best is None or key < best[0]:
                    best = (key, s)
        if best is not None:
            return best[1]
    return list(range(nb))


def test_select_matches_brute_force():
    rng = np.random.default_rng(7)
    checked = 0
    for trial in range(300):
        nb = int(rng.integers(2, 11))
        logits = rng.standard_normal(nb) * rng.uniform(0.3, 3.0)
        p = np.exp(logits) / np.exp(logits).sum()
        i = int(rng.integers(0, nb))
        tau = float(rng.choice([0.5, 0.8, 0.85, 0.9, 0.95, 0.99, 1.0, rng.uniform(0.05, 1.0)]))
        if O.selection_margin(p, i, tau) < 1e-9:      # exact ties at the cut: rounding decides
            continue
        assert O.select_row(p, i, tau) == _brute_force(p, i, tau), (p, i, tau)
        checked += 1
    assert checked > 250


def test_select_tiny_config_brute_force_and_invariants():
    wl = get_config("tiny")
    q, k, _ = make_qkv(wl)
    geom = wl.schemes[0].as_tuple()
    P = O.estimate(O.summarize(q.double().numpy(), geom), O.summarize(k.double().numpy(), geom))
    for h in range(wl.heads):
        for i in range(P.shape[1]):
            prev = None
            for tau in (0.3, 0.5, 0.8, 0.9, 0.95, 1.0):
                kept = O.select_row(P[h, i], i, tau)
                assert i in kept and kept == sorted(set(kept))
                assert kept == _brute_force(P[h, i], i, tau)
                if prev is not None:
                    assert set(prev) <= set(kept)           # monotone in tau
                prev = kept
            assert O.select_row(P[h, i], i, 1.0) == list(range(P.shape[1]))
    cnt, idx = O.select(P, [0.8] * wl.heads)
    assert (cnt >= 1).all()
    for h in range(wl.heads):
        for i in range(P.shape[1]):
            assert i in idx[h, i, : cnt[h, i]]
            assert (idx[h, i, cnt[h, i]:] == -1).all()


# -------------------------------------------------------------- attention ---

def _token_block_ids(geom):
    T, H, W, bt, bh, bw = geom
    n = np.arange(T * H * W)
    t, y, x = n // (H * W), (n // W) % H, n % W
    return ((t // bt) * (-(-H // bh)) + (y // bh)) * (-(-W // bw)) + (x // bw)


def _sdpa(q, k, v, mask=None):
    """torch's scaled_dot_product_attention in fp64 per head; mask[n_q, n_k] bool."""
    out = np.empty_like(q, dtype=np.float64)
    for h in range(q.shape[1]):
        qq = torch.from_numpy(q[:, h]).double()[None]
        kk = torch.from_numpy(k[:, h]).double()[None]
        vv = torch.from_numpy(v[:, h]).double()[None]
        m = None if mask is None else torch.from_numpy(mask[h] if mask.ndim == 3 else mask)[None]
        out[:, h] = torch.nn.functional.scaled_dot_product_attention(qq, kk, vv, attn_mask=m)[0].numpy()
    return out


def _small_case(seed=0, geom=(3, 5, 7, 2, 4, 4), heads=2, d=16, text=0):
    rng = np.random.default_rng(seed)
    n = geom[0] * geom[1] * geom[2] + text
    return [rng.standard_normal((n, heads, d)) * s for s in (1.0, 1.0, 1.0)]


def test_attention_tau1_equals_dense_sdpa():
    geom = (3, 5, 7, 2, 4, 4)
    q, k, v = _small_case()
    res = O.pipeline(q, k, v, [geom], [0, 0], [1.0, 1.0], [False, False])
    assert np.abs(res["out"] - _sdpa(q, k, v)).max() <= 1e-12
    assert np.abs(O.dense_attention(q, k, v) - _sdpa(q, k, v)).max() <= 1e-12


def test_attention_arbitrary_mask_matches_masked_sdpa():
    """Random kept lists (diagonal included) with ragged edge blocks and text
    tokens: equals SDPA under the token mask built from integer block ids."""
    geom = (3, 5, 7, 2, 4, 4)
    text = 5
    q, k, v = _small_case(seed=4, text=text)
    N = 3 * 5 * 7
    bid = _token_block_ids(geom)
    nb = int(bid.max()) + 1
    rng = np.random.default_rng(5)
    kept = []
    mask = np.zeros((2, N + text, N + text), dtype=bool)
    for h in range(2):
        kh = []
        for i in range(nb):
            s = sorted(set([i] + [int(j) for j in rng.choice(nb, size=int(rng.integers(0, nb)), replace=False)]))
            kh.append(s)
            rows = np.nonzero(bid == i)[0]
            cols = np.nonzero(np.isin(bid, s))[0]
            mask[h][np.ix_(rows, cols)] = True
            mask[h][np.ix_(rows, np.arange(N, N + text))] = True
        mask[h][N:, :] = True                                   # text rows are dense
        kept.append(kh)
    out = O.block_sparse_attention(q, k, v, [geom, geom], kept, text_tokens=text)
    assert np.abs(out - _sdpa(q, k, v, mask)).max() <= 1e-12


def test_attention_block_local_and_onehot_v():
    geom = (2, 4, 4, 1, 2, 2)
    q, k, v = _small_case(seed=2, geom=geom, heads=1, d=8)
    N = 32
    bid = _token_block_ids(geom)
    nb = int(bid.max()) + 1
    kept = [[[i] for i in range(nb)]]
    out = O.block_sparse_attention(q, k, v, [geom], kept)
    mask = bid[:, None] == bid[None, :]
    assert np.abs(out - _sdpa(q, k, v, mask)).max() <= 1e-12
    # V = one-hot rows over keys: the output rows are the softmax weights
    v1 = np.eye(N).reshape(N, 1, N)
    q1 = q[:, :, :8]
    k1 = k[:, :, :8]
    qq = np.concatenate([q1, np.zeros((N, 1, N - 8))], axis=2)
    kk = np.concatenate([k1, np.zeros((N, 1, N - 8))], axis=2)
    out = O.block_sparse_attention(qq, kk, v1, [geom], [[list(range(nb))] * nb])
    s = (q1[:, 0] @ k1[:, 0].T) / math.sqrt(N)
    w = torch.softmax(torch.from_numpy(s), dim=1).numpy()
    assert np.abs(out[:, 0] - w).max() <= 1e-14


def test_attention_scale_pin():
    """Two keys with scores 0 and ln(3)*sqrt(d) / sqrt(d) = ln 3 after scaling:
    weights 1/4, 3/4 exactly; catches a missing or wrong 1/sqrt(d)."""
    d = 4
    q = np.zeros((2, 1, d)); q[:, 0, 0] = 1.0
    k = np.zeros((2, 1, d)); k[1, 0, 0] = math.log(3) * math.sqrt(d)
    v = np.zeros((2, 1, d)); v[0, 0, 1] = 1.0; v[1, 0, 2] = 1.0
    out = O.block_sparse_attention(q, k, v, [(1, 1, 2, 1, 1, 2)], [[[0]]])
    assert out[0, 0, 1] == pytest.approx(0.25, abs=1e-15)
    assert out[0, 0, 2] == pytest.approx(0.75, abs=1e-15)


def test_kept_token_pairs_counts():
    geom = (3, 5, 7, 2, 4, 4)
    vc = O.valid_counts(geom)
    nb = len(vc)
    kept = [[[i] for i in range(nb)]]
    assert O.kept_token_pairs([geom], kept) == int((vc ** 2).sum())
    assert O.kept_token_pairs([geom], [None]) == int(vc.sum()) ** 2
    assert O.kept_token_pairs([geom], [None], text_tokens=3) == (int(vc.sum()) + 3) ** 2


# ------------------------------------------------ planted mistakes fail ---

def test_planted_mistakes_are_caught(golden_dir, monkeypatch):
    """Each variant below is a plausible slip; a pin above must reject it."""
    g = _load(golden_dir, "select_hand.json")

    def strict_cut(p, i, tau):                  # '>' instead of '>='
        if tau >= 1.0:
            return list(range(len(p)))
        kept, mass = [i], p[i]
        for j in sorted((j for j in range(len(p)) if j != i), key=lambda j: (-p[j], j)):
            if mass > tau:
                break
            kept.append(j); mass += p[j]
        return sorted(kept)

    def topset_union_diag(p, i, tau):           # top-mass set first, diagonal added after
        kept, mass = [], 0.0
        for j in sorted(range(len(p)), key=lambda j: (-p[j], j)):
            if mass >= tau:
                break
            kept.append(j); mass += p[j]
        return sorted(set(kept) | {i})

    for bad in (strict_cut, topset_union_diag):
        assert any(bad(np.array(r["p"]), r["i"], r["tau"]) != r["kept"] for r in g["rows"]), bad

    # a mean over the padded box size instead of the valid count
    geom = (3, 5, 7, 2, 4, 4)
    xx = np.ones((105, 1, 1))
    blocks = O.block_tokens(*geom)
    padded_mean = np.array([len(t) / 32.0 for t, _ in blocks])
    assert not np.allclose(padded_mean, O.summarize(xx, geom)[0, :, 0])


# ---- Summarizer variants (max / min reduces) ----

def test_summarize_max_min_properties():
    """max/min are attained by a valid token of the block, bound every valid
    token and bracket the mean; padding never takes part (an all-negative
    ragged input would show a padded zero as the max)."""
    rng = np.random.default_rng(11)
    geom = (3, 5, 7, 2, 4, 4)                       # ragged in every dimension
    x = -np.abs(rng.standard_normal((3 * 5 * 7, 2, 6))) - 0.1
    mx, mn, me = (O.summarize(x, geom, m) for m in ("max", "min", "mean"))
    for b, (toks, _) in enumerate(O.block_tokens(*geom)):
        xb = x[toks]                                  # [n, heads, d]
        for h in range(2):
            for c in range(6):
                col = xb[:, h, c]
                assert mx[h, b, c] in set(col.tolist()) and mn[h, b, c] in set(col.tolist())
                assert (col <= mx[h, b, c]).all() and (col >= mn[h, b, c]).all()
                assert mn[h, b, c] <= me[h, b, c] <= mx[h, b, c]
    assert (mx < 0).all()


def test_summarize_modes_agree_on_constant_blocks():
    geom = (4, 4, 4, 2, 2, 2)
    vals = np.arange(8, dtype=np.float64)
    x = np.zeros((64, 1, 3))
    for b, (toks, _) in enumerate(O.block_tokens(*geom)):
        x[toks] = vals[b]
    for m in ("mean", "max", "min"):
        assert np.allclose(O.summarize(x, geom, m)[0, :, 0], vals)


# ---- static windows merged with dynamic selection ----

def test_window_blocks_by_coordinates():
    geom = (5, 9, 10, 2, 4, 4)                       # 3 x 3 x 3 blocks
    assert O.window_blocks(geom, 13, (0, 0, 0)) == [13]
    assert O.window_blocks(geom, 13, (1, 1, 1)) == list(range(27))   # the centre block's neighbourhood is all
    assert O.window_blocks(geom, 0, (0, 0, 1)) == [0, 1]
    assert O.window_blocks(geom, 0, (1, 0, 0)) == [0, 9]
    assert O.window_blocks(geom, 26, (0, 1, 1)) == [22, 23, 25, 26]


def test_select_with_radius_zero_window_is_the_diagonal_rule():
    rng = np.random.default_rng(12)
    geom = (4, 8, 8, 2, 4, 4)
    for _ in range(20):
        p = rng.dirichlet(np.full(8, 0.4))
        i = int(rng.integers(0, 8))
        tau = float(rng.uniform(0.3, 0.99))
        assert O.select_row(p, i, tau, O.window_blocks(geom, i, (0, 0, 0))) == O.select_row(p, i, tau)


def test_select_with_window_brute_force():
    """The kept set is the smallest superset of the window whose mass reaches
    tau, ties broken toward the larger mass then the lexicographically
    smaller ids -- checked by enumerating every superset."""
    import itertools
    rng = np.random.default_rng(13)
    geom = (4, 8, 8, 2, 4, 4)                        # 8 blocks
    for _ in range(30):
        p = rng.dirichlet(np.full(8, 0.5))
        i = int(rng.integers(0, 8))
        win = O.window_blocks(geom, i, (0, 1, 0))
        tau = float(rng.uniform(0.3, 0.98))
        got = O.select_row(p, i, tau, win)
        rest = [j for j in range(8) if j not in win]
        best = None
        for r in range(len(rest) + 1):
            for extra in itertools.combinations(rest, r):
                s = sorted(win + list(extra))
                m = float(p[s].sum())
                if m >= tau or len(s) == 8:
                    key = (len(s), -m, s)
                    best = key if best is None or key < best else best
            if best is not None:
                break
        assert got == best[2], (p, i, tau, got, best)
        assert set(win) <= set(got)
