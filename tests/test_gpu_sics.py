"""Scheme generation on the GPU (spade_sics) against the oracle's pairwise
definition of the Sum of Intra-block Cosine Similarities."""
import numpy as np
import pytest
import torch

import oracle as O
from input_adaptive_block_b200 import api
from spade_workloads import Scheme, Workload, make_qkv

from helpers import to_np

pytestmark = pytest.mark.gpu

SCORE_REL = 1e-4      # fp32 sums of ~128 unit vectors vs fp64


def _wl(T, H, W, heads, d, dtype, cid=21):
    return Workload("sics", cid, T, H, W, heads, d, dtype, 0, (Scheme(T, H, W, 1, 1, 1),),
                    (0,) * heads, (0.9,) * heads, (False,) * heads)


def _check(q, k, cands):
    scores, choice = api.sics(q, k, cands)
    torch.cuda.synchronize()
    ref_s, ref_c = O.choose_schemes(to_np(q), to_np(k), cands)
    got = to_np(scores)
    assert np.allclose(got, ref_s, rtol=SCORE_REL, atol=1e-3), np.abs(got - ref_s).max()
    ch = choice.cpu().numpy()
    for h in range(ref_s.shape[0]):
        srt = np.sort(ref_s[h])[::-1]
        if len(srt) == 1 or (srt[0] - srt[1]) > 1e-3 * abs(srt[0]):
            assert ch[h] == ref_c[h], (h, ref_s[h], got[h])
    return scores, choice


@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("bf16", 64), ("f32", 64), ("f32", 128)])
def test_sics_matches_oracle_ragged(dtype, d):
    T, H, W = 5, 9, 10
    wl = _wl(T, H, W, 2 if d == 128 or dtype == "f32" else 4, d, dtype)
    q, k, _ = make_qkv(wl, device="cuda")
    cands = [(T, H, W, 2, 4, 4), (T, H, W, 1, 8, 8), (T, H, W, 4, 2, 4)]
    _check(q, k, cands)


def test_sics_odd_head_count():
    T, H, W = 4, 8, 8
    wl = _wl(T, H, W, 3, 128, "bf16", cid=22)       # 3 x 16 lanes: a partial warp group
    q, k, _ = make_qkv(wl, device="cuda")
    _check(q, k, [(T, H, W, 2, 4, 4), (T, H, W, 4, 8, 2)])


def test_sics_single_token_cells():
    """Candidates 1x1x2, 1x1x3 and 2x1x1: their common refinement has
    single-token cells in 2x1x6 regions (a ragged last region along x and
    t), so every block sums cells of one token."""
    T, H, W = 3, 5, 20
    wl = _wl(T, H, W, 3, 128, "bf16", cid=26)
    q, k, _ = make_qkv(wl, device="cuda")
    _check(q, k, [(T, H, W, 1, 1, 2), (T, H, W, 1, 1, 3), (T, H, W, 2, 1, 1)])


def test_sics_four_candidates():
    """The most candidates a call takes (four), on a ragged grid: their
    common refinement is 32 cells of 1x2x4 tokens in 4x8x8 regions."""
    T, H, W = 5, 9, 10
    wl = _wl(T, H, W, 2, 128, "bf16", cid=27)
    q, k, _ = make_qkv(wl, device="cuda")
    _check(q, k, [(T, H, W, 2, 4, 4), (T, H, W, 1, 8, 8), (T, H, W, 4, 2, 4), (T, H, W, 2, 2, 8)])


def test_sics_candidates_on_different_grids():
    """Candidates only need the same number of tokens: here the 192 tokens
    are read as a 4x6x8 and as an 8x6x4 grid (each candidate walks the token
    order of its own grid), which takes one pass per candidate."""
    wl = _wl(4, 6, 8, 2, 64, "bf16", cid=28)
    q, k, _ = make_qkv(wl, device="cuda")
    _check(q, k, [(4, 6, 8, 2, 3, 4), (8, 6, 4, 4, 3, 2)])


def test_sics_per_candidate_path():
    """Candidates whose common refinement has more cells than the one-pass
    kernel keeps on chip (8x4x8 cells of 1x2x2 tokens per 8x8x16 region) run
    one launch per candidate; same check against the oracle."""
    T, H, W = 9, 10, 18
    wl = _wl(T, H, W, 3, 128, "bf16", cid=25)
    q, k, _ = make_qkv(wl, device="cuda")
    _check(q, k, [(T, H, W, 1, 2, 16), (T, H, W, 8, 8, 2)])


def test_sics_picks_the_constructed_scheme():
    rng = np.random.default_rng(4)
    T, H, W, heads, d = 4, 8, 8, 2, 64
    A = (T, H, W, 2, 4, 4)
    cands = [(T, H, W, 4, 2, 4), A, (T, H, W, 1, 8, 8)]
    q = np.zeros((T * H * W, heads, d), dtype=np.float32)
    k = np.zeros_like(q)
    for x in (q, k):
        for ids, _ in O.block_tokens(*A):
            for h in range(heads):
                x[ids, h] = np.outer(rng.uniform(0.5, 2.0, len(ids)), rng.standard_normal(d))
    scores, choice = _check(torch.from_numpy(q).cuda(), torch.from_numpy(k).cuda(), cands)
    assert choice.cpu().tolist() == [1] * heads


def test_sics_deterministic():
    T, H, W = 6, 16, 16
    wl = _wl(T, H, W, 4, 128, "bf16", cid=23)
    q, k, _ = make_qkv(wl, device="cuda")
    cands = [(T, H, W, 2, 8, 8), (T, H, W, 1, 8, 16), (T, H, W, 6, 4, 4)]
    a = api.sics(q, k, cands)
    b = api.sics(q, k, cands)
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_sics_full_size_sampled_blocks():
    """Wan-14B shape, 40 heads, the three candidates of the mixed policy:
    per-block values (read from the workspace) against the oracle's pairwise
    sum on sampled (candidate, head, block) triples; the per-head scores are
    the fixed-order sums of those values."""
    from spade_workloads import get_config
    wl = get_config("wan14b")
    q, k, _ = make_qkv(wl, device="cuda")
    T, H, W = wl.T, wl.H, wl.W
    cands = [(T, H, W, 2, 8, 8), (T, H, W, 1, 8, 16), (T, H, W, 8, 4, 4)]
    ws = torch.zeros(api.sics_workspace_bytes(cands, wl.heads), dtype=torch.uint8, device="cuda")
    scores, choice = api.sics(q, k, cands, workspace=ws)
    torch.cuda.synchronize()
    vals = ws.view(torch.float32).cpu().numpy().astype(np.float64)
    rng = np.random.default_rng(7)
    off = 0
    for c, g in enumerate(cands):
        blocks = O.block_tokens(*g)
        nb = len(blocks)
        per = vals[off: off + wl.heads * nb].reshape(wl.heads, nb)
        assert np.allclose(per.sum(axis=1), to_np(scores)[:, c], rtol=1e-5)
        for h in rng.choice(wl.heads, 2, replace=False):
            for b in rng.choice(nb, 2, replace=False):
                ids = blocks[b][0]
                ref = O.block_sics(to_np(q[ids, h])) + O.block_sics(to_np(k[ids, h]))
                assert per[h, b] == pytest.approx(ref, rel=SCORE_REL), (c, h, b)
        off += wl.heads * nb
    best = to_np(scores).argmax(axis=1)
    assert (choice.cpu().numpy() == best).all()


def test_computed_scheme_table_drives_the_grouped_launch():
    """Scheme generation feeding step a6: the per-head scheme table comes from
    spade_sics, the layer runs through one grouped launch, and the result is
    checked against the oracle under the same table (its own choice where the
    score margin is clear, attention under the GPU's masks)."""
    from helpers import (ATTN_MAX_ABS_BF16, ATTN_MEAN_ABS_BF16, attn_errors, compare_kept,
                         oracle_selection, run_grouped)
    T, H, W, heads = 8, 16, 32, 6
    cands = (Scheme(T, H, W, 2, 8, 8), Scheme(T, H, W, 1, 8, 16), Scheme(T, H, W, 8, 4, 4))
    wl0 = Workload("sics-table", 24, T, H, W, heads, 128, "bf16", 0, cands, (0,) * heads,
                   (0.85, 0.9, 0.95, 0.85, 0.9, 0.95), (False,) * heads)
    q, k, v = make_qkv(wl0, device="cuda")
    scores, choice = api.sics(q, k, [c.as_tuple() for c in cands])
    torch.cuda.synchronize()
    ref_s, ref_c = O.choose_schemes(to_np(q), to_np(k), [c.as_tuple() for c in cands])
    ch = [int(c) for c in choice.cpu().tolist()]
    for h in range(heads):
        srt = np.sort(ref_s[h])[::-1]
        if srt[0] - srt[1] > 1e-3 * abs(srt[0]):
            assert ch[h] == ref_c[h]
    wl = Workload("sics-table", 24, T, H, W, heads, 128, "bf16", 0, cands, tuple(ch), wl0.head_tau,
                  (False,) * heads)
    out, _, kept = run_grouped(wl, q, k, v)
    qn, kn, vn = to_np(q), to_np(k), to_np(v)
    head_geom = [cands[ch[h]].as_tuple() for h in range(heads)]
    ref = O.block_sparse_attention(qn, kn, vn, head_geom, [kept(h) for h in range(heads)], 0)
    mx, mean, n = attn_errors(to_np(out), ref)
    assert n == wl.N * heads * wl.d
    assert mx <= ATTN_MAX_ABS_BF16 and mean <= ATTN_MEAN_ABS_BF16, (mx, mean)
    for h in range(heads):
        P, ok, mg = oracle_selection(wl, qn[:, h: h + 1], kn[:, h: h + 1], h)
        _, bad, _ = compare_kept(kept(h), ok, mg, P=P, tau=wl.head_tau[h])
        assert not bad, (h, bad[:5])
