"""Pins of the oracle's scheme-generation score (SICS) against facts that do
not come from the oracle itself: the cosine-sum identity, closed-form special
cases, invariances, and a constructed input whose best blocking scheme is
known by construction."""
import numpy as np
import pytest

import oracle as O


def _norm_sum_sq(xb):
    """sum_{i,j} cos(x_i, x_j) = || sum_i x_i / ||x_i|| ||^2 (zero rows skipped)."""
    n = np.linalg.norm(xb, axis=1)
    u = (xb[n > 0] / n[n > 0, None]).sum(axis=0)
    return float(u @ u)


@pytest.mark.parametrize("n,d", [(1, 4), (7, 3), (32, 16), (50, 64)])
def test_block_sics_matches_unit_vector_identity(n, d):
    rng = np.random.default_rng(n * 100 + d)
    xb = rng.standard_normal((n, d))
    assert O.block_sics(xb) == pytest.approx(_norm_sum_sq(xb), rel=1e-12, abs=1e-12)


def test_block_sics_special_cases():
    rng = np.random.default_rng(1)
    v = rng.standard_normal(8)
    same = np.outer(rng.uniform(0.1, 5.0, 10), v)             # one direction, positive scales
    assert O.block_sics(same) == pytest.approx(100.0, rel=1e-12)
    mixed = np.vstack([np.outer(rng.uniform(0.1, 2, 6), v), -np.outer(rng.uniform(0.1, 2, 2), v)])
    assert O.block_sics(mixed) == pytest.approx((6 - 2) ** 2, rel=1e-12)
    ortho = np.eye(8)[:5] * rng.uniform(0.5, 3.0, (5, 1))     # pairwise orthogonal: only i = j counts
    assert O.block_sics(ortho) == pytest.approx(5.0, rel=1e-12)
    with_zero = np.vstack([same[:3], np.zeros(8)])             # a zero vector adds nothing
    assert O.block_sics(with_zero) == pytest.approx(9.0, rel=1e-12)


def test_block_sics_scale_and_order_invariant():
    rng = np.random.default_rng(2)
    xb = rng.standard_normal((12, 6))
    ref = O.block_sics(xb)
    assert O.block_sics(xb * rng.uniform(0.01, 100, (12, 1))) == pytest.approx(ref, rel=1e-10)
    assert O.block_sics(xb[rng.permutation(12)]) == pytest.approx(ref, rel=1e-10)


def test_sics_sums_over_blocks_of_the_scheme():
    rng = np.random.default_rng(3)
    T, H, W = 3, 5, 6
    x = rng.standard_normal((T * H * W, 2, 4))
    geom = (T, H, W, 2, 2, 4)
    total = np.zeros(2)
    for ids, _ in O.block_tokens(*geom):
        for h in range(2):
            total[h] += _norm_sum_sq(x[ids, h])
    assert np.allclose(O.sics(x, geom), total, rtol=1e-12)
    # one block covering the whole grid: the whole-tensor identity
    whole = (T, H, W, T, H, W)
    assert np.allclose(O.sics(x, whole), [_norm_sum_sq(x[:, h]) for h in range(2)], rtol=1e-12)


def test_choose_schemes_finds_the_constructed_scheme():
    """Every block of scheme A holds one direction (random positive scales),
    different per block and per head; the other candidates mix blocks of A,
    so A must win with SICS = sum of squared block sizes."""
    rng = np.random.default_rng(4)
    T, H, W, heads, d = 4, 8, 8, 3, 16
    A = (T, H, W, 2, 4, 4)
    cands = [(T, H, W, 4, 2, 4), A, (T, H, W, 1, 8, 8)]
    q = np.zeros((T * H * W, heads, d))
    k = np.zeros_like(q)
    for x in (q, k):
        for ids, _ in O.block_tokens(*A):
            for h in range(heads):
                x[ids, h] = np.outer(rng.uniform(0.5, 2.0, len(ids)), rng.standard_normal(d))
    scores, choice = O.choose_schemes(q, k, cands)
    assert list(choice) == [1] * heads
    assert np.allclose(scores[:, 1], 2 * 8 * 32 ** 2)          # Q and K: 8 blocks of 32 aligned tokens
    assert (scores[:, [0, 2]] < scores[:, [1]] - 1.0).all()


def test_choose_schemes_ties_take_the_lower_index():
    rng = np.random.default_rng(5)
    q = rng.standard_normal((4 * 4 * 4, 2, 8))
    g = (4, 4, 4, 2, 2, 2)
    scores, choice = O.choose_schemes(q, q, [g, g])
    assert list(choice) == [0, 0] and np.allclose(scores[:, 0], scores[:, 1])
