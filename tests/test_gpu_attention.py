"""GPU parity of the block-sparse attention (and the whole grouped layer)
against the oracle evaluated under the GPU's own kept lists: max abs error
<= 2e-2 and mean abs error <= 2e-3 for bf16 I/O (fp32 accumulation); fp32
data (CUDA-core path) at 1e-4.  Cases span several key tiles, ragged edge
blocks in t, y and x, ragged text blocks, dense heads, tau = 1, d = 64 and
mixed schemes in one launch."""
import numpy as np
import pytest
import torch

import oracle as O
from input_adaptive_block_b200 import api
from spade_workloads import Scheme, Workload, flat_scheme, get_config, make_qkv

from helpers import (ATTN_MAX_ABS_BF16, ATTN_MAX_ABS_F32, ATTN_MEAN_ABS_BF16, attn_errors,
                     compare_kept, oracle_selection, run_grouped, to_np)

pytestmark = pytest.mark.gpu


def _wl(name, T, H, W, heads, d, dtype, block, tau=0.9, text=0):
    return Workload(name, 8, T, H, W, heads, d, dtype, text, (Scheme(T, H, W, *block),),
                    (0,) * heads, (tau,) * heads, (False,) * heads)


def _mixed_small():
    T, H, W, heads = 9, 18, 33, 6
    N = T * H * W
    schemes = (flat_scheme(N), Scheme(T, H, W, 1, 8, 16), Scheme(T, H, W, 8, 4, 4))
    return Workload("mixed-small", 9, T, H, W, heads, 128, "bf16", 0, schemes,
                    (0, 0, 1, 1, 2, 2), (1.0, 1.0, 0.85, 0.9, 0.95, 0.85),
                    (True, True, False, False, False, False))


CASES = [
    _wl("ragged-2x8x8", 6, 20, 28, 2, 128, "bf16", (2, 8, 8)),
    _wl("ragged-d64", 5, 19, 23, 2, 64, "bf16", (2, 8, 8), tau=0.8),
    # every edge case of a 2x8x8 block (t, y, x and their combinations), with
    # valid-token counts that are not multiples of 16 (24, 42, 21, ...)
    _wl("ragged-all-edges-d128", 5, 19, 23, 3, 128, "bf16", (2, 8, 8), tau=0.85),
    _wl("text-200", 4, 16, 24, 2, 128, "bf16", (2, 8, 8), text=200),
    _wl("tau1-dense-equivalent", 3, 16, 17, 2, 128, "bf16", (2, 8, 8), tau=1.0),
    _wl("one-block", 1, 4, 4, 2, 128, "bf16", (2, 8, 8)),
    # tau -> 0: every row keeps its diagonal block only, so the 1152 items
    # (about eight per persistent CTA) have one key block each and the CTA's
    # block counter steps through every score slot from item to item
    _wl("diagonal-only", 8, 48, 64, 6, 128, "bf16", (2, 8, 8), tau=1e-6),
    _mixed_small(),
    get_config("tiny"),
]


def _check(wl, q, k, v, out, kept, heads=None, q_blocks=None):
    qn, kn, vn = to_np(q), to_np(k), to_np(v)
    hs = list(range(wl.heads)) if heads is None else heads
    head_geom = [wl.schemes[wl.head_scheme[h]].as_tuple() for h in range(wl.heads)]
    gk = [kept(h) if h in hs else [[0]] * wl.schemes[wl.head_scheme[h]].nb for h in range(wl.heads)]
    qsel = {h: (q_blocks[h] if q_blocks else list(range(wl.schemes[wl.head_scheme[h]].nb +
                                                         (1 if wl.text_tokens else 0)))) for h in hs}
    ref = O.block_sparse_attention(qn, kn, vn, head_geom, gk, wl.text_tokens, qsel)
    mx, mean, n = attn_errors(to_np(out), ref)
    if wl.dtype == "f32":
        assert mx <= ATTN_MAX_ABS_F32, (mx, mean)
    else:
        assert mx <= ATTN_MAX_ABS_BF16 and mean <= ATTN_MEAN_ABS_BF16, (mx, mean)
    return n


@pytest.mark.parametrize("wl", CASES, ids=lambda w: w.name)
def test_grouped_layer_parity(wl):
    q, k, v = make_qkv(wl, device="cuda")
    out, _, kept = run_grouped(wl, q, k, v)
    assert torch.isfinite(out.float()).all()
    n = _check(wl, q, k, v, out, kept)
    assert n == wl.n_total * wl.heads * wl.d            # every output row compared
    # the GPU's masks match the oracle's selection wherever the margin is clear
    qn, kn = to_np(q), to_np(k)
    for h in range(wl.heads):
        if wl.head_dense[h]:
            continue
        P, ok, mg = oracle_selection(wl, qn[:, h: h + 1], kn[:, h: h + 1], h)
        _, bad, _ = compare_kept(kept(h), ok, mg, P=P, tau=wl.head_tau[h])
        assert not bad, (h, bad[:5])


def test_tau1_equals_dense_attention():
    wl = _wl("tau1", 3, 16, 17, 2, 128, "bf16", (2, 8, 8), tau=1.0)
    q, k, v = make_qkv(wl, device="cuda")
    out, _, kept = run_grouped(wl, q, k, v)
    ref = O.dense_attention(to_np(q), to_np(k), to_np(v))
    mx, mean, _ = attn_errors(to_np(out), ref)
    assert mx <= ATTN_MAX_ABS_BF16 and mean <= ATTN_MEAN_ABS_BF16, (mx, mean)


def test_block_sparse_attn_entry_with_given_lists():
    """spade_block_sparse_attn with caller-made lists: only the diagonal, all
    blocks, and a random subset per row (ascending, diagonal included)."""
    wl = _wl("given", 4, 24, 24, 2, 128, "bf16", (2, 8, 8))
    geom = wl.schemes[0].as_tuple()
    nb = wl.schemes[0].nb
    q, k, v = make_qkv(wl, device="cuda")
    rng = np.random.default_rng(3)
    for mode in ("diag", "all", "random"):
        cnt = np.zeros((wl.heads, nb), np.int32)
        idx = np.full((wl.heads, nb, nb), -1, np.int32)
        lists = []
        for h in range(wl.heads):
            lh = []
            for i in range(nb):
                if mode == "diag":
                    s = [i]
                elif mode == "all":
                    s = list(range(nb))
                else:
                    s = sorted(set([i] + list(rng.choice(nb, int(rng.integers(0, nb)), replace=False))))
                lh.append(s)
                cnt[h, i] = len(s)
                idx[h, i, : len(s)] = s
            lists.append(lh)
        out = api.block_sparse_attn(q, k, v, torch.from_numpy(cnt).cuda(), torch.from_numpy(idx).cuda(), geom)
        torch.cuda.synchronize()
        ref = O.block_sparse_attention(to_np(q), to_np(k), to_np(v), [geom] * wl.heads, lists)
        mx, mean, _ = attn_errors(to_np(out), ref)
        assert mx <= ATTN_MAX_ABS_BF16 and mean <= ATTN_MEAN_ABS_BF16, (mode, mx, mean)
    # cnt = NULL: every head dense
    out = api.block_sparse_attn(q, k, v, None, None, geom)
    torch.cuda.synchronize()
    ref = O.dense_attention(to_np(q), to_np(k), to_np(v))
    mx, mean, _ = attn_errors(to_np(out), ref)
    assert mx <= ATTN_MAX_ABS_BF16 and mean <= ATTN_MEAN_ABS_BF16, (mx, mean)


def test_repeat_calls_identical():
    """Scheduling does not change results: two calls give identical bits."""
    wl = _mixed_small()
    q, k, v = make_qkv(wl, device="cuda")
    a, _, _ = run_grouped(wl, q, k, v)
    b, _, _ = run_grouped(wl, q, k, v)
    assert torch.equal(a, b)
