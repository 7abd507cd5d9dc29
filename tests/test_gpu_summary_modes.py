"""Summarizer variants (Methodology 1 names max / min / mean reduces) on the
GPU: the standalone pass bit-exact against the oracle, and whole grouped
layers whose estimator scores max / min summaries."""
import numpy as np
import pytest
import torch

import oracle as O
from input_adaptive_block_b200 import api
from spade_workloads import Scheme, Workload, make_qkv

from helpers import (ATTN_MAX_ABS_BF16, ATTN_MEAN_ABS_BF16, MARGIN, attn_errors, compare_kept, table_of,
                     to_np)

pytestmark = pytest.mark.gpu


def _wl(T, H, W, heads, d, dtype, block, cid=31, tau=0.9):
    return Workload("modes", cid, T, H, W, heads, d, dtype, 0, (Scheme(T, H, W, *block),),
                    (0,) * heads, (tau,) * heads, (False,) * heads)


@pytest.mark.parametrize("mode", ["max", "min"])
@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("bf16", 64), ("f32", 64)])
def test_summarize_mode_bit_exact(mode, dtype, d):
    wl = _wl(5, 19, 23, 3, d, dtype, (2, 8, 8))
    q, _, _ = make_qkv(wl, device="cuda")
    g = wl.schemes[0].as_tuple()
    got = api.summarize(q, g, mode=mode)
    torch.cuda.synchronize()
    ref = O.summarize(to_np(q), g, mode)
    assert np.array_equal(to_np(got), ref)          # max / min of exactly representable values: no rounding


@pytest.mark.parametrize("summary", [("max", "mean"), ("min", "max")])
def test_grouped_layer_with_summary_modes(summary):
    wl = _wl(6, 20, 28, 2, 128, "bf16", (2, 8, 8), cid=32)
    q, k, v = make_qkv(wl, device="cuda")
    schemes = [s.as_tuple() for s in wl.schemes]
    table = table_of(wl)
    ws = torch.zeros(api.grouped_workspace_bytes(schemes, table, wl.d, 0), dtype=torch.uint8, device="cuda")
    out = api.grouped_attn(q, k, v, schemes, table, 0, workspace=ws, summary=summary)
    torch.cuda.synchronize()
    assert api.last_device_status() == 0
    qn, kn, vn = to_np(q), to_np(k), to_np(v)
    g = schemes[0]
    nb = wl.schemes[0].nb
    kept = []
    for h in range(wl.heads):
        co, io = api.grouped_head_lists(schemes, table, wl.d, 0, h)
        cnt = ws[co: co + 4 * nb].view(torch.int32).cpu().numpy()
        idx = ws[io: io + 4 * nb * nb].view(torch.int32).view(nb, nb).cpu().numpy()
        kept.append([list(map(int, idx[i, : cnt[i]])) for i in range(nb)])
        qm = O.summarize(qn[:, h: h + 1], g, summary[0])
        km = O.summarize(kn[:, h: h + 1], g, summary[1])
        P = O.estimate(qm, km)[0]
        ok = [O.select_row(P[i], i, wl.head_tau[h]) for i in range(nb)]
        mg = np.array([O.selection_margin(P[i], i, wl.head_tau[h]) for i in range(nb)])
        checked, bad, _ = compare_kept(kept[h], ok, mg, thr=MARGIN, P=P, tau=wl.head_tau[h])
        assert not bad and checked > 0, (h, bad[:5])
    ref = O.block_sparse_attention(qn, kn, vn, [g] * wl.heads, kept, 0)
    mx, mean, n = attn_errors(to_np(out), ref)
    assert n == wl.N * wl.heads * wl.d
    assert mx <= ATTN_MAX_ABS_BF16 and mean <= ATTN_MEAN_ABS_BF16, (mx, mean)
