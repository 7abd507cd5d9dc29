"""The five workload configurations at full size, in the launch configuration
bench.py times (one grouped call over all heads): kept lists against the fp64
oracle chain on sampled heads (bit-exact where the margin exceeds 1e-3), and
attention outputs on sampled query blocks (interior, every kind of edge block,
text rows) under the GPU's own mask."""
import numpy as np
import pytest
import torch

import oracle as O
from spade_workloads import get_config, make_qkv

from helpers import (ATTN_MAX_ABS_BF16, ATTN_MAX_ABS_F32, ATTN_MEAN_ABS_BF16, attn_errors,
                     compare_kept, oracle_selection, run_grouped, to_np)

pytestmark = pytest.mark.gpu

SAMPLE_HEADS = {
    "tiny": [0, 1],
    "wan1.3b": list(range(12)),
    "wan14b": [0, 13, 27, 39],
    "hunyuan": [0, 11, 23],
    "mixed": [0, 12, 13, 20, 26, 27, 33, 39],
}


def _sample_qblocks(wl, h, rng):
    sc = wl.schemes[wl.head_scheme[h]]
    nb = sc.nb
    vc = O.valid_counts(sc.as_tuple())
    edges = [b for b in range(nb) if vc[b] < sc.bs]
    picks = {0, nb - 1, nb // 2}
    if edges:
        picks.update(rng.choice(edges, size=min(2, len(edges)), replace=False).tolist())
    if wl.text_tokens:
        picks.add(nb)                                   # the text query rows
    return sorted(int(b) for b in picks)


# Wan-14B is also run at the ends of its tau sweep: 0.8 gives the shortest
# kept lists, 0.95 the longest, and both move the selection cut the most.
@pytest.mark.parametrize("name,tau", [("tiny", None), ("wan1.3b", None), ("wan14b", None), ("wan14b", 0.8),
                                      ("wan14b", 0.95), ("hunyuan", None), ("mixed", None)],
                         ids=["tiny", "wan1.3b", "wan14b", "wan14b@tau=0.8", "wan14b@tau=0.95", "hunyuan", "mixed"])
def test_full_config(name, tau):
    wl = get_config(name)
    if tau is not None:
        wl = wl.with_tau(tau)
    q, k, v = make_qkv(wl, device="cuda")
    out, _, kept = run_grouped(wl, q, k, v)
    assert torch.isfinite(out.float()).all()
    rng = np.random.default_rng(wl.config_id)
    checked_rows, skipped_rows = 0, 0
    for h in SAMPLE_HEADS[name]:
        qh, kh, vh = to_np(q[:, h: h + 1]), to_np(k[:, h: h + 1]), to_np(v[:, h: h + 1])
        geom = wl.schemes[wl.head_scheme[h]].as_tuple()
        gk = kept(h)
        if gk is not None:
            P, ok, mg = oracle_selection(wl, qh, kh, h)
            c, bad, s = compare_kept(gk, ok, mg, P=P, tau=wl.head_tau[h])
            assert not bad, (name, h, bad[:5])
            checked_rows += c
            skipped_rows += s
        qb = _sample_qblocks(wl, h, rng)
        ref = O.block_sparse_attention(qh, kh, vh, [geom], [gk], wl.text_tokens, {0: qb})
        mx, mean, n = attn_errors(to_np(out[:, h: h + 1]), ref)
        assert n > 0
        if wl.dtype == "f32":
            assert mx <= ATTN_MAX_ABS_F32, (name, h, mx)
        else:
            assert mx <= ATTN_MAX_ABS_BF16 and mean <= ATTN_MEAN_ABS_BF16, (name, h, mx, mean)
    if any(not wl.head_dense[h] for h in SAMPLE_HEADS[name]):
        assert checked_rows >= 0.5 * (checked_rows + skipped_rows)

