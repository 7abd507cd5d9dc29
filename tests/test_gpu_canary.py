"""Out-of-bounds writes, checked without a memory sanitizer: every output and
workspace buffer of every entry point sits between two 4 KB guard regions
filled with a byte pattern; after the call the guards must be intact.  The
index search must also leave every entry of a kept-list row past its count
as it was (the interface promises those entries are untouched).  Shapes:
ragged grids (edge blocks in every direction, nb not a multiple of 4), a
multi-tile grid with nb a multiple of 4 (the vectorised paths), text tokens,
and the fp32 tiny configuration."""
import numpy as np
import pytest
import torch

from input_adaptive_block_b200 import api
from spade_workloads import Scheme, Workload, get_config, make_qkv

pytestmark = pytest.mark.gpu

GUARD = 4096
FILL = 0xA5


class Guarded:
    """A tensor of `shape` inside a byte buffer with guard regions around it."""

    def __init__(self, shape, dtype, value=None):
        n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        self.buf = torch.full((GUARD + n + GUARD,), FILL, dtype=torch.uint8, device="cuda")
        self.t = self.buf[GUARD: GUARD + n].view(dtype).view(*shape)
        if value is not None:
            self.t.fill_(value)

    def intact(self) -> bool:
        torch.cuda.synchronize()
        return bool((self.buf[:GUARD] == FILL).all()) and bool((self.buf[-GUARD:] == FILL).all())


def _wl(name, T, H, W, heads, text=0, block=(2, 8, 8), dtype="bf16"):
    return Workload(name, 23, T, H, W, heads, 128, dtype, text, (Scheme(T, H, W, *block),),
                    (0,) * heads, (0.9,) * heads, (False,) * heads)


CASES = [
    _wl("ragged", 5, 19, 23, 3),                  # nb = 27, edges in t, y and x
    _wl("multi-tile", 16, 32, 60, 2),             # nb = 256 (two 128-block tiles), x edges
    _wl("text", 4, 16, 24, 2, text=200),          # text tokens appended
    get_config("tiny"),                           # fp32
]


@pytest.mark.parametrize("wl", CASES, ids=lambda w: w.name)
def test_outputs_stay_in_bounds(wl):
    q, k, v = make_qkv(wl, device="cuda")
    g = wl.schemes[0].as_tuple()
    sc = wl.schemes[0]
    heads, d, nb = wl.heads, wl.d, sc.nb
    dt = q.dtype

    xt = Guarded((heads, nb, sc.bs, d), dt)
    api.tile3d(q, g, out=xt.t)
    assert xt.intact(), "tile3d"

    qm, km = Guarded((heads, nb, d), torch.float32), Guarded((heads, nb, d), torch.float32)
    api.summarize(q, g, out=qm.t)
    assert qm.intact(), "summarize"
    qm2, km2 = Guarded((heads, nb, d), torch.float32), Guarded((heads, nb, d), torch.float32)
    api.summarize_qk(q, k, g, qout=qm2.t, kout=km2.t)
    assert qm2.intact() and km2.intact(), "summarize_qk"
    api.summarize(k, g, out=km.t)

    pr = Guarded((heads, nb, nb), torch.float32)
    api.estimate(qm.t, km.t, out=pr.t)
    assert pr.intact(), "estimate"
    sco = Guarded((heads, nb, nb), torch.float32)
    api.estimate_scores(qm.t, km.t, out=sco.t)
    assert sco.intact(), "estimate_scores"

    for name, fn, src in (("select", api.select, pr.t), ("select_scores", api.select_scores, sco.t)):
        cnt = Guarded((heads, nb), torch.int32, value=-3)
        idx = Guarded((heads, nb, nb), torch.int32, value=-7)
        fn(src, wl.head_tau, cnt=cnt.t, idx=idx.t)
        assert cnt.intact() and idx.intact(), name
        c, ix = cnt.t.cpu().numpy(), idx.t.cpu().numpy()
        assert (c >= 1).all() and (c <= nb).all(), name
        for h in range(heads):
            for i in range(nb):
                assert (ix[h, i, c[h, i]:] == -7).all(), (name, h, i)

    cnt = torch.empty(heads, nb, dtype=torch.int32, device="cuda")
    idx = torch.empty(heads, nb, nb, dtype=torch.int32, device="cuda")
    api.select_scores(sco.t, wl.head_tau, cnt=cnt, idx=idx)
    out = Guarded(tuple(q.shape), dt)
    ws = Guarded((max(api.attn_workspace_bytes(g, heads, d, wl.text_tokens), 256),), torch.uint8)
    api.block_sparse_attn(q, k, v, cnt, idx, g, wl.text_tokens, out=out.t, workspace=ws.t)
    assert out.intact() and ws.intact(), "block_sparse_attn"

    schemes = [s.as_tuple() for s in wl.schemes]
    table = [(wl.head_scheme[h], wl.head_tau[h], wl.head_dense[h]) for h in range(heads)]
    out2 = Guarded(tuple(q.shape), dt)
    gws = Guarded((max(api.grouped_workspace_bytes(schemes, table, d, wl.text_tokens), 256),), torch.uint8)
    api.grouped_attn(q, k, v, schemes, table, wl.text_tokens, out=out2.t, workspace=gws.t)
    assert out2.intact() and gws.intact(), "grouped_attn"
    assert api.last_device_status() == 0
    assert torch.isfinite(out2.t.float()).all()


def test_scheme_generation_stays_in_bounds():
    wl = _wl("sics", 6, 16, 24, 2)
    q, k, _ = make_qkv(wl, device="cuda")
    T, H, W = wl.T, wl.H, wl.W
    cands = [(T, H, W, 2, 8, 8), (T, H, W, 1, 8, 16), (T, H, W, 8, 4, 4)]
    ws = Guarded((max(api.sics_workspace_bytes(cands, wl.heads), 256),), torch.uint8)
    scores, choice = api.sics(q, k, cands, workspace=ws.t)
    assert ws.intact()
    assert choice.min().item() >= 0 and choice.max().item() < len(cands)
