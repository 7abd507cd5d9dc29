"""spade_block_sparse_attn_noalloc: the attention entry point for callers that
cannot allocate device memory (the library keeps the scratch in a fixed
device array instead of taking a workspace).  Its output must match the
regular entry point's on the same inputs, on consecutive calls that reuse the
fixed array.  Its host-side refusals (oversized calls, bad arguments) are
checked without a GPU in test_abi_cpu.py, with a pointer that is never
dereferenced, so no GPU process ever hands it a mis-sized buffer.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test.
"""
import numpy as np
import pytest
import torch

from input_adaptive_block_b200 import api
from spade_workloads import Scheme, Workload, make_qkv

from helpers import ATTN_MAX_ABS_BF16, ATTN_MEAN_ABS_BF16, to_np

pytestmark = pytest.mark.gpu


def _case(T, H, W, heads, text):
    return Workload("noalloc", 11, T, H, W, heads, 128, "bf16", text, (Scheme(T, H, W, 2, 8, 8),),
                    (0,) * heads, (0.9,) * heads, (False,) * heads)


@pytest.mark.parametrize("text", [0, 200])
def test_noalloc_matches_workspace_entry_point(text):
    wl = _case(6, 20, 28, 3, text)
    geom = wl.schemes[0].as_tuple()
    q, k, v = make_qkv(wl, device="cuda")
    # kept lists from the library's own index search
    P = api.estimate(api.summarize(q, geom), api.summarize(k, geom))
    cnt, idx = api.select(P, wl.head_tau)
    ref = api.block_sparse_attn(q, k, v, cnt, idx, geom, text_tokens=text)
    outs = []
    for _ in range(2):                                  # the second call reuses the fixed scratch
        outs.append(api.block_sparse_attn_noalloc(q, k, v, cnt, idx, geom, text_tokens=text))
    torch.cuda.synchronize()
    assert api.last_device_status() == 0
    r = to_np(ref)
    for o in outs:
        diff = np.abs(to_np(o) - r)
        assert diff.max() <= ATTN_MAX_ABS_BF16 and diff.mean() <= ATTN_MEAN_ABS_BF16, (diff.max(), diff.mean())
    assert torch.equal(outs[0], outs[1])


def test_noalloc_dense_heads():
    wl = _case(3, 16, 17, 2, 0)
    geom = wl.schemes[0].as_tuple()
    q, k, v = make_qkv(wl, device="cuda")
    ref = api.block_sparse_attn(q, k, v, None, None, geom)
    a = api.block_sparse_attn_noalloc(q, k, v, None, None, geom)
    b = api.block_sparse_attn_noalloc(q, k, v, None, None, geom)
    torch.cuda.synchronize()
    diff = np.abs(to_np(a) - to_np(ref))
    assert diff.max() <= ATTN_MAX_ABS_BF16 and diff.mean() <= ATTN_MEAN_ABS_BF16
    assert torch.equal(a, b)
