"""spade_grouped_attn_lists runs step 5 alone under the kept lists an earlier
grouped call left in its workspace.  The kept lists depend on Q and K only,
so re-running the attention with a new V under the old lists must give
exactly what a whole grouped call on the new V gives."""
import pytest
import torch

from input_adaptive_block_b200 import api
from spade_workloads import Scheme, Workload, make_qkv

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("text", [0, 100])
def test_lists_entry_reuses_the_mask(text):
    T, H, W, heads = 5, 16, 24, 5
    wl = Workload("lists", 63, T, H, W, heads, 128, "bf16", text,
                  (Scheme(T, H, W, 2, 8, 8), Scheme(T, H, W, 1, 8, 16)),
                  (0, 1, 0, 1, 0), (0.85, 0.9, 0.95, 0.85, 0.9), (True, False, False, False, False))
    q, k, v = make_qkv(wl, device="cuda")
    v2 = torch.flip(v, dims=[0]).contiguous()
    schemes = [sc.as_tuple() for sc in wl.schemes]
    table = [(wl.head_scheme[h], wl.head_tau[h], wl.head_dense[h]) for h in range(heads)]
    ws = torch.zeros(api.grouped_workspace_bytes(schemes, table, wl.d, text), dtype=torch.uint8, device="cuda")
    first = api.grouped_attn(q, k, v, schemes, table, text, workspace=ws)
    again = api.grouped_attn_lists(q, k, v, schemes, table, ws, text)
    swapped = api.grouped_attn_lists(q, k, v2, schemes, table, ws, text)
    ref2 = api.grouped_attn(q, k, v2, schemes, table, text)
    torch.cuda.synchronize()
    assert api.last_device_status() == 0
    assert torch.equal(first, again)
    assert torch.equal(swapped, ref2)
