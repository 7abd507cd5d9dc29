"""The pipelined host-memory entry (grouped_attn_from_host) moves data only:
its output must equal the device-resident grouped call, for even and uneven
head groups and with text tokens."""
import pytest
import torch

from input_adaptive_block_b200 import api
from spade_workloads import Scheme, Workload, make_qkv

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("chunk,text,slots,streams", [(2, 0, 3, 2), (3, 0, 2, 1), (4, 64, 3, 2), (1, 0, 4, 3)])
def test_from_host_equals_device_call(chunk, text, slots, streams):
    T, H, W, heads = 5, 16, 24, 6
    wl = Workload("from-host", 61, T, H, W, heads, 128, "bf16", text, (Scheme(T, H, W, 2, 8, 8),),
                  (0,) * heads, (0.85, 0.9, 0.95, 0.85, 0.9, 0.95), (False,) * heads)
    q, k, v = make_qkv(wl, device="cuda")
    schemes = [wl.schemes[0].as_tuple()]
    table = [(0, wl.head_tau[h], False) for h in range(heads)]
    ref = api.grouped_attn(q, k, v, schemes, table, text)
    qh, kh, vh = (t.cpu().pin_memory() for t in (q, k, v))
    oh = torch.empty(qh.shape, dtype=qh.dtype).pin_memory()
    api.grouped_attn_from_host(qh, kh, vh, oh, schemes, table, text, head_chunk=chunk, slots=slots,
                               compute_streams=streams)
    torch.cuda.synchronize()
    assert api.last_device_status() == 0
    assert torch.equal(oh, ref.cpu())
