"""The host-memory entry (spade_grouped_attn_host, through
api.grouped_attn_from_host) moves data only: its output must equal the
device-resident grouped call, for even and uneven head groups, with text
tokens and mixed schemes, on consecutive calls that reuse the library's
streams and the caller's workspace."""
import pytest
import torch

from input_adaptive_block_b200 import api
from spade_workloads import Scheme, Workload, make_qkv

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("chunk,text", [(2, 0), (3, 0), (4, 64), (1, 0), (6, 0)])
def test_from_host_equals_device_call(chunk, text):
    T, H, W, heads = 5, 16, 24, 6
    wl = Workload("from-host", 61, T, H, W, heads, 128, "bf16", text,
                  (Scheme(T, H, W, 2, 8, 8), Scheme(T, H, W, 1, 8, 16)),
                  (0, 1, 0, 1, 0, 0), (0.85, 0.9, 0.95, 0.85, 0.9, 0.95), (False, False, False, False, True, False))
    q, k, v = make_qkv(wl, device="cuda")
    schemes = [sc.as_tuple() for sc in wl.schemes]
    table = [(wl.head_scheme[h], wl.head_tau[h], wl.head_dense[h]) for h in range(heads)]
    ref = api.grouped_attn(q, k, v, schemes, table, text)
    qh, kh, vh = (t.cpu().pin_memory() for t in (q, k, v))
    ws = torch.empty(api.grouped_host_workspace_bytes(schemes, table, wl.d, text, q.dtype, chunk),
                     dtype=torch.uint8, device="cuda")
    for _ in range(2):
        oh = torch.full(qh.shape, float("nan"), dtype=qh.dtype).pin_memory()
        api.grouped_attn_from_host(qh, kh, vh, oh, schemes, table, text, head_chunk=chunk, workspace=ws)
        torch.cuda.synchronize()
        assert api.last_device_status() == 0
        assert torch.equal(oh, ref.cpu())


def test_from_host_fp32_tiny():
    """The fp32 configuration (CUDA-core attention path) through the host entry."""
    from spade_workloads import get_config
    wl = get_config("tiny")
    q, k, v = make_qkv(wl, device="cuda")
    schemes = [sc.as_tuple() for sc in wl.schemes]
    table = [(wl.head_scheme[h], wl.head_tau[h], wl.head_dense[h]) for h in range(wl.heads)]
    ref = api.grouped_attn(q, k, v, schemes, table, wl.text_tokens)
    qh, kh, vh = (t.cpu().pin_memory() for t in (q, k, v))
    oh = torch.empty(qh.shape, dtype=qh.dtype).pin_memory()
    api.grouped_attn_from_host(qh, kh, vh, oh, schemes, table, wl.text_tokens, head_chunk=1)
    torch.cuda.synchronize()
    assert api.last_device_status() == 0
    assert torch.equal(oh, ref.cpu())
