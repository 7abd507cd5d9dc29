"""The head-sharded wrapper on the GPU: an NCCL process group of one rank
runs the grouped launch through both all-to-all exchanges; the result must
equal the direct grouped call (the exchanges only move data)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist

from input_adaptive_block_b200 import api
from input_adaptive_block_b200.sharded import grouped_attn_layer, head_sharded_layer
from spade_workloads import Scheme, Workload, make_qkv

pytestmark = pytest.mark.gpu


def test_head_sharded_grouped_layer_single_rank_nccl():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("nccl", rank=0, world_size=1)
    try:
        T, H, W, heads = 6, 20, 28, 4
        wl = Workload("sharded-gpu", 52, T, H, W, heads, 128, "bf16", 0, (Scheme(T, H, W, 2, 8, 8),),
                      (0,) * heads, (0.9,) * heads, (False,) * heads)
        q, k, v = make_qkv(wl, device="cuda")
        schemes = [wl.schemes[0].as_tuple()]
        table = [(0, 0.9, False)] * heads
        ref = api.grouped_attn(q, k, v, schemes, table)
        out = head_sharded_layer(q, k, v, grouped_attn_layer(schemes, table))
        torch.cuda.synchronize()
        assert torch.equal(out, ref)
    finally:
        dist.destroy_process_group()
