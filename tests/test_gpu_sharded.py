"""The head-sharded wrapper on the GPU: an NCCL process group of one rank runs
the grouped launch through both all-to-all exchanges (head plan, token
splits, text rows and all), and the result is checked against the oracle
under the kept lists the GPU chose."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import oracle as O
from input_adaptive_block_b200 import api
from input_adaptive_block_b200.sharded import grouped_attn_layer, head_costs, head_sharded_layer, plan_heads, \
    token_splits
from spade_workloads import Scheme, Workload, make_qkv

from helpers import ATTN_MAX_ABS_BF16, ATTN_MEAN_ABS_BF16, attn_errors, to_np

pytestmark = pytest.mark.gpu


def test_head_sharded_grouped_layer_single_rank_nccl():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("nccl", rank=0, world_size=1)
    try:
        T, H, W, heads, text = 6, 20, 28, 4, 150
        wl = Workload("sharded-gpu", 52, T, H, W, heads, 128, "bf16", text,
                      (Scheme(T, H, W, 2, 8, 8), Scheme(T, H, W, 1, 8, 16)),
                      (0, 1, 0, 1), (0.9, 0.85, 0.95, 0.9), (True, False, False, False))
        q, k, v = make_qkv(wl, device="cuda")
        schemes = [sc.as_tuple() for sc in wl.schemes]
        table = [(wl.head_scheme[h], wl.head_tau[h], wl.head_dense[h]) for h in range(heads)]
        plan = plan_heads(head_costs(wl.N, text, wl.d, table), 1)
        splits = token_splits(wl.N, 1)
        rows = [table[h] for h in plan[0]]
        ws = torch.zeros(api.grouped_workspace_bytes(schemes, rows, wl.d, text), dtype=torch.uint8, device="cuda")
        out = head_sharded_layer(q, k, v, grouped_attn_layer(schemes, table, text, workspace=ws), plan, splits, text)
        torch.cuda.synchronize()
        assert api.last_device_status() == 0
        qn, kn, vn = to_np(q), to_np(k), to_np(v)
        kept, geoms = [], []
        for lh, h in enumerate(plan[0]):
            geoms.append(schemes[wl.head_scheme[h]])
            if wl.head_dense[h]:
                kept.append(None)
                continue
            co, io = api.grouped_head_lists(schemes, rows, wl.d, text, lh)
            nb = wl.schemes[wl.head_scheme[h]].nb
            cnt = ws[co: co + 4 * nb].view(torch.int32).cpu().numpy()
            idx = ws[io: io + 4 * nb * nb].view(torch.int32).view(nb, nb).cpu().numpy()
            kept.append([list(map(int, idx[i, : cnt[i]])) for i in range(nb)])
        order = list(plan[0])
        ref = O.block_sparse_attention(qn[:, order], kn[:, order], vn[:, order], geoms, kept, text)
        mx, mean, n = attn_errors(to_np(out)[:, order], ref)
        assert n == ref.size and mx <= ATTN_MAX_ABS_BF16 and mean <= ATTN_MEAN_ABS_BF16, (mx, mean)
        assert np.isfinite(to_np(out)).all()
    finally:
        dist.destroy_process_group()
