"""Head-sharded execution across two gloo ranks on CPU: the two all-to-all
exchanges are exact inverses, and a layer run head-sharded equals the same
layer run on one process (the per-head work is the oracle here, on CPU)."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle as O
from spade_workloads import Scheme, Workload, make_qkv


def _port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _wl():
    T, H, W, heads = 4, 8, 8, 4
    return Workload("sharded", 51, T, H, W, heads, 16, "f32", 0, (Scheme(T, H, W, 2, 4, 4),),
                    (0,) * heads, (0.8, 0.9, 0.85, 0.95), (False,) * heads)


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from input_adaptive_block_b200.sharded import head_sharded_layer, heads_to_seq, seq_to_heads
        wl = _wl()
        q, k, v = make_qkv(wl)                        # every rank builds the same full tensors
        nl = wl.N // world
        sl = slice(rank * nl, (rank + 1) * nl)
        # round trip
        back = heads_to_seq(seq_to_heads(q[sl].contiguous()))
        out[f"roundtrip{rank}"] = bool(torch.equal(back, q[sl]))
        # the head slice this rank receives is the global head range
        hl = wl.heads // world
        out[f"heads{rank}"] = bool(torch.equal(seq_to_heads(k[sl].contiguous()), k[:, rank * hl:(rank + 1) * hl]))

        def layer(qh, kh, vh, head0):                 # oracle pipeline on this rank's heads (test only)
            hs = list(range(head0, head0 + qh.shape[1]))
            res = O.pipeline(qh.double().numpy(), kh.double().numpy(), vh.double().numpy(),
                             [wl.schemes[0].as_tuple()], [0] * len(hs), [wl.head_tau[h] for h in hs],
                             [False] * len(hs))
            return torch.from_numpy(res["out"]).to(qh.dtype)
        y = head_sharded_layer(q[sl].contiguous(), k[sl].contiguous(), v[sl].contiguous(), layer)
        out[f"y{rank}"] = y.numpy()
    finally:
        dist.destroy_process_group()


def test_head_sharded_layer_two_ranks():
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    mp.start_processes(_worker, args=(2, _port(), out), nprocs=2, join=True, start_method="spawn")
    assert out["roundtrip0"] and out["roundtrip1"] and out["heads0"] and out["heads1"]
    wl = _wl()
    q, k, v = make_qkv(wl)
    ref = O.pipeline(q.double().numpy(), k.double().numpy(), v.double().numpy(), [wl.schemes[0].as_tuple()],
                     [0] * wl.heads, wl.head_tau, [False] * wl.heads)["out"]
    y = np.concatenate([out["y0"], out["y1"]], axis=0)
    assert np.allclose(y, ref.astype(np.float32), atol=1e-6)
