"""bench.py host logic without a GPU: the max-over-ranks reduction on a
world-size-2 gloo group, the JSON line's contract fields, and the kept-pair
FLOP count (against the oracle's own pair count)."""
import json
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import oracle as O
from spade_workloads import Scheme, Workload, get_config


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        got = bench.reduce_max(10.0 + rank * 5.5, world)
        out[rank] = got
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_reduce_max_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    port = _free_port()
    mp.start_processes(_worker, args=(2, port, out), nprocs=2, join=True, start_method="spawn")
    assert out[0] == out[1] == 15.5


def test_reduce_max_single_rank_is_identity():
    assert bench.reduce_max(3.25, 1) == 3.25


def test_assemble_line_contract():
    line = bench.assemble_line(value=500.0, unit="TFLOP/s", n_gpus=2, steps=10, warmup=3, ms=12.5,
                               config={"workload": "x"}, extra={"roofline": {"frac": 0.3}})
    s = json.loads(json.dumps(line))
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "roofline"):
        assert key in s
    assert s["scaling"] == "weak" and s["higher_is_better"] is True and s["vs_baseline"] is None


@pytest.mark.parametrize("text", [0, 37])
def test_kept_pair_flops_matches_oracle_pair_count(text):
    T, H, W = 3, 5, 7
    sc = Scheme(T, H, W, 2, 4, 4)
    wl = Workload("w", 5, T, H, W, 2, 16, "bf16", text, (sc, Scheme(1, 1, T * H * W, 1, 1, 128)),
                  (0, 1), (0.9, 1.0), (False, True))
    rng = np.random.default_rng(0)
    kept0 = [sorted(set([i] + list(rng.choice(sc.nb, 3, replace=False)))) for i in range(sc.nb)]
    flops = bench.kept_pair_flops(wl, [[np.array(k) for k in kept0], None])
    pairs = O.kept_token_pairs([sc.as_tuple(), wl.schemes[1].as_tuple()], [kept0, None], text)
    assert flops == 4 * wl.d * pairs
    assert (bench._valid_counts(sc) == O.valid_counts(sc.as_tuple())).all()


def test_launches_per_step():
    """Kernels of one grouped call, counted from the head table."""
    wl = get_config("mixed")
    table = [(wl.head_scheme[h], wl.head_tau[h], wl.head_dense[h]) for h in range(wl.heads)]
    # dense heads: no selection; two sparse schemes, one run of heads each: (1 + 2) x 2, + work list + attention
    assert bench.launches_per_step(table, 3) == 8
    assert bench.launches_per_step([(0, 0.9, False)] * 40, 1) == 5
    # a run of heads broken in two by a dense head: two summarize launches
    assert bench.launches_per_step([(0, 0.9, False), (0, 0.9, True), (0, 0.9, False)], 1) == 6
    assert bench.launches_per_step([(0, 0.9, True)] * 3, 1) == 2
