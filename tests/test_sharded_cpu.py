"""Head-sharded execution on CPU: the LPT head plan, and the layer run across
two and three gloo ranks against the same layer run on one process (the
per-head work is the oracle here).  The cases carry a mixed head policy with
the dense heads first, a head count the world size does not divide, a token
count it does not divide, and text tokens that every rank holds whole."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle as O
from input_adaptive_block_b200.sharded import head_costs, plan_heads, token_splits
from spade_workloads import Scheme, Workload, get_config, make_qkv


def _port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _imbalance(costs, plan):
    loads = [sum(costs[h] for h in p) for p in plan]
    return max(loads) / (sum(loads) / len(loads)) - 1.0


def test_plan_covers_every_head_once_and_is_deterministic():
    costs = [5.0, 1.0, 1.0, 3.0, 3.0, 2.0, 2.0]
    for world in (1, 2, 3, 4, 9):
        plan = plan_heads(costs, world)
        assert len(plan) == world
        assert sorted(h for p in plan for h in p) == list(range(len(costs)))
        assert all(p == sorted(p) for p in plan)
        assert plan == plan_heads(costs, world)
    assert plan_heads(costs, 9)[8] == []                     # more ranks than heads: some hold none
    # LPT by hand, heads in the order 0 (5), 3, 4 (3), 5, 6 (2), 1, 2 (1): h0 -> r0 (5), h3 -> r1 (3),
    # h4 -> r1 (6), h5 -> r0 (7), h6 -> r1 (8), h1 -> r0 (8), h2 -> r0 (tie at 8: lower rank; 9)
    assert plan_heads(costs, 2) == [[0, 1, 2, 5], [3, 4, 6]]


@pytest.mark.parametrize("world", [2, 3, 4])
def test_plan_balances_the_mixed_policy(world):
    """Heads 0-12 of the mixed configuration are dense: an equal split of
    contiguous heads would give rank 0 all of them.  The cost plan keeps
    every rank within 10 % of the mean, from tau alone and from measured
    kept fractions."""
    wl = get_config("mixed")
    table = [(wl.head_scheme[h], wl.head_tau[h], wl.head_dense[h]) for h in range(wl.heads)]
    contiguous = [list(range(r * wl.heads // world, (r + 1) * wl.heads // world)) for r in range(world)]
    for kept in (None, [None if wl.head_dense[h] else 0.35 + 0.01 * (h % 7) for h in range(wl.heads)]):
        costs = head_costs(wl.N, wl.text_tokens, wl.d, table, kept)
        plan = plan_heads(costs, world)
        assert _imbalance(costs, plan) <= 0.10, (world, plan)
        assert _imbalance(costs, plan) <= _imbalance(costs, contiguous)
    # with the measured fractions (sparse heads at ~40 % of a dense head) the
    # contiguous split is far off and the plan is not
    assert _imbalance(costs, contiguous) > 0.2 and _imbalance(costs, plan) < 0.05
    dense_ranks = {r for r, p in enumerate(plan) for h in p if wl.head_dense[h]}
    assert len(dense_ranks) == world                        # the dense heads are spread over every rank


def test_head_costs():
    table = [(0, 0.9, True), (0, 0.9, False), (0, 2.0, False)]
    c = head_costs(100, 28, 64, table)
    full = 4 * 64 * 128 * 128
    assert c == [full, pytest.approx(0.9 * full), full]
    assert head_costs(100, 28, 64, table, [None, 0.25, None])[1] == pytest.approx(0.25 * full)
    assert token_splits(10, 3) == [4, 3, 3] and token_splits(9, 3) == [3, 3, 3]


def _wl():
    # 7 heads: 2 dense first, then sparse heads of two schemes; 10*8*8 = 640
    # video tokens (not divisible by 3) and 40 text tokens
    T, H, W, heads = 10, 8, 8, 7
    return Workload("sharded", 51, T, H, W, heads, 16, "f32", 40,
                    (Scheme(T, H, W, 2, 4, 4), Scheme(T, H, W, 1, 4, 8)),
                    (0, 0, 0, 1, 0, 1, 1), (0.9, 0.9, 0.8, 0.9, 0.85, 0.95, 0.8),
                    (True, True, False, False, False, False, False))


def _oracle_layer(wl, q, k, v, heads):
    """The oracle pipeline on the given global heads (q, k, v hold only them)."""
    res = O.pipeline(q.double().numpy(), k.double().numpy(), v.double().numpy(),
                     [s.as_tuple() for s in wl.schemes], [wl.head_scheme[h] for h in heads],
                     [wl.head_tau[h] for h in heads], [wl.head_dense[h] for h in heads], wl.text_tokens)
    return torch.from_numpy(res["out"]).to(q.dtype)


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from input_adaptive_block_b200.sharded import head_sharded_layer, heads_to_seq, seq_to_heads
        wl = _wl()
        q, k, v = make_qkv(wl)                        # every rank builds the same full tensors
        table = [(wl.head_scheme[h], wl.head_tau[h], wl.head_dense[h]) for h in range(wl.heads)]
        plan = plan_heads(head_costs(wl.N, wl.text_tokens, wl.d, table), world)
        splits = token_splits(wl.N, world)
        s0 = sum(splits[:rank])
        rows = list(range(s0, s0 + splits[rank])) + list(range(wl.N, wl.n_total))

        def local(x):                                 # this rank's video slice + the text rows
            return x[rows].contiguous()
        # the forward exchange gives every token of this rank's heads ...
        got = seq_to_heads(local(k), plan, splits, wl.text_tokens)
        out[f"heads{rank}"] = bool(torch.equal(got, k[:, plan[rank]]))
        # ... and the inverse exchange undoes it
        back = heads_to_seq(seq_to_heads(local(q), plan, splits, wl.text_tokens), plan, splits, wl.heads,
                            wl.text_tokens)
        out[f"roundtrip{rank}"] = bool(torch.equal(back, local(q)))
        y = head_sharded_layer(local(q), local(k), local(v),
                               lambda qh, kh, vh, hs: _oracle_layer(wl, qh, kh, vh, hs), plan, splits,
                               wl.text_tokens)
        out[f"y{rank}"] = y.numpy()
        out[f"plan{rank}"] = plan
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_head_sharded_layer(world):
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    mp.start_processes(_worker, args=(world, _port(), out), nprocs=world, join=True, start_method="spawn")
    for r in range(world):
        assert out[f"heads{r}"] and out[f"roundtrip{r}"], r
        assert out[f"plan{r}"] == out["plan0"]
    wl = _wl()
    q, k, v = make_qkv(wl)
    ref = _oracle_layer(wl, q, k, v, list(range(wl.heads))).numpy()
    splits = token_splits(wl.N, world)
    video = np.concatenate([out[f"y{r}"][: splits[r]] for r in range(world)], axis=0)
    assert np.allclose(video, ref[: wl.N], atol=1e-6)
    for r in range(world):                            # every rank holds the text output of every head
        assert np.allclose(out[f"y{r}"][splits[r]:], ref[wl.N:], atol=1e-6)
    # the plan is not the contiguous split: the two dense heads sit on different ranks
    assert all(len([h for h in out["plan0"][r] if wl.head_dense[h]]) <= 1 for r in range(world))
