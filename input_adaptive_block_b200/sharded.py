"""Head-sharded execution of one layer across ranks (one process per GPU).

Every step of the executor -- block summaries, estimate, index search,
attention -- reads one head's Q/K/V only (technical summary, Methodology 3,
"Head Grouping": heads are the unit the executor groups and schedules), so a
layer whose tokens are sharded across ranks (sequence parallelism, the usual
layout of a DiT between attention layers) is run by re-sharding it by heads:

  1. plan: heads are assigned to ranks by their attention cost, longest
     first, each to the least-loaded rank (LPT).  A dense head costs
     4 (N+text)^2 d FLOPs, a sparse head that times its kept fraction (from a
     previous call's kept lists, or tau as the prior), so a rank holding the
     dense heads of a mixed policy gets fewer heads.  Any number of heads and
     ranks works.
  2. exchange: one all_to_all_single sends each rank's token slice of every
     other rank's heads (NCCL over NVLink on GPUs); the text tokens, which
     every rank holds whole, need no exchange.
  3. the rank runs the layer on its heads (the grouped launch on the GPU).
  4. a second all_to_all_single returns each rank's token slice of every
     head, text rows included (each rank then holds the text output of every
     head, as it holds the text input).

The exchanges are layout moves around the attention, with no arithmetic to
fuse them with; the per-head work is untouched.
"""
from __future__ import annotations

from typing import Callable, List, Optional, Sequence

import torch
import torch.distributed as dist

__all__ = ["head_costs", "kept_fraction_from_counts", "plan_heads", "token_splits", "seq_to_heads",
           "heads_to_seq", "head_sharded_layer", "grouped_attn_layer"]


def head_costs(n_video: int, text_tokens: int, d: int, table: Sequence,
               kept_fraction: Optional[Sequence[Optional[float]]] = None) -> List[float]:
    """Attention FLOPs of each head of a layer: 4 d (N + text)^2 for a dense
    head; for a sparse head, that times its kept fraction of key blocks --
    kept_fraction[h] when given (e.g. kept_fraction_from_counts of an earlier
    call on the same layer), else tau, the fraction a flat block distribution
    would keep.  table: (scheme, tau, dense) rows, one per head."""
    n = n_video + text_tokens
    full = 4.0 * d * n * n
    out = []
    for h, (_, tau, dense) in enumerate(table):
        if dense:
            out.append(full)
            continue
        f = kept_fraction[h] if kept_fraction is not None and kept_fraction[h] is not None else min(float(tau), 1.0)
        out.append(full * max(float(f), 1e-6))
    return out


def kept_fraction_from_counts(cnt: torch.Tensor) -> float:
    """Kept fraction of key blocks of one head from its kept counts [nb]."""
    nb = cnt.numel()
    return float(cnt.sum().item()) / float(nb * nb)


def plan_heads(costs: Sequence[float], world: int) -> List[List[int]]:
    """LPT assignment: heads by descending cost (ties: lower head first), each
    to the rank with the least assigned cost (ties: lower rank).  Returns the
    ascending head list of every rank; deterministic, so every rank computes
    the same plan from the same costs."""
    if world < 1:
        raise ValueError("world must be >= 1")
    load = [0.0] * world
    plan: List[List[int]] = [[] for _ in range(world)]
    for h in sorted(range(len(costs)), key=lambda i: (-costs[i], i)):
        r = min(range(world), key=lambda j: (load[j], j))
        plan[r].append(h)
        load[r] += costs[h]
    return [sorted(p) for p in plan]


def token_splits(n_video: int, world: int) -> List[int]:
    """Video tokens of each rank's contiguous slice: the first n % world ranks
    hold one more."""
    base, extra = divmod(n_video, world)
    return [base + (1 if r < extra else 0) for r in range(world)]


def seq_to_heads(x_local: torch.Tensor, plan: Sequence[Sequence[int]], splits: Sequence[int],
                 text_tokens: int = 0, group=None) -> torch.Tensor:
    """This rank's token slice [splits[rank] + text, heads, d] (video rows,
    then the text rows every rank holds) -> [N + text, len(plan[rank]), d]:
    every token of this rank's heads, in global token order."""
    rank, world = dist.get_rank(group), dist.get_world_size(group)
    nl = splits[rank]
    d = x_local.shape[2]
    mine = list(plan[rank])
    video = x_local[:nl]
    send = torch.cat([video[:, list(plan[r])].reshape(-1) for r in range(world)])
    recv = torch.empty(sum(splits) * len(mine) * d, dtype=x_local.dtype, device=x_local.device)
    dist.all_to_all_single(recv, send.contiguous(),
                           output_split_sizes=[splits[s] * len(mine) * d for s in range(world)],
                           input_split_sizes=[nl * len(plan[r]) * d for r in range(world)], group=group)
    out = recv.view(sum(splits), len(mine), d)
    if text_tokens:
        out = torch.cat([out, x_local[nl:nl + text_tokens][:, mine]], dim=0)
    return out.contiguous()


def heads_to_seq(y_heads: torch.Tensor, plan: Sequence[Sequence[int]], splits: Sequence[int], heads: int,
                 text_tokens: int = 0, group=None) -> torch.Tensor:
    """Inverse exchange: this rank's heads over every token
    [N + text, len(plan[rank]), d] -> its token slice of every head
    [splits[rank] + text, heads, d] (text rows of every head included)."""
    rank, world = dist.get_rank(group), dist.get_world_size(group)
    mine = list(plan[rank])
    nl = splits[rank]
    d = y_heads.shape[2]
    starts = [sum(splits[:r]) for r in range(world)]
    text = y_heads[sum(splits):]
    # to rank r: its video slice of my heads, then the text rows of my heads
    send = torch.cat([torch.cat([y_heads[starts[r]:starts[r] + splits[r]], text], dim=0).reshape(-1)
                      for r in range(world)])
    recv = torch.empty((nl + text_tokens) * heads * d, dtype=y_heads.dtype, device=y_heads.device)
    sizes_in = [(splits[r] + text_tokens) * len(mine) * d for r in range(world)]
    sizes_out = [(nl + text_tokens) * len(plan[s]) * d for s in range(world)]
    dist.all_to_all_single(recv, send.contiguous(), output_split_sizes=sizes_out, input_split_sizes=sizes_in,
                           group=group)
    out = torch.empty(nl + text_tokens, heads, d, dtype=y_heads.dtype, device=y_heads.device)
    off = 0
    for s in range(world):
        hs = list(plan[s])
        n = (nl + text_tokens) * len(hs) * d
        if hs:
            out[:, hs] = recv[off:off + n].view(nl + text_tokens, len(hs), d)
        off += n
    return out


def head_sharded_layer(q_local: torch.Tensor, k_local: torch.Tensor, v_local: torch.Tensor,
                       layer_fn: Callable[[torch.Tensor, torch.Tensor, torch.Tensor, Sequence[int]], torch.Tensor],
                       plan: Sequence[Sequence[int]], splits: Sequence[int], text_tokens: int = 0,
                       group=None) -> torch.Tensor:
    """Runs layer_fn(q, k, v, heads) on this rank's heads (plan[rank], every
    token, text rows last) and returns the output in the token slicing of the
    inputs ([splits[rank] + text, heads, d]).  plan and splits must be the
    same on every rank (plan_heads, token_splits)."""
    rank = dist.get_rank(group)
    heads = q_local.shape[1]
    mine = list(plan[rank])
    q_h, k_h, v_h = (seq_to_heads(t, plan, splits, text_tokens, group) for t in (q_local, k_local, v_local))
    if mine:
        out_h = layer_fn(q_h, k_h, v_h, mine)
    else:
        out_h = q_h.new_empty(q_h.shape)
    return heads_to_seq(out_h, plan, splits, heads, text_tokens, group)


def grouped_attn_layer(schemes: Sequence, table: Sequence, text_tokens: int = 0,
                       workspace: Optional[torch.Tensor] = None, **kw):
    """layer_fn for head_sharded_layer that runs spade_grouped_attn on the
    rank's heads; table holds one (scheme, tau, dense) row per GLOBAL head.
    A workspace, when given, must hold grouped_workspace_bytes of the rank's
    rows."""
    from . import api

    def fn(q, k, v, heads):
        rows = [table[h] for h in heads]
        return api.grouped_attn(q, k, v, schemes, rows, text_tokens, workspace=workspace, **kw)
    return fn
