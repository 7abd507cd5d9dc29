"""Head-sharded execution of one layer across ranks (one process per GPU).

The executor's work is independent per head (every step -- summaries,
estimate, selection, attention -- reads one head's Q/K/V only), so a layer
whose tokens are sharded across ranks (sequence parallelism, the usual
layout of a DiT between attention layers) is run by re-sharding it by
heads: one all-to-all turns each rank's [N/world, heads, d] token slice into
[N, heads/world, d] (all tokens of this rank's heads), the rank runs the
layer on its heads (the grouped launch on the GPU), and a second all-to-all
returns the output to the token slicing.  The exchange is
torch.distributed's all_to_all_single (NCCL over NVLink on GPUs); the
per-head work itself is untouched.

Limits: N and heads divisible by the world size; no text tokens (the text
tail would have to be replicated, which the token slicing does not give).
"""
from __future__ import annotations

from typing import Callable, Optional, Sequence

import torch
import torch.distributed as dist

__all__ = ["seq_to_heads", "heads_to_seq", "head_sharded_layer", "grouped_attn_layer"]


def _world(group) -> int:
    return dist.get_world_size(group)


def seq_to_heads(x_local: torch.Tensor, group=None) -> torch.Tensor:
    """[N/world, heads, d] (this rank's token slice, slices in rank order)
    -> [N, heads/world, d] (every token, this rank's contiguous head range)."""
    world = _world(group)
    nl, heads, d = x_local.shape
    if heads % world:
        raise ValueError(f"heads={heads} not divisible by world={world}")
    hl = heads // world
    # chunk j (heads j*hl..) goes to rank j: [world, nl, hl, d]
    send = x_local.reshape(nl, world, hl, d).permute(1, 0, 2, 3).contiguous()
    recv = torch.empty_like(send)
    dist.all_to_all_single(recv, send, group=group)
    # recv[j] = rank j's token slice of my heads -> tokens in rank order
    return recv.reshape(world * nl, hl, d)


def heads_to_seq(y_heads: torch.Tensor, group=None) -> torch.Tensor:
    """Inverse of seq_to_heads: [N, heads/world, d] -> [N/world, heads, d]."""
    world = _world(group)
    n, hl, d = y_heads.shape
    if n % world:
        raise ValueError(f"N={n} not divisible by world={world}")
    nl = n // world
    send = y_heads.reshape(world, nl, hl, d).contiguous()      # token slice j goes to rank j
    recv = torch.empty_like(send)
    dist.all_to_all_single(recv, send, group=group)
    # recv[j] = my token slice of rank j's heads -> heads in rank order
    return recv.permute(1, 0, 2, 3).reshape(nl, world * hl, d)


def head_sharded_layer(q_local: torch.Tensor, k_local: torch.Tensor, v_local: torch.Tensor,
                       layer_fn: Callable[[torch.Tensor, torch.Tensor, torch.Tensor, int], torch.Tensor],
                       group=None) -> torch.Tensor:
    """Runs layer_fn(q, k, v, head0) on this rank's heads (all tokens) and
    returns the output in the token slicing of the inputs.  head0 is the
    first global head index this rank holds."""
    world = _world(group)
    rank = dist.get_rank(group)
    heads = q_local.shape[1]
    q_h, k_h, v_h = (seq_to_heads(t, group) for t in (q_local, k_local, v_local))
    out_h = layer_fn(q_h, k_h, v_h, rank * (heads // world))
    return heads_to_seq(out_h, group)


def grouped_attn_layer(schemes: Sequence, table: Sequence, workspace: Optional[torch.Tensor] = None, **kw):
    """layer_fn for head_sharded_layer that runs spade_grouped_attn on the
    rank's heads; table holds one (scheme, tau, dense) row per GLOBAL head."""
    from . import api

    def fn(q, k, v, head0):
        hl = q.shape[1]
        rows = list(table[head0: head0 + hl])
        return api.grouped_attn(q, k, v, schemes, rows, 0, workspace=workspace, **kw)
    return fn
