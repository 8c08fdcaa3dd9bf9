"""Linear attention with the sequence split across ranks (one process per GPU).

Rank r of a group of P holds tokens [r*n, (r+1)*n) of every head: q, k, v,
dO of shape [B, H, n, D] (shards may differ in length).  The states S and z
are sums over tokens ("Efficient Transformers Survey", Proposition "Linear
Attention via Kernel Decomposition", Statement; "Why It Matters": the state
is carried along the sequence), so the only exchange is one state record
per head and rank: an all-gather of [B, H, D*D + D] float32 records,
followed by a sum over the ranks before (causal prefix), after (the
backward's causal suffix) or all of them (non-causal), taken by
la_state_range_sum.  Every other step is this rank's own kernel calls
(``api.la_state_local``, ``la_forward_sp``, ``la_backward_sp_dq``,
``la_backward_sp_dkdv``); the records cross ranks through
``torch.distributed`` (NCCL on GPUs; with the gloo backend they are staged
through host memory).

    o, g = forward(q, k, v, causal, phi, group)
    dq, dk, dv = backward(q, k, v, dO, o, g, causal, phi, group)

Ranks must call both in the same order (they are collectives).
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import api


def prefix_range(rank: int, world: int, causal: bool) -> tuple[int, int]:
    """Ranks whose records a rank's forward (and dQ step) starts from."""
    return (0, rank) if causal else (0, world)


def suffix_range(rank: int, world: int, causal: bool) -> tuple[int, int]:
    """Ranks whose query-side records a rank's dK/dV step starts from."""
    return (rank + 1, world) if causal else (0, world)


def gather_records(rec: torch.Tensor, group=None) -> torch.Tensor:
    """All ranks' records in rank order: [P, *rec.shape]."""
    world = dist.get_world_size(group)
    staged = rec
    if dist.get_backend(group) == "gloo" and rec.is_cuda:
        staged = rec.cpu()
    out = torch.empty((world * staged.shape[0], *staged.shape[1:]), dtype=staged.dtype,
                      device=staged.device)
    dist.all_gather_into_tensor(out, staged.contiguous(), group=group)
    out = out.view(world, *staged.shape)
    return out.to(rec.device) if out.device != rec.device else out


def exchange(rec: torch.Tensor, rng: tuple[int, int], group=None, combine=None) -> torch.Tensor:
    """Sum of the gathered records of ranks rng[0] .. rng[1]-1.  ``combine``
    (gathered, lo, hi) -> sum defaults to the library's la_state_range_sum."""
    gathered = gather_records(rec, group)
    combine = combine or (lambda g, lo, hi: api.la_state_range_sum(g, lo, hi))
    return combine(gathered, *rng)


def forward(q, k, v, causal: bool = True, phi="elu1", group=None):
    """This rank's outputs o [B, H, n, D] and denominators g [B, H, n]."""
    rank, world = dist.get_rank(group), dist.get_world_size(group)
    B, H, n, _ = q.shape
    rec = api.la_state_local(k, v, phi)
    state_in = exchange(rec, prefix_range(rank, world, causal), group)
    g = torch.empty((B, H, n), dtype=torch.float32, device=q.device)
    o = api.la_forward_sp(q, k, v, state_in, causal, phi, g=g)
    return o, g


def backward(q, k, v, dO, o, g, causal: bool = True, phi="elu1", group=None):
    """dq, dk, dv of this rank's shard for L = sum over all ranks of
    sum(dO * O), given this rank's forward o and g."""
    rank, world = dist.get_rank(group), dist.get_world_size(group)
    rec = api.la_state_local(k, v, phi, centred=True)
    state_in = exchange(rec, prefix_range(rank, world, causal), group)
    dq, rrec, ws = api.la_backward_sp_dq(q, k, v, dO, o, g, state_in, causal, phi)
    r_in = exchange(rrec, suffix_range(rank, world, causal), group)
    dk, dv = api.la_backward_sp_dkdv(q, k, v, dO, g, r_in, ws, causal, phi)
    return dq, dk, dv


class SequenceParallelLinearAttention(torch.autograd.Function):
    """torch autograd wrapper of forward/backward above (every rank of the
    group calls it on its shard; the backward exchanges records too)."""

    @staticmethod
    def forward(ctx, q, k, v, causal=True, phi="elu1", group=None):
        q, k, v = q.contiguous(), k.contiguous(), v.contiguous()
        o, g = forward(q, k, v, causal, phi, group)
        ctx.save_for_backward(q, k, v, o, g)
        ctx.causal, ctx.phi, ctx.group = causal, phi, group
        return o

    @staticmethod
    def backward(ctx, dO):
        q, k, v, o, g = ctx.saved_tensors
        dq, dk, dv = backward(q, k, v, dO.contiguous(), o, g, ctx.causal, ctx.phi, ctx.group)
        return dq, dk, dv, None, None, None
