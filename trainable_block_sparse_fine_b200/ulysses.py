"""Ulysses resharding around the VSA2 attention: sequence shards <-> head shards.

A model that keeps its activations sharded along the sequence gives each of P ranks a contiguous
1/P of the cube-major tokens of every head. VSA2 needs whole sequences per head: the softmaxes of
Eq. 2, 6 and 12 run over all tiles of a head, and the TopK budget of Eq. 8-9 is per sequence.
Ulysses sequence parallelism gathers the full sequence on each rank and shards the heads, and
because VSA2 gives every head the same budget, the work stays balanced ("Improving Video Sparse
Attention with Fine-grained Router and Sparse Rebasing", App. E). So:
  1. one all-to-all regroups the sequence shards by head: rank g then holds heads
     [g*H/P, (g+1)*H/P) over the full sequence;
  2. the per-head path (router, TopK, both branches, merge) runs with no further exchange;
  3. a second all-to-all returns the output to sequence shards.
The exchange is `torch.distributed.all_to_all_single` (NCCL on GPUs, gloo on CPU). Each
regrouping is a permutation of elements, so its gradient is the inverse regrouping; both are
autograd functions, and a backward pass through `ulysses_attention` runs the two all-to-alls in
reverse. No arithmetic of the method happens here.
"""
from __future__ import annotations

from typing import Callable, Sequence

import torch
import torch.distributed as dist


def _world(group) -> int:
    return dist.get_world_size(group)


def _seq_to_heads(x: torch.Tensor, group) -> torch.Tensor:
    P = _world(group)
    B, H, Ls = x.shape[:3]
    rest = tuple(x.shape[3:])
    if H % P:
        raise ValueError(f"{H} heads do not split over {P} ranks")
    send = x.reshape(B, P, H // P, Ls, *rest).transpose(0, 1).contiguous()  # [P dst, B, H/P, Ls, ...]
    recv = torch.empty_like(send)
    dist.all_to_all_single(recv, send, group=group)  # recv[r] = rank r's shard of my heads
    dims = (1, 2, 0, 3) + tuple(range(4, 4 + len(rest)))
    return recv.permute(*dims).reshape(B, H // P, P * Ls, *rest).contiguous()


def _heads_to_seq(y: torch.Tensor, group) -> torch.Tensor:
    P = _world(group)
    B, Hg, L = y.shape[:3]
    rest = tuple(y.shape[3:])
    if L % P:
        raise ValueError(f"{L} tokens do not split over {P} ranks")
    send = y.reshape(B, Hg, P, L // P, *rest)
    send = send.permute(2, 0, 1, 3, *range(4, 4 + len(rest))).contiguous()  # [P dst, B, Hg, L/P, ...]
    recv = torch.empty_like(send)
    dist.all_to_all_single(recv, send, group=group)  # recv[g] = my shard of head group g
    dims = (1, 0, 2, 3) + tuple(range(4, 4 + len(rest)))
    return recv.permute(*dims).reshape(B, P * Hg, L // P, *rest).contiguous()


class _SeqToHeads(torch.autograd.Function):
    @staticmethod
    def forward(ctx, x, group):
        ctx.group = group
        return _seq_to_heads(x.contiguous(), group)

    @staticmethod
    def backward(ctx, g):
        return _heads_to_seq(g.contiguous(), ctx.group), None


class _HeadsToSeq(torch.autograd.Function):
    @staticmethod
    def forward(ctx, y, group):
        ctx.group = group
        return _heads_to_seq(y.contiguous(), group)

    @staticmethod
    def backward(ctx, g):
        return _seq_to_heads(g.contiguous(), ctx.group), None


def seq_to_heads(x: torch.Tensor, group=None) -> torch.Tensor:
    """[B, H, L/P, ...] (this rank's sequence shard of every head) -> [B, H/P, L, ...] (this rank's
    head group over the whole sequence, shards concatenated in rank order). Differentiable."""
    return _SeqToHeads.apply(x, group)


def heads_to_seq(y: torch.Tensor, group=None) -> torch.Tensor:
    """Inverse of seq_to_heads: [B, H/P, L, ...] -> [B, H, L/P, ...]. Differentiable."""
    return _HeadsToSeq.apply(y, group)


def ulysses_attention(attn_fn: Callable[..., torch.Tensor], seq_shards: Sequence[torch.Tensor],
                      group=None) -> torch.Tensor:
    """Run `attn_fn` on whole sequences of this rank's head group and return its output as this
    rank's sequence shard.

    seq_shards: tensors laid out [B, H, L/P, ...] (Q, K, V, and e.g. the gate logits of Eq. 13),
    each regrouped with seq_to_heads before the call. attn_fn receives them as [B, H/P, L, ...]
    and returns [B, H/P, L, D] (for VSA2: `lambda q, k, v, g: vsa2_attention(q, k, v, g, engine)`
    with an engine built for H/P heads and the full grid)."""
    full = [seq_to_heads(t, group) for t in seq_shards]
    return heads_to_seq(attn_fn(*full), group)
