"""Sequence-sharded (context-parallel) parallel form over torch.distributed.

The parallel form's state after a run of chunks is the initial state plus a sum of
independent per-chunk deltas ("Test-Time Training with KV Binding Is Secretly Linear
Attention", 前置知识 / 前缀扫描; the In-Place TTT notes' context-parallel form): so a
sequence split into contiguous shards, one per rank, needs only each earlier shard's total
delta. Rank r

  1. runs the layer on its shard from a zero state; the final state is its total delta T_r
     (the outputs of this pass are discarded);
  2. all-gathers the totals and forms the exclusive prefix P_r = sum_{r' < r} T_r';
  3. runs the layer on its shard from W1 + P_r: its outputs are those of the unsharded
     sequence, and on the last rank the final state is the sequence's final state.

Every rank issues the same collective (one all_gather of [B, H, m, h] fp32) in the same
order. Shards must be whole chunks (N_r a multiple of chunk on every rank but the last).
Pass 1 costs a full layer call; a state-only first pass would halve the extra work.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def exclusive_prefix(total: torch.Tensor, group=None) -> torch.Tensor:
    """Sum of `total` over the ranks below this one (zeros on rank 0). All ranks call it."""
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    parts = [torch.empty_like(total) for _ in range(world)]
    dist.all_gather(parts, total.contiguous(), group=group)
    out = torch.zeros_like(total)
    for r in range(rank):
        out += parts[r]
    return out


def la_parallel_fwd_cp(q, k, v, eta, W0, W2, W1, chunk, *, order="update_apply", sign=1,
                       group=None, local_fn=None):
    """Parallel form on this rank's contiguous shard of the sequence (q, k, v [B,H,N_r,h],
    eta [B,H,N_r]); W0, W2, W1 per head as for ``layer.la_parallel_fwd``. Returns (out
    [B,H,N_r,h], the state after this shard [B,H,m,h]; on the last rank that is the
    sequence's final state). ``local_fn`` runs the single-device layer (defaults to the
    library's ``layer.la_parallel_fwd``)."""
    if local_fn is None:
        from . import layer
        local_fn = layer.la_parallel_fwd
    N_r = q.shape[2]
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    if rank < world - 1 and N_r % chunk != 0:
        raise ValueError(f"shard of {N_r} tokens is not a whole number of {chunk}-token chunks")
    zero = torch.zeros_like(W1)
    _, total = local_fn(q, k, v, eta, W0, W2, zero, chunk, order=order, sign=sign)
    prefix = exclusive_prefix(total, group)            # [B, H, m, h]
    # per-(b, head) initial states: the library takes per-head W1, so run per batch entry
    B = q.shape[0]
    outs, states = [], []
    for b in range(B):
        W1b = (W1 + prefix[b]).contiguous()
        o, s = local_fn(q[b:b + 1].contiguous(), k[b:b + 1].contiguous(),
                        v[b:b + 1].contiguous(), eta[b:b + 1].contiguous(), W0, W2, W1b, chunk,
                        order=order, sign=sign)
        outs.append(o)
        states.append(s)
    return torch.cat(outs, 0), torch.cat(states, 0)
