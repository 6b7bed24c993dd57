"""Sequence-sharded (context-parallel) parallel form over torch.distributed.

The parallel form's state after a run of chunks is the initial state plus a sum of
independent per-chunk deltas ("Test-Time Training with KV Binding Is Secretly Linear
Attention", 前置知识 / 前缀扫描; the In-Place TTT notes' context-parallel form, section 3.4):
so a sequence split into contiguous shards, one per rank, needs only each earlier shard's
total delta. Rank r

  1. forms its shard's total delta T_r: the state-only library call from a zero state (the
     key side and the scan; no query side, no outputs);
  2. all-gathers the totals (one collective of [B, H, m, h] fp32 per rank, NCCL over
     NVLink on GPUs);
  3. runs its shard from W1 plus T_0 + ... + T_{r-1}: the library adds the gathered totals
     of the earlier ranks into each (batch, head)'s initial state inside its scan kernel,
     reusing the chunk deltas of step 1 (left in the shared workspace), so the key side
     runs once per shard. The outputs are those of the unsharded sequence, and on the last
     rank the final state is the sequence's final state.

Every rank issues the same collective in the same order. Shards must be whole chunks (N_r a
multiple of chunk on every rank but the last).
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def gather_totals(total: torch.Tensor, group=None) -> torch.Tensor:
    """The totals of every rank, in rank order: [world, *total.shape]. All ranks call it."""
    world = dist.get_world_size(group)
    flat = torch.empty(world * total.numel(), dtype=total.dtype, device=total.device)
    dist.all_gather_into_tensor(flat, total.contiguous().reshape(-1), group=group)
    return flat.view((world,) + tuple(total.shape))


def la_parallel_fwd_cp(q, k, v, eta, W0, W2, W1, chunk, *, order="update_apply", sign=1,
                       w_in_layout=0, w1_layout=0, group=None, shard_fn=None):
    """Parallel form on this rank's contiguous shard of the sequence (q, k, v [B,H,N_r,h],
    eta [B,H,N_r]); W0, W2, W1 per head as for ``layer.la_parallel_fwd``. Returns (out
    [B,H,N_r,h], the state after this shard [B,H,m,h] (W1's layout); on the last rank that
    is the sequence's final state). ``shard_fn`` runs one shard on this device (defaults to
    the library: its state-only pass, then the outputs pass that reuses its chunk deltas)."""
    reuse = shard_fn is None
    if shard_fn is None:
        from . import layer
        shard_fn = layer.la_parallel_fwd_shard
    N_r = q.shape[2]
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    if rank < world - 1 and N_r % chunk != 0:
        raise ValueError(f"shard of {N_r} tokens is not a whole number of {chunk}-token chunks")
    m = W1.shape[1] if w1_layout == 0 else W1.shape[2]
    kw = dict(order=order, sign=sign, w_in_layout=w_in_layout, w1_layout=w1_layout, m=m)
    if not reuse:
        _, total = shard_fn(q, k, v, eta, W0, W2, None, chunk, state_only=True, **kw)
        totals = gather_totals(total, group)
        prior = totals[:rank] if rank > 0 else None
        return shard_fn(q, k, v, eta, W0, W2, W1, chunk, prior=prior, **kw)
    from . import abi
    desc = layer.parallel_desc(q, W1, chunk, order, sign, w_in_layout, w1_layout)
    ws = layer.workspace(abi.ttt_workspace_bytes(desc, abi.TTT_PATH_PARALLEL), q.device)
    _, total = layer.la_parallel_fwd_shard(q, k, v, eta, W0, W2, None, chunk, state_only=True,
                                           ws=ws, **kw)
    totals = gather_totals(total, group)
    prior = totals[:rank] if rank > 0 else None
    try:
        return layer.la_parallel_fwd_shard_outputs(
            q, W1, chunk, ws, prior=prior, order=order, sign=sign, w_in_layout=w_in_layout,
            w1_layout=w1_layout)
    except abi.TTTError as e:
        if e.status != abi.TTT_ERR_UNSUPPORTED:   # the sequential schedule keeps no deltas
            raise
    return layer.la_parallel_fwd_shard(q, k, v, eta, W0, W2, W1, chunk, prior=prior, ws=ws,
                                       **kw)
