"""Host logic of the sequence-sharded parallel form with 2 and 3 gloo ranks on the CPU: each
rank runs its shard (the fp64 oracle stands in for the GPU library's shard call here: the
state-only total from a zero state, then the shard from W1 plus the gathered totals of the
earlier ranks); the outputs and the last rank's final state equal the unsharded run. The
GPU tests run the same decomposition through the library on one device."""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from oracle import ttt_oracle as O
from ttt_inputs import WORKLOADS, make_layer_inputs


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _oracle_shard(q, k, v, eta, W0, W2, W1, chunk, *, prior=None, state_only=False,
                  order="update_apply", sign=1, w_in_layout=0, w1_layout=0, m=None):
    """One shard on one device, computed by the oracle (torch CPU tensors in and out): the
    parallel form from W1 (zeros when None) plus the sum of the prior totals."""
    assert w_in_layout == 0 and w1_layout == 0
    ordv = O.UPDATE_APPLY if order == "update_apply" else O.APPLY_UPDATE
    B, H = q.shape[:2]
    h = q.shape[3]
    m = W1.shape[1] if m is None else m
    S0 = np.zeros((B, H, m, h)) if W1 is None else np.repeat(W1.numpy()[None], B, axis=0)
    if prior is not None:
        S0 = S0 + prior.numpy().sum(axis=0)
    outs, Ss = [], []
    for b in range(B):
        o, S = O.la_parallel_batched(q.numpy()[b:b + 1], k.numpy()[b:b + 1], v.numpy()[b:b + 1],
                                     eta.numpy()[b:b + 1], W0.numpy(), W2.numpy(), S0[b], chunk,
                                     order=ordv, sign=sign)
        outs.append(o)
        Ss.append(S)
    out = torch.from_numpy(np.concatenate(outs, 0))
    return (None if state_only else out), torch.from_numpy(np.concatenate(Ss, 0))


def _inputs():
    wl = WORKLOADS["tiny"].scaled(B=2, H=2, N=192, h=8, m=12, chunk=32)
    x = make_layer_inputs(wl, seed=5)
    return wl, {n: torch.from_numpy(np.asarray(x[n], np.float64)) for n in
                ("q", "k", "v", "eta", "W0", "W2", "W1")}


def _rank_main(rank, world, port, order, queue):
    torch.set_num_threads(1)
    import torch.distributed as dist
    from test_weight_layers_ttt_b200.context_parallel import la_parallel_fwd_cp
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    wl, x = _inputs()
    # whole chunks on every rank but the last, which takes the ragged rest
    n = wl.N // world // wl.chunk * wl.chunk
    sl = slice(rank * n, (rank + 1) * n if rank < world - 1 else wl.N)
    out, S = la_parallel_fwd_cp(x["q"][:, :, sl], x["k"][:, :, sl], x["v"][:, :, sl],
                                x["eta"][:, :, sl], x["W0"], x["W2"], x["W1"], wl.chunk,
                                order=order, shard_fn=_oracle_shard)
    dist.barrier()
    dist.destroy_process_group()
    queue.put((rank, out.numpy(), S.numpy()))


@pytest.mark.parametrize("order,world", [("update_apply", 2), ("apply_update", 2),
                                         ("update_apply", 3)])
def test_shards_equal_the_unsharded_sequence(order, world):
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, order, queue))
             for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((queue.get(timeout=180) for _ in procs), key=lambda t: t[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    wl, x = _inputs()
    ordv = O.UPDATE_APPLY if order == "update_apply" else O.APPLY_UPDATE
    ref, Sref = O.la_parallel_batched(*(x[n].numpy() for n in ("q", "k", "v", "eta", "W0",
                                                                "W2", "W1")),
                                      wl.chunk, order=ordv)
    out = np.concatenate([r[1] for r in res], axis=2)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12 * np.abs(ref).max())
    np.testing.assert_allclose(res[-1][2], Sref, rtol=0, atol=1e-12 * np.abs(Sref).max())


def test_single_rank_is_the_single_device_layer():
    import torch.distributed as dist
    from test_weight_layers_ttt_b200.context_parallel import la_parallel_fwd_cp
    port = _free_port()
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    store = dist.TCPStore("127.0.0.1", port, 1, True, timeout=datetime.timedelta(seconds=30))
    dist.init_process_group("gloo", rank=0, world_size=1, store=store)
    try:
        wl, x = _inputs()
        # one rank is the last rank: a ragged shard is allowed and the result is the
        # single-device one
        out, S = la_parallel_fwd_cp(x["q"][:, :, :100], x["k"][:, :, :100], x["v"][:, :, :100],
                                    x["eta"][:, :, :100], x["W0"], x["W2"], x["W1"], wl.chunk,
                                    shard_fn=_oracle_shard)
        ref, Sref = O.la_parallel_batched(*(x[n][:, :, :100].numpy() for n in ("q", "k", "v",
                                                                               "eta")),
                                          x["W0"].numpy(), x["W2"].numpy(), x["W1"].numpy(),
                                          wl.chunk)
        out, S, ref, Sref = (np.asarray(t) for t in (out, S, ref, Sref))
        assert np.allclose(out, ref, rtol=0, atol=1e-12) and np.allclose(S, Sref, rtol=0,
                                                                         atol=1e-12)
    finally:
        dist.destroy_process_group()
