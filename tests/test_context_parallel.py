"""Host logic of the sequence-sharded parallel form with 2 gloo ranks on the CPU: each rank
runs the single-device layer (the fp64 oracle stands in for the GPU library here) on its
shard; the collective prefix makes the shards' outputs and the last rank's final state
equal to the unsharded run. The GPU test runs the same decomposition through the library
on one device."""
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


def _oracle_local(q, k, v, eta, W0, W2, W1, chunk, *, order="update_apply", sign=1):
    """The layer on one device, computed by the oracle (torch CPU tensors in and out)."""
    ordv = O.UPDATE_APPLY if order == "update_apply" else O.APPLY_UPDATE
    out, S = O.la_parallel_batched(q.numpy(), k.numpy(), v.numpy(), eta.numpy(), W0.numpy(),
                                   W2.numpy(), W1.numpy(), chunk, order=ordv, sign=sign)
    return torch.from_numpy(out), torch.from_numpy(S)


def _inputs():
    wl = WORKLOADS["tiny"].scaled(B=2, H=2, N=192, h=8, m=12, chunk=32)
    x = make_layer_inputs(wl, seed=5)
    return wl, {n: torch.from_numpy(np.asarray(x[n], np.float64)) for n in
                ("q", "k", "v", "eta", "W0", "W2", "W1")}


def _rank_main(rank, world, port, order, queue):
    import torch.distributed as dist
    from test_weight_layers_ttt_b200.context_parallel import la_parallel_fwd_cp
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    wl, x = _inputs()
    n = wl.N // world
    sl = slice(rank * n, (rank + 1) * n)
    out, S = la_parallel_fwd_cp(x["q"][:, :, sl], x["k"][:, :, sl], x["v"][:, :, sl],
                                x["eta"][:, :, sl], x["W0"], x["W2"], x["W1"], wl.chunk,
                                order=order, local_fn=_oracle_local)
    dist.barrier()
    dist.destroy_process_group()
    queue.put((rank, out.numpy(), S.numpy()))


@pytest.mark.parametrize("order", ["update_apply", "apply_update"])
def test_two_shards_equal_the_unsharded_sequence(order):
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, order, queue)) for r in range(2)]
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
    out = np.concatenate([res[0][1], res[1][1]], axis=2)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12 * np.abs(ref).max())
    np.testing.assert_allclose(res[1][2], Sref, rtol=0, atol=1e-12 * np.abs(Sref).max())


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
                                    local_fn=_oracle_local)
        ref, Sref = _oracle_local(x["q"][:, :, :100], x["k"][:, :, :100], x["v"][:, :, :100],
                                  x["eta"][:, :, :100], x["W0"], x["W2"], x["W1"], wl.chunk)
        assert torch.allclose(out, ref, rtol=0, atol=1e-12) and torch.allclose(S, Sref)
    finally:
        dist.destroy_process_group()
