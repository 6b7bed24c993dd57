"""The allocation-free parallel entry point against the regular one.

ttt_la_parallel_fwd_noalloc serves callers that cannot allocate device memory (a plug-in
whose host runtime owns every allocation, a real-time loop that must not call cudaMalloc
after start-up). It takes no workspace and runs in the library's built-in scratch. Here it
must give the regular entry point's results on two calls in a row with different inputs
(so nothing left in the shared scratch by one call leaks into the next), and it must turn
down problems larger than its scratch before enqueueing anything.

This file is collected last on purpose; it also passes when run alone in a fresh process.
"""
import numpy as np
import pytest
import torch

from test_weight_layers_ttt_b200 import abi, layer
from ttt_inputs import WORKLOADS, make_layer_inputs

from gpu_helpers import TOL, dev, host, rel

pytestmark = pytest.mark.gpu


def _problem(dtype, B, H, N, h, m, chunk, seed):
    base = WORKLOADS["tiny" if dtype == "fp32" else "lm"]
    wl = base.scaled(B=B, H=H, N=N, h=h, m=m, chunk=chunk, dtype=dtype)
    x = make_layer_inputs(wl, seed=seed)
    td = torch.bfloat16 if dtype == "bf16" else torch.float32
    return ([dev(x[n], td) for n in ("q", "k", "v")] +
            [dev(x[n]) for n in ("eta", "W0", "W2", "W1")])


def _regular(args, chunk, order):
    q = args[0]
    desc = layer.parallel_desc(q, args[6], chunk, order)
    out = torch.empty_like(q)
    S = torch.empty((q.shape[0], q.shape[1], desc.m, desc.h), dtype=torch.float32,
                    device="cuda")
    ws = layer.workspace(abi.ttt_workspace_bytes(desc, abi.TTT_PATH_PARALLEL), "cuda")
    abi.ttt_la_parallel_fwd(desc, *args, out, S, ws)
    return desc, out, S


def _noalloc(desc, args):
    q = args[0]
    out = torch.full_like(q, float("nan"))
    S = torch.full((q.shape[0], q.shape[1], desc.m, desc.h), float("nan"),
                   dtype=torch.float32, device="cuda")
    abi.ttt_la_parallel_fwd_noalloc(desc, *args, out, S)
    return out, S


@pytest.mark.parametrize("dtype,shape,order", [
    ("bf16", (2, 3, 1000, 64, 200, 256), "update_apply"),
    ("fp32", (1, 2, 203, 12, 20, 50), "apply_update"),
])
def test_noalloc_matches_regular_entry_point_twice(dtype, shape, order):
    first = _problem(dtype, *shape, seed=71)
    second = _problem(dtype, *shape, seed=72)
    chunk = shape[-1]
    for args in (first, second):       # two calls in a row, different inputs
        desc, ref_out, ref_S = _regular(args, chunk, order)
        assert abi.ttt_workspace_bytes(desc, 0) <= abi.TTT_STATIC_SCRATCH_BYTES
        out, S = _noalloc(desc, args)
        abi.ttt_last_device_status()
        tol = TOL[dtype]
        assert rel(host(out), host(ref_out)) <= tol
        assert rel(host(S), host(ref_S)) <= tol
        assert np.isfinite(host(out)).all() and np.isfinite(host(S)).all()


def test_noalloc_rejects_problems_beyond_its_scratch():
    desc = abi.ttt_desc(B=2, H=4, N=32768, h=256, m=512, chunk=2048, dtype=abi.TTT_DTYPE_BF16)
    assert abi.ttt_workspace_bytes(desc, 0) > abi.TTT_STATIC_SCRATCH_BYTES
    with pytest.raises(abi.TTTError) as ei:
        abi.ttt_la_parallel_fwd_noalloc(desc, 256, 256, 256, 256, 256, 256, 256, 256, None)
    assert ei.value.status == abi.TTT_ERR_WORKSPACE
    assert "built-in scratch" in abi.ttt_last_error_message()
