"""GPU tests of the library's debug checks and of the single tensor-core engine in bf16 mode.

* With TTT_CHECK_GUARDS | TTT_CHECK_FINITE on, every form runs on shifted workspace layouts
  (guards between regions) and still matches the oracle, with a clean device status.
* A guard changed from the host between two checks, and a NaN fed to the layer, are
  reported as TTT_ERR_DEVICE (failures made on the host: nothing faults or hangs).
* No contraction of a bf16 call runs on the CUDA cores: every traced GEMM of every form in
  bf16 mode ran on the tcgen05 engine.
"""
import numpy as np
import pytest
import torch

from oracle import ttt_oracle as O
from test_weight_layers_ttt_b200 import abi, layer
from ttt_inputs import WORKLOADS, make_layer_inputs

from gpu_helpers import TOL, dev, host, rel

pytestmark = pytest.mark.gpu


def _inputs(B, H, N, h, m, chunk, seed, dtype="bf16"):
    wl = WORKLOADS["lm"].scaled(B=B, H=H, N=N, h=h, m=m, chunk=chunk, dtype=dtype)
    x = make_layer_inputs(wl, seed=seed)
    td = torch.bfloat16 if dtype == "bf16" else torch.float32
    g = [dev(x[n], td) for n in ("q", "k", "v")] + [dev(x[n]) for n in ("eta", "W0", "W2", "W1")]
    return x, g


@pytest.fixture
def checks():
    abi.ttt_set_debug_checks(abi.TTT_CHECK_GUARDS | abi.TTT_CHECK_FINITE)
    try:
        yield
    finally:
        abi.ttt_set_debug_checks(0)


def _guard_pattern():
    i = np.arange(64, dtype=np.uint64)
    return (np.uint64(0x7E57C0DE) ^ ((i * np.uint64(0x9E3779B1)) & np.uint64(0xFFFFFFFF))
            ).astype(np.uint32)


def _guard_offsets(ws):
    """Byte offsets of the guards in a workspace (16-byte aligned runs of the pattern)."""
    words = ws.cpu().numpy().view(np.uint32)
    pat = _guard_pattern()
    cand = np.nonzero(words[: len(words) - 63] == pat[0])[0]
    return [int(c) * 4 for c in cand if c % 4 == 0 and np.array_equal(words[c:c + 64], pat)]


def test_every_form_is_clean_and_correct_with_guards(checks):
    x, (q, k, v, eta, W0, W2, W1) = _inputs(2, 2, 1000, 128, 256, 256, seed=71)
    ref, Sref = O.la_parallel_batched(x["q"], x["k"], x["v"], x["eta"], x["W0"], x["W2"],
                                      x["W1"], 256)
    out, S = layer.la_parallel_fwd(q, k, v, eta, W0, W2, W1, 256)
    abi.ttt_last_device_status()
    assert rel(host(out), ref) <= TOL["bf16"] and rel(host(S), Sref) <= TOL["bf16"]
    alpha = torch.full((2, 2, 4), 0.8, dtype=torch.float32, device="cuda")
    ref, Wref, _ = O.lact_recurrent_batched(x["q"], x["k"], x["v"], x["eta"], x["W0"], x["W2"],
                                            x["W1"], 256, update=("W1",),
                                            alpha=host(alpha), ns_steps=5)
    out, S = layer.la_parallel_momentum_fwd(q, k, v, eta, W0, W2, W1, 256, alpha=alpha,
                                            ns_steps=5)
    abi.ttt_last_device_status()
    assert rel(host(out), ref) <= TOL["bf16"] and rel(host(S), Wref["W1"]) <= TOL["bf16"]
    ref, Wref, _ = O.lact_recurrent_batched(x["q"], x["k"], x["v"], x["eta"], x["W0"], x["W2"],
                                            x["W1"], 256, renorm=True)
    out, Wf, _ = layer.lact_recurrent_fwd(q, k, v, eta, W0, W2, W1, 256, renorm=True)
    abi.ttt_last_device_status()
    assert rel(host(out), ref) <= TOL["bf16"]
    dO = torch.randn_like(q)
    grads = layer.la_parallel_bwd(q, k, v, eta, W0, W2, W1, dO, 256)
    abi.ttt_last_device_status()
    assert all(torch.isfinite(g.float()).all() for g in grads)
    S0 = W1[:, :128, :].contiguous()
    refl, _ = O.linear_attention_batched(x["q"], x["k"], x["v"], x["eta"], host(S0), 256)
    outl, _ = layer.linear_attn_fwd(q, k, v, eta, S0, 256)
    abi.ttt_last_device_status()
    assert rel(host(outl), refl) <= TOL["bf16"]


def test_overwritten_guard_is_reported(checks):
    x, (q, k, v, eta, W0, W2, W1) = _inputs(1, 2, 512, 128, 256, 128, seed=72)
    desc = layer.parallel_desc(q, W1, 128)
    ws = layer.workspace(abi.ttt_workspace_bytes(desc, abi.TTT_PATH_PARALLEL), "cuda")
    layer.la_parallel_fwd(q, k, v, eta, W0, W2, W1, 128, ws=ws)
    abi.ttt_last_device_status()
    offs = _guard_offsets(ws)
    assert len(offs) == 6           # one in front, one after each of the five regions
    abi.ttt_debug_check_workspace(desc, abi.TTT_PATH_PARALLEL, ws)
    abi.ttt_last_device_status()    # intact
    ws[offs[3] + 100] ^= 0x5A       # a stray byte written just past the deltas
    abi.ttt_debug_check_workspace(desc, abi.TTT_PATH_PARALLEL, ws)
    with pytest.raises(abi.TTTError) as ei:
        abi.ttt_last_device_status()
    assert ei.value.status == abi.TTT_ERR_DEVICE and "guard" in str(ei.value)
    # the next call rewrites the guards; the word was cleared by the read
    layer.la_parallel_fwd(q, k, v, eta, W0, W2, W1, 128, ws=ws)
    abi.ttt_last_device_status()


def test_non_finite_output_is_reported(checks):
    x, (q, k, v, eta, W0, W2, W1) = _inputs(1, 1, 256, 64, 128, 64, seed=73)
    q[0, 0, 70, 3] = float("nan")
    layer.la_parallel_fwd(q, k, v, eta, W0, W2, W1, 64)
    with pytest.raises(abi.TTTError) as ei:
        abi.ttt_last_device_status()
    assert ei.value.status == abi.TTT_ERR_DEVICE and "NaN" in str(ei.value)
    q[0, 0, 70, 3] = 0.0
    layer.la_parallel_fwd(q, k, v, eta, W0, W2, W1, 64)
    abi.ttt_last_device_status()


def test_bf16_calls_run_every_contraction_on_the_tensor_cores():
    x, (q, k, v, eta, W0, W2, W1) = _inputs(1, 2, 1000, 128, 256, 256, seed=74)
    alpha = torch.full((1, 2, 4), 0.8, dtype=torch.float32, device="cuda")
    abi.ttt_trace_enable(4096)
    try:
        layer.la_parallel_fwd(q, k, v, eta, W0, W2, W1, 256)
        layer.la_parallel_fwd(q, q, v, eta, W0, W2, W1, 256, order="apply_update")
        layer.la_parallel_momentum_fwd(q, k, v, eta, W0, W2, W1, 256, alpha=alpha, ns_steps=5)
        layer.lact_recurrent_fwd(q, k, v, eta, W0, W2, W1, 256, renorm=True, alpha=alpha,
                                 ns_steps=5)
        layer.la_parallel_bwd(q, k, v, eta, W0, W2, W1, torch.randn_like(q), 256)
        layer.linear_attn_fwd(q, k, v, eta, W1[:, :128].contiguous(), 256)
        torch.cuda.synchronize()
        names = [abi.ttt_trace_get(i)[0] for i in range(abi.ttt_trace_count())]
    finally:
        abi.ttt_trace_disable()
    abi.ttt_last_device_status()
    assert any(n.endswith("@tcgen05") for n in names)
    assert not [n for n in names if n.endswith("@simt")]
