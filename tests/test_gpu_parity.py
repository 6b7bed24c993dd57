"""GPU parity of the C-ABI path against the fp64 oracle on small seeded inputs.

Sizes are chosen so that the oracle finishes in seconds while the GPU kernels still run
several tiles with ragged edges (m and N not multiples of the 128-row tiles, a short last
chunk, N < chunk). Tolerance: max|err| / max|ref| <= 1e-4 (fp32 mode) / 2e-2 (bf16 mode).
"""
import numpy as np
import pytest
import torch

from oracle import ttt_oracle as O
from test_weight_layers_ttt_b200 import abi, layer
from ttt_inputs import WORKLOADS, bf16_round, make_layer_inputs, make_inplace_inputs

from gpu_helpers import TOL, dev, host, rel, torch_dtype

pytestmark = pytest.mark.gpu

ORD = {"update_apply": O.UPDATE_APPLY, "apply_update": O.APPLY_UPDATE}


def layer_inputs(kind, dtype, B, H, N, h, m, chunk, seed, momentum=False):
    base = WORKLOADS["tiny" if kind == "tiny" else "lm"]
    wl = base.scaled(B=B, H=H, N=N, h=h, m=m, chunk=chunk, dtype=dtype, momentum=momentum)
    return wl, make_layer_inputs(wl, seed=seed)


def gpu_args(inp, dtype):
    td = torch_dtype(dtype)
    return (dev(inp["q"], td), dev(inp["k"], td), dev(inp["v"], td), dev(inp["eta"]),
            dev(inp["W0"]), dev(inp["W2"]), dev(inp["W1"]))


# ----------------------------------------------------------------------------- parallel
PAR_CASES = [
    # kind, dtype, B, H, N, h, m, chunk
    ("tiny", "fp32", 1, 1, 256, 16, 16, 64),
    ("tiny", "fp32", 2, 2, 203, 12, 20, 50),
    ("lm", "bf16", 2, 3, 1000, 64, 200, 256),
    ("lm", "bf16", 1, 2, 640, 128, 512, 128),
    ("lm", "bf16", 1, 1, 300, 256, 256, 512),
]


@pytest.mark.parametrize("case", PAR_CASES, ids=lambda c: "-".join(map(str, c)))
@pytest.mark.parametrize("order", ["update_apply", "apply_update"])
def test_parallel_matches_oracle(case, order):
    kind, dtype, B, H, N, h, m, chunk = case
    wl, inp = layer_inputs(kind, dtype, B, H, N, h, m, chunk, seed=1000 + N)
    ref, Sref = O.la_parallel_batched(inp["q"], inp["k"], inp["v"], inp["eta"], inp["W0"],
                                      inp["W2"], inp["W1"], chunk, order=ORD[order])
    q, k, v, eta, W0, W2, W1 = gpu_args(inp, dtype)
    out, S = layer.la_parallel_fwd(q, k, v, eta, W0, W2, W1, chunk, order=order)
    abi.ttt_last_device_status()
    tol = TOL[dtype]
    assert rel(host(out), ref) <= tol
    assert rel(host(S), Sref) <= tol
    # the state-driven part alone: start from a zero state
    Z = np.zeros_like(inp["W1"])
    ref0, Sref0 = O.la_parallel_batched(inp["q"], inp["k"], inp["v"], inp["eta"], inp["W0"],
                                        inp["W2"], Z, chunk, order=ORD[order])
    out0, S0 = layer.la_parallel_fwd(q, k, v, eta, W0, W2, dev(Z), chunk, order=order)
    assert rel(host(out0), ref0) <= tol
    assert rel(host(S0), Sref0) <= tol


@pytest.mark.parametrize("case", [
    # B, H, N, h, m, chunk: odd number of 128-column phi blocks and more tiles than SMs;
    # ragged m (zero-padded phi block, state rows past m) and ragged N (the last tile's
    # rows partly, or a 32-row store box wholly, past N)
    (2, 4, 4096, 128, 384, 512),
    (1, 2, 1000, 256, 200, 256),
    (1, 3, 1100, 256, 512, 512),
    (2, 1, 700, 128, 256, 384),
], ids=lambda c: "-".join(map(str, c)))
def test_fused_query_side_matches_oracle_and_unfused(case, monkeypatch):
    """phi(Q_c) S_c computed with phi kept in shared memory (h = 128 or 256, chunk a
    multiple of 128) against the oracle and against the unfused feature + output GEMMs."""
    B, H, N, h, m, chunk = case
    wl, inp = layer_inputs("lm", "bf16", B, H, N, h, m, chunk, seed=90 + N)
    ref, Sref = O.la_parallel_batched(inp["q"], inp["k"], inp["v"], inp["eta"], inp["W0"],
                                      inp["W2"], inp["W1"], chunk)
    q, k, v, eta, W0, W2, W1 = gpu_args(inp, "bf16")
    monkeypatch.delenv("TTT_NO_FUSED_APPLY", raising=False)
    abi.ttt_trace_enable(256)
    try:
        fused, Sf = layer.la_parallel_fwd(q, k, v, eta, W0, W2, W1, chunk)
        torch.cuda.synchronize()
        names = [abi.ttt_trace_get(i)[0] for i in range(abi.ttt_trace_count())]
    finally:
        abi.ttt_trace_disable()
    assert "fused_apply@tcgen05" in names
    monkeypatch.setenv("TTT_NO_FUSED_APPLY", "1")
    plain, Sp = layer.la_parallel_fwd(q, k, v, eta, W0, W2, W1, chunk)
    abi.ttt_last_device_status()
    assert rel(host(fused), ref) <= TOL["bf16"] and rel(host(Sf), Sref) <= TOL["bf16"]
    assert rel(host(fused), host(plain)) <= 1e-2
    assert torch.equal(Sf, Sp)


@pytest.mark.parametrize("case", [
    # B, H, N, h, m, chunk, order, sign: more (b, head, chunk) pairs than CTA groups,
    # ragged m (zero-padded phi block), a chunk that is not a multiple of the 128-token
    # tile, a short last chunk, N < chunk
    (2, 4, 4096, 256, 512, 512, "update_apply", 1),
    (1, 3, 1000, 128, 200, 200, "apply_update", -1),
    (2, 2, 1300, 256, 384, 256, "update_apply", 1),
    (1, 2, 100, 128, 256, 256, "update_apply", 1),
], ids=lambda c: "-".join(map(str, c)))
def test_fused_key_side_matches_oracle_and_unfused(case, monkeypatch):
    """Delta S_c = sign phi(K_c)^T diag(eta_c) V_c computed with phi(K) eta kept in shared
    memory (h = 128 or 256) against the oracle and against the unfused feature and
    state-delta GEMMs."""
    B, H, N, h, m, chunk, order, sign = case
    wl, inp = layer_inputs("lm", "bf16", B, H, N, h, m, chunk, seed=190 + N)
    ref, Sref = O.la_parallel_batched(inp["q"], inp["k"], inp["v"], inp["eta"], inp["W0"],
                                      inp["W2"], inp["W1"], chunk, order=ORD[order], sign=sign)
    Z = np.zeros_like(inp["W1"])
    ref0, Sref0 = O.la_parallel_batched(inp["q"], inp["k"], inp["v"], inp["eta"], inp["W0"],
                                        inp["W2"], Z, chunk, order=ORD[order], sign=sign)
    q, k, v, eta, W0, W2, W1 = gpu_args(inp, "bf16")
    monkeypatch.delenv("TTT_NO_FUSED_DELTA", raising=False)
    fused, Sf = layer.la_parallel_fwd(q, k, v, eta, W0, W2, W1, chunk, order=order, sign=sign)
    fused0, Sf0 = layer.la_parallel_fwd(q, k, v, eta, W0, W2, dev(Z), chunk, order=order,
                                        sign=sign)
    monkeypatch.setenv("TTT_NO_FUSED_DELTA", "1")
    plain, Sp = layer.la_parallel_fwd(q, k, v, eta, W0, W2, W1, chunk, order=order, sign=sign)
    abi.ttt_last_device_status()
    assert rel(host(fused), ref) <= TOL["bf16"] and rel(host(Sf), Sref) <= TOL["bf16"]
    assert rel(host(fused0), ref0) <= TOL["bf16"] and rel(host(Sf0), Sref0) <= TOL["bf16"]
    assert rel(host(Sf) - host(W1)[None], host(Sp) - host(W1)[None]) <= 1e-2
    assert rel(host(fused), host(plain)) <= 1e-2


@pytest.mark.parametrize("case", [
    # B, H, N, h, m, chunk, order, sign, w1_layout: ragged last chunk, both state layouts
    (2, 2, 1000, 128, 256, 256, "update_apply", 1, 0),
    (1, 3, 700, 64, 192, 128, "apply_update", -1, 1),
], ids=lambda c: "-".join(map(str, c)))
def test_sequential_schedule_matches_oracle_and_prefix(case, monkeypatch):
    """The parallel form's sequential schedule (one fp32 state per (b, head); per chunk an
    apply GEMM on its bf16 copy and an update GEMM into it) against the oracle and against
    the prefix schedule, with a zero initial state too (the state-driven part alone)."""
    B, H, N, h, m, chunk, order, sign, lay = case
    wl, inp = layer_inputs("lm", "bf16", B, H, N, h, m, chunk, seed=290 + N)
    q, k, v, eta, W0, W2, W1 = gpu_args(inp, "bf16")
    W1d = W1.transpose(1, 2).contiguous() if lay else W1

    def run(W):
        return layer.la_parallel_fwd(q, k, v, eta, W0, W2, W, chunk, order=order, sign=sign,
                                     w1_layout=lay)

    def st(S):
        return np.swapaxes(host(S), 2, 3) if lay else host(S)

    monkeypatch.setenv("TTT_SEQUENTIAL", "1")
    out, S = run(W1d)
    out0, S0 = run(torch.zeros_like(W1d))
    monkeypatch.setenv("TTT_SEQUENTIAL", "0")
    pout, pS = run(W1d)
    abi.ttt_last_device_status()
    ref, Sref = O.la_parallel_batched(inp["q"], inp["k"], inp["v"], inp["eta"], inp["W0"],
                                      inp["W2"], inp["W1"], chunk, order=ORD[order], sign=sign)
    Z = np.zeros_like(inp["W1"])
    ref0, Sref0 = O.la_parallel_batched(inp["q"], inp["k"], inp["v"], inp["eta"], inp["W0"],
                                        inp["W2"], Z, chunk, order=ORD[order], sign=sign)
    assert rel(host(out), ref) <= TOL["bf16"] and rel(st(S), Sref) <= TOL["bf16"]
    assert rel(host(out0), ref0) <= TOL["bf16"] and rel(st(S0), Sref0) <= TOL["bf16"]
    assert rel(host(out), host(pout)) <= 1e-2 and rel(st(S), st(pS)) <= 1e-3


def test_parallel_ascent_equals_descent_with_negated_values():
    wl, inp = layer_inputs("lm", "bf16", 1, 2, 512, 64, 128, 128, seed=7)
    q, k, v, eta, W0, W2, W1 = gpu_args(inp, "bf16")
    a, Sa = layer.la_parallel_fwd(q, k, v, eta, W0, W2, W1, 128, sign=-1)
    d, Sd = layer.la_parallel_fwd(q, k, (-v).contiguous(), eta, W0, W2, W1, 128, sign=1)
    assert torch.equal(a, d) and torch.equal(Sa, Sd)


def test_parallel_edge_sizes():
    wl, inp = layer_inputs("lm", "bf16", 1, 2, 64, 64, 128, 128, seed=11)   # N < chunk
    q, k, v, eta, W0, W2, W1 = gpu_args(inp, "bf16")
    out, S = layer.la_parallel_fwd(q, k, v, eta, W0, W2, W1, 128)
    ref, Sref = O.la_parallel_batched(inp["q"], inp["k"], inp["v"], inp["eta"], inp["W0"],
                                      inp["W2"], inp["W1"], 128)
    assert rel(host(out), ref) <= TOL["bf16"] and rel(host(S), Sref) <= TOL["bf16"]
    # N = 0: no output rows, the final state is the initial one (per (b, head))
    e = torch.empty((1, 2, 0, 64), dtype=torch.bfloat16, device="cuda")
    eta0 = torch.empty((1, 2, 0), dtype=torch.float32, device="cuda")
    _, S0 = layer.la_parallel_fwd(e, e, e, eta0, W0, W2, W1, 128)
    assert torch.equal(S0[0], W1)
    # chunk = 1 (per-token) in fp32 mode
    wl, inp = layer_inputs("tiny", "fp32", 1, 1, 40, 8, 12, 1, seed=12)
    q, k, v, eta, W0, W2, W1 = gpu_args(inp, "fp32")
    out, S = layer.la_parallel_fwd(q, k, v, eta, W0, W2, W1, 1)
    ref, Sref = O.la_parallel_batched(inp["q"], inp["k"], inp["v"], inp["eta"], inp["W0"],
                                      inp["W2"], inp["W1"], 1)
    assert rel(host(out), ref) <= TOL["fp32"] and rel(host(S), Sref) <= TOL["fp32"]
    abi.ttt_last_device_status()


def test_parallel_rejects_misaligned_pointer_on_device():
    wl, inp = layer_inputs("lm", "bf16", 1, 1, 128, 64, 128, 64, seed=13)
    q, k, v, eta, W0, W2, W1 = gpu_args(inp, "bf16")
    desc = layer.parallel_desc(q, W1, 64)
    ws = layer.workspace(abi.ttt_workspace_bytes(desc, 0), "cuda")
    out = torch.empty_like(q)
    with pytest.raises(abi.TTTError) as ei:
        abi.ttt_la_parallel_fwd(desc, q.data_ptr() + 2, k, v, eta, W0, W2, W1, out, None, ws)
    assert ei.value.status == abi.TTT_ERR_INVALID_ARG


# ----------------------------------------------------------------------------- backward
BWD_CASES = [
    # kind, dtype, B, H, N, h, m, chunk, order, sign, with dS_final
    ("tiny", "fp32", 1, 2, 150, 16, 24, 40, "update_apply", 1, True),
    ("lm", "bf16", 2, 2, 1000, 128, 256, 256, "update_apply", 1, True),
    ("lm", "bf16", 1, 3, 640, 64, 192, 128, "apply_update", -1, False),
]


@pytest.mark.parametrize("case", BWD_CASES, ids=lambda c: "-".join(map(str, c)))
def test_parallel_backward_matches_oracle(case):
    """Every gradient of the parallel form (inputs, step sizes, weights summed over the batch)
    against the oracle's chain rule."""
    kind, dtype, B, H, N, h, m, chunk, order, sign, with_sf = case
    wl, inp = layer_inputs(kind, dtype, B, H, N, h, m, chunk, seed=5000 + N)
    rng = np.random.default_rng(N)
    dO = rng.standard_normal((B, H, N, h))
    if dtype == "bf16":
        dO = bf16_round(dO.astype(np.float32)).astype(np.float64)
    dSf = rng.standard_normal((B, H, m, h)) if with_sf else None
    ref = {key: [] for key in ("dq", "dk", "dv", "deta")}
    wsum = {key: 0.0 for key in ("dW0", "dW2", "dW1")}
    for b in range(B):
        for hd in range(H):
            g = O.la_parallel_backward(inp["q"][b, hd], inp["k"][b, hd], inp["v"][b, hd],
                                       inp["eta"][b, hd], inp["W0"][hd], inp["W2"][hd],
                                       inp["W1"][hd], dO[b, hd], chunk, order=ORD[order],
                                       sign=sign, dS_final=None if dSf is None else dSf[b, hd])
            for key in ref:
                ref[key].append(g[key])
            for key in wsum:
                wsum[key] = wsum[key] + np.eye(H)[hd][:, None, None] * g[key][None]
    q, k, v, eta, W0, W2, W1 = gpu_args(inp, dtype)
    td = torch_dtype(dtype)
    grads = layer.la_parallel_bwd(q, k, v, eta, W0, W2, W1, dev(dO, td), chunk, order=order,
                                  sign=sign, dS_final=None if dSf is None else dev(dSf))
    abi.ttt_last_device_status()
    tol = TOL[dtype]
    for key, got in zip(("dq", "dk", "dv", "deta"), grads[:4]):
        want = np.stack(ref[key]).reshape(host(got).shape)
        assert rel(host(got), want) <= tol, key
    for key, got in zip(("dW0", "dW2", "dW1"), grads[4:]):
        assert rel(host(got), wsum[key]) <= tol, key


# ----------------------------------------------------------------------------- identity features
LIN_CASES = [
    # dtype, B, H, N, h, chunk, s_layout, sign
    ("fp32", 1, 2, 200, 24, 48, 0, 1),
    ("bf16", 2, 2, 1000, 128, 256, 0, 1),
    ("bf16", 1, 3, 700, 64, 128, 1, -1),
]


@pytest.mark.parametrize("case", LIN_CASES, ids=lambda c: "-".join(map(str, c)))
@pytest.mark.parametrize("order", ["update_apply", "apply_update"])
def test_linear_attention_matches_oracle(case, order):
    """phi = identity (variants 3-6 of the simplification ladder): plain chunked linear
    attention with per-token eta, multi-tile and ragged last chunk, both state layouts."""
    dtype, B, H, N, h, chunk, s_layout, sign = case
    wl, inp = layer_inputs("lm", dtype, B, H, N, h, h, chunk, seed=3000 + N)
    S0 = inp["W1"]                        # [H, h, h]
    ref, Sref = O.linear_attention_batched(inp["q"], inp["k"], inp["v"], inp["eta"], S0, chunk,
                                           order=ORD[order], sign=sign)
    td = torch_dtype(dtype)
    q, k, v = (dev(inp[n], td) for n in ("q", "k", "v"))
    eta = dev(inp["eta"])
    S0_dev = dev(np.ascontiguousarray(np.swapaxes(S0, 1, 2)) if s_layout else S0)
    out, S = layer.linear_attn_fwd(q, k, v, eta, S0_dev, chunk, order=order, sign=sign,
                                   s_layout=s_layout)
    abi.ttt_last_device_status()
    Sh = host(S)
    if s_layout:
        Sh = np.swapaxes(Sh, 2, 3)
    assert rel(host(out), ref) <= TOL[dtype]
    assert rel(Sh, Sref) <= TOL[dtype]
    # state-driven part alone (zero initial state)
    Z = np.zeros_like(S0)
    ref0, Sref0 = O.linear_attention_batched(inp["q"], inp["k"], inp["v"], inp["eta"], Z, chunk,
                                             order=ORD[order], sign=sign)
    out0, S0r = layer.linear_attn_fwd(q, k, v, eta, dev(Z), chunk, order=order, sign=sign)
    assert rel(host(out0), ref0) <= TOL[dtype]


# ----------------------------------------------------------------------------- momentum + NS
MOM_CASES = [
    # kind, dtype, B, H, N, h, m, chunk, momentum, ns_steps
    ("tiny", "fp32", 1, 2, 200, 16, 24, 48, True, 5),      # CUDA-core Newton-Schulz
    ("lm", "bf16", 2, 1, 1000, 128, 256, 256, True, 5),    # tensor-core Newton-Schulz
    ("lm", "bf16", 1, 2, 640, 64, 192, 128, False, 5),
    ("lm", "bf16", 1, 2, 640, 64, 192, 128, True, 0),
    # bf16 with 136 x 256 matrices (over the one-CTA limit): three tf32 GEMMs per step,
    # K = 136 not a multiple of the 32-wide k-block (zero-filled tail)
    ("lm", "bf16", 1, 1, 512, 256, 136, 128, True, 3),
    # the lm shape: 256 x 512 matrices, five steps (the first reads the momentum itself,
    # normalised through per-matrix GEMM scales); one step (a scaled copy first)
    ("lm", "bf16", 1, 1, 1024, 256, 512, 256, True, 5),
    ("lm", "bf16", 1, 2, 512, 256, 512, 256, True, 1),
    # no momentum: the norms come from their own pass, not from the momentum scan
    ("lm", "bf16", 1, 1, 512, 256, 512, 256, False, 5),
]


@pytest.mark.parametrize("case", MOM_CASES, ids=lambda c: "-".join(map(str, c[:10])))
@pytest.mark.parametrize("order", ["update_apply", "apply_update"])
def test_parallel_momentum_matches_recurrent_oracle(case, order):
    """The parallel form with W1 momentum and Newton-Schulz equals the recurrent form with
    only W1 fast, the same momentum and steps and no renormalisation (oracle)."""
    kind, dtype, B, H, N, h, m, chunk, momentum, ns = case
    wl, inp = layer_inputs(kind, dtype, B, H, N, h, m, chunk, seed=4000 + N + h, momentum=True)
    ref, Wref, _ = O.lact_recurrent_batched(
        inp["q"], inp["k"], inp["v"], inp["eta"], inp["W0"], inp["W2"], inp["W1"], chunk,
        order=ORD[order], update=("W1",), alpha=inp["alpha"] if momentum else None,
        ns_steps=ns)
    q, k, v, eta, W0, W2, W1 = gpu_args(inp, dtype)
    alpha = dev(inp["alpha"]) if momentum else None
    out, S = layer.la_parallel_momentum_fwd(q, k, v, eta, W0, W2, W1, chunk, order=order,
                                            alpha=alpha, ns_steps=ns)
    abi.ttt_last_device_status()
    tol = TOL[dtype]
    assert rel(host(out), ref) <= tol
    assert rel(host(S), Wref["W1"]) <= tol
    init = inp["W1"][None].repeat(B, axis=0)
    assert rel(host(S) - init, Wref["W1"] - init) <= 5 * tol


def test_parallel_momentum_without_options_is_the_parallel_form():
    wl, inp = layer_inputs("lm", "bf16", 1, 2, 512, 64, 128, 128, seed=41)
    q, k, v, eta, W0, W2, W1 = gpu_args(inp, "bf16")
    a, Sa = layer.la_parallel_fwd(q, k, v, eta, W0, W2, W1, 128)
    b, Sb = layer.la_parallel_momentum_fwd(q, k, v, eta, W0, W2, W1, 128)
    assert torch.equal(a, b) and torch.equal(Sa, Sb)


# ----------------------------------------------------------------------------- context parallel
@pytest.mark.parametrize("case", [
    # B, H, N, h, m, chunk, shard bounds, order, q == k with the In-Place weight layouts
    (2, 2, 1024, 128, 256, 128, (0, 384, 768, 1024), "update_apply", False),
    (1, 3, 1000, 256, 200, 256, (0, 256, 768, 1000), "apply_update", False),
    (1, 1, 768, 128, 384, 128, (0, 256, 768), "apply_update", True),
], ids=lambda c: "-".join(map(str, c[:6])) + "-" + c[7] + ("-qk" if c[8] else ""))
def test_sequence_shards_through_the_library_match_the_oracle(case):
    """The context-parallel decomposition on one device, through the library's shard call:
    each shard's state-only total from a zero state, then each shard from W1 plus the
    totals of the shards before it. Outputs and the last shard's final state against the
    oracle on the unsharded sequence."""
    B, H, N, h, m, chunk, bounds, order, qk = case
    wl, inp = layer_inputs("lm", "bf16", B, H, N, h, m, chunk, seed=61 + N)
    if qk:
        inp["k"] = inp["q"]
    ref, Sref = O.la_parallel_batched(inp["q"], inp["k"], inp["v"], inp["eta"], inp["W0"],
                                      inp["W2"], inp["W1"], chunk, order=ORD[order])
    q, k, v, eta, W0, W2, W1 = gpu_args(inp, "bf16")
    lay = dict(order=order)
    if qk:   # In-Place layouts: gate / up as [m, h], the state transposed [h, m]
        k = q
        W0 = W0.transpose(1, 2).contiguous()
        W2 = W2.transpose(1, 2).contiguous()
        W1 = W1.transpose(1, 2).contiguous()
        lay.update(w_in_layout=1, w1_layout=1)
    shards = [slice(a, b) for a, b in zip(bounds[:-1], bounds[1:])]
    totals = []
    for sl in shards:
        args = [t[:, :, sl].contiguous() for t in (q, k, v, eta)]
        if qk:
            args[1] = args[0]
        _, T = layer.la_parallel_fwd_shard(*args, W0, W2, None, chunk, state_only=True, m=m,
                                           **lay)
        totals.append(T)
    outs = []
    for r, sl in enumerate(shards):
        args = [t[:, :, sl].contiguous() for t in (q, k, v, eta)]
        if qk:
            args[1] = args[0]
        prior = torch.stack(totals[:r]) if r else None
        o, S = layer.la_parallel_fwd_shard(*args, W0, W2, W1, chunk, prior=prior, **lay)
        outs.append(o)
    abi.ttt_last_device_status()
    Sh = host(S)
    if qk:
        Sh = np.swapaxes(Sh, 2, 3)
    assert rel(host(torch.cat(outs, 2)), ref) <= TOL["bf16"]
    assert rel(Sh, Sref) <= TOL["bf16"]
    # the state-only call's final state is the full call's (bit for bit when both take the
    # same key-side kernels; with q == k the full call forms phi once for both sides)
    _, Sfull = layer.la_parallel_fwd_shard(q, k, v, eta, W0, W2, W1, chunk, **lay)
    _, Sonly = layer.la_parallel_fwd_shard(q, k, v, eta, W0, W2, W1, chunk, state_only=True,
                                           m=m, **lay)
    if qk:
        assert rel(host(Sonly), host(Sfull)) <= 1e-3
    else:
        assert torch.equal(Sfull, Sonly)
    # each shard's outputs pass reusing the chunk deltas its state-only pass left in the
    # workspace: against the oracle, and (without q == k, where the full call forms phi once
    # for both sides) bit for bit the second full pass's outputs
    outs2 = []
    for r, sl in enumerate(shards):
        args = [t[:, :, sl].contiguous() for t in (q, k, v, eta)]
        if qk:
            args[1] = args[0]
        desc = layer.parallel_desc(args[0], W1, chunk, order=order,
                                   w_in_layout=lay.get("w_in_layout", 0),
                                   w1_layout=lay.get("w1_layout", 0))
        ws = layer.workspace(abi.ttt_workspace_bytes(desc, abi.TTT_PATH_PARALLEL), q.device)
        layer.la_parallel_fwd_shard(*args, W0, W2, None, chunk, state_only=True, m=m, ws=ws,
                                    **lay)
        prior = torch.stack(totals[:r]) if r else None
        o2, S2 = layer.la_parallel_fwd_shard_outputs(args[0], W1, chunk, ws, prior=prior, **lay)
        outs2.append(o2)
        if not qk:
            assert torch.equal(o2, outs[r])
    abi.ttt_last_device_status()
    assert rel(host(torch.cat(outs2, 2)), ref) <= TOL["bf16"]
    S2h = np.swapaxes(host(S2), 2, 3) if qk else host(S2)
    assert rel(S2h, Sref) <= TOL["bf16"]
    with pytest.raises(abi.TTTError):   # the outputs pass consumed the state-only record
        layer.la_parallel_fwd_shard_outputs(args[0], W1, chunk, ws, prior=prior, **lay)


def test_context_parallel_single_rank_nccl_matches_the_oracle():
    import datetime
    import socket
    import torch.distributed as dist
    from test_weight_layers_ttt_b200.context_parallel import la_parallel_fwd_cp
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    store = dist.TCPStore("127.0.0.1", port, 1, True, timeout=datetime.timedelta(seconds=30))
    dist.init_process_group("nccl", rank=0, world_size=1, store=store,
                            timeout=datetime.timedelta(seconds=60))
    try:
        wl, inp = layer_inputs("lm", "bf16", 1, 2, 512, 128, 256, 128, seed=62)
        q, k, v, eta, W0, W2, W1 = gpu_args(inp, "bf16")
        out, S = la_parallel_fwd_cp(q, k, v, eta, W0, W2, W1, 128)
        ref, Sref = O.la_parallel_batched(inp["q"], inp["k"], inp["v"], inp["eta"], inp["W0"],
                                          inp["W2"], inp["W1"], 128)
        assert rel(host(out), ref) <= TOL["bf16"] and rel(host(S), Sref) <= TOL["bf16"]
    finally:
        dist.destroy_process_group()

# ----------------------------------------------------------------------------- recurrent
REC_CASES = [
    # kind, dtype, B, H, N, h, m, chunk, opts
    ("tiny", "fp32", 1, 1, 256, 16, 16, 64, dict()),
    ("tiny", "fp32", 1, 2, 150, 16, 24, 40, dict(renorm=True, momentum=True, ns_steps=5)),
    ("lm", "bf16", 1, 2, 768, 64, 128, 256, dict(renorm=True)),
    ("lm", "bf16", 2, 1, 600, 128, 256, 256, dict(renorm=True, momentum=True, ns_steps=5)),
    ("lm", "bf16", 1, 2, 512, 64, 192, 128, dict(update_mask=abi.TTT_UPDATE_W1)),
    ("lm", "bf16", 1, 1, 512, 128, 64, 256, dict(update_mask=5, ns_steps=5)),
    # ragged matrices for the tensor-core Newton-Schulz (zero padding inside the CTA)
    ("lm", "bf16", 1, 2, 320, 40, 200, 96, dict(renorm=True, momentum=True, ns_steps=5)),
    # min(h, m) > 128: bf16 mode runs Newton-Schulz as three tf32 GEMMs per step; 3 steps
    ("lm", "bf16", 1, 1, 256, 256, 136, 128, dict(ns_steps=3)),
]


@pytest.mark.parametrize("case", REC_CASES, ids=lambda c: "-".join(map(str, c[:8])))
@pytest.mark.parametrize("order", ["update_apply", "apply_update"])
def test_recurrent_matches_oracle(case, order):
    kind, dtype, B, H, N, h, m, chunk, opts = case
    momentum = opts.get("momentum", False)
    wl, inp = layer_inputs(kind, dtype, B, H, N, h, m, chunk, seed=2000 + N, momentum=momentum)
    mask = opts.get("update_mask", 7)
    upd = tuple(n for bit, n in ((1, "W0"), (2, "W1"), (4, "W2")) if mask & bit)
    ref, Wref, Mref = O.lact_recurrent_batched(
        inp["q"], inp["k"], inp["v"], inp["eta"], inp["W0"], inp["W2"], inp["W1"], chunk,
        order=ORD[order], update=upd, renorm=opts.get("renorm", False),
        alpha=inp["alpha"] if momentum else None, ns_steps=opts.get("ns_steps", 0))
    q, k, v, eta, W0, W2, W1 = gpu_args(inp, dtype)
    alpha = dev(inp["alpha"]) if momentum else None
    out, Wf, M = layer.lact_recurrent_fwd(q, k, v, eta, W0, W2, W1, chunk, order=order,
                                          update_mask=mask, renorm=opts.get("renorm", False),
                                          alpha=alpha, ns_steps=opts.get("ns_steps", 0),
                                          return_momentum=momentum)
    abi.ttt_last_device_status()
    tol = TOL[dtype]
    assert rel(host(out), ref) <= tol
    for got, name in zip(Wf, ("W0", "W2", "W1")):
        assert rel(host(got), Wref[name]) <= tol, name
        # the change of each fast matrix, relative to the oracle's change
        init = inp[name][None].repeat(B, axis=0)
        if name in upd:
            assert rel(host(got) - init, Wref[name] - init) <= 5 * tol, name
        else:
            assert np.array_equal(host(got), np.broadcast_to(init, host(got).shape))
    if momentum:
        hm = h * m
        Mh = host(M)
        for pidx, name in enumerate(("W0", "W1", "W2")):
            if name in upd:
                assert rel(Mh[..., pidx * hm:(pidx + 1) * hm].reshape(Mref[name].shape),
                           Mref[name]) <= 5 * tol, name


def test_recurrent_ascent_equals_descent_with_negated_values():
    wl, inp = layer_inputs("lm", "bf16", 1, 2, 512, 64, 128, 128, seed=21, momentum=True)
    q, k, v, eta, W0, W2, W1 = gpu_args(inp, "bf16")
    alpha = dev(inp["alpha"])
    kw = dict(renorm=True, alpha=alpha, ns_steps=5)
    a, Wa, _ = layer.lact_recurrent_fwd(q, k, v, eta, W0, W2, W1, 128, sign=-1, **kw)
    d, Wd, _ = layer.lact_recurrent_fwd(q, k, (-v).contiguous(), eta, W0, W2, W1, 128, sign=1,
                                        **kw)
    assert torch.equal(a, d)
    for x, y in zip(Wa, Wd):
        assert torch.equal(x, y)


def test_recurrent_resume_equals_full_run():
    wl, inp = layer_inputs("lm", "bf16", 1, 2, 1024, 64, 128, 256, seed=22, momentum=True)
    q, k, v, eta, W0, W2, W1 = gpu_args(inp, "bf16")
    alpha = dev(inp["alpha"])
    kw = dict(renorm=True, ns_steps=5, return_momentum=True)
    full, Wf, Mf = layer.lact_recurrent_fwd(q, k, v, eta, W0, W2, W1, 256, alpha=alpha, **kw)
    h1 = slice(0, 512)
    h2 = slice(512, 1024)
    a, Wa, Ma = layer.lact_recurrent_fwd(q[:, :, h1].contiguous(), k[:, :, h1].contiguous(),
                                         v[:, :, h1].contiguous(), eta[:, :, h1].contiguous(),
                                         W0, W2, W1, 256, alpha=alpha[:, :, :2].contiguous(), **kw)
    # resume from the carried state (one batch element: the per-(b, head) weights are the
    # per-head weights of the next call)
    b, Wb, Mb = layer.lact_recurrent_fwd(q[:, :, h2].contiguous(), k[:, :, h2].contiguous(),
                                         v[:, :, h2].contiguous(), eta[:, :, h2].contiguous(),
                                         Wa[0][0].contiguous(), Wa[1][0].contiguous(),
                                         Wa[2][0].contiguous(), 256,
                                         alpha=alpha[:, :, 2:].contiguous(), M_init=Ma, **kw)
    # renorm targets are the column norms at the start of each call, equal up to rounding
    assert rel(host(torch.cat([a, b], dim=2)), host(full)) <= TOL["bf16"]
    for x, y in zip(Wb, Wf):
        assert rel(host(x), host(y)) <= TOL["bf16"]


@pytest.mark.parametrize("order", ["update_apply", "apply_update"])
def test_recurrent_graph_replay_equals_eager(order):
    """The recurrent form forks its applies and the W1 gradient onto a second stream and
    joins it before returning; captured into a CUDA graph from the caller's stream and
    replayed, it gives the eager call's results bit for bit (no kernel depends on the
    interleaving of the two streams). NS on the one-CTA path, momentum, renorm, 5 chunks."""
    wl, inp = layer_inputs("lm", "bf16", 1, 2, 1280, 128, 256, 256, seed=23, momentum=True)
    q, k, v, eta, W0, W2, W1 = gpu_args(inp, "bf16")
    alpha = dev(inp["alpha"])
    kw = dict(order=order, renorm=True, alpha=alpha, ns_steps=5)
    ref, Wr, _ = layer.lact_recurrent_fwd(q, k, v, eta, W0, W2, W1, 256, **kw)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        layer.lact_recurrent_fwd(q, k, v, eta, W0, W2, W1, 256, **kw)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    with torch.cuda.graph(g):
        out, Wf, _ = layer.lact_recurrent_fwd(q, k, v, eta, W0, W2, W1, 256, **kw)
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    abi.ttt_last_device_status()
    assert torch.equal(out, ref)
    for x, y in zip(Wf, Wr):
        assert torch.equal(x, y)
    del g


# ----------------------------------------------------------------------------- In-Place form
def test_inplace_shaped_update_matches_oracle():
    """q = k = H, W0 = Wg^T, W2 = Wu^T given as [m,h]; W1 = W_down^T given as [h,m];
    apply then update with constant eta (In-Place TTT, sections 3.1 and 3.4)."""
    wl = WORKLOADS["inplace"].scaled(N=640, h=256, m=384, chunk=128)
    inp = make_inplace_inputs(wl, seed=31)
    Vbar = O.lm_target(inp["X0"], inp["conv_w"], inp["W_target"])
    ref, Wref = O.inplace_sequential(inp["Hs"], inp["Wg"], inp["Wu"], inp["W_down"], Vbar,
                                     wl.chunk, 1e-3)
    Hs = dev(inp["Hs"], torch.bfloat16)[None, None]
    vb = layer.lm_target(dev(inp["X0"], torch.bfloat16), dev(inp["conv_w"]),
                         dev(inp["W_target"], torch.bfloat16))
    assert rel(host(vb), Vbar) <= TOL["bf16"]
    eta = torch.full((1, 1, wl.N), 1e-3, dtype=torch.float32, device="cuda")
    out, S = layer.la_parallel_fwd(Hs, Hs, vb[None, None].contiguous(), eta,
                                   dev(inp["Wg"])[None], dev(inp["Wu"])[None],
                                   dev(inp["W_down"])[None], wl.chunk, order="apply_update",
                                   w_in_layout=1, w1_layout=1)
    abi.ttt_last_device_status()
    assert rel(host(out[0, 0]), ref) <= TOL["bf16"]
    assert rel(host(S[0, 0]), Wref) <= TOL["bf16"]
    assert rel(host(S[0, 0]) - inp["W_down"], Wref - inp["W_down"]) <= TOL["bf16"]


def test_lm_target_matches_oracle():
    rng = np.random.Generator(np.random.PCG64(41))
    N, d = 300, 64
    from ttt_inputs import bf16_round
    X0 = bf16_round(rng.standard_normal((N, d), dtype=np.float32))
    cw = rng.standard_normal((4, d), dtype=np.float32)
    Wt = bf16_round((rng.standard_normal((d, d)) / 8).astype(np.float32))
    got = layer.lm_target(dev(X0, torch.bfloat16), dev(cw), dev(Wt, torch.bfloat16))
    assert rel(host(got), O.lm_target(X0, cw, Wt)) <= TOL["bf16"]
    shift = np.zeros((4, d), np.float32)
    shift[1] = 1.0
    got = layer.lm_target(dev(X0, torch.bfloat16), dev(shift),
                          dev(np.eye(d, dtype=np.float32), torch.bfloat16))
    assert np.array_equal(host(got)[1:], X0[:-1]) and not host(got)[0].any()


# ----------------------------------------------------------------------------- failure path
def test_bounded_wait_reports_timeout_and_context_survives():
    abi.ttt_debug_wait_timeout(2_000_000)   # 2 ms: the barrier is never completed
    with pytest.raises(abi.TTTError) as ei:
        abi.ttt_last_device_status()
    assert ei.value.status == abi.TTT_ERR_TIMEOUT
    abi.ttt_last_device_status()            # the word was cleared
    wl, inp = layer_inputs("tiny", "fp32", 1, 1, 64, 16, 16, 32, seed=51)
    out, _ = layer.la_parallel_fwd(*gpu_args(inp, "fp32"), 32)
    ref, _ = O.la_parallel_batched(inp["q"], inp["k"], inp["v"], inp["eta"], inp["W0"],
                                   inp["W2"], inp["W1"], 32)
    assert rel(host(out), ref) <= TOL["fp32"]
