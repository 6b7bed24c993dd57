"""GPU parity at the workloads' full sizes, in the launch configuration bench.py times.

Where the fp64 oracle cannot redo a whole workload in seconds, the comparison is on outputs
it can compute one by one (sampled token rows, every chunk state formed in full), on a
leading part of the sequence, or on properties that hold at any size (bitwise resume,
renormalisation invariants). Tolerance max|err| / max|ref| as in the small cases.
"""
import numpy as np
import pytest
import torch

from oracle import ttt_oracle as O
from test_weight_layers_ttt_b200 import abi, layer
from ttt_inputs import WORKLOADS, make_inplace_inputs, make_layer_inputs

from gpu_helpers import TOL, dev, host, rel

pytestmark = pytest.mark.gpu


def gpu_layer_args(x, dtype=torch.bfloat16):
    return ([dev(x[n], dtype) for n in ("q", "k", "v")] +
            [dev(x[n]) for n in ("eta", "W0", "W2", "W1")])


def sample_rows(N, chunk, n_random, seed):
    rng = np.random.Generator(np.random.PCG64(seed))
    rows = {0, N - 1}
    for c in range(0, N, chunk):
        rows.update({c, min(N - 1, c + chunk - 1)})
    rows.update(rng.integers(0, N, n_random).tolist())
    return np.array(sorted(rows))


@pytest.fixture(scope="module")
def lm():
    wl = WORKLOADS["lm"]
    return wl, make_layer_inputs(wl)


def test_lm_parallel_full_size(lm):
    wl, x = lm
    args = gpu_layer_args(x)
    out, S = layer.la_parallel_fwd(*args, wl.chunk)
    abi.ttt_last_device_status()
    Oh, Sh = host(out), host(S)
    assert np.isfinite(Oh).all()
    for b in range(wl.B):
        for hd in range(wl.H):
            rows = sample_rows(wl.N, wl.chunk, 48, seed=b * 16 + hd)
            ref, Sref = O.la_parallel_rows(x["q"][b, hd], x["k"][b, hd], x["v"][b, hd],
                                           x["eta"][b, hd], x["W0"][hd], x["W2"][hd],
                                           x["W1"][hd], wl.chunk, rows)
            assert rel(Oh[b, hd, rows], ref) <= TOL["bf16"], (b, hd)
            assert rel(Sh[b, hd], Sref) <= TOL["bf16"], (b, hd)
            # the accumulated deltas alone
            assert rel(Sh[b, hd] - x["W1"][hd], Sref - x["W1"][hd]) <= TOL["bf16"], (b, hd)


def test_lm_parallel_resume_is_bitwise(lm):
    """Running [0, N/2) and then [N/2, N) from the carried state equals one run."""
    wl, x = lm
    q, k, v, eta, W0, W2, W1 = gpu_layer_args(x)
    full, Sf = layer.la_parallel_fwd(q, k, v, eta, W0, W2, W1, wl.chunk)
    h = wl.N // 2
    a, Sa = layer.la_parallel_fwd(q[:, :, :h].contiguous(), k[:, :, :h].contiguous(),
                                  v[:, :, :h].contiguous(), eta[:, :, :h].contiguous(),
                                  W0, W2, W1, wl.chunk)
    for b in range(wl.B):   # the carried state differs per batch element
        sl = slice(b, b + 1)
        o2, S2 = layer.la_parallel_fwd(q[sl, :, h:].contiguous(), k[sl, :, h:].contiguous(),
                                       v[sl, :, h:].contiguous(), eta[sl, :, h:].contiguous(),
                                       W0, W2, Sa[b].contiguous(), wl.chunk)
        assert torch.equal(o2[0], full[b, :, h:])
        assert torch.equal(S2[0], Sf[b])
    assert torch.equal(a, full[:, :, :h])


def test_lm_recurrent_full_size(lm):
    wl, x = lm
    out, Wf, _ = layer.lact_recurrent_fwd(*gpu_layer_args(x), wl.chunk, renorm=True)
    abi.ttt_last_device_status()
    Oh = host(out)
    for b, hd in ((0, 0), (1, 3)):
        ref, Wref, _ = O.lact_recurrent(x["q"][b, hd], x["k"][b, hd], x["v"][b, hd],
                                        x["eta"][b, hd], x["W0"][hd], x["W2"][hd], x["W1"][hd],
                                        wl.chunk, renorm=True)
        assert rel(Oh[b, hd], ref) <= TOL["bf16"], (b, hd)
        for got, name in zip(Wf, ("W0", "W2", "W1")):
            g = host(got)[b, hd]
            assert rel(g, Wref[name]) <= TOL["bf16"], name
            assert rel(g - x[name][hd], Wref[name] - x[name][hd]) <= 5 * TOL["bf16"], name


def test_long_parallel_full_size():
    wl = WORKLOADS["long"]
    x = make_layer_inputs(wl)
    out, S = layer.la_parallel_fwd(*gpu_layer_args(x), wl.chunk)
    abi.ttt_last_device_status()
    Oh, Sh = host(out), host(S)
    assert np.isfinite(Oh).all()
    for hd in (0, 5):
        rows = sample_rows(wl.N, wl.chunk, 32, seed=hd)
        ref, Sref = O.la_parallel_rows(x["q"][0, hd], x["k"][0, hd], x["v"][0, hd],
                                       x["eta"][0, hd], x["W0"][hd], x["W2"][hd], x["W1"][hd],
                                       wl.chunk, rows)
        assert rel(Oh[0, hd, rows], ref) <= TOL["bf16"], hd
        assert rel(Sh[0, hd], Sref) <= TOL["bf16"], hd
        assert rel(Sh[0, hd] - x["W1"][hd], Sref - x["W1"][hd]) <= TOL["bf16"], hd


@pytest.fixture(scope="module")
def nvs():
    wl = WORKLOADS["nvs"]
    return wl, make_layer_inputs(wl)


def test_nvs_recurrent_bf16_leading_chunks_and_invariants(nvs):
    """bf16 operands: the leading chunks match the oracle; the whole run keeps every
    column norm at its initial value (renormalisation) and stays finite."""
    wl, x = nvs
    args = gpu_layer_args(x)
    out, Wf, _ = layer.lact_recurrent_fwd(*args, wl.chunk, renorm=True, alpha=dev(x["alpha"]),
                                          ns_steps=5)
    abi.ttt_last_device_status()
    Oh = host(out)
    assert np.isfinite(Oh).all()
    lead = 4 * wl.chunk
    for hd in (0, 5):
        ref, _, _ = O.lact_recurrent(x["q"][0, hd, :lead], x["k"][0, hd, :lead],
                                     x["v"][0, hd, :lead], x["eta"][0, hd, :lead], x["W0"][hd],
                                     x["W2"][hd], x["W1"][hd], wl.chunk, renorm=True,
                                     alpha=x["alpha"][0, hd, :4], ns_steps=5)
        assert rel(Oh[0, hd, :lead], ref) <= TOL["bf16"], hd
    for got, name in zip(Wf, ("W0", "W2", "W1")):
        g = host(got)
        n0 = np.sqrt(np.sum(x[name].astype(np.float64) ** 2, axis=1))       # [H, cols]
        n1 = np.sqrt(np.sum(g ** 2, axis=2))                               # [B, H, cols]
        assert np.max(np.abs(n1 / n0[None] - 1.0)) < 1e-4, name


def test_nvs_recurrent_fp32_full_length(nvs):
    """fp32 operands (the same bf16-valued inputs): the full 48-chunk trajectory of two
    heads matches the oracle."""
    wl, x = nvs
    args = gpu_layer_args(x, torch.float32)
    out, Wf, _ = layer.lact_recurrent_fwd(*args, wl.chunk, renorm=True, alpha=dev(x["alpha"]),
                                          ns_steps=5)
    abi.ttt_last_device_status()
    Oh = host(out)
    for hd in (0, 3):
        ref, Wref, _ = O.lact_recurrent(x["q"][0, hd], x["k"][0, hd], x["v"][0, hd],
                                        x["eta"][0, hd], x["W0"][hd], x["W2"][hd], x["W1"][hd],
                                        wl.chunk, renorm=True, alpha=x["alpha"][0, hd],
                                        ns_steps=5)
        assert rel(Oh[0, hd], ref) <= TOL["bf16"], hd
        # the first ten chunks hold the fp32 bound
        assert rel(Oh[0, hd, :10 * wl.chunk], ref[:10 * wl.chunk]) <= TOL["fp32"], hd
        for got, name in zip(Wf, ("W0", "W2", "W1")):
            assert rel(host(got)[0, hd], Wref[name]) <= TOL["bf16"], name


def _inplace_gpu(x, N, wl):
    Hs = dev(x["Hs"][:N], torch.bfloat16)[None, None]
    vb = layer.lm_target(dev(x["X0"][:N], torch.bfloat16), dev(x["conv_w"]),
                         dev(x["W_target"], torch.bfloat16))
    eta = torch.full((1, 1, N), 1e-3, dtype=torch.float32, device="cuda")
    out, S = layer.la_parallel_fwd(Hs, Hs, vb[None, None].contiguous(), eta,
                                   dev(x["Wg"])[None], dev(x["Wu"])[None],
                                   dev(x["W_down"])[None], wl.chunk, order="apply_update",
                                   w_in_layout=1, w1_layout=1)
    return vb, out, S


@pytest.fixture(scope="module")
def inplace():
    wl = WORKLOADS["inplace"]
    return wl, make_inplace_inputs(wl)


def test_inplace_full_width_two_chunks(inplace):
    """Full d = 4096 and d_H = 11008, the first two chunks (2048 tokens)."""
    wl, x = inplace
    n = 2 * wl.chunk
    vb, out, S = _inplace_gpu(x, n, wl)
    abi.ttt_last_device_status()
    Vref = O.lm_target(x["X0"][:n], x["conv_w"], x["W_target"])
    assert rel(host(vb), Vref) <= TOL["bf16"]
    ref, Wref = O.inplace_sequential(x["Hs"][:n], x["Wg"], x["Wu"], x["W_down"], Vref,
                                     wl.chunk, 1e-3)
    assert rel(host(out[0, 0]), ref) <= TOL["bf16"]
    assert rel(host(S[0, 0]), Wref) <= TOL["bf16"]
    assert rel(host(S[0, 0]) - x["W_down"], Wref - x["W_down"]) <= TOL["bf16"]


def test_inplace_reduced_width_all_chunks_match_the_oracle(inplace):
    """All 32 chunks of the In-Place workload (N = 32768, chunk 1024, q = k, apply->update,
    the exclusive scan over 32 chunk states) at reduced width d = 512, d_H = 1408 against
    the oracle's sequential apply-then-update route."""
    wl = WORKLOADS["inplace"].scaled(h=512, m=1408)
    x = make_inplace_inputs(wl, seed=777)
    vb, out, S = _inplace_gpu(x, wl.N, wl)
    abi.ttt_last_device_status()
    Vref = O.lm_target(x["X0"], x["conv_w"], x["W_target"])
    assert rel(host(vb), Vref) <= TOL["bf16"]
    ref, Wref = O.inplace_sequential(x["Hs"], x["Wg"], x["Wu"], x["W_down"], Vref, wl.chunk,
                                     1e-3)
    Oh = host(out[0, 0])
    assert rel(Oh, ref) <= TOL["bf16"]
    assert rel(host(S[0, 0]), Wref) <= TOL["bf16"]
    assert rel(host(S[0, 0]) - x["W_down"], Wref - x["W_down"]) <= TOL["bf16"]
    # the last chunk's outputs alone (read the state after 31 exclusive-scan steps)
    last = slice(wl.N - wl.chunk, wl.N)
    assert rel(Oh[last], ref[last]) <= TOL["bf16"]


def test_inplace_reduced_width_sequential_schedule_matches_the_oracle(inplace, monkeypatch):
    """The same 32 chunks through the sequential schedule (one fp32 state, per chunk an
    apply GEMM on its bf16 copy and an update GEMM into it), which the library takes for
    states too large to materialise per chunk, against the oracle's sequential route."""
    monkeypatch.setenv("TTT_SEQUENTIAL", "1")
    wl = WORKLOADS["inplace"].scaled(h=512, m=1408)
    x = make_inplace_inputs(wl, seed=778)
    vb, out, S = _inplace_gpu(x, wl.N, wl)
    abi.ttt_last_device_status()
    Vref = O.lm_target(x["X0"], x["conv_w"], x["W_target"])
    ref, Wref = O.inplace_sequential(x["Hs"], x["Wg"], x["Wu"], x["W_down"], Vref, wl.chunk,
                                     1e-3)
    assert rel(host(out[0, 0]), ref) <= TOL["bf16"]
    assert rel(host(S[0, 0]), Wref) <= TOL["bf16"]
    assert rel(host(S[0, 0]) - x["W_down"], Wref - x["W_down"]) <= TOL["bf16"]


def test_inplace_full_length_resume_is_bitwise(inplace):
    wl, x = inplace
    vb, out, S = _inplace_gpu(x, wl.N, wl)
    abi.ttt_last_device_status()
    assert torch.isfinite(out).all() and torch.isfinite(S).all()
    h = wl.N // 2
    Hs = dev(x["Hs"], torch.bfloat16)[None, None]
    eta = torch.full((1, 1, h), 1e-3, dtype=torch.float32, device="cuda")
    Wg, Wu = dev(x["Wg"])[None], dev(x["Wu"])[None]
    kw = dict(order="apply_update", w_in_layout=1, w1_layout=1)
    a, Sa = layer.la_parallel_fwd(Hs[:, :, :h].contiguous(), Hs[:, :, :h].contiguous(),
                                  vb[None, None, :h].contiguous(), eta, Wg, Wu,
                                  dev(x["W_down"])[None], wl.chunk, **kw)
    b, Sb = layer.la_parallel_fwd(Hs[:, :, h:].contiguous(), Hs[:, :, h:].contiguous(),
                                  vb[None, None, h:].contiguous(), eta, Wg, Wu, Sa[0].contiguous(),
                                  wl.chunk, **kw)
    assert torch.equal(a[0, 0], out[0, 0, :h]) and torch.equal(b[0, 0], out[0, 0, h:])
    assert torch.equal(Sb, S)
