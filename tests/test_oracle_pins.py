"""Pins of the fp64 oracle against what the pages and the mathematics fix.

Each test checks the oracle against something other than itself: a textbook closed form,
an independent route (attention-matrix form, torch autograd, finite differences, a
spectral identity), an exact symmetry, or a value worked by hand from the pages.
All run on CPU in well under a minute.
"""
import math
import os

import numpy as np
import pytest
import torch

from oracle import ttt_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed):
    return np.random.Generator(np.random.PCG64(seed))


def _layer(seed, N=37, h=5, m=7, eta_scale=0.3, unit=False):
    r = _rng(seed)
    q = r.standard_normal((N, h))
    k = r.standard_normal((N, h))
    v = r.standard_normal((N, h))
    if unit:
        q, k, v = (x / np.linalg.norm(x, axis=1, keepdims=True) for x in (q, k, v))
    eta = eta_scale * (1.0 / (1.0 + np.exp(-r.standard_normal(N))))
    W0 = r.standard_normal((h, m)) / math.sqrt(h)
    W2 = r.standard_normal((h, m)) / math.sqrt(h)
    W1 = r.standard_normal((m, h)) / math.sqrt(m)
    return q, k, v, eta, W0, W2, W1


# --------------------------------------------------------------------------- activations
def test_silu_special_values():
    a = np.array([0.0, 1.0, -1.0, 30.0, -30.0])
    s = O.silu(a)
    assert s[0] == 0.0
    assert abs(s[1] - 1.0 / (1.0 + math.exp(-1.0))) < 1e-15
    assert abs(s[2] + math.exp(-1.0) / (1.0 + math.exp(-1.0))) < 1e-15
    assert abs(s[3] - 30.0) < 1e-10 and abs(s[4]) < 1e-10
    assert abs(O.silu_prime(np.array([0.0]))[0] - 0.5) < 1e-15
    # derivative against a central difference of silu itself
    x = np.linspace(-6, 6, 25)
    eps = 1e-6
    fd = (O.silu(x + eps) - O.silu(x - eps)) / (2 * eps)
    assert np.max(np.abs(fd - O.silu_prime(x))) < 1e-9


# --------------------------------------------------------------------------- (1) linear attention
def test_chunk1_identity_features_is_causal_linear_attention():
    """phi = identity, zero initial state, one token per chunk: the layer is causal linear
    attention o_t = q_t sum_{i<=t} eta_i k_i^T v_i (brute-force triple loop)."""
    r = _rng(1)
    N, h = 9, 3
    q, k, v = r.standard_normal((N, h)), r.standard_normal((N, h)), r.standard_normal((N, h))
    eta = r.uniform(0.1, 1.0, N)
    expect = np.zeros((N, h))
    for t in range(N):
        for i in range(t + 1):
            score = sum(q[t, a] * k[i, a] for a in range(h))
            for j in range(h):
                expect[t, j] += eta[i] * score * v[i, j]
    got, S = O.chunked_linear_attention(q, k, v, eta, np.zeros((h, h)), 1, O.UPDATE_APPLY)
    assert np.max(np.abs(got - expect)) < 1e-12
    assert np.max(np.abs(S - sum(eta[i] * np.outer(k[i], v[i]) for i in range(N)))) < 1e-12


@pytest.mark.parametrize("order", [O.UPDATE_APPLY, O.APPLY_UPDATE])
@pytest.mark.parametrize("chunk", [1, 4, 7, 37, 50])
def test_chunked_scan_equals_masked_form(order, chunk):
    """Prefix-sum route == attention-matrix (dual) route, any chunk size, ragged tail."""
    q, k, v, eta, W0, W2, W1 = _layer(2)
    pq, pk = O.swiglu_features(q, W0, W2), O.swiglu_features(k, W0, W2)
    got, _ = O.chunked_linear_attention(pq, pk, v, eta, W1, chunk, order)
    ref = O.la_masked(pq, pk, v, eta, W1, chunk, order)
    assert np.max(np.abs(got - ref)) <= 1e-12 * max(1.0, np.max(np.abs(ref)))


def test_teaching_example_golden():
    rows = {}
    final = None
    with open(os.path.join(GOLDEN, "teaching_chunk4.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            parts = line.split()
            if parts[0] == "final_state":
                final = float(parts[1])
                continue
            rows.setdefault(parts[0], []).append([float(x) for x in parts[1:]])
    for order, data in rows.items():
        data = np.array(data)
        q, k, v, eta, expect = data[:, 1:2], data[:, 2:3], data[:, 3:4], data[:, 4], data[:, 5]
        got, S = O.chunked_linear_attention(q, k, v, eta, np.zeros((1, 1)), 4, order)
        assert np.array_equal(got[:, 0], expect), order
        assert S[0, 0] == final
        assert np.array_equal(O.la_masked(q, k, v, eta, np.zeros((1, 1)), 4, order)[:, 0], expect)


# --------------------------------------------------------------------------- (2) parallel == recurrent
@pytest.mark.parametrize("order", [O.UPDATE_APPLY, O.APPLY_UPDATE])
@pytest.mark.parametrize("chunk", [1, 6, 16])
def test_parallel_equals_recurrent_last_layer_only(order, chunk):
    q, k, v, eta, W0, W2, W1 = _layer(3)
    Op, S = O.la_parallel(q, k, v, eta, W0, W2, W1, chunk, order=order)
    Or, W, _ = O.lact_recurrent(q, k, v, eta, W0, W2, W1, chunk, order=order, update=("W1",))
    assert np.max(np.abs(Op - Or)) < 1e-12
    assert np.max(np.abs(S - W["W1"])) < 1e-12
    assert np.array_equal(W["W0"], W0) and np.array_equal(W["W2"], W2)


def test_parallel_rows_matches_full():
    q, k, v, eta, W0, W2, W1 = _layer(4, N=40)
    for order in (O.UPDATE_APPLY, O.APPLY_UPDATE):
        full, S = O.la_parallel(q, k, v, eta, W0, W2, W1, 8, order=order)
        rows = np.array([0, 7, 8, 21, 39])
        part, S2 = O.la_parallel_rows(q, k, v, eta, W0, W2, W1, 8, rows, order=order)
        assert np.max(np.abs(part - full[rows])) < 1e-13
        assert np.max(np.abs(S - S2)) < 1e-13


# --------------------------------------------------------------------------- (3) ascent == negated v
@pytest.mark.parametrize("opts", [
    dict(), dict(renorm=True), dict(ns_steps=5), dict(renorm=True, ns_steps=5, momentum=True),
])
def test_ascent_equals_descent_with_negated_values(opts):
    q, k, v, eta, W0, W2, W1 = _layer(5)
    alpha = _rng(6).uniform(0.2, 0.9, 7) if opts.get("momentum") else None
    kw = dict(renorm=opts.get("renorm", False), ns_steps=opts.get("ns_steps", 0), alpha=alpha)
    oa, Wa, Ma = O.lact_recurrent(q, k, v, eta, W0, W2, W1, 6, sign=-1, **kw)
    od, Wd, Md = O.lact_recurrent(q, k, -v, eta, W0, W2, W1, 6, sign=1, **kw)
    assert np.array_equal(oa, od)
    for n in O.WEIGHTS:
        assert np.array_equal(Wa[n], Wd[n])
    pa, Sa = O.la_parallel(q, k, v, eta, W0, W2, W1, 6, sign=-1)
    pd, Sd = O.la_parallel(q, k, -v, eta, W0, W2, W1, 6, sign=1)
    assert np.array_equal(pa, pd) and np.array_equal(Sa, Sd)
    # and ascent really moves differently from descent with the same values
    o_plain, _, _ = O.lact_recurrent(q, k, v, eta, W0, W2, W1, 6, sign=1, **kw)
    assert np.max(np.abs(o_plain - oa)) > 1e-6


# --------------------------------------------------------------------------- (4) chunk 1 == per-token
def _per_token_autograd(q, k, v, eta, W0, W2, W1, renorm):
    """Independent per-token TTT loop: gradients by torch autograd in float64."""
    t64 = lambda a: torch.tensor(a, dtype=torch.float64)  # noqa: E731
    W = [t64(W0), t64(W2), t64(W1)]
    n0 = [w.norm(dim=0) for w in W]
    out = []
    for t in range(q.shape[0]):
        Ws = [w.clone().requires_grad_(True) for w in W]
        kt, vt, qt = t64(k[t:t + 1]), t64(v[t:t + 1]), t64(q[t:t + 1])
        f = (torch.nn.functional.silu(kt @ Ws[0]) * (kt @ Ws[1])) @ Ws[2]
        loss = -(float(eta[t]) * (f * vt).sum())
        grads = torch.autograd.grad(loss, Ws)
        W = [w - g for w, g in zip(W, grads)]
        if renorm:
            W = [w * (n / w.norm(dim=0)) for w, n in zip(W, n0)]
        o = (torch.nn.functional.silu(qt @ W[0]) * (qt @ W[1])) @ W[2]
        out.append(o.detach().numpy()[0])
    return np.array(out), [w.numpy() for w in W]


@pytest.mark.parametrize("renorm", [False, True])
def test_chunk1_recurrent_equals_per_token_autograd_loop(renorm):
    q, k, v, eta, W0, W2, W1 = _layer(7, N=23, eta_scale=1.0, unit=True)
    ref, Wref = _per_token_autograd(q, k, v, eta, W0, W2, W1, renorm)
    got, W, _ = O.lact_recurrent(q, k, v, eta, W0, W2, W1, 1, renorm=renorm)
    assert np.max(np.abs(got - ref)) < 1e-12
    for name, w in zip(("W0", "W2", "W1"), Wref):
        assert np.max(np.abs(W[name] - w)) < 1e-12


def test_chunked_grads_equal_autograd():
    q, k, v, eta, W0, W2, W1 = _layer(8, N=16)
    g = O.inner_grads(W0, W2, W1, k, v, eta)
    Ws = [torch.tensor(w, requires_grad=True) for w in (W0, W2, W1)]
    kt = torch.tensor(k)
    f = (torch.nn.functional.silu(kt @ Ws[0]) * (kt @ Ws[1])) @ Ws[2]
    loss = -(torch.tensor(eta)[:, None] * f * torch.tensor(v)).sum()
    ag = torch.autograd.grad(loss, Ws)
    for name, a in zip(("W0", "W2", "W1"), ag):
        assert np.max(np.abs(g[name] - a.numpy())) < 1e-13


# --------------------------------------------------------------------------- (5) finite differences
def test_inner_gradient_finite_differences():
    q, k, v, eta, W0, W2, W1 = _layer(9, N=5, h=3, m=4, eta_scale=1.0)
    g = O.inner_grads(W0, W2, W1, k, v, eta)
    eps = 1e-6
    Ws = {"W0": W0, "W2": W2, "W1": W1}
    for name in O.WEIGHTS:
        fd = np.zeros_like(Ws[name])
        for idx in np.ndindex(Ws[name].shape):
            plus = {n: w.copy() for n, w in Ws.items()}
            minus = {n: w.copy() for n, w in Ws.items()}
            plus[name][idx] += eps
            minus[name][idx] -= eps
            lp = O.inner_loss(plus["W0"], plus["W2"], plus["W1"], k, v, eta)
            lm = O.inner_loss(minus["W0"], minus["W2"], minus["W1"], k, v, eta)
            fd[idx] = (lp - lm) / (2 * eps)
        rel = np.max(np.abs(fd - g[name])) / np.max(np.abs(g[name]))
        assert rel <= 1e-7, (name, rel)


# --------------------------------------------------------------------------- Theorem 5.3: momentum
@pytest.mark.parametrize("order", [O.UPDATE_APPLY, O.APPLY_UPDATE])
def test_momentum_is_value_reweighting_closed_form(order):
    """Frozen W0, W2, momentum on W1, no orthogonalisation: the W1 increment of chunk i
    enters the chunk-c state with weight sum_{j=i}^{c} prod_{l=i+1}^{j} alpha_l."""
    q, k, v, eta, W0, W2, W1 = _layer(10, N=30)
    chunk = 5
    C = 6
    alpha = _rng(11).uniform(0.1, 0.95, C)
    dS = O.chunk_state_deltas(O.swiglu_features(k, W0, W2), v, eta, chunk)
    states = []
    for c in range(C):
        S = W1.copy()
        for i in range(c + 1):
            coef = 0.0
            for j in range(i, c + 1):
                prod = 1.0
                for l in range(i + 1, j + 1):
                    prod *= alpha[l]
                coef += prod
            S = S + coef * dS[i]
        states.append(S)
    pq = O.swiglu_features(q, W0, W2)
    expect = np.empty_like(q)
    for c in range(C):
        sl = slice(c * chunk, (c + 1) * chunk)
        Sc = states[c] if order == O.UPDATE_APPLY else (W1 if c == 0 else states[c - 1])
        expect[sl] = pq[sl] @ Sc
    got, W, M = O.lact_recurrent(q, k, v, eta, W0, W2, W1, chunk, order=order, update=("W1",),
                                 alpha=alpha)
    assert np.max(np.abs(W["W1"] - states[-1])) < 1e-12
    assert np.max(np.abs(got - expect)) < 1e-12
    # alpha = 0 is plain gradient descent
    g0, W0r, _ = O.lact_recurrent(q, k, v, eta, W0, W2, W1, chunk, update=("W1",),
                                  alpha=np.zeros(C))
    g1, W1r, _ = O.lact_recurrent(q, k, v, eta, W0, W2, W1, chunk, update=("W1",))
    assert np.max(np.abs(g0 - g1)) < 1e-13


def _ns5_spectral(G):
    """Five Newton-Schulz steps written on the singular values: for G = U diag(s) V^T the
    iteration only maps s / (||G||_F + 1e-7) through p(x) = a x + b x^3 + c x^5 five times
    (an SVD route, independent of the oracle's matrix iteration)."""
    a, b, c = 3.4445, -4.7750, 2.0315
    U, s, Vt = np.linalg.svd(G, full_matrices=False)
    x = s / (math.sqrt(float(np.sum(s * s))) + 1e-7)
    for _ in range(5):
        x = a * x + b * x ** 3 + c * x ** 5
    return U @ np.diag(x) @ Vt


@pytest.mark.parametrize("order", [O.UPDATE_APPLY, O.APPLY_UPDATE])
def test_momentum_then_newton_schulz_order(order):
    """Momentum before orthogonalisation ("Test-Time Training Done Right" notes, section
    2.2: the momentum buffer accumulates raw gradients, Muon orthogonalises the buffer):
    with W0, W2 frozen and only W1 fast, M_c = sum_{i <= c} (prod_{l=i+1}^{c} alpha_l) g_i
    (nested loops over the raw chunk gradients g_i = -Delta S_i), U_c = NS5(M_c) by the
    spectral route, W1_c = W1 - sum_{c' <= c} U_c'. The two plausible mistakes (NS before
    the momentum, NS fed the raw gradient) give different weights and fail this pin."""
    q, k, v, eta, W0, W2, W1 = _layer(21, N=24, h=4, m=6)
    chunk, C = 4, 6
    alpha = _rng(22).uniform(0.3, 0.95, C)
    g = [-d for d in O.chunk_state_deltas(O.swiglu_features(k, W0, W2), v, eta, chunk)]
    states = []
    S = W1.copy()
    for c in range(C):
        M = np.zeros_like(W1)
        for i in range(c + 1):
            prod = 1.0
            for l in range(i + 1, c + 1):
                prod *= alpha[l]
            M = M + prod * g[i]
        S = S - _ns5_spectral(M)
        states.append(S)
    pq = O.swiglu_features(q, W0, W2)
    expect = np.empty_like(q)
    for c in range(C):
        sl = slice(c * chunk, (c + 1) * chunk)
        Sc = states[c] if order == O.UPDATE_APPLY else (W1 if c == 0 else states[c - 1])
        expect[sl] = pq[sl] @ Sc
    got, W, M = O.lact_recurrent(q, k, v, eta, W0, W2, W1, chunk, order=order, update=("W1",),
                                 alpha=alpha, ns_steps=5)
    assert np.max(np.abs(W["W1"] - states[-1])) < 1e-10
    assert np.max(np.abs(got - expect)) < 1e-10
    # the pin separates the orders: NS before momentum / NS of the raw gradient differ
    Mw, Sw1, Sw2 = np.zeros_like(W1), W1.copy(), W1.copy()
    for c in range(C):
        Mw = alpha[c] * Mw + _ns5_spectral(g[c])
        Sw1 = Sw1 - Mw
        Sw2 = Sw2 - _ns5_spectral(g[c])
    assert np.max(np.abs(Sw1 - states[-1])) > 1e-2
    assert np.max(np.abs(Sw2 - states[-1])) > 1e-2


# --------------------------------------------------------------------------- Newton-Schulz
@pytest.mark.parametrize("shape", [(6, 9), (9, 6), (7, 7)])
def test_newton_schulz_acts_on_singular_values(shape):
    """NS5(U diag(s) V^T) = U diag(p^5(s / ||s||)) V^T with p(x) = a x + b x^3 + c x^5."""
    p, r = shape
    n = min(p, r)
    rng = _rng(12)
    U, _ = np.linalg.qr(rng.standard_normal((p, n)))
    V, _ = np.linalg.qr(rng.standard_normal((r, n)))
    sig = np.array([3.0, 1.5, 1.0, 0.5, 0.2, 0.05, 0.01])[:n]
    G = U @ np.diag(sig) @ V.T
    a, b, c = 3.4445, -4.7750, 2.0315
    s = sig / (math.sqrt(float(np.sum(sig ** 2))) + 1e-7)
    for _ in range(5):
        s = a * s + b * s ** 3 + c * s ** 5
    expect = U @ np.diag(s) @ V.T
    got = O.newton_schulz(G, 5)
    assert np.max(np.abs(got - expect)) < 1e-12
    assert np.array_equal(O.newton_schulz(-G, 5), -got)
    assert np.max(np.abs(O.newton_schulz(1e3 * G, 5) - got)) < 1e-6  # invariant up to the eps term


# --------------------------------------------------------------------------- renormalisation
def test_renorm_keeps_initial_column_norms_every_chunk():
    q, k, v, eta, W0, W2, W1 = _layer(13, N=40, eta_scale=2.0)
    n0 = {"W0": O.column_norms(W0), "W1": O.column_norms(W1), "W2": O.column_norms(W2)}
    W = {"W0": W0, "W1": W1, "W2": W2}
    for c in range(5):
        sl = slice(8 * c, 8 * c + 8)
        _, W, _ = O.lact_recurrent(q[sl], k[sl], v[sl], eta[sl], W["W0"], W["W2"], W["W1"], 8,
                                   renorm=True, target_norms=n0)
        for name in O.WEIGHTS:
            assert np.max(np.abs(O.column_norms(W[name]) / n0[name] - 1)) < 1e-12
    # closed form: columns along the axes are rescaled exactly
    Wd = np.diag([2.0, 3.0, 4.0])
    assert np.allclose(O.renormalize_columns(Wd, [1.0, 1.0, 2.0]), np.diag([1.0, 1.0, 2.0]),
                       atol=0, rtol=1e-15)


# --------------------------------------------------------------------------- resume
def test_resume_split_equals_full_run():
    q, k, v, eta, W0, W2, W1 = _layer(14, N=48)
    alpha = _rng(15).uniform(0.3, 0.9, 6)
    kw = dict(renorm=True, ns_steps=5)
    full, Wf, Mf = O.lact_recurrent(q, k, v, eta, W0, W2, W1, 8, alpha=alpha, **kw)
    n0 = {n: O.column_norms(w) for n, w in (("W0", W0), ("W1", W1), ("W2", W2))}
    a, Wa, Ma = O.lact_recurrent(q[:24], k[:24], v[:24], eta[:24], W0, W2, W1, 8,
                                 alpha=alpha[:3], **kw)
    b, Wb, Mb = O.lact_recurrent(q[24:], k[24:], v[24:], eta[24:], Wa["W0"], Wa["W2"], Wa["W1"],
                                 8, alpha=alpha[3:], M_init=Ma, target_norms=n0, **kw)
    assert np.max(np.abs(np.concatenate([a, b]) - full)) < 1e-12
    for n in O.WEIGHTS:
        assert np.max(np.abs(Wb[n] - Wf[n])) < 1e-12
        assert np.max(np.abs(Mb[n] - Mf[n])) < 1e-12
    pf, Sf = O.la_parallel(q, k, v, eta, W0, W2, W1, 8)
    pa, Sa = O.la_parallel(q[:24], k[:24], v[:24], eta[:24], W0, W2, W1, 8)
    pb, Sb = O.la_parallel(q[24:], k[24:], v[24:], eta[24:], W0, W2, Sa, 8)
    assert np.max(np.abs(np.concatenate([pa, pb]) - pf)) < 1e-13
    assert np.max(np.abs(Sb - Sf)) < 1e-13


# --------------------------------------------------------------------------- In-Place TTT
def _inplace_small(seed=16, N=20, d=5, dH=7):
    r = _rng(seed)
    Hs = r.standard_normal((N, d))
    Wg = r.standard_normal((dH, d)) / math.sqrt(d)
    Wu = r.standard_normal((dH, d)) / math.sqrt(d)
    Wd = r.standard_normal((d, dH)) / math.sqrt(dH)
    X0 = r.standard_normal((N, d))
    cw = r.standard_normal((4, d)) * math.sqrt(0.5)
    Wt = r.standard_normal((d, d)) / math.sqrt(d)
    return Hs, Wg, Wu, Wd, X0, cw, Wt


def test_inplace_sequential_equals_prefix_and_generic_parallel():
    Hs, Wg, Wu, Wd, X0, cw, Wt = _inplace_small()
    Vbar = O.lm_target(X0, cw, Wt)
    eta = 1e-3
    os_, Ws = O.inplace_sequential(Hs, Wg, Wu, Wd, Vbar, 6, eta)
    op, Wp = O.inplace_prefix(Hs, Wg, Wu, Wd, Vbar, 6, eta)
    assert np.max(np.abs(os_ - op)) < 1e-13 and np.max(np.abs(Ws - Wp)) < 1e-13
    # the generic parallel layer with q = k = H, W0 = Wg^T, W2 = Wu^T, W1 = W_down^T,
    # v = Vbar, constant eta, apply-then-update computes the same thing
    og, Sg = O.la_parallel(Hs, Hs, Vbar, np.full(len(Hs), eta), Wg.T, Wu.T, Wd.T, 6,
                           order=O.APPLY_UPDATE)
    assert np.max(np.abs(og - os_)) < 1e-13 and np.max(np.abs(Sg.T - Ws)) < 1e-13


def test_lm_target_conv_brute_force_and_shift():
    Hs, Wg, Wu, Wd, X0, cw, Wt = _inplace_small(N=6, d=3)
    N, d = X0.shape
    conv = [[0.0] * d for _ in range(N)]
    for t in range(N):
        for i in range(d):
            for j in range(4):
                if t - j >= 0:
                    conv[t][i] += cw[j, i] * X0[t - j, i]
    assert np.max(np.abs(O.lm_target(X0, cw, Wt) - np.array(conv) @ Wt)) < 1e-13
    shift = np.zeros((4, d))
    shift[1] = 1.0
    got = O.lm_target(X0, shift, np.eye(d))
    assert np.array_equal(got[1:], X0[:-1]) and np.array_equal(got[0], np.zeros(d))
    ident = np.zeros((4, d))
    ident[0] = 1.0
    assert np.array_equal(O.lm_target(X0, ident, np.eye(d)), X0)


# ----------------------------------------------------------------------------- backward
@pytest.mark.parametrize("order", [O.UPDATE_APPLY, O.APPLY_UPDATE])
@pytest.mark.parametrize("sign", [1, -1])
def test_parallel_backward_matches_finite_differences(order, sign):
    """Every gradient of the parallel form against central differences of the forward
    oracle (fp64) on a tiny ragged problem, through a random linear functional of the
    outputs and of the final state."""
    rng = np.random.default_rng(17)
    N, h, m, chunk = 11, 3, 4, 4
    x = dict(q=rng.standard_normal((N, h)), k=rng.standard_normal((N, h)),
             v=rng.standard_normal((N, h)), eta=rng.uniform(0.1, 0.9, N),
             W0=rng.standard_normal((h, m)) * 0.5, W2=rng.standard_normal((h, m)) * 0.5,
             W1=rng.standard_normal((m, h)) * 0.5)
    dO = rng.standard_normal((N, h))
    dSf = rng.standard_normal((m, h))

    def loss(**kw):
        a = dict(x)
        a.update(kw)
        O_, S_ = O.la_parallel(a["q"], a["k"], a["v"], a["eta"], a["W0"], a["W2"], a["W1"],
                               chunk, order=order, sign=sign)
        return float(np.sum(O_ * dO) + np.sum(S_ * dSf))

    g = O.la_parallel_backward(x["q"], x["k"], x["v"], x["eta"], x["W0"], x["W2"], x["W1"], dO,
                               chunk, order=order, sign=sign, dS_final=dSf)
    eps = 1e-6
    for name, key in (("q", "dq"), ("k", "dk"), ("v", "dv"), ("eta", "deta"), ("W0", "dW0"),
                      ("W2", "dW2"), ("W1", "dW1")):
        base = x[name]
        num = np.empty_like(base)
        for idx in np.ndindex(base.shape):
            up, dn = base.copy(), base.copy()
            up[idx] += eps
            dn[idx] -= eps
            num[idx] = (loss(**{name: up}) - loss(**{name: dn})) / (2 * eps)
        assert np.allclose(g[key], num, rtol=1e-6, atol=1e-7), key


def test_parallel_backward_w1_gradient_is_the_output_functional():
    """The outputs are linear in W1 with every state containing it once: dW1 is the sum over
    chunks of phi(Q_c)^T dO_c (plus the final-state cotangent), in both orders."""
    rng = np.random.default_rng(3)
    N, h, m, chunk = 9, 2, 3, 3
    q, k, v = (rng.standard_normal((N, h)) for _ in range(3))
    eta = np.full(N, 0.5)
    W0, W2, W1 = rng.standard_normal((h, m)), rng.standard_normal((h, m)), rng.standard_normal((m, h))
    dO = rng.standard_normal((N, h))
    phiQ = O.swiglu_features(q, W0, W2)
    for order in (O.UPDATE_APPLY, O.APPLY_UPDATE):
        g = O.la_parallel_backward(q, k, v, eta, W0, W2, W1, dO, chunk, order=order)
        assert np.allclose(g["dW1"], phiQ.T @ dO, rtol=1e-12, atol=1e-12)
