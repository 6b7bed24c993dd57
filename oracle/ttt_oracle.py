"""Plain fp64 CPU oracle for the chunked TTT-KVB fast-weight layer.

TEST INFRASTRUCTURE ONLY. This module is the correctness reference for the CUDA path.
Only the test suite, the smoke check in ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import it. The product
path (the C-ABI library and its Python binding) never calls into it, and it shares no
code, tables or helpers with that path.

Everything is float64 NumPy, written for a reader who checks it against the pages by eye:
no blocking, fusion or reordering beyond what the definitions state. Library matmuls,
``cumsum`` and ``linalg.norm`` serve as single steps.

Notation (row vectors, one (batch, head) at a time): q, k, v in R^{N x h}, eta in R^N.
W0, W2 in R^{h x m} (input side), W1 in R^{m x h} (the last, linear layer). Chunk c holds
rows [c*b, (c+1)*b); the last chunk may be shorter.

Sources (pages and sections):
* "Test-Time Training with KV Binding Is Secretly Linear Attention" (paper notes),
  sections "前置知识 / LaCT" (the SwiGLU inner map f(x)=silu(xW0)*(xW2)W1 and the loss
  L=-<f(k),v>), "前置知识 / 线性注意力" (o = phi(q) S, S = S0 + sum phi(k)^T v),
  "前置知识 / 前缀扫描" (prefix sums over an associative update), and
  "方法步骤详情" (Theorems 5.1-5.3 and the six simplification steps).
* "NVIDIA团队揭秘：测试时训练的真实面目原来如此不同", section 四 (the parallel form over
  chunks; weight normalisation breaks associativity).
* "Test-Time Training Done Right: 中文精读笔记", sections 2.1 (symbols, per-token eta),
  2.2 (gradient / Muon writes, per-input-dim weight normalisation, momentum, five
  Newton-Schulz steps with 3.4445, -4.7750, 2.0315), 2.3 (update/apply orders).
* "In-Place Test-Time Training", sections 3.1 (eq. 2, chunk-wise apply-then-update of
  W_down), 3.2 (eq. 3 target V = Conv1D(X0) W_target, eq. 4 update), 3.4 (the
  context-parallel exclusive prefix-sum form).

Readings of points the pages leave open (each is listed in the design notes):
* step size: eta sits inside the loss and the step size is 1;
* renormalisation: after each step every column (output unit) of an updated matrix is
  rescaled over the input dimension to the column norm it had at the start of the
  sequence; no epsilon;
* momentum: M <- alpha_c M + g with M = 0 at the start, applied to the raw gradient,
  before orthogonalisation; the momentum buffer itself is never orthogonalised;
* Newton-Schulz: X = G / (||G||_F + 1e-7); iterate on the wide orientation (rows <= cols)
  X <- a X + (b A + c A^2) X with A = X X^T; no post-scaling;
* ascent (sign = -1) moves the weights along +g instead of -g;
* the causal Conv1D of the In-Place target uses taps t, t-1, t-2, t-3 (tap j multiplies
  X0[t-j]) with zero padding before the first token.
"""
from __future__ import annotations

import numpy as np

UPDATE_APPLY = "update_apply"   # a chunk's queries read the weights after its own update
APPLY_UPDATE = "apply_update"   # a chunk's queries read the weights from before its update
NS_COEFFS = (3.4445, -4.7750, 2.0315)
NS_EPS = 1e-7
WEIGHTS = ("W0", "W1", "W2")


def _f64(x):
    return np.asarray(x, dtype=np.float64)


# ----------------------------------------------------------------------------- activations
def sigmoid(a):
    a = _f64(a)
    out = np.empty_like(a)
    pos = a >= 0
    out[pos] = 1.0 / (1.0 + np.exp(-a[pos]))
    e = np.exp(a[~pos])
    out[~pos] = e / (1.0 + e)
    return out


def silu(a):
    """silu(a) = a * sigmoid(a)."""
    a = _f64(a)
    return a * sigmoid(a)


def silu_prime(a):
    """d silu / da = s (1 + a (1 - s)) with s = sigmoid(a)."""
    a = _f64(a)
    s = sigmoid(a)
    return s * (1.0 + a * (1.0 - s))


# ----------------------------------------------------------------------------- inner model
def swiglu_features(X, W0, W2):
    """phi(X) = silu(X W0) * (X W2): the hidden layer of LaCT's bias-free SwiGLU fast
    weight ("Test-Time Training with KV Binding Is Secretly Linear Attention", 前置知识 /
    LaCT; "Test-Time Training Done Right" notes, section 2.1)."""
    X = _f64(X)
    return silu(X @ _f64(W0)) * (X @ _f64(W2))


def fast_weight_forward(X, W0, W2, W1):
    """f(X) = phi(X) W1, the inner map read by the queries."""
    return swiglu_features(X, W0, W2) @ _f64(W1)


def inner_loss(W0, W2, W1, K, V, eta):
    """Chunk loss L = -sum_i eta_i <f(k_i), v_i> (negative dot-product / Frobenius inner
    product objective, per-token learning rate eta_i)."""
    F = fast_weight_forward(K, W0, W2, W1)
    return -float(np.sum(_f64(eta)[:, None] * F * _f64(V)))


def inner_grads(W0, W2, W1, K, V, eta):
    """Gradients of the chunk loss w.r.t. W0, W1, W2 at fixed weights (chain rule).

    G = dL/df = -diag(eta) V;  dW1 = phi^T G;  D = dL/dphi = G W1^T;
    dW2 = K^T (D * silu(A));  dW0 = K^T (D * B * silu'(A));  A = K W0, B = K W2.
    """
    K, V, eta = _f64(K), _f64(V), _f64(eta)
    W0, W2, W1 = _f64(W0), _f64(W2), _f64(W1)
    A = K @ W0
    Bm = K @ W2
    sA = silu(A)
    phi = sA * Bm
    G = -(eta[:, None] * V)
    D = G @ W1.T
    return {
        "W0": K.T @ (D * Bm * silu_prime(A)),
        "W1": phi.T @ G,
        "W2": K.T @ (D * sA),
    }


# ----------------------------------------------------------------------------- update operators
def newton_schulz(G, steps=5, coeffs=NS_COEFFS, eps=NS_EPS):
    """Approximate orthogonalisation of an update matrix by ``steps`` quintic
    Newton-Schulz iterations with coefficients (3.4445, -4.7750, 2.0315)
    ("Test-Time Training Done Right" notes, section 2.2 / appendix A).

    X = G / (||G||_F + eps), taken in the orientation with rows <= cols;
    X <- a X + (b A + c A^2) X with A = X X^T.
    """
    a, b, c = coeffs
    G = _f64(G)
    X = G / (np.linalg.norm(G) + eps)
    transposed = X.shape[0] > X.shape[1]
    if transposed:
        X = X.T
    for _ in range(steps):
        A = X @ X.T
        X = a * X + (b * A + c * (A @ A)) @ X
    return X.T if transposed else X


def column_norms(W):
    """Norm of every column (output unit) taken over the rows (the input dimension)."""
    W = _f64(W)
    return np.sqrt(np.sum(W * W, axis=0))


def renormalize_columns(W, target_norms):
    """Rescale each column of W to ``target_norms`` (weight normalisation along the input
    dimension, "Test-Time Training Done Right" notes, section 2.2)."""
    W = _f64(W)
    return W * (_f64(target_norms) / column_norms(W))[None, :]


# ----------------------------------------------------------------------------- recurrent form
def chunk_slices(N, chunk):
    return [slice(s, min(N, s + chunk)) for s in range(0, N, chunk)]


def lact_recurrent(q, k, v, eta, W0, W2, W1, chunk, *, order=UPDATE_APPLY, sign=1,
                   update=WEIGHTS, renorm=False, alpha=None, ns_steps=0, M_init=None,
                   target_norms=None):
    """Recurrent LaCT form for one (batch, head).

    For each chunk, at the chunk-start weights: gradient of the chunk loss for every
    updated matrix -> optional momentum (M <- alpha_c M + g) -> optional Newton-Schulz
    -> step W <- W - sign * u -> optional column renormalisation to the sequence-start
    column norms. The chunk's queries read f(q) with the weights after the update
    (update_apply) or before it (apply_update).

    Returns (O [N,h], weights dict, momentum dict or None).
    """
    q, k, v, eta = _f64(q), _f64(k), _f64(v), _f64(eta)
    W = {"W0": _f64(W0).copy(), "W1": _f64(W1).copy(), "W2": _f64(W2).copy()}
    if target_norms is None:
        target_norms = {name: column_norms(W[name]) for name in update}
    M = None
    if alpha is not None:
        M = {name: (np.zeros_like(W[name]) if M_init is None else _f64(M_init[name]).copy())
             for name in update}
    N, h = q.shape
    O = np.empty((N, h))
    for c, sl in enumerate(chunk_slices(N, chunk)):
        if order == APPLY_UPDATE:
            O[sl] = fast_weight_forward(q[sl], W["W0"], W["W2"], W["W1"])
        g = inner_grads(W["W0"], W["W2"], W["W1"], k[sl], v[sl], eta[sl])
        for name in update:
            u = g[name]
            if M is not None:
                M[name] = float(alpha[c]) * M[name] + u
                u = M[name]
            if ns_steps:
                u = newton_schulz(u, ns_steps)
            W[name] = W[name] - sign * u
            if renorm:
                W[name] = renormalize_columns(W[name], target_norms[name])
        if order == UPDATE_APPLY:
            O[sl] = fast_weight_forward(q[sl], W["W0"], W["W2"], W["W1"])
    return O, W, M


# ----------------------------------------------------------------------------- parallel form
def chunk_state_deltas(phiK, V, eta, chunk, sign=1):
    """Delta S_c = sign * phi(K_c)^T diag(eta_c) V_c for every chunk (the last-layer
    update of one chunk written as a sum of outer products; Theorem 5.2)."""
    phiK, V, eta = _f64(phiK), _f64(V), _f64(eta)
    return [sign * (phiK[sl].T @ (eta[sl, None] * V[sl])) for sl in chunk_slices(len(V), chunk)]


def chunked_linear_attention(phiQ, phiK, V, eta, S0, chunk, order=UPDATE_APPLY, sign=1):
    """Chunked linear attention with static features: S_c = S0 + sum_{c' <= c} Delta S_c'
    (inclusive, update_apply) or sum over c' < c (exclusive, apply_update);
    O_c = phi(Q_c) S_c.  Returns (O [N,h], S after the last chunk)."""
    phiQ = _f64(phiQ)
    dS = chunk_state_deltas(phiK, V, eta, chunk, sign)
    S = _f64(S0).copy()
    O = np.empty((phiQ.shape[0], S.shape[1]))
    for c, sl in enumerate(chunk_slices(phiQ.shape[0], chunk)):
        if order == APPLY_UPDATE:
            O[sl] = phiQ[sl] @ S
            S = S + dS[c]
        else:
            S = S + dS[c]
            O[sl] = phiQ[sl] @ S
    return O, S


def la_parallel(q, k, v, eta, W0, W2, W1, chunk, *, order=UPDATE_APPLY, sign=1):
    """Parallel last-layer-only form: W0, W2 frozen, no renormalisation, so the features
    are static and the W1 updates add up (associative); phi(K) and phi(Q) for all chunks,
    state deltas, prefix sum over chunks, outputs phi(Q_c) S_c."""
    phiK = swiglu_features(k, W0, W2)
    phiQ = swiglu_features(q, W0, W2)
    return chunked_linear_attention(phiQ, phiK, v, eta, W1, chunk, order, sign)


def la_parallel_backward(q, k, v, eta, W0, W2, W1, dO, chunk, *, order=UPDATE_APPLY, sign=1,
                         dS_final=None):
    """Gradients of the parallel form's outputs (and of its final state, when dS_final is
    given) for one (batch, head): the chain rule through O_c = phi(Q_c) S_c, the prefix sum
    S_c = W1 + sum ΔS_c' and ΔS_c = sign phi(K_c)^T diag(eta_c) V_c (TTT≡LA notes,
    方法步骤详情), then through phi = silu(X W0) * (X W2). Returns dq, dk, dv, deta, dW0, dW2,
    dW1 in the shapes of the inputs.

    With R_c = dS_final + sum_{c' >= c} phi(Q_c')^T dO_c' (suffix sum), the gradient of
    ΔS_c is G_c = R_c (update_apply: chunk c's own delta reaches its own outputs) or R_{c+1}
    (apply_update), and dW1 = R_0."""
    q, k, v, eta, dO = _f64(q), _f64(k), _f64(v), _f64(eta), _f64(dO)
    W0, W2, W1 = _f64(W0), _f64(W2), _f64(W1)
    N = len(q)
    Aq, Bq, Ak, Bk = q @ W0, q @ W2, k @ W0, k @ W2
    phiQ, phiK = silu(Aq) * Bq, silu(Ak) * Bk
    sl = chunk_slices(N, chunk)
    dS = [sign * (phiK[c].T @ (eta[c, None] * v[c])) for c in sl]
    # the state each chunk reads
    S, Sc = W1.copy(), []
    for d in dS:
        if order == APPLY_UPDATE:
            Sc.append(S.copy())
            S = S + d
        else:
            S = S + d
            Sc.append(S.copy())
    R = np.zeros_like(W1) if dS_final is None else _f64(dS_final).copy()
    Rs = [None] * (len(sl) + 1)
    Rs[len(sl)] = R.copy()
    for ci in range(len(sl) - 1, -1, -1):
        R = R + phiQ[sl[ci]].T @ dO[sl[ci]]
        Rs[ci] = R.copy()
    dphiQ = np.empty_like(phiQ)
    dphiK = np.empty_like(phiK)
    dv = np.empty_like(v)
    deta = np.empty_like(eta)
    for ci, c in enumerate(sl):
        G = Rs[ci] if order == UPDATE_APPLY else Rs[ci + 1]
        dphiQ[c] = dO[c] @ Sc[ci].T
        T = phiK[c] @ G                              # [L, h]
        dv[c] = sign * eta[c, None] * T
        deta[c] = sign * np.sum(T * v[c], axis=1)
        dphiK[c] = sign * eta[c, None] * (v[c] @ G.T)
    out = {"dW1": Rs[0]}
    dW0 = np.zeros_like(W0)
    dW2 = np.zeros_like(W2)
    for X, A, B, dphi, name in ((q, Aq, Bq, dphiQ, "dq"), (k, Ak, Bk, dphiK, "dk")):
        dA = dphi * B * silu_prime(A)
        dB = dphi * silu(A)
        out[name] = dA @ W0.T + dB @ W2.T
        dW0 += X.T @ dA
        dW2 += X.T @ dB
    out.update(dv=dv, deta=deta, dW0=dW0, dW2=dW2)
    return out


def la_parallel_rows(q, k, v, eta, W0, W2, W1, chunk, rows, *, order=UPDATE_APPLY, sign=1):
    """Outputs of the parallel form at the given token rows only, plus the final state.
    Every chunk state up to the last needed chunk is formed in full; only the query side
    is restricted to ``rows``."""
    rows = np.asarray(rows)
    N = len(v)
    dS = chunk_state_deltas(swiglu_features(k, W0, W2), v, eta, chunk, sign)
    incl = []
    S = _f64(W1).copy()
    for d in dS:
        S = S + d
        incl.append(S)
    c_of = rows // chunk
    phiQ = swiglu_features(_f64(q)[rows], W0, W2)
    O = np.empty((len(rows), _f64(W1).shape[1]))
    for i, c in enumerate(c_of):
        if order == APPLY_UPDATE:
            Sc = _f64(W1) if c == 0 else incl[c - 1]
        else:
            Sc = incl[c]
        O[i] = phiQ[i] @ Sc
    assert len(incl) == -(-N // chunk)
    return O, incl[-1]


def la_masked(phiQ, phiK, V, eta, S0, chunk, order=UPDATE_APPLY, sign=1):
    """The same chunked linear attention in its masked (attention-matrix) form:
    O = phi(Q) S0 + sign * ((phi(Q) phi(K)^T) * M) diag(eta) V, with M[t,i] = 1 when
    token i's chunk is at or before (update_apply) / strictly before (apply_update)
    token t's chunk."""
    phiQ, phiK, V, eta = _f64(phiQ), _f64(phiK), _f64(V), _f64(eta)
    cid = np.arange(len(V)) // chunk
    if order == APPLY_UPDATE:
        Mask = cid[:, None] > cid[None, :]
    else:
        Mask = cid[:, None] >= cid[None, :]
    return phiQ @ _f64(S0) + sign * ((phiQ @ phiK.T) * Mask) @ (eta[:, None] * V)


# ----------------------------------------------------------------------------- In-Place TTT
def lm_target(X0, conv_w, W_target):
    """LM-aligned value target V = Conv1D(X0) W_target with a causal depthwise Conv1D:
    (Conv1D(X0))_t = sum_j conv_w[j] * X0[t-j], X0[t-j] = 0 for t-j < 0
    ("In-Place Test-Time Training", section 3.2, eq. 3)."""
    X0, conv_w = _f64(X0), _f64(conv_w)
    N = X0.shape[0]
    Xc = np.zeros_like(X0)
    for j in range(conv_w.shape[0]):
        if j < N:
            Xc[j:] += conv_w[j][None, :] * X0[:N - j]
    return Xc @ _f64(W_target)


def inplace_intermediate(Hs, Wg, Wu):
    """Z = silu(H Wg^T) * (H Wu^T) (In-Place TTT, section 3.1, eq. 2)."""
    Hs = _f64(Hs)
    return silu(Hs @ _f64(Wg).T) * (Hs @ _f64(Wu).T)


def inplace_sequential(Hs, Wg, Wu, W_down, Vbar, chunk, eta):
    """Chunk-wise apply then update of the fast W_down (In-Place TTT, section 3.1):
    O_[i] = Z_[i] W_down^T, then W_down += eta Vbar_[i]^T Z_[i] (eq. 4).
    Returns (O [N,d], W_down after the last chunk)."""
    Z = inplace_intermediate(Hs, Wg, Wu)
    Vbar = _f64(Vbar)
    W = _f64(W_down).copy()
    O = np.empty((Z.shape[0], W.shape[0]))
    for sl in chunk_slices(Z.shape[0], chunk):
        O[sl] = Z[sl] @ W.T
        W = W + eta * (Vbar[sl].T @ Z[sl])
    return O, W


def inplace_prefix(Hs, Wg, Wu, W_down, Vbar, chunk, eta):
    """Context-parallel form (In-Place TTT, section 3.4): all Delta W_j = Vbar_[j]^T Z_[j]
    at once, exclusive prefix sums, W_i = W_down + eta * sum_{j<i} Delta W_j, then all
    outputs O_[i] = Z_[i] W_i^T at once."""
    Z = inplace_intermediate(Hs, Wg, Wu)
    Vbar = _f64(Vbar)
    sls = chunk_slices(Z.shape[0], chunk)
    dW = np.stack([Vbar[sl].T @ Z[sl] for sl in sls])
    excl = np.concatenate([np.zeros_like(dW[:1]), np.cumsum(dW, axis=0)[:-1]], axis=0)
    O = np.empty((Z.shape[0], _f64(W_down).shape[0]))
    for i, sl in enumerate(sls):
        O[sl] = Z[sl] @ (_f64(W_down) + eta * excl[i]).T
    return O, _f64(W_down) + eta * np.sum(dW, axis=0)


# ----------------------------------------------------------------------------- batched wrappers
def la_parallel_batched(q, k, v, eta, W0, W2, W1, chunk, *, order=UPDATE_APPLY, sign=1):
    """la_parallel over [B,H,...] inputs with per-head weights [H,...].
    Returns O [B,H,N,h] and the final states [B,H,m,h]."""
    B, H, N, h = q.shape
    m = W1.shape[1]
    O = np.empty((B, H, N, h))
    S = np.empty((B, H, m, h))
    for b in range(B):
        for hd in range(H):
            O[b, hd], S[b, hd] = la_parallel(q[b, hd], k[b, hd], v[b, hd], eta[b, hd],
                                             W0[hd], W2[hd], W1[hd], chunk, order=order,
                                             sign=sign)
    return O, S


def linear_attention_batched(q, k, v, eta, S0, chunk, *, order=UPDATE_APPLY, sign=1):
    """The parallel form with identity features over [B,H,...] inputs (TTT≡LA notes,
    方法步骤详情, variants 3-6: phi(x) = x), per-head initial states S0 [H,h,h].
    Returns O [B,H,N,h] and the final states [B,H,h,h]."""
    B, H, N, h = q.shape
    O = np.empty((B, H, N, h))
    S = np.empty((B, H, h, h))
    for b in range(B):
        for hd in range(H):
            O[b, hd], S[b, hd] = chunked_linear_attention(q[b, hd], k[b, hd], v[b, hd],
                                                          eta[b, hd], S0[hd], chunk, order,
                                                          sign)
    return O, S


def lact_recurrent_batched(q, k, v, eta, W0, W2, W1, chunk, *, order=UPDATE_APPLY, sign=1,
                           update=WEIGHTS, renorm=False, alpha=None, ns_steps=0):
    """lact_recurrent over [B,H,...] inputs. Returns O [B,H,N,h], final weights
    {W0: [B,H,h,m], W1: [B,H,m,h], W2: [B,H,h,m]} and final momentum (or None)."""
    B, H, N, h = q.shape
    O = np.empty((B, H, N, h))
    Wf = {"W0": np.empty((B, H) + W0.shape[1:]), "W1": np.empty((B, H) + W1.shape[1:]),
          "W2": np.empty((B, H) + W2.shape[1:])}
    Mf = None
    if alpha is not None:
        Mf = {name: np.zeros((B, H) + Wf[name].shape[2:]) for name in WEIGHTS}
    for b in range(B):
        for hd in range(H):
            o, W, M = lact_recurrent(q[b, hd], k[b, hd], v[b, hd], eta[b, hd], W0[hd], W2[hd],
                                     W1[hd], chunk, order=order, sign=sign, update=update,
                                     renorm=renorm,
                                     alpha=None if alpha is None else alpha[b, hd],
                                     ns_steps=ns_steps)
            O[b, hd] = o
            for name in WEIGHTS:
                Wf[name][b, hd] = W[name]
            if M is not None:
                for name in M:
                    Mf[name][b, hd] = M[name]
    return O, Wf, Mf
