"""Torch-tensor front end of the C ABI: builds the ``ttt_desc``, allocates outputs and the
workspace with torch, and calls the library. No arithmetic of the layer happens here.

Shapes (see include/ttt.h): q, k, v [B,H,N,h] (bf16 or fp32, contiguous, on the GPU);
eta [B,H,N] fp32; W0, W2 [H,h,m] fp32 ([H,m,h] with w_in_layout=1); W1 [H,m,h] fp32
([H,h,m] with w1_layout=1).
"""
from __future__ import annotations

import torch

from . import abi

ORDERS = {"update_apply": abi.TTT_ORDER_UPDATE_APPLY, "apply_update": abi.TTT_ORDER_APPLY_UPDATE}


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return abi.TTT_DTYPE_BF16
    if t.dtype == torch.float32:
        return abi.TTT_DTYPE_FP32
    raise TypeError(f"q/k/v must be bfloat16 or float32, got {t.dtype}")


def _need(t, name, dtype=None):
    if t is None:
        return
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")


def workspace(nbytes: int, device) -> torch.Tensor:
    """A device byte buffer of at least ``nbytes`` (torch allocations are 512-byte aligned)."""
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def parallel_desc(q, W1, chunk, order="update_apply", sign=1, w_in_layout=0, w1_layout=0):
    B, H, N, h = q.shape
    m = W1.shape[1] if w1_layout == 0 else W1.shape[2]
    return abi.ttt_desc(B=B, H=H, N=N, h=h, m=m, chunk=chunk, dtype=_dtype_code(q),
                        order=ORDERS[order], sign=sign, w_in_layout=w_in_layout,
                        w1_layout=w1_layout)


def la_parallel_fwd(q, k, v, eta, W0, W2, W1, chunk, *, order="update_apply", sign=1,
                    w_in_layout=0, w1_layout=0, return_state=True, out=None, ws=None,
                    stream=None):
    """Parallel last-layer-only form. Returns (out [B,H,N,h], final state or None)."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n, q.dtype)
    _need(eta, "eta", torch.float32)
    for t, n in ((W0, "W0"), (W2, "W2"), (W1, "W1")):
        _need(t, n, torch.float32)
    desc = parallel_desc(q, W1, chunk, order, sign, w_in_layout, w1_layout)
    B, H, N, h = q.shape
    m = desc.m
    if out is None:
        out = torch.empty_like(q)
    S = None
    if return_state:
        shape = (B, H, m, h) if w1_layout == 0 else (B, H, h, m)
        S = torch.empty(shape, dtype=torch.float32, device=q.device)
    if ws is None:
        ws = workspace(abi.ttt_workspace_bytes(desc, abi.TTT_PATH_PARALLEL), q.device)
    abi.ttt_la_parallel_fwd(desc, q, k, v, eta, W0, W2, W1, out, S, ws, stream=stream)
    return out, S


def la_parallel_fwd_shard(q, k, v, eta, W0, W2, W1, chunk, *, prior=None, state_only=False,
                          order="update_apply", sign=1, w_in_layout=0, w1_layout=0, m=None,
                          out=None, ws=None, stream=None):
    """One contiguous shard of a sequence (context parallelism): the parallel form from the
    initial state W1 (zeros when None) plus the sum of ``prior`` [n, B, H, m, h] (W1's
    layout per entry) along its first axis. ``state_only`` skips the outputs. Returns
    (out or None, final state). ``m`` is needed when W1 is None."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n, q.dtype)
    _need(eta, "eta", torch.float32)
    for t, n in ((W0, "W0"), (W2, "W2"), (W1, "W1"), (prior, "prior")):
        _need(t, n, torch.float32)
    B, H, N, h = q.shape
    if m is None:
        m = W1.shape[1] if w1_layout == 0 else W1.shape[2]
    desc = abi.ttt_desc(B=B, H=H, N=N, h=h, m=m, chunk=chunk, dtype=_dtype_code(q),
                        order=ORDERS[order], sign=sign, w_in_layout=w_in_layout,
                        w1_layout=w1_layout)
    if out is None and not state_only:
        out = torch.empty_like(q)
    S = torch.empty((B, H, m, h) if w1_layout == 0 else (B, H, h, m), dtype=torch.float32,
                    device=q.device)
    if ws is None:
        ws = workspace(abi.ttt_workspace_bytes(desc, abi.TTT_PATH_PARALLEL), q.device)
    n_prior = 0 if prior is None else prior.shape[0]
    abi.ttt_la_parallel_fwd_shard(desc, q, k, v, eta, W0, W2, W1, prior if n_prior else None,
                                  n_prior, None if state_only else out, S, ws, stream=stream)
    return (None if state_only else out), S


def la_parallel_fwd_shard_outputs(q, W1, chunk, ws, *, prior=None, order="update_apply",
                                  sign=1, w_in_layout=0, w1_layout=0, m=None, out=None,
                                  stream=None):
    """The outputs pass of a shard after its state-only pass ``la_parallel_fwd_shard(...,
    state_only=True, ws=ws)`` on this thread: reuses that call's chunk deltas (left in
    ``ws``) and forms the states from W1 (zeros when None) plus the sum of ``prior``, then
    the outputs. Returns (out, final state). ``m`` is needed when W1 is None."""
    _need(q, "q", q.dtype)
    for t, n in ((W1, "W1"), (prior, "prior")):
        _need(t, n, torch.float32)
    B, H, N, h = q.shape
    if m is None:
        m = W1.shape[1] if w1_layout == 0 else W1.shape[2]
    desc = abi.ttt_desc(B=B, H=H, N=N, h=h, m=m, chunk=chunk, dtype=_dtype_code(q),
                        order=ORDERS[order], sign=sign, w_in_layout=w_in_layout,
                        w1_layout=w1_layout)
    if out is None:
        out = torch.empty_like(q)
    S = torch.empty((B, H, m, h) if w1_layout == 0 else (B, H, h, m), dtype=torch.float32,
                    device=q.device)
    n_prior = 0 if prior is None else prior.shape[0]
    abi.ttt_la_parallel_fwd_shard_outputs(desc, q, W1, prior if n_prior else None, n_prior,
                                          out, S, ws, stream=stream)
    return out, S


def la_parallel_momentum_fwd(q, k, v, eta, W0, W2, W1, chunk, *, order="update_apply", sign=1,
                             alpha=None, ns_steps=0, w_in_layout=0, return_state=True,
                             out=None, ws=None, stream=None):
    """Parallel form with W1 momentum (when ``alpha`` [B,H,C] is given) and Newton-Schulz.
    Returns (out [B,H,N,h], final state [B,H,m,h] or None)."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n, q.dtype)
    _need(eta, "eta", torch.float32)
    _need(alpha, "alpha", torch.float32)
    desc = parallel_desc(q, W1, chunk, order, sign, w_in_layout, 0)
    desc.momentum = int(alpha is not None)
    desc.ns_steps = ns_steps
    B, H, N, h = q.shape
    if out is None:
        out = torch.empty_like(q)
    S = torch.empty((B, H, desc.m, h), dtype=torch.float32, device=q.device) if return_state else None
    if ws is None:
        ws = workspace(abi.ttt_workspace_bytes(desc, abi.TTT_PATH_PARALLEL_MOMENTUM), q.device)
    abi.ttt_la_parallel_momentum_fwd(desc, q, k, v, eta, alpha, W0, W2, W1, out, S, ws,
                                     stream=stream)
    return out, S


def la_parallel_bwd(q, k, v, eta, W0, W2, W1, dout, chunk, *, order="update_apply", sign=1,
                    dS_final=None, ws=None, stream=None):
    """Backward of la_parallel_fwd. Returns dq, dk, dv (q's dtype), deta, dW0, dW2, dW1
    (fp32; weight gradients per head, summed over the batch)."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (dout, "dout")):
        _need(t, n, q.dtype)
    _need(eta, "eta", torch.float32)
    _need(dS_final, "dS_final", torch.float32)
    desc = parallel_desc(q, W1, chunk, order, sign)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    deta = torch.empty_like(eta)
    dW0, dW2, dW1 = torch.empty_like(W0), torch.empty_like(W2), torch.empty_like(W1)
    if ws is None:
        ws = workspace(abi.ttt_workspace_bytes(desc, abi.TTT_PATH_PARALLEL_BWD), q.device)
    abi.ttt_la_parallel_bwd(desc, q, k, v, eta, W0, W2, W1, dout, dS_final, dq, dk, dv, deta,
                            dW0, dW2, dW1, ws, stream=stream)
    return dq, dk, dv, deta, dW0, dW2, dW1


def linear_attn_fwd(q, k, v, eta, S0, chunk, *, order="update_apply", sign=1, s_layout=0,
                    return_state=True, out=None, ws=None, stream=None):
    """Parallel form with identity features (plain chunked linear attention with per-token
    eta). S0 [H,h,h] fp32. Returns (out [B,H,N,h], final state [B,H,h,h] or None)."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n, q.dtype)
    _need(eta, "eta", torch.float32)
    _need(S0, "S0", torch.float32)
    B, H, N, h = q.shape
    desc = abi.ttt_desc(B=B, H=H, N=N, h=h, m=h, chunk=chunk, dtype=_dtype_code(q),
                        order=ORDERS[order], sign=sign, w1_layout=s_layout)
    if out is None:
        out = torch.empty_like(q)
    S = torch.empty((B, H, h, h), dtype=torch.float32, device=q.device) if return_state else None
    if ws is None:
        ws = workspace(abi.ttt_workspace_bytes(desc, abi.TTT_PATH_LINEAR), q.device)
    abi.ttt_linear_attn_fwd(desc, q, k, v, eta, S0, out, S, ws, stream=stream)
    return out, S


def recurrent_desc(q, W1, chunk, order="update_apply", sign=1, update_mask=abi.TTT_UPDATE_ALL,
                   renorm=False, momentum=False, ns_steps=0):
    B, H, N, h = q.shape
    return abi.ttt_desc(B=B, H=H, N=N, h=h, m=W1.shape[1], chunk=chunk, dtype=_dtype_code(q),
                        order=ORDERS[order], sign=sign, update_mask=update_mask,
                        renorm=int(renorm), momentum=int(momentum), ns_steps=ns_steps)


def lact_recurrent_fwd(q, k, v, eta, W0, W2, W1, chunk, *, order="update_apply", sign=1,
                       update_mask=abi.TTT_UPDATE_ALL, renorm=False, alpha=None, ns_steps=0,
                       M_init=None, return_weights=True, return_momentum=False, out=None,
                       ws=None, stream=None):
    """Recurrent LaCT form. Returns (out, (W0, W2, W1) finals or None, momentum or None).
    Momentum is on when ``alpha`` [B,H,C] is given; ``M_init`` [B,H,3hm] resumes it."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n, q.dtype)
    _need(eta, "eta", torch.float32)
    _need(alpha, "alpha", torch.float32)
    for t, n in ((W0, "W0"), (W2, "W2"), (W1, "W1")):
        _need(t, n, torch.float32)
    momentum = alpha is not None
    desc = recurrent_desc(q, W1, chunk, order, sign, update_mask, renorm, momentum, ns_steps)
    B, H, N, h = q.shape
    m = desc.m
    dev = q.device
    if out is None:
        out = torch.empty_like(q)
    Wf = None
    if return_weights:
        Wf = (torch.empty((B, H, h, m), dtype=torch.float32, device=dev),
              torch.empty((B, H, h, m), dtype=torch.float32, device=dev),
              torch.empty((B, H, m, h), dtype=torch.float32, device=dev))
    M = None
    if momentum and (return_momentum or M_init is not None):
        M = torch.zeros((B, H, 3 * h * m), dtype=torch.float32, device=dev)
        if M_init is not None:
            M.copy_(M_init)
    if ws is None:
        ws = workspace(abi.ttt_workspace_bytes(desc, abi.TTT_PATH_RECURRENT), dev)
    abi.ttt_lact_recurrent_fwd(desc, q, k, v, eta, alpha, W0, W2, W1, out,
                               Wf[0] if Wf else None, Wf[1] if Wf else None,
                               Wf[2] if Wf else None, M, ws, stream=stream)
    return out, Wf, M


def lm_target(X0, conv_w, W_target, *, out=None, ws=None, stream=None):
    """LM-aligned target Vbar = Conv1D(X0) W_target (bf16 [N,d])."""
    _need(X0, "X0", torch.bfloat16)
    _need(conv_w, "conv_w", torch.float32)
    _need(W_target, "W_target", torch.bfloat16)
    N, d = X0.shape
    if out is None:
        out = torch.empty_like(X0)
    if ws is None:
        ws = workspace(abi.ttt_lm_target_workspace_bytes(N, d), X0.device)
    abi.ttt_lm_target(N, d, X0, conv_w, W_target, out, ws, stream=stream)
    return out
