"""Seeded synthetic workloads for the chunked TTT-KVB layer.

This module only draws random numbers and shapes them into the inputs of the five
workloads (tiny check, LM-shaped LaCT layer, long context, NVS-shaped recurrent LaCT,
In-Place-TTT-shaped last-layer update). It holds none of the layer's arithmetic: no
features, no gradients, no scans. Both the fp64 oracle's tests and the CUDA path's
tests and benchmark take their inputs from here, so the two sides see identical values.

Conventions
-----------
* Generator: numpy PCG64, one generator per workload, seed = 20261202 + workload index
  (callers may pass another seed for reduced test shapes).
* ``N(mu, s2)`` in a recipe is read with ``s2`` as the VARIANCE, so ``N(0, 1/h)`` is the
  usual fan-in initialisation; ``N(-2, 0.5)`` has standard deviation sqrt(0.5).
* q, k, v are drawn N(0,1) and L2-normalised per token in float64, then cast to float32.
* "bf16" inputs are rounded to bfloat16 by round-to-nearest-even on the float32 bit
  pattern; arrays are returned as float32 holding exactly representable bf16 values, and
  ``bf16_bits`` gives the raw 16-bit patterns for upload.
* Layout of per-head tensors: q, k, v [B, H, N, h]; eta [B, H, N]; alpha [B, H, C];
  W0, W2 [H, h, m]; W1 [H, m, h] (row-vector convention: phi(x) = silu(x W0) * (x W2),
  f(x) = phi(x) W1).
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

BASE_SEED = 20261202


# ----------------------------------------------------------------------------- bf16 bits
def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even); returns float32."""
    return bf16_from_bits(bf16_bits(x))


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Raw bfloat16 bit patterns (uint16) of float32 values, round-to-nearest-even."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    r = (u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_from_bits(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


# ----------------------------------------------------------------------------- workloads
@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape and input recipe of one workload.

    ``kind`` selects the value recipe: "tiny" (eta = 0.1 sigmoid(N(0,1))), "lm"
    (eta = softplus(N(-2, 0.5))), "inplace" (the In-Place-TTT-shaped MLP update).
    """
    name: str
    index: int
    B: int
    H: int
    N: int
    h: int
    m: int
    chunk: int
    dtype: str                 # "fp32" or "bf16": element type of q, k, v and of the output
    kind: str                  # "tiny" | "lm" | "inplace"
    paths: tuple               # which forms run on this workload
    renorm: bool = False       # recurrent form: per-column weight renormalisation
    momentum: bool = False     # recurrent form: M <- alpha_c M + g
    ns_steps: int = 0          # recurrent form: Newton-Schulz steps (0 or 5)
    order: str = "update_apply"

    @property
    def C(self) -> int:
        return -(-self.N // self.chunk)

    @property
    def tokens(self) -> int:
        return self.B * self.N

    @property
    def seed(self) -> int:
        return BASE_SEED + self.index

    def scaled(self, **kw) -> "Workload":
        """A copy with some sizes replaced (reduced test shapes keep the recipe)."""
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    "tiny": Workload("tiny", 0, B=1, H=1, N=256, h=16, m=16, chunk=64, dtype="fp32",
                     kind="tiny", paths=("parallel", "recurrent")),
    "lm": Workload("lm", 1, B=2, H=4, N=32768, h=256, m=512, chunk=2048, dtype="bf16",
                   kind="lm", paths=("parallel", "recurrent"), renorm=True),
    "long": Workload("long", 2, B=1, H=8, N=131072, h=128, m=512, chunk=4096, dtype="bf16",
                     kind="lm", paths=("parallel",)),
    "nvs": Workload("nvs", 3, B=1, H=6, N=196608, h=128, m=256, chunk=4096, dtype="bf16",
                    kind="lm", paths=("recurrent",), renorm=True, momentum=True, ns_steps=5),
    "inplace": Workload("inplace", 4, B=1, H=1, N=32768, h=4096, m=11008, chunk=1024,
                        dtype="bf16", kind="inplace", paths=("parallel",),
                        order="apply_update"),
}

INPLACE_ETA = 1e-3
INPLACE_CONV_K = 4


# ----------------------------------------------------------------------------- drawing
def _normal(rng, shape, mean=0.0, var=1.0):
    x = rng.standard_normal(size=shape, dtype=np.float32)
    if var != 1.0:
        x *= np.float32(math.sqrt(var))
    if mean != 0.0:
        x += np.float32(mean)
    return x


def _l2_tokens(x: np.ndarray) -> np.ndarray:
    """Per-token L2 normalisation (last axis) in float64, returned as float32."""
    out = np.empty_like(x)
    step = 1 << 20
    flat = x.reshape(-1, x.shape[-1])
    oflat = out.reshape(-1, x.shape[-1])
    rows = max(1, step // x.shape[-1])
    for s in range(0, flat.shape[0], rows):
        blk = flat[s:s + rows].astype(np.float64)
        blk /= np.sqrt(np.sum(blk * blk, axis=1, keepdims=True))
        oflat[s:s + rows] = blk.astype(np.float32)
    return out


def _sigmoid64(x):
    x = x.astype(np.float64)
    return 1.0 / (1.0 + np.exp(-x))


def _softplus64(x):
    x = x.astype(np.float64)
    return np.logaddexp(0.0, x)


def make_layer_inputs(wl: Workload, seed: int | None = None) -> dict:
    """Inputs of the TTT layer for workload ``wl`` (kinds "tiny" and "lm").

    Returns float32 arrays: q, k, v [B,H,N,h] (bf16-representable when wl.dtype is
    "bf16"), eta [B,H,N], alpha [B,H,C] (momentum workloads only, else None),
    W0, W2 [H,h,m] and W1 [H,m,h] (fp32 state, never rounded).
    """
    if wl.kind not in ("tiny", "lm"):
        raise ValueError("make_layer_inputs handles the per-head layer workloads")
    rng = np.random.Generator(np.random.PCG64(wl.seed if seed is None else seed))
    B, H, N, h, m = wl.B, wl.H, wl.N, wl.h, wl.m
    q = _l2_tokens(_normal(rng, (B, H, N, h)))
    k = _l2_tokens(_normal(rng, (B, H, N, h)))
    v = _l2_tokens(_normal(rng, (B, H, N, h)))
    if wl.dtype == "bf16":
        q, k, v = bf16_round(q), bf16_round(k), bf16_round(v)
    if wl.kind == "tiny":
        eta = (0.1 * _sigmoid64(_normal(rng, (B, H, N)))).astype(np.float32)
    else:
        eta = _softplus64(_normal(rng, (B, H, N), mean=-2.0, var=0.5)).astype(np.float32)
    W0 = _normal(rng, (H, h, m), var=1.0 / h)
    W2 = _normal(rng, (H, h, m), var=1.0 / h)
    W1 = _normal(rng, (H, m, h), var=1.0 / m)
    alpha = None
    if wl.momentum:
        alpha = _sigmoid64(_normal(rng, (B, H, wl.C), mean=1.0, var=0.5)).astype(np.float32)
    return dict(q=q, k=k, v=v, eta=eta, alpha=alpha, W0=W0, W2=W2, W1=W1)


def make_inplace_inputs(wl: Workload, seed: int | None = None) -> dict:
    """Inputs of the In-Place-TTT-shaped update (kind "inplace").

    d = wl.h (model width), dH = wl.m (MLP width). Returns float32 arrays:
    Hs [N,d] hidden states, Wg, Wu [dH,d] frozen gate/up projections, W_down [d,dH]
    fast weight (fp32, unrounded), X0 [N,d] token embeddings, conv_w [4,d] depthwise
    causal taps (tap j multiplies X0[t-j]), W_target [d,d]. Everything except W_down and
    conv_w is bf16-representable.
    """
    if wl.kind != "inplace":
        raise ValueError("make_inplace_inputs handles the inplace workload")
    rng = np.random.Generator(np.random.PCG64(wl.seed if seed is None else seed))
    N, d, dH = wl.N, wl.h, wl.m
    Hs = bf16_round(_normal(rng, (N, d)))
    Wg = bf16_round(_normal(rng, (dH, d), var=1.0 / d))
    Wu = bf16_round(_normal(rng, (dH, d), var=1.0 / d))
    W_down = _normal(rng, (d, dH), var=1.0 / dH)
    X0 = bf16_round(_normal(rng, (N, d)))
    conv_w = _normal(rng, (INPLACE_CONV_K, d), var=0.5)
    W_target = bf16_round(_normal(rng, (d, d), var=1.0 / d))
    return dict(Hs=Hs, Wg=Wg, Wu=Wu, W_down=W_down, X0=X0, conv_w=conv_w, W_target=W_target,
                eta=np.full((N,), INPLACE_ETA, dtype=np.float32))
