"""Shared helpers of the GPU parity tests: upload seeded host inputs, download results,
and the parity metric max|err| / max|ref|."""
import numpy as np
import torch

TOL = {"fp32": 1e-4, "bf16": 2e-2}


def dev(x, dtype=torch.float32):
    """Host float array -> CUDA tensor. bf16 inputs hold bf16-representable values, so the
    cast is exact."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to("cuda")
    return t.to(dtype).contiguous()


def host(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def rel(got, ref):
    ref = np.asarray(ref, dtype=np.float64)
    den = float(np.max(np.abs(ref))) if ref.size else 0.0
    if den == 0.0:
        return float(np.max(np.abs(got))) if np.size(got) else 0.0
    return float(np.max(np.abs(np.asarray(got, dtype=np.float64) - ref)) / den)


def torch_dtype(name):
    return torch.bfloat16 if name == "bf16" else torch.float32
