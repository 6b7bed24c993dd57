#!/usr/bin/env python
"""Benchmark of the chunked TTT-KVB layer on B200: TTT-layer tokens/s of the parallel and
the recurrent form, and the fraction of roofline.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload lm] [--impl reference]

A step is one pass of the layer over one batch of the workload with inputs resident in
HBM. The headline ``value`` is the parallel form's tokens/s summed over all ranks; the
recurrent form is timed the same way and reported under ``forms``. With N > 1 (launched
by torchrun) every rank runs its own replica of the workload (independent (batch, head)
problems, no collective on the data path): weak scaling, time = max over ranks.

``--impl reference`` times the fp64 CPU oracle on a bounded sample of the same workload
(the pages ship no runnable implementation); only rank 0 runs it.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "TTT-layer tokens/sec at 1 B200 (parallel vs recurrent) and % of roofline"
L2_BYTES = 126 * 2 ** 20
# dense tf32 over dense bf16 tensor throughput (nominal 1.1 against 2.25 PFLOP/s): the peak
# of a tf32 product is the measured bf16 peak times this ratio
TF32_RATIO = 1.1 / 2.25


# ----------------------------------------------------------------------------- cost model
def state_size(d: int, n_heads: int, r: int) -> int:
    """Fast-weight elements of one LaCT layer: three matrices of h x rh per head,
    n_heads heads, h = d / n_heads  ->  3 r d^2 / n_heads."""
    return 3 * r * d * d // n_heads


def layer_flops(wl, form: str) -> float:
    """Algorithmic FLOPs of one pass of the layer over the workload (matmuls only)."""
    T = wl.B * wl.H * wl.N
    hm = wl.h * wl.m
    if form == "parallel":
        feats = 4 * hm * T if wl.kind == "inplace" else 8 * hm * T   # q == k: once
        return float(feats + 2 * hm * T + 2 * hm * T)
    if form == "linear":   # identity features: state deltas and outputs, [h, h] states
        return 4.0 * wl.h * wl.h * T
    if form == "train":   # forward 12hm + backward: recomputed forward 10hm, 4 chunk GEMMs
        # 8hm, SwiGLU backward GEMMs 8hm, dX 8hm, dW 8hm per token-head
        return 54.0 * hm * T
    if form == "parallel_momentum":   # parallel form + Newton-Schulz 5 on every chunk's W1 step
        r, c = min(wl.h, wl.m), max(wl.h, wl.m)
        return 12.0 * hm * T + 5 * (4.0 * r * r * c + 2.0 * r ** 3) * wl.B * wl.H * wl.C
    flops = 18.0 * hm * T   # 9 matmuls: K features (2), D, 3 gradients, Q features (2), out
    if wl.ns_steps:
        r, c = min(wl.h, wl.m), max(wl.h, wl.m)
        per = wl.ns_steps * (2 * r * r * c + 2 * r ** 3 + 2 * r * r * c)
        # one CTA per matrix: three bf16 terms per product; larger matrices: tf32 products
        flops += (3.0 if ns_one_cta(r, c) else 1.0) * per * wl.B * wl.H * wl.C
    return flops


def ns_one_cta(r: int, c: int) -> bool:
    """The library's Newton-Schulz on one CTA per matrix (split bf16 operands) fits."""
    return r <= 128 and c <= 256


def tf32_flops(wl, form: str) -> float:
    """The part of layer_flops that runs as tf32 products: Newton-Schulz on matrices too
    large for one CTA (bf16 mode)."""
    r, c = min(wl.h, wl.m), max(wl.h, wl.m)
    if wl.dtype != "bf16" or ns_one_cta(r, c):
        return 0.0
    if form == "parallel_momentum":
        return 5 * (4.0 * r * r * c + 2.0 * r ** 3) * wl.B * wl.H * wl.C
    if form == "recurrent" and wl.ns_steps:
        return wl.ns_steps * (4.0 * r * r * c + 2.0 * r ** 3) * wl.B * wl.H * wl.C
    return 0.0


def tensor_seconds(wl, form: str, flops: float, peak_tflops: float) -> float:
    """Tensor-core time bound of `flops` algorithmic FLOPs of which tf32_flops run at the
    tf32 rate."""
    f32 = tf32_flops(wl, form)
    return (flops - f32) / (peak_tflops * 1e12) + f32 / (peak_tflops * TF32_RATIO * 1e12)


def layer_bytes(wl, form: str) -> float:
    """Algorithmic HBM bytes: each input read once, each output written once, weights."""
    es = 2 if wl.dtype == "bf16" else 4
    T = wl.B * wl.H * wl.N
    hm = wl.h * wl.m
    n_in = 1 if wl.kind == "inplace" else 2          # q and k (aliased for in-place)
    act = (n_in + 1) * T * wl.h * es + T * wl.h * es + T * 4      # q,k,v in, O out, eta
    if form == "linear":
        hh = wl.h * wl.h
        return float(act + hh * 4 * wl.H + hh * 4 * wl.B * wl.H)
    weights = 3 * hm * 4 * wl.H
    state_out = hm * 4 * wl.B * wl.H
    return float(act + weights + state_out)


def _ns_work(wl, r, c, matrices):
    """Step-level work of the Newton-Schulz kernels on `matrices` [r, c] matrices (r <= c):
    tensor FLOPs of the one-CTA kernel (three bf16 terms hi*hi + hi*lo + lo*hi per fp32
    product), of the tf32 GEMMs (one term, at the tf32 rate), and the HBM bytes of the fp32
    set-up (read U, write the scaled X; or only its norms, the scaling then riding on the
    first step's epilogues) and write-back."""
    steps = wl.ns_steps if wl.ns_steps else 5
    Z = float(matrices)
    return {
        "ns_mma": ("tensor", 3.0 * steps * (4.0 * r * r * c + 2.0 * r ** 3) * Z),
        "ns_gram": ("tensor_tf32", steps * 2.0 * r * r * c * Z),
        "ns_poly": ("tensor_tf32", steps * 2.0 * r ** 3 * Z),
        "ns_apply": ("tensor_tf32", steps * 2.0 * r * r * c * Z),
        "ns_normalize": ("hbm", 8.0 * r * c * Z),
        "ns_sumsq": ("hbm", 4.0 * r * c * Z),
        "ns_writeback": ("hbm", 8.0 * r * c * Z),
    }


def rec_splits(wl) -> int:
    """Token splits of the recurrent form's gradient GEMMs, as the library chooses them:
    the largest power of two dividing the chunk with splits of at least 256 tokens (a
    multiple of 64), one wave of tiles and at most 32 MB of fp32 partials."""
    BH, L = wl.B * wl.H, wl.chunk
    tiles = BH * (-(-2 * wl.m // 128)) * (-(-wl.h // 256))   # the merged W0 / W2 gradient GEMM
    partial = BH * 3 * wl.h * wl.m * 4
    best, sp = 1, 2
    while sp <= 64:
        if L % sp or (L // sp) % 64 or L // sp < 256 or tiles * sp > 148 or \
                sp * partial > 32 << 20:
            break
        best, sp = sp, sp * 2
    return best


def kernel_work(name: str, wl, form: str):
    """(bound, algorithmic work of one whole step) of a traced kernel: FLOP for tensor
    kernels, HBM bytes for memory-bound ones. Per-launch work = this / launches per step.
    Every kernel the library launches for a form has an entry."""
    base = name.split("@")[0]
    BH, h, m, H, C = wl.B * wl.H, wl.h, wl.m, wl.H, wl.C
    T = BH * wl.N
    hm = h * m
    es = 2 if wl.dtype == "bf16" else 4
    mpad = -(-m // 128) * 128
    r, c = min(h, m), max(h, m)
    if form == "linear":
        hh = h * h
        table = {
            "gemm_state_delta": ("tensor", 2.0 * hh * T),
            "gemm_output": ("tensor", 2.0 * hh * T),
            "scale_rows": ("hbm", T * h * 2.0 * es + T * 4.0),
            "chunk_scan": ("hbm", BH * C * hh * (4.0 + es) + 2 * 4.0 * BH * hh),
        }
        return table.get(base, (None, None))
    if form == "lm_target":
        # Vbar = conv4(X0) W_target: one [N,d]x[d,d] product; the conv reads X0, writes bf16
        table = {
            "gemm_lm_target": ("tensor", 2.0 * wl.N * h * h),
            "conv4_causal": ("hbm", 2.0 * 2 * wl.N * h),
        }
        return table.get(base, (None, None))
    if form == "recurrent":
        # per chunk: fp32 masters W (3hm), update U (3hm), momentum M (3hm) per (b, head)
        sp = rec_splits(wl)
        mom = 2.0 * 3 * hm * 4 if wl.momentum else 0.0
        # the step reads the update U after Newton-Schulz, else the split partials (and
        # updates the momentum) itself; it reads and writes W and writes the bf16 operands
        upd = 3 * hm * 4.0 if wl.ns_steps else sp * 3 * hm * 4.0 + mom
        table = {
            "gemm_features_k": ("tensor", 4.0 * hm * T),
            "gemm_features_q": ("tensor", 4.0 * hm * T),
            "gemm_v_w1t": ("tensor", 2.0 * hm * T),
            "gemm_grad_w1": ("tensor", 2.0 * hm * T),
            "gemm_grad_w0": ("tensor", 2.0 * hm * T),
            "gemm_grad_w2": ("tensor", 2.0 * hm * T),
            "gemm_grad_w02": ("tensor", 4.0 * hm * T),
            "gemm_output": ("tensor", 2.0 * hm * T),
            # split-K partials in, U out (and M in / out)
            "reduce_momentum": ("hbm", C * BH * (sp * 3 * hm * 4.0 + 3 * hm * 4.0 + mom)),
            "step_renorm": ("hbm", C * BH * (2 * 3 * hm * 4.0 + upd + (2 * mpad * h + hm) * es)),
            "rec_init": ("hbm", 3 * hm * 4.0 * H + BH * (3 * hm * 4.0 + hm * es)),
            "col_norms": ("hbm", 3 * hm * 4.0 * H),
            "prep_weights": ("hbm", 2 * hm * 4.0 * H + BH * 2 * mpad * h * es),
            "rec_finish": ("hbm", 2 * BH * 3 * hm * 4.0),
        }
        table.update(_ns_work(wl, r, c, 3 * BH * C))
        return table.get(base, (None, None))
    # parallel forms; the training step runs the forward kernels twice (forward call and
    # the backward's recomputation)
    fw = 2 if form == "train" else 1
    # the forward's key side runs as one fused kernel (phi(K) eta on chip) for bf16 with
    # h = 128 or 256 and distinct q, k; the backward always recomputes it unfused
    fused_key = wl.dtype == "bf16" and h in (128, 256) and wl.kind != "inplace"
    unfused_k = fw - (1 if fused_key else 0)
    scan = BH * C * hm * (4.0 + es) + 2 * 4.0 * BH * hm
    table = {
        "prep_weights": ("hbm", fw * (2 * hm * 4.0 * H + 2 * mpad * h * es * H)),
        "fused_delta": ("tensor", 6.0 * hm * T),   # phi(K) (4hm) and phi(K)^T eta V (2hm)
        "gemm_features_k": ("tensor", unfused_k * 4.0 * hm * T),
        "gemm_state_delta": ("tensor", unfused_k * 2.0 * hm * T),
        "chunk_scan": ("hbm", fw * scan),
        "fused_apply": ("tensor", 6.0 * hm * T),   # phi(Q) (4hm) and phi(Q) S_c (2hm)
        # sequential schedule (large states): per chunk the update phi(K)^T eta V into the
        # fp32 state, and the state's set-up
        "gemm_state_update": ("tensor", 2.0 * hm * T),
        "seq_init": ("hbm", BH * hm * (4.0 + 4.0 + es)),
        "gemm_features_q": ("tensor", 4.0 * hm * T),
        "gemm_output": ("tensor", 2.0 * hm * T),
        "momentum_scan": ("hbm", 2 * 4.0 * BH * C * hm + 4.0 * BH * C),
    }
    if form == "parallel_momentum":
        table.update(_ns_work(wl, r, c, BH * C))
    if form == "train":
        table.update({
            "cast_weights": ("hbm", 2 * hm * 4.0 * H + 2 * hm * es * H),
            "gemm_bwd_state": ("tensor", 2.0 * hm * T),
            "suffix_scan": ("hbm", BH * C * hm * (4.0 + es) + 4.0 * BH * hm),
            "gemm_bwd_dphi_q": ("tensor", 2.0 * hm * T),
            "scale_rows": ("hbm", T * h * 2.0 * es + T * 4.0),
            "gemm_bwd_dphi_k": ("tensor", 2.0 * hm * T),
            "gemm_bwd_t": ("tensor", 2.0 * hm * T),
            "row_grads": ("hbm", T * h * (4.0 + 2 * es) + 8.0 * T),
            "fill": ("hbm", 4.0 * T),
            "gemm_bwd_swiglu_k": ("tensor", 4.0 * hm * T),
            "gemm_bwd_swiglu_q": ("tensor", 4.0 * hm * T),
            "gemm_bwd_dx": ("tensor", 2 * 4.0 * hm * T),     # k side and q side
            "gemm_bwd_dw": ("tensor", 2 * 4.0 * hm * T),
            # split partials of [dW0 | dW2] and the batch's R0 in, weight gradients out
            "sum_batches": ("hbm", 4.0 * (2 * hm * BH * 2 + 2 * hm * H + hm * BH + hm * H)),
        })
    return table.get(base, (None, None))


# ----------------------------------------------------------------------------- environment
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained",
                                                     p["bf16_tflops"])),
                "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for ln in getattr(self, "lines", []):
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[3:7]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm)}


def gpu_id(local, torch):
    """nvidia-smi selector of the torch device: its UUID when torch exposes it."""
    try:
        u = str(torch.cuda.get_device_properties(local).uuid)
        if u:
            return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        pass
    return str(local)


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        info = [d for d in threadpool_info() if d.get("user_api") == "blas"]
        if info:
            return int(max(d.get("num_threads", 1) for d in info))
    except Exception:
        pass
    return os.cpu_count() or 1


# ----------------------------------------------------------------------------- ranks
def dist_setup(ngpus: int, backend: str):
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if world > 1 and not dist.is_initialized():
        import datetime
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=300))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, local, world


def max_over_ranks(value: float, world: int, device=None) -> float:
    """Max of a per-rank float over all ranks (identity when world == 1)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: float, world: int, seconds: float) -> float:
    """Whole-job throughput: units every rank processed divided by the slowest rank's time."""
    return units_per_rank * world / seconds


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ----------------------------------------------------------------------------- GPU arm
def _gpu_inputs(wl, seed, torch):
    """Device inputs of the workload. For the In-Place workload q = k = H (one tensor),
    v = the LM-aligned target computed on the GPU from X0 (see lm_target), the gate/up
    projections and W_down in their own layouts."""
    from ttt_inputs import make_inplace_inputs, make_layer_inputs

    def dev(a, dt=torch.float32):
        return torch.from_numpy(a).cuda().to(dt).contiguous()

    if wl.kind == "inplace":
        x = make_inplace_inputs(wl, seed=seed)
        bf = torch.bfloat16
        g = {"X0": dev(x["X0"], bf), "conv_w": dev(x["conv_w"]), "W_target": dev(x["W_target"], bf)}
        g["q"] = dev(x["Hs"], bf)[None, None].contiguous()
        g["k"] = g["q"]
        g["v"] = torch.empty_like(g["q"])
        g["eta"] = dev(x["eta"])[None, None].contiguous()
        g["W0"], g["W2"] = dev(x["Wg"])[None].contiguous(), dev(x["Wu"])[None].contiguous()
        g["W1"] = dev(x["W_down"])[None].contiguous()
        g["alpha"] = None
        g["layouts"] = (1, 1)
        return x, g
    x = make_layer_inputs(wl, seed=seed)
    td = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    g = {n: dev(x[n], td) for n in ("q", "k", "v")}
    g.update({n: dev(x[n]) for n in ("eta", "W0", "W2", "W1")})
    g["alpha"] = dev(x["alpha"]) if x["alpha"] is not None else None
    g["layouts"] = (0, 0)
    return x, g


def _timed(fn, steps, warmup, world, torch, trace_capacity=0):
    from test_weight_layers_ttt_b200 import abi
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    if trace_capacity:
        abi.ttt_trace_enable(trace_capacity)
    s = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s)
    for _ in range(steps):
        fn()
    e1.record(s)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    barrier(world)
    torch.cuda.synchronize()
    trace = []
    if trace_capacity:
        n = abi.ttt_trace_count()
        trace = [abi.ttt_trace_get(i) for i in range(n)]
        abi.ttt_trace_disable()
    return ms, trace


def _timed_graph(fn, steps, warmup, world, torch):
    """The same steps replayed from one CUDA graph capture of `fn` (the kernels and their
    arguments are baked at capture; replays launch them without host work). Returns
    (ms over `steps` replays) or None when `fn` cannot be captured."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    try:
        g = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            fn()                     # one eager call on the capture stream first
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        with torch.cuda.graph(g, capture_error_mode="thread_local"):
            fn()
        torch.cuda.synchronize()
    except Exception:
        torch.cuda.synchronize()
        return None
    for _ in range(max(1, warmup)):
        g.replay()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    s = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s)
    for _ in range(steps):
        g.replay()
    e1.record(s)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    barrier(world)
    torch.cuda.synchronize()
    del g
    return ms


def _kernel_table(trace, steps):
    tot = sum(ms for _, ms in trace) or 1.0
    table = {}
    for name, ms in trace:
        e = table.setdefault(name, {"launches": 0, "ms_total": 0.0})
        e["launches"] += 1
        e["ms_total"] += ms
    for e in table.values():
        e["share"] = e["ms_total"] / tot
        e["ms_avg"] = e["ms_total"] / e["launches"]
    return dict(sorted(table.items(), key=lambda kv: -kv[1]["ms_total"]))


def _traffic(workload: str, kernel: str):
    """DRAM bytes per launch recorded from an ncu capture (profiles/traffic.txt), or None
    when there is none or the kernel's source changed since the capture."""
    import hashlib
    try:
        lines = open(os.path.join(ROOT, "profiles", "traffic.txt")).read().splitlines()
    except OSError:
        return None
    for ln in lines:
        f = ln.split()
        if len(f) < 4 or ln.startswith("#") or f[0] != workload or f[1] != kernel:
            continue
        src, want = f[3].split(":")
        path = os.path.join(ROOT, "test_weight_layers_ttt_b200", "csrc", src)
        try:
            have = hashlib.sha256(open(path, "rb").read()).hexdigest()[:len(want)]
        except OSError:
            return None
        return float(f[2]) if have == want else None
    return None


def _roofline(table, wl, peaks, form, steps):
    """Roofline of the dominant kernel: the one with the largest share of the traced step.
    Its algorithmic work per launch is the form's per-step work (kernel_work) over its
    launches per step; a kernel without an entry is reported with null figures."""
    if not table:
        return None
    name, e = next(iter(table.items()))
    bound, step_work = kernel_work(name, wl, form)
    if bound is None:
        return {"kernel": name, "bound": None, "achieved": None, "peak": None, "unit": None,
                "frac": None, "traffic": None, "work_per_launch": None,
                "share": round(e["share"], 4), "peak_source": peaks["source"]}
    work = step_work / (e["launches"] / steps)
    secs = e["ms_avg"] / 1e3
    if bound in ("tensor", "tensor_tf32"):
        achieved = work / secs / 1e12
        peak = peaks["bf16_tflops"] * (TF32_RATIO if bound == "tensor_tf32" else 1.0)
        unit = "TFLOP/s"
    else:
        achieved = work / secs / 1e9
        peak = peaks["hbm_gbs"]
        unit = "GB/s"
    return {"kernel": name, "bound": "hbm" if bound == "hbm" else "tensor",
            "dtype": "tf32" if bound == "tensor_tf32" else ("bf16" if bound == "tensor" else None),
            "achieved": round(achieved, 2), "peak": round(peak, 2), "unit": unit,
            "frac": round(achieved / peak, 4),
            # captures exist for the parallel form's kernels and the momentum form's
            # Newton-Schulz GEMMs (names that no other form launches)
            "traffic": (_traffic(wl.name, name)
                        if (form == "parallel" or name.startswith("ns_"))
                        and wl == WORKLOADS_REF().get(wl.name) else None),
            "work_per_launch": work, "share": round(e["share"], 4),
            "peak_source": peaks["source"] + " (burst)"}


def run_gpu(args, rank, local, world):
    import torch

    from test_weight_layers_ttt_b200 import abi, layer
    from ttt_inputs import WORKLOADS

    torch.cuda.set_device(local)
    wl = workload_from_args(args)
    peaks = load_peaks()
    x, g = _gpu_inputs(wl, wl.seed + rank, torch)
    tokens = wl.B * wl.N
    result = {"forms": {}}

    # ---- parallel form (headline)
    forms = [f for f in ("parallel", "recurrent") if f in wl.paths]
    if wl.kind == "lm" and "parallel" in forms:
        forms.insert(1, "linear")   # identity features (plain chunked linear attention)
        # W1 momentum + Newton-Schulz 5 (simplification variant 2)
        forms.insert(2, "parallel_momentum")
        # one training step of the layer: parallel forward + backward
        forms.insert(3, "train")
    if args.forms:
        keep = set(args.forms.split(","))
        forms = [f for f in forms if f in keep]
    lin, l1 = g["layouts"]
    if wl.kind == "inplace":
        # the value target is part of the In-Place step; timed on its own below
        layer.lm_target(g["X0"], g["conv_w"], g["W_target"], out=g["v"][0, 0])
        forms = ["lm_target"] + forms
    for form in forms:
        if form == "lm_target":
            tws = layer.workspace(abi.ttt_lm_target_workspace_bytes(wl.N, wl.h), "cuda")

            def step():
                abi.ttt_lm_target(wl.N, wl.h, g["X0"], g["conv_w"], g["W_target"], g["v"], tws)
        elif form == "linear":
            ldesc = abi.ttt_desc(B=wl.B, H=wl.H, N=wl.N, h=wl.h, m=wl.h, chunk=wl.chunk,
                                 dtype=abi.TTT_DTYPE_BF16 if wl.dtype == "bf16" else 0,
                                 order=layer.ORDERS[wl.order], sign=1)
            lws = layer.workspace(abi.ttt_workspace_bytes(ldesc, abi.TTT_PATH_LINEAR), "cuda")
            lS0 = torch.zeros((wl.H, wl.h, wl.h), dtype=torch.float32, device="cuda")
            lS0[:, :, :] = g["W1"][:, :wl.h, :]
            lout = torch.empty_like(g["q"])

            def step():
                abi.ttt_linear_attn_fwd(ldesc, g["q"], g["k"], g["v"], g["eta"], lS0, lout,
                                        None, lws)
        elif form == "train":
            tdesc = layer.parallel_desc(g["q"], g["W1"], wl.chunk, wl.order)
            tws = layer.workspace(max(abi.ttt_workspace_bytes(tdesc, abi.TTT_PATH_PARALLEL_BWD),
                                      abi.ttt_workspace_bytes(tdesc, abi.TTT_PATH_PARALLEL)),
                                  "cuda")
            tout = torch.empty_like(g["q"])
            tdo = torch.randn_like(g["q"])
            tgr = [torch.empty_like(g[n]) for n in ("q", "k", "v", "eta", "W0", "W2", "W1")]

            def step():
                abi.ttt_la_parallel_fwd(tdesc, g["q"], g["k"], g["v"], g["eta"], g["W0"],
                                        g["W2"], g["W1"], tout, None, tws)
                abi.ttt_la_parallel_bwd(tdesc, g["q"], g["k"], g["v"], g["eta"], g["W0"],
                                        g["W2"], g["W1"], tdo, None, *tgr, tws)
        elif form == "parallel_momentum":
            mdesc = layer.parallel_desc(g["q"], g["W1"], wl.chunk, wl.order, 1, lin, l1)
            mdesc.momentum, mdesc.ns_steps = 1, 5
            mws = layer.workspace(
                abi.ttt_workspace_bytes(mdesc, abi.TTT_PATH_PARALLEL_MOMENTUM), "cuda")
            malpha = g["alpha"] if g["alpha"] is not None else torch.full(
                (wl.B, wl.H, wl.C), 0.9, dtype=torch.float32, device="cuda")
            mout = torch.empty_like(g["q"])

            def step():
                abi.ttt_la_parallel_momentum_fwd(mdesc, g["q"], g["k"], g["v"], g["eta"], malpha,
                                                 g["W0"], g["W2"], g["W1"], mout, None, mws)
        elif form == "parallel":
            desc = layer.parallel_desc(g["q"], g["W1"], wl.chunk, wl.order, 1, lin, l1)
            ws = layer.workspace(abi.ttt_workspace_bytes(desc, abi.TTT_PATH_PARALLEL), "cuda")
            out = torch.empty_like(g["q"])
            S = torch.empty((wl.B, wl.H, wl.m, wl.h) if l1 == 0 else (wl.B, wl.H, wl.h, wl.m),
                            dtype=torch.float32, device="cuda")

            def step():
                abi.ttt_la_parallel_fwd(desc, g["q"], g["k"], g["v"], g["eta"], g["W0"],
                                        g["W2"], g["W1"], out, S, ws)
        else:
            desc = layer.recurrent_desc(g["q"], g["W1"], wl.chunk, wl.order, 1, 7, wl.renorm,
                                        wl.momentum, wl.ns_steps)
            ws = layer.workspace(abi.ttt_workspace_bytes(desc, abi.TTT_PATH_RECURRENT), "cuda")
            out = torch.empty_like(g["q"])

            def step():
                abi.ttt_lact_recurrent_fwd(desc, g["q"], g["k"], g["v"], g["eta"], g["alpha"],
                                           g["W0"], g["W2"], g["W1"], out, None, None, None,
                                           None, ws)
        steps = args.steps if form in ("parallel", "linear") else max(3, args.steps // 4)
        # timed region: the step replayed from a CUDA graph (eager launches when the step
        # cannot be captured); the per-kernel table comes from a separate traced eager pass
        with ClockSampler(gpu_id(local, torch)) as clk:
            ms = _timed_graph(step, steps, args.warmup, world, torch)
            mode = "cuda_graph"
            if ms is None:
                ms, _ = _timed(step, steps, args.warmup, world, torch)
                mode = "eager"
        abi.ttt_last_device_status()
        ms_max = max_over_ranks(ms, world, "cuda")
        per_step = ms_max / steps
        tsteps = min(steps, 5)
        _, trace = _timed(step, tsteps, 1, world, torch, trace_capacity=16384)
        table = _kernel_table(trace, tsteps)
        if form == "lm_target":
            flops = 2.0 * wl.N * wl.h * wl.h
            nbytes = 2.0 * (2 * wl.N * wl.h + wl.h * wl.h) + 16.0 * wl.h
        else:
            flops, nbytes = layer_flops(wl, form), layer_bytes(wl, form)
        t_roof = max(tensor_seconds(wl, form, flops, peaks["bf16_tflops"]),
                     nbytes / (peaks["hbm_gbs"] * 1e9))
        result["forms"][form] = {
            "tokens_per_s": job_throughput(tokens, world, per_step / 1e3),
            "ms_per_step": per_step, "steps": steps,
            "flop_per_step": flops, "bytes_per_step": nbytes,
            "roofline_frac": t_roof / (per_step / 1e3),
            "roofline_frac_sustained": max(
                tensor_seconds(wl, form, flops, peaks["bf16_tflops_sustained"]),
                nbytes / (peaks["hbm_gbs"] * 1e9)) / (per_step / 1e3),
            "gpu_launches": len(trace) * steps // tsteps,
            "launch_mode": mode,
            "kernels": {k: {kk: (round(vv, 5) if isinstance(vv, float) else vv)
                            for kk, vv in v.items()} for k, v in table.items()},
            "roofline": _roofline(table, wl, peaks, form, tsteps),
            "clocks": clk.summary(),
        }

    # ---- end to end through the public API, host buffers, copies inside the timed region
    e2e = None
    if "parallel" in forms and wl.kind == "inplace":
        hq = {n: g[n].cpu().pin_memory() for n in ("q", "X0")}
        dq = {n: torch.empty_like(g[n]) for n in hq}
        hout = torch.empty(g["q"].shape, dtype=g["q"].dtype).pin_memory()
        dout = torch.empty_like(g["q"])
        dv = torch.empty_like(g["v"])
        ws = layer.workspace(abi.ttt_workspace_bytes(
            layer.parallel_desc(g["q"], g["W1"], wl.chunk, wl.order, 1, lin, l1), 0), "cuda")
        tws = layer.workspace(abi.ttt_lm_target_workspace_bytes(wl.N, wl.h), "cuda")

        def e2e_step():
            for n in dq:
                dq[n].copy_(hq[n], non_blocking=True)
            layer.lm_target(dq["X0"], g["conv_w"], g["W_target"], out=dv[0, 0], ws=tws)
            layer.la_parallel_fwd(dq["q"], dq["q"], dv, g["eta"], g["W0"], g["W2"], g["W1"],
                                  wl.chunk, order=wl.order, w_in_layout=lin, w1_layout=l1,
                                  return_state=False, out=dout, ws=ws)
            hout.copy_(dout, non_blocking=True)

        steps = max(3, args.steps // 2)
        ms, _ = _timed(e2e_step, steps, args.warmup, world, torch)
        ms = max_over_ranks(ms, world, "cuda")
        e2e = {"value": job_throughput(tokens, world, ms / steps / 1e3), "unit": "tokens/s",
               "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in hq.values()),
               "d2h_bytes_per_step": hout.numel() * hout.element_size(),
               "ms_per_step": ms / steps}
    elif "parallel" in forms:
        hq = {n: g[n].cpu().pin_memory() for n in ("q", "k", "v", "eta")}
        dq = {n: torch.empty_like(g[n]) for n in ("q", "k", "v", "eta")}
        hout = torch.empty(g["q"].shape, dtype=g["q"].dtype).pin_memory()
        dout = torch.empty_like(g["q"])
        # The step as one layer call per (batch element, head), alternating between two
        # streams: the (batch, head) problems are independent, so the host-to-device copies
        # of one overlap the kernels and the device-to-host copy of another (the copy
        # engines of the two directions run at the same time).
        streams = [torch.cuda.Stream() for _ in range(2)]
        one = lambda t, b, hh: t[b:b + 1, hh:hh + 1]
        ws1 = [layer.workspace(abi.ttt_workspace_bytes(layer.parallel_desc(
            one(g["q"], 0, 0), g["W1"][:1], wl.chunk, wl.order), 0), "cuda") for _ in streams]

        def e2e_step():
            cur = torch.cuda.current_stream()
            for st in streams:
                st.wait_stream(cur)
            for i in range(wl.B * wl.H):
                b, hh = divmod(i, wl.H)
                st = streams[i % 2]
                with torch.cuda.stream(st):
                    for n in dq:
                        one(dq[n], b, hh).copy_(one(hq[n], b, hh), non_blocking=True)
                    layer.la_parallel_fwd(
                        one(dq["q"], b, hh), one(dq["k"], b, hh), one(dq["v"], b, hh),
                        one(dq["eta"], b, hh), g["W0"][hh:hh + 1], g["W2"][hh:hh + 1],
                        g["W1"][hh:hh + 1], wl.chunk, order=wl.order, return_state=False,
                        out=one(dout, b, hh), ws=ws1[i % 2])
                    one(hout, b, hh).copy_(one(dout, b, hh), non_blocking=True)
            for st in streams:
                cur.wait_stream(st)

        steps = max(3, args.steps // 2)
        ms, _ = _timed(e2e_step, steps, args.warmup, world, torch)
        ms = max_over_ranks(ms, world, "cuda")
        h2d = sum(t.numel() * t.element_size() for t in hq.values())
        d2h = hout.numel() * hout.element_size()
        e2e = {"value": job_throughput(tokens, world, ms / steps / 1e3), "unit": "tokens/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "ms_per_step": ms / steps}
    result["e2e"] = e2e
    return wl, peaks, result, x


# ----------------------------------------------------------------------------- CPU oracle
def oracle_time(wl, x, n: int, form: str = "parallel") -> float:
    """Seconds the fp64 oracle takes for the first ``n`` tokens of batch element 0 through
    all H heads of the layer, so that n / seconds counts layer tokens like the GPU arm's
    ``value`` (for the In-Place workload: the target prologue and the sequential update on
    n tokens)."""
    from oracle import ttt_oracle as O
    if wl.kind == "inplace":
        t0 = time.perf_counter()
        vbar = O.lm_target(x["X0"][:n], x["conv_w"], x["W_target"])
        O.inplace_sequential(x["Hs"][:n], x["Wg"], x["Wu"], x["W_down"], vbar, wl.chunk,
                             float(x["eta"][0]))
        return time.perf_counter() - t0
    heads = x["q"].shape[1]
    t0 = time.perf_counter()
    for hd in range(heads):
        q, k, v, eta = (x[name][0, hd, :n].astype("float64") for name in ("q", "k", "v", "eta"))
        W0, W2, W1 = x["W0"][hd], x["W2"][hd], x["W1"][hd]
        if form == "parallel":
            O.la_parallel(q, k, v, eta, W0, W2, W1, wl.chunk, order=wl.order)
        else:
            alpha = x["alpha"][0, hd] if x.get("alpha") is not None else None
            O.lact_recurrent(q, k, v, eta, W0, W2, W1, wl.chunk, order=wl.order,
                             renorm=wl.renorm, alpha=alpha, ns_steps=wl.ns_steps)
    return time.perf_counter() - t0


def oracle_sample(wl, x, target_s: float, form: str = "parallel"):
    """Time the fp64 oracle on batch element 0, all heads, with as many leading whole
    chunks as fit about ``target_s`` seconds; returns (tokens, seconds, description)."""
    n = min(wl.N, wl.chunk)
    t = oracle_time(wl, x, n, form)
    if t < target_s / 2 and n < wl.N:
        n2 = min(wl.N, max(wl.chunk, int(n * target_s / max(t, 1e-3)) // wl.chunk * wl.chunk))
        if n2 > n:
            n, t = n2, oracle_time(wl, x, n2, form)
    if wl.kind == "inplace":
        what = "the target prologue and the sequential update"
    else:
        what = f"all {x['q'].shape[1]} heads of batch element 0"
    desc = (f"{form} form, fp64 oracle, {what} of the '{wl.name}' workload, first {n} of "
            f"{wl.N} tokens; layer tokens/s (each token through every head)")
    return n, t, desc


def workload_from_args(args):
    from ttt_inputs import WORKLOADS
    wl = WORKLOADS[args.workload]
    if args.override:
        kw = {}
        for item in args.override.split(","):
            key, val = item.split("=")
            kw[key.strip()] = type(getattr(wl, key.strip()))(val)
        wl = wl.scaled(**kw)
    return wl


def run_reference(args):
    """Reference arm: the fp64 CPU oracle as it stands, on bounded samples."""
    from ttt_inputs import make_inplace_inputs, make_layer_inputs
    wl = workload_from_args(args)
    if wl.kind == "inplace":
        x = make_inplace_inputs(wl, seed=wl.seed)
    else:
        x = make_layer_inputs(wl.scaled(B=1), seed=wl.seed)
    form = "parallel" if "parallel" in wl.paths else "recurrent"
    n, t, desc = oracle_sample(wl, x, 2.0, form)
    times = []
    for i in range(args.warmup + args.steps):
        ti = oracle_time(wl, x, n, form)
        if i >= args.warmup:
            times.append(ti)
    secs = sum(times)
    value = n * len(times) / secs
    cores = blas_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": secs / len(times) * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(wl, form),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": desc + " per step"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))


def workload_config(wl, form):
    """The workload's sizes and the options of `form` (the recurrent options only on the
    recurrent form's line)."""
    cfg = {"workload": wl.name if wl == WORKLOADS_REF().get(wl.name) else wl.name + "*",
           "form": form, "B": wl.B, "H": wl.H, "N": wl.N, "h": wl.h,
           "m": wl.m, "chunk": wl.chunk, "order": wl.order}
    if form == "recurrent":
        cfg.update({"renorm": wl.renorm, "momentum": wl.momentum, "ns_steps": wl.ns_steps})
    cfg.update({"parallelism": "replicas",
                "l2": "no flush: the per-step inputs exceed the 126 MB L2"})
    return cfg


def WORKLOADS_REF():
    from ttt_inputs import WORKLOADS
    return WORKLOADS


# ----------------------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="lm")
    ap.add_argument("--impl", default="ours", choices=("ours", "reference"))
    ap.add_argument("--cpu-seconds", type=float, default=15.0,
                    help="target seconds of the CPU oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--override", default="",
                    help="comma-separated workload field overrides for profiling, e.g. B=1,H=4")
    ap.add_argument("--forms", default="",
                    help="comma-separated subset of the forms to time (profiling), e.g. "
                         "parallel; the default times every form of the workload")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)

    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            run_reference(args)
        return

    import torch
    rank, local, world = dist_setup(args.gpus, "nccl" if torch.cuda.is_available() else "gloo")
    from test_weight_layers_ttt_b200 import build as tbuild
    if not os.path.exists(tbuild.LIB_PATH):
        tbuild.build()
    wl, peaks, res, x = run_gpu(args, rank, local, world)
    if rank == 0:
        form = next((f for f in ("parallel", "recurrent") if f in res["forms"]),
                    next(iter(res["forms"])))
        head = dict(res["forms"][form])
        if "lm_target" in res["forms"]:
            # In-Place step = target prologue + parallel update/apply
            pro = res["forms"]["lm_target"]
            ms = head["ms_per_step"] + pro["ms_per_step"]
            head["tokens_per_s"] = job_throughput(wl.B * wl.N, world, ms / 1e3)
            head["ms_per_step"] = ms
            head["roofline_frac"] = (res["forms"][form]["roofline_frac"] *
                                     res["forms"][form]["ms_per_step"] +
                                     pro["roofline_frac"] * pro["ms_per_step"]) / ms
        line = {
            "metric": METRIC, "value": head["tokens_per_s"], "unit": "tokens/s",
            "n_gpus": world, "steps": head["steps"], "warmup": args.warmup,
            "ms_per_step": head["ms_per_step"], "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": wl.dtype, "data": "synthetic",
            "config": workload_config(wl, form),
            "roofline": head["roofline"],
            "step_roofline_frac": head["roofline_frac"],
            "gpu_launches": sum(f["gpu_launches"] for f in res["forms"].values()),
            "clocks": head["clocks"],
            "e2e": res["e2e"],
            "forms": res["forms"],
        }
        if "parallel" in res["forms"] and "recurrent" in res["forms"]:
            line["parallel_over_recurrent"] = (res["forms"]["parallel"]["tokens_per_s"] /
                                               res["forms"]["recurrent"]["tokens_per_s"])
        if world == 1 and not args.no_cpu_baseline:
            n, secs, desc = oracle_sample(wl, x, args.cpu_seconds, form)
            line["cpu_baseline"] = {"value": n / secs, "unit": "tokens/s",
                                    "cores": blas_threads(), "kind": "oracle", "sample": desc}
        print(json.dumps(line))
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
