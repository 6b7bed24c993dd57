"""Host-side logic of bench.py: the cost model against numbers the pages print, and the
multi-rank timing reduction (max over ranks, whole-job throughput) with 2 gloo ranks."""
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench
from ttt_inputs import WORKLOADS

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "state_size.txt")


def test_state_size_matches_pages():
    rows = [l.split() for l in open(GOLDEN) if l.strip() and not l.startswith("#")]
    assert rows
    for d, nh, r, layers, expect in rows:
        assert bench.state_size(int(d), int(nh), int(r)) * int(layers) == int(expect)
    assert abs(bench.state_size(768, 1, 2) * 24 / 1e6 - 84.9) < 0.05
    assert bench.state_size(768, 4, 1) == 0.75 * 768 ** 2


@pytest.mark.parametrize("name", ["lm", "nvs", "tiny"])
def test_recurrent_flops_are_six_n_s(name):
    wl = WORKLOADS[name].scaled(ns_steps=0)
    n = wl.B * wl.N                                  # tokens through the layer
    S = bench.state_size(wl.H * wl.h, wl.H, wl.m // wl.h)
    assert bench.layer_flops(wl, "recurrent") == 6 * n * S


def test_parallel_flops_and_bytes():
    wl = WORKLOADS["lm"]
    T = wl.B * wl.H * wl.N
    assert bench.layer_flops(wl, "parallel") == 12 * wl.h * wl.m * T
    ip = WORKLOADS["inplace"]
    assert bench.layer_flops(ip, "parallel") == 8 * ip.h * ip.m * ip.N   # features once
    # q, k, v in and O out (bf16), eta, weights, final state
    expect = 4 * T * wl.h * 2 + 4 * T + 3 * wl.h * wl.m * 4 * wl.H + wl.h * wl.m * 4 * wl.B * wl.H
    assert bench.layer_bytes(wl, "parallel") == expect


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    r, local, w = bench.dist_setup(world, "gloo")
    ms = 10.0 + 5.0 * r                        # rank 1 is the slow one
    slowest = bench.max_over_ranks(ms, w)
    value = bench.job_throughput(65536, w, slowest / 1e3)
    bench.barrier(w)
    import torch.distributed as dist
    dist.destroy_process_group()
    q.put((r, w, slowest, value))


def test_max_over_ranks_with_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r, w, slowest, value in res:
        assert w == 2 and slowest == 15.0
        assert value == pytest.approx(2 * 65536 / 0.015)


def test_roofline_per_launch_work():
    """The dominant kernel (largest share) is reported; its algorithmic work per launch is
    the form's per-step work over its launches per step. In the training step the forward
    kernels run twice per step (forward pass and the backward's recomputation), each launch
    doing the forward form's whole work."""
    wl = WORKLOADS["lm"]
    T = wl.B * wl.H * wl.N
    peaks = {"bf16_tflops": 1000.0, "hbm_gbs": 5000.0, "source": "test"}
    table = {"gemm_features_k@tcgen05": {"launches": 10, "ms_avg": 0.1, "share": 0.6},
             "no_such_kernel": {"launches": 5, "ms_avg": 1.0, "share": 0.1}}
    r = bench._roofline(table, wl, peaks, "train", 5)             # two launches per step
    assert r["kernel"] == "gemm_features_k@tcgen05"
    # lm: the forward's key side is fused, so only the backward's recomputation launches it
    assert r["work_per_launch"] == 4.0 * wl.h * wl.m * T / 2
    t = bench._roofline({"gemm_features_k@tcgen05": {"launches": 5, "ms_avg": 0.1,
                                                      "share": 0.6}}, wl, peaks, "train", 5)
    assert t["work_per_launch"] == 4.0 * wl.h * wl.m * T
    assert abs(t["achieved"] - 4.0 * wl.h * wl.m * T / 1e-4 / 1e12) < 0.01
    assert abs(t["frac"] - t["achieved"] / 1000.0) < 1e-4
    assert t["bound"] == "tensor" and t["unit"] == "TFLOP/s"
    # a dominant kernel without known work is still the one reported, with null figures
    u = bench._roofline({"no_such_kernel": {"launches": 5, "ms_avg": 1.0, "share": 0.9}},
                        wl, peaks, "parallel", 5)
    assert u["kernel"] == "no_such_kernel" and u["achieved"] is None


def test_every_traced_kernel_has_algorithmic_work():
    """Every kernel name the library traces (the names passed to its trace scopes) has an
    entry in the work table of each form that launches it."""
    import re
    src = open(os.path.join(os.path.dirname(bench.__file__), "test_weight_layers_ttt_b200",
                            "csrc", "ttt_api.cu")).read()
    names = set(re.findall(r'(?:TTT_OP|run_gemm|run_simt|run_swiglu|TraceScope ts)\(\s*"(\w+)',
                           src))
    names |= set(re.findall(r'"(gemm_\w+|fused_apply)(?:@tcgen05)?"', src))
    assert {"gemm_features_k", "ns_mma", "step_renorm", "fused_apply"} <= names
    forms = {"parallel": WORKLOADS["lm"], "parallel_momentum": WORKLOADS["lm"],
             "train": WORKLOADS["lm"], "recurrent": WORKLOADS["nvs"],
             "linear": WORKLOADS["lm"], "lm_target": WORKLOADS["inplace"]}
    known = set()
    for form, wl in forms.items():
        known |= {n for n in names if bench.kernel_work(n, wl, form)[0] is not None}
    # the failure-path probe and the debug-check kernels are not part of any timed form
    missing = names - known - {"wait_timeout_probe", "guards_fill", "guards_check",
                               "finite_scan"}
    assert not missing, missing


def test_traffic_only_while_the_captured_source_is_unchanged():
    import hashlib
    path = os.path.join(os.path.dirname(bench.__file__), "profiles", "traffic.txt")
    rows = [l.split() for l in open(path) if l.strip() and not l.startswith("#")]
    assert rows
    for wl, kernel, value, src in (r[:4] for r in rows):
        name, want = src.split(":")
        f = os.path.join(os.path.dirname(bench.__file__), "test_weight_layers_ttt_b200", "csrc",
                         name)
        have = hashlib.sha256(open(f, "rb").read()).hexdigest()[:len(want)]
        assert bench._traffic(wl, kernel) == (float(value) if have == want else None)
    assert bench._traffic("lm", "no_such_kernel") is None


def test_tf32_products_are_measured_against_the_tf32_peak():
    """The batched Newton-Schulz GEMMs run as tf32 products: their work is one product per
    step (not three split-bf16 terms) and their peak is the bf16 peak times the nominal
    tf32 / bf16 ratio; the step roofline charges the Newton-Schulz FLOPs at that rate."""
    wl = WORKLOADS["lm"]
    r, c = min(wl.h, wl.m), max(wl.h, wl.m)
    Z = wl.B * wl.H * wl.C
    bound, work = bench.kernel_work("ns_apply@tcgen05", wl, "parallel_momentum")
    assert bound == "tensor_tf32" and work == 5 * 2.0 * r * r * c * Z
    peaks = {"bf16_tflops": 1000.0, "hbm_gbs": 5000.0, "source": "test"}
    t = bench._roofline({"ns_apply@tcgen05": {"launches": 5, "ms_avg": 0.05, "share": 0.3}},
                        wl, peaks, "parallel_momentum", 1)
    assert t["bound"] == "tensor" and t["dtype"] == "tf32"
    assert abs(t["peak"] - 1000.0 * 1.1 / 2.25) < 0.01
    assert abs(t["frac"] - t["achieved"] / t["peak"]) < 1e-3
    # the one-CTA kernel (matrices up to 128 x 256) stays a bf16 (three-term) product
    nvs = WORKLOADS["nvs"]
    assert bench.kernel_work("ns_mma", nvs, "recurrent")[0] == "tensor"
    assert bench.tf32_flops(nvs, "recurrent") == 0.0
    f = bench.layer_flops(wl, "parallel_momentum")
    nsf = bench.tf32_flops(wl, "parallel_momentum")
    assert 0 < nsf < f
    s = bench.tensor_seconds(wl, "parallel_momentum", f, 1000.0)
    assert abs(s - ((f - nsf) / 1e15 + nsf / (1e15 * 1.1 / 2.25))) < 1e-12
