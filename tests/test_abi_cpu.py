"""Host-side checks of the C-ABI library that need no GPU: it loads, exports every symbol
include/ttt.h declares, sizes workspaces, and rejects bad arguments before enqueueing
anything (so none of these calls reaches the CUDA driver)."""
import ctypes
import os
import re
import subprocess

import pytest

from test_weight_layers_ttt_b200 import abi
from test_weight_layers_ttt_b200 import build as tbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ttt.h")


@pytest.fixture(scope="module", autouse=True)
def built():
    tbuild.build()
    return abi.lib()


def header_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return set(re.findall(r"\b(ttt_[a-z0-9_]+)\s*\(", src))


def test_every_declared_symbol_is_exported():
    declared = header_functions()
    assert declared == set(abi.EXPORTED)
    out = subprocess.run(["nm", "-D", "--defined-only", tbuild.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (ttt_[a-z0-9_]+)$", out, flags=re.M))
    assert declared <= exported, declared - exported
    for name in declared:
        assert getattr(abi.lib(), name) is not None


def test_status_strings_and_version():
    for st, name in [(0, "TTT_OK"), (1, "TTT_ERR_INVALID_ARG"), (2, "TTT_ERR_UNSUPPORTED"),
                     (3, "TTT_ERR_WORKSPACE"), (4, "TTT_ERR_CUDA"), (5, "TTT_ERR_TIMEOUT"),
                     (6, "TTT_ERR_DEVICE")]:
        assert abi.ttt_status_str(st) == name
    assert abi.ttt_status_str(99) == "TTT_ERR_UNKNOWN"
    assert abi.ttt_version() == 100
    assert ctypes.sizeof(abi.ttt_desc) == 15 * 4


def lm_desc(**kw):
    base = dict(B=2, H=4, N=32768, h=256, m=512, chunk=2048, dtype=abi.TTT_DTYPE_BF16)
    base.update(kw)
    return abi.ttt_desc(**base)


def test_workspace_sizes():
    par = abi.ttt_workspace_bytes(lm_desc(), abi.TTT_PATH_PARALLEL)
    # blocked bf16 weights + two bf16 feature buffers + fp32 deltas + bf16 chunk states
    BH, N, h, m, C = 8, 32768, 256, 512, 16
    expect = 2 * 2 * m * h * 4 + 2 * (2 * BH * N * m) + BH * C * m * h * 6
    assert expect <= par <= expect + 6 * 256
    assert abi.ttt_workspace_bytes(lm_desc(N=65536), 0) > par
    rec = abi.ttt_workspace_bytes(lm_desc(update_mask=7, renorm=1), abi.TTT_PATH_RECURRENT)
    assert rec > 0
    with_ns = abi.ttt_workspace_bytes(lm_desc(update_mask=7, ns_steps=5, momentum=1), 1)
    assert with_ns > rec
    # invalid descriptions size to 0
    assert abi.ttt_workspace_bytes(lm_desc(sign=0), 0) == 0
    assert abi.ttt_workspace_bytes(lm_desc(update_mask=7), 0) == 0      # parallel takes no mask
    assert abi.ttt_workspace_bytes(lm_desc(), 1) == 0                   # recurrent needs a mask
    assert abi.ttt_workspace_bytes(lm_desc(), 7) == 0


@pytest.mark.parametrize("field,value,status", [
    ("sign", 0, abi.TTT_ERR_INVALID_ARG),
    ("dtype", 5, abi.TTT_ERR_INVALID_ARG),
    ("order", 2, abi.TTT_ERR_INVALID_ARG),
    ("h", 0, abi.TTT_ERR_INVALID_ARG),
    ("chunk", 0, abi.TTT_ERR_INVALID_ARG),
    ("N", -1, abi.TTT_ERR_INVALID_ARG),
    ("renorm", 1, abi.TTT_ERR_INVALID_ARG),
    ("w_in_layout", 2, abi.TTT_ERR_INVALID_ARG),
    ("h", 100, abi.TTT_ERR_UNSUPPORTED),   # bf16 needs multiples of 8
])
def test_parallel_rejects_bad_desc(field, value, status):
    d = lm_desc(**{field: value})
    with pytest.raises(abi.TTTError) as ei:
        abi.ttt_la_parallel_fwd(d, 256, 256, 256, 256, 256, 256, 256, 256, None, 256, 1 << 40,
                                stream=0)
    assert ei.value.status == status


def test_parallel_rejects_pointers_and_workspace():
    d = lm_desc()
    need = abi.ttt_workspace_bytes(d, 0)
    with pytest.raises(abi.TTTError) as ei:   # NULL q
        abi.ttt_la_parallel_fwd(d, None, 256, 256, 256, 256, 256, 256, 256, None, 256, need,
                                stream=0)
    assert ei.value.status == abi.TTT_ERR_INVALID_ARG
    with pytest.raises(abi.TTTError) as ei:   # misaligned k
        abi.ttt_la_parallel_fwd(d, 256, 258, 256, 256, 256, 256, 256, 256, None, 256, need,
                                stream=0)
    assert ei.value.status == abi.TTT_ERR_INVALID_ARG
    with pytest.raises(abi.TTTError) as ei:   # workspace too small
        abi.ttt_la_parallel_fwd(d, 256, 256, 256, 256, 256, 256, 256, 256, None, 256, need - 1,
                                stream=0)
    assert ei.value.status == abi.TTT_ERR_WORKSPACE
    with pytest.raises(abi.TTTError) as ei:   # misaligned workspace
        abi.ttt_la_parallel_fwd(d, 256, 256, 256, 256, 256, 256, 256, 256, None, 272, need,
                                stream=0)
    assert ei.value.status == abi.TTT_ERR_WORKSPACE
    assert "256-byte" in abi.ttt_last_error_message()


def test_shard_outputs_pass_needs_a_state_only_call_first():
    """The outputs pass reuses what a state-only shard call left in the workspace: without
    one just before on this thread (or after a failed one) it is refused."""
    d = lm_desc()
    need = abi.ttt_workspace_bytes(d, abi.TTT_PATH_PARALLEL)
    with pytest.raises(abi.TTTError) as ei:
        abi.ttt_la_parallel_fwd_shard_outputs(d, 256, 256, None, 0, 256, None, 256, need,
                                              stream=0)
    assert ei.value.status == abi.TTT_ERR_INVALID_ARG
    assert "state-only" in abi.ttt_last_error_message()
    with pytest.raises(abi.TTTError):   # a state-only call that fails (NULL q) marks nothing
        abi.ttt_la_parallel_fwd_shard(d, None, 256, 256, 256, 256, 256, None, None, 0, None,
                                      256, 256, need, stream=0)
    with pytest.raises(abi.TTTError) as ei:
        abi.ttt_la_parallel_fwd_shard_outputs(d, 256, 256, None, 0, 256, None, 256, need,
                                              stream=0)
    assert ei.value.status == abi.TTT_ERR_INVALID_ARG


def test_linear_attention_workspace_and_checks():
    d = lm_desc(m=256)   # identity features: the state is [h, h]
    BH, N, h, C = 8, 32768, 256, 16
    expect = 2 * BH * N * h + 4 * BH * C * h * h + 2 * BH * C * h * h
    got = abi.ttt_workspace_bytes(d, abi.TTT_PATH_LINEAR)
    assert expect <= got <= expect + 3 * 256
    assert abi.ttt_workspace_bytes(lm_desc(), abi.TTT_PATH_LINEAR) == 0        # m != h
    assert abi.ttt_workspace_bytes(lm_desc(m=256, w_in_layout=1), 2) == 0
    with pytest.raises(abi.TTTError) as ei:
        abi.ttt_linear_attn_fwd(lm_desc(), 256, 256, 256, 256, 256, 256, None, 256, 1 << 40,
                                stream=0)
    assert ei.value.status == abi.TTT_ERR_INVALID_ARG
    with pytest.raises(abi.TTTError) as ei:   # NULL S0
        abi.ttt_linear_attn_fwd(d, 256, 256, 256, 256, None, 256, None, 256, got, stream=0)
    assert ei.value.status == abi.TTT_ERR_INVALID_ARG
    with pytest.raises(abi.TTTError) as ei:   # workspace too small
        abi.ttt_linear_attn_fwd(d, 256, 256, 256, 256, 256, 256, None, 256, got - 1, stream=0)
    assert ei.value.status == abi.TTT_ERR_WORKSPACE
    abi.ttt_linear_attn_fwd(lm_desc(B=0, m=256), None, None, None, None, None, None, None,
                            None, 0, stream=0)


def test_parallel_momentum_workspace_and_checks():
    P = abi.TTT_PATH_PARALLEL_MOMENTUM
    plain = abi.ttt_workspace_bytes(lm_desc(), abi.TTT_PATH_PARALLEL)
    assert abi.ttt_workspace_bytes(lm_desc(momentum=1), P) >= plain
    # min(h, m) = 256 > 128: the CUDA-core Newton-Schulz needs its scratch
    assert abi.ttt_workspace_bytes(lm_desc(momentum=1, ns_steps=5), P) > plain
    # an NVS-shaped state fits the tensor-core Newton-Schulz: no extra scratch
    small = dict(h=128, m=256)
    assert (abi.ttt_workspace_bytes(lm_desc(ns_steps=5, **small), P) ==
            abi.ttt_workspace_bytes(lm_desc(**small), P))
    for bad in (dict(renorm=1), dict(update_mask=2), dict(ns_steps=9), dict(w1_layout=1)):
        assert abi.ttt_workspace_bytes(lm_desc(**bad), P) == 0
    with pytest.raises(abi.TTTError) as ei:   # momentum without alpha
        abi.ttt_la_parallel_momentum_fwd(lm_desc(momentum=1), 256, 256, 256, 256, None, 256,
                                         256, 256, 256, None, 256, 1 << 40, stream=0)
    assert ei.value.status == abi.TTT_ERR_INVALID_ARG


def test_backward_workspace_and_checks():
    P = abi.TTT_PATH_PARALLEL_BWD
    assert abi.ttt_workspace_bytes(lm_desc(), P) > abi.ttt_workspace_bytes(lm_desc(), 0)
    assert abi.ttt_workspace_bytes(lm_desc(w_in_layout=1), P) == 0
    assert abi.ttt_workspace_bytes(lm_desc(momentum=1), P) == 0
    d = lm_desc()
    need = abi.ttt_workspace_bytes(d, P)
    with pytest.raises(abi.TTTError) as ei:   # q aliased with k
        abi.ttt_la_parallel_bwd(d, 256, 256, 256, 256, 256, 256, 256, 256, None, 512, 768, 1024,
                                1280, 256, 256, 256, 256, need, stream=0)
    assert ei.value.status == abi.TTT_ERR_INVALID_ARG
    with pytest.raises(abi.TTTError) as ei:   # missing weight gradient
        abi.ttt_la_parallel_bwd(d, 256, 512, 256, 256, 256, 256, 256, 256, None, 512, 768, 1024,
                                1280, None, 256, 256, 256, need, stream=0)
    assert ei.value.status == abi.TTT_ERR_INVALID_ARG


def test_recurrent_rejects_bad_args():
    d = lm_desc(update_mask=7, momentum=1)
    need = abi.ttt_workspace_bytes(d, 1)
    with pytest.raises(abi.TTTError) as ei:   # momentum without alpha
        abi.ttt_lact_recurrent_fwd(d, 256, 256, 256, 256, None, 256, 256, 256, 256, None, None,
                                   None, None, 256, need, stream=0)
    assert ei.value.status == abi.TTT_ERR_INVALID_ARG
    d2 = lm_desc(update_mask=7, w1_layout=1)
    with pytest.raises(abi.TTTError) as ei:
        abi.ttt_lact_recurrent_fwd(d2, 256, 256, 256, 256, None, 256, 256, 256, 256, None, None,
                                   None, None, 256, 1 << 40, stream=0)
    assert ei.value.status == abi.TTT_ERR_UNSUPPORTED
    for bad in (dict(update_mask=8), dict(update_mask=7, ns_steps=9)):
        with pytest.raises(abi.TTTError):
            abi.ttt_lact_recurrent_fwd(lm_desc(**bad), 256, 256, 256, 256, None, 256, 256, 256,
                                       256, None, None, None, None, 256, 1 << 40, stream=0)


def test_empty_batch_is_a_no_op():
    # B * H == 0 returns before touching the device.
    abi.ttt_la_parallel_fwd(lm_desc(B=0), None, None, None, None, None, None, None, None, None,
                            None, 0, stream=0)
    abi.ttt_lact_recurrent_fwd(lm_desc(H=0, update_mask=7), None, None, None, None, None, None,
                               None, None, None, None, None, None, None, None, 0, stream=0)


def test_lm_target_host_checks():
    assert abi.ttt_lm_target_workspace_bytes(32768, 4096) >= 2 * 32768 * 4096
    assert abi.ttt_lm_target_workspace_bytes(-1, 8) == 0
    abi.ttt_lm_target(0, 64, None, None, None, None, None, 0, stream=0)   # empty: no-op
    with pytest.raises(abi.TTTError) as ei:
        abi.ttt_lm_target(16, 12, 256, 256, 256, 256, 256, 1 << 20, stream=0)
    assert ei.value.status == abi.TTT_ERR_UNSUPPORTED
    with pytest.raises(abi.TTTError) as ei:
        abi.ttt_debug_wait_timeout(10, stream=0)
    assert ei.value.status == abi.TTT_ERR_INVALID_ARG


def test_debug_checks_setting_and_guarded_workspace_sizes():
    """TTT_CHECK_GUARDS adds a 256-byte guard in front of the first workspace region and
    after each region; the setting is process-wide and unknown flags are refused (all host
    logic: nothing reaches the driver)."""
    assert abi.ttt_get_debug_checks() == 0
    plain = {p: abi.ttt_workspace_bytes(lm_desc(), p)
             for p in (abi.TTT_PATH_PARALLEL, abi.TTT_PATH_PARALLEL_BWD)}
    rec = abi.ttt_workspace_bytes(lm_desc(update_mask=7), abi.TTT_PATH_RECURRENT)
    assert rec > 0
    tgt = abi.ttt_lm_target_workspace_bytes(1000, 64)
    with pytest.raises(abi.TTTError) as ei:
        abi.ttt_set_debug_checks(8)
    assert ei.value.status == abi.TTT_ERR_INVALID_ARG
    try:
        abi.ttt_set_debug_checks(abi.TTT_CHECK_GUARDS | abi.TTT_CHECK_FINITE)
        assert abi.ttt_get_debug_checks() == 3
        par = abi.ttt_workspace_bytes(lm_desc(), abi.TTT_PATH_PARALLEL)
        # 5 regions at lm (blocked weights, two feature buffers, deltas, chunk states):
        # 6 guards, each region end rounded to 16 bytes and the next region to 256
        assert plain[abi.TTT_PATH_PARALLEL] + 6 * 256 <= par <= \
            plain[abi.TTT_PATH_PARALLEL] + 6 * 256 + 6 * 256
        assert abi.ttt_workspace_bytes(lm_desc(), abi.TTT_PATH_PARALLEL_BWD) > \
            plain[abi.TTT_PATH_PARALLEL_BWD]
        assert abi.ttt_workspace_bytes(lm_desc(update_mask=7), abi.TTT_PATH_RECURRENT) > rec
        assert abi.ttt_lm_target_workspace_bytes(1000, 64) >= tgt + 2 * 256
        # a workspace sized with guards off is refused with guards on, before any launch
        d = lm_desc()
        with pytest.raises(abi.TTTError) as ei:
            abi.ttt_la_parallel_fwd(d, 256, 512, 768, 1024, 2048, 4096, 8192, 16384, None,
                                    1 << 20, plain[abi.TTT_PATH_PARALLEL], 0)
        assert ei.value.status == abi.TTT_ERR_WORKSPACE
        abi.ttt_set_debug_checks(0)
        with pytest.raises(abi.TTTError) as ei:   # guards off: nothing to compare
            abi.ttt_debug_check_workspace(d, abi.TTT_PATH_PARALLEL, 1 << 20, 1 << 30, 0)
        assert ei.value.status == abi.TTT_ERR_INVALID_ARG
    finally:
        abi.ttt_set_debug_checks(0)
    assert abi.ttt_workspace_bytes(lm_desc(), abi.TTT_PATH_PARALLEL) == \
        plain[abi.TTT_PATH_PARALLEL]


def test_bf16_mode_refuses_shapes_the_tensor_cores_cannot_take():
    """bf16 mode has one engine: a request it cannot take is refused up front with
    TTT_ERR_UNSUPPORTED (never rerouted to the CUDA cores)."""
    for h, m in ((12, 64), (64, 20)):
        d = lm_desc(B=1, H=1, N=256, h=h, m=m, chunk=64)
        assert abi.ttt_workspace_bytes(d, abi.TTT_PATH_PARALLEL) == 0
        with pytest.raises(abi.TTTError) as ei:
            abi.ttt_la_parallel_fwd(d, 256, 512, 768, 1024, 2048, 4096, 8192, 16384, None,
                                    1 << 20, 1 << 30, 0)
        assert ei.value.status == abi.TTT_ERR_UNSUPPORTED
