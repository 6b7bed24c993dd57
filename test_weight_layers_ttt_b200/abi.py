"""Thin Python binding of the C ABI in include/ttt.h (argument marshalling only).

Every function has the name and argument order of its C counterpart. Tensor arguments
may be torch tensors (their ``data_ptr()`` is passed), plain integers (raw device
pointers) or None (NULL). ``stream`` may be a ``torch.cuda.Stream``, a raw handle or None
(the current torch stream of the current device). A non-OK status raises ``TTTError``
carrying the status and the library's message. All computation happens in the CUDA
library; nothing here falls back to another implementation, and loading fails loudly
when the library has not been built.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libttt_b200.so")

TTT_OK = 0
TTT_ERR_INVALID_ARG = 1
TTT_ERR_UNSUPPORTED = 2
TTT_ERR_WORKSPACE = 3
TTT_ERR_CUDA = 4
TTT_ERR_TIMEOUT = 5
TTT_ERR_DEVICE = 6

TTT_DTYPE_FP32 = 0
TTT_DTYPE_BF16 = 1
TTT_ORDER_UPDATE_APPLY = 0
TTT_ORDER_APPLY_UPDATE = 1
TTT_UPDATE_W0 = 1
TTT_UPDATE_W1 = 2
TTT_UPDATE_W2 = 4
TTT_UPDATE_ALL = 7
TTT_PATH_PARALLEL = 0
TTT_PATH_RECURRENT = 1
TTT_PATH_LINEAR = 2
TTT_PATH_PARALLEL_MOMENTUM = 3
TTT_PATH_PARALLEL_BWD = 4
TTT_STATIC_SCRATCH_BYTES = 64 << 20
TTT_CHECK_GUARDS = 1
TTT_CHECK_FINITE = 2

# Every symbol include/ttt.h declares.
EXPORTED = (
    "ttt_workspace_bytes", "ttt_la_parallel_fwd", "ttt_la_parallel_fwd_noalloc",
    "ttt_la_parallel_fwd_shard", "ttt_la_parallel_fwd_shard_outputs",
    "ttt_linear_attn_fwd", "ttt_la_parallel_momentum_fwd", "ttt_la_parallel_bwd",
    "ttt_lact_recurrent_fwd",
    "ttt_lm_target_workspace_bytes", "ttt_lm_target", "ttt_last_device_status",
    "ttt_set_debug_checks", "ttt_get_debug_checks", "ttt_debug_check_workspace",
    "ttt_debug_wait_timeout", "ttt_trace_enable", "ttt_trace_disable", "ttt_trace_count",
    "ttt_trace_get", "ttt_status_str", "ttt_last_error_message", "ttt_version",
)


class TTTError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{status_name(status)}: {message}")
        self.status = status


class ttt_desc(ctypes.Structure):
    _fields_ = [(name, ctypes.c_int32) for name in (
        "B", "H", "N", "h", "m", "chunk", "dtype", "order", "sign", "update_mask", "renorm",
        "momentum", "ns_steps", "w_in_layout", "w1_layout")]

    def __init__(self, **kw):
        kw.setdefault("sign", 1)
        super().__init__(**kw)

    def __repr__(self):
        return "ttt_desc(" + ", ".join(f"{n}={getattr(self, n)}" for n, _ in self._fields_) + ")"


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded CUDA library; raises when it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m test_weight_layers_ttt_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, S, I32, I64 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int32, ctypes.c_int64
        D = ctypes.POINTER(ttt_desc)
        L.ttt_workspace_bytes.argtypes = [D, I32]
        L.ttt_workspace_bytes.restype = S
        L.ttt_la_parallel_fwd.argtypes = [D] + [P] * 10 + [S, P]
        L.ttt_la_parallel_fwd.restype = I32
        L.ttt_la_parallel_fwd_shard.argtypes = [D] + [P] * 8 + [I32, P, P, P, S, P]
        L.ttt_la_parallel_fwd_shard.restype = I32
        L.ttt_la_parallel_fwd_shard_outputs.argtypes = [D] + [P] * 3 + [I32, P, P, P, S, P]
        L.ttt_la_parallel_fwd_shard_outputs.restype = I32
        L.ttt_la_parallel_fwd_noalloc.argtypes = [D] + [P] * 10
        L.ttt_la_parallel_fwd_noalloc.restype = I32
        L.ttt_linear_attn_fwd.argtypes = [D] + [P] * 8 + [S, P]
        L.ttt_linear_attn_fwd.restype = I32
        L.ttt_la_parallel_momentum_fwd.argtypes = [D] + [P] * 11 + [S, P]
        L.ttt_la_parallel_momentum_fwd.restype = I32
        L.ttt_la_parallel_bwd.argtypes = [D] + [P] * 17 + [S, P]
        L.ttt_la_parallel_bwd.restype = I32
        L.ttt_lact_recurrent_fwd.argtypes = [D] + [P] * 14 + [S, P]
        L.ttt_lact_recurrent_fwd.restype = I32
        L.ttt_lm_target_workspace_bytes.argtypes = [I32, I32]
        L.ttt_lm_target_workspace_bytes.restype = S
        L.ttt_lm_target.argtypes = [I32, I32, P, P, P, P, P, S, P]
        L.ttt_lm_target.restype = I32
        L.ttt_last_device_status.argtypes = [P]
        L.ttt_last_device_status.restype = I32
        L.ttt_set_debug_checks.argtypes = [I32]
        L.ttt_set_debug_checks.restype = I32
        L.ttt_get_debug_checks.argtypes = []
        L.ttt_get_debug_checks.restype = I32
        L.ttt_debug_check_workspace.argtypes = [D, I32, P, S, P]
        L.ttt_debug_check_workspace.restype = I32
        L.ttt_debug_wait_timeout.argtypes = [I64, P]
        L.ttt_debug_wait_timeout.restype = I32
        L.ttt_trace_enable.argtypes = [I32]
        L.ttt_trace_enable.restype = I32
        L.ttt_trace_disable.argtypes = []
        L.ttt_trace_disable.restype = I32
        L.ttt_trace_count.argtypes = []
        L.ttt_trace_count.restype = I32
        L.ttt_trace_get.argtypes = [I32, ctypes.POINTER(ctypes.c_char_p),
                                    ctypes.POINTER(ctypes.c_float)]
        L.ttt_trace_get.restype = I32
        L.ttt_status_str.argtypes = [I32]
        L.ttt_status_str.restype = ctypes.c_char_p
        L.ttt_last_error_message.argtypes = []
        L.ttt_last_error_message.restype = ctypes.c_char_p
        L.ttt_version.argtypes = []
        L.ttt_version.restype = I32
        _lib = L
    return _lib


def status_name(status: int) -> str:
    names = {0: "TTT_OK", 1: "TTT_ERR_INVALID_ARG", 2: "TTT_ERR_UNSUPPORTED",
             3: "TTT_ERR_WORKSPACE", 4: "TTT_ERR_CUDA", 5: "TTT_ERR_TIMEOUT",
             6: "TTT_ERR_DEVICE"}
    return names.get(int(status), f"status {status}")


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(s):
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _check(status: int):
    if status != TTT_OK:
        msg = lib().ttt_last_error_message().decode(errors="replace")
        raise TTTError(status, msg)


def _nbytes(x):
    if x is None:
        return 0
    if isinstance(x, int):
        raise TypeError("pass workspace_bytes explicitly with a raw workspace pointer")
    return x.numel() * x.element_size()


# ----------------------------------------------------------------------------- entry points
def ttt_workspace_bytes(desc: ttt_desc, path: int) -> int:
    return int(lib().ttt_workspace_bytes(ctypes.byref(desc), path))


def ttt_la_parallel_fwd(desc, q, k, v, eta, W0, W2, W1, out, S_final, workspace,
                        workspace_bytes=None, stream=None):
    wb = _nbytes(workspace) if workspace_bytes is None else workspace_bytes
    _check(lib().ttt_la_parallel_fwd(
        ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(eta), _ptr(W0), _ptr(W2), _ptr(W1),
        _ptr(out), _ptr(S_final), _ptr(workspace), wb, _stream(stream)))


def ttt_la_parallel_fwd_shard(desc, q, k, v, eta, W0, W2, W1, prior, n_prior, out, S_final,
                              workspace, workspace_bytes=None, stream=None):
    wb = _nbytes(workspace) if workspace_bytes is None else workspace_bytes
    _check(lib().ttt_la_parallel_fwd_shard(
        ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(eta), _ptr(W0), _ptr(W2), _ptr(W1),
        _ptr(prior), int(n_prior), _ptr(out), _ptr(S_final), _ptr(workspace), wb,
        _stream(stream)))


def ttt_la_parallel_fwd_shard_outputs(desc, q, W1, prior, n_prior, out, S_final, workspace,
                                      workspace_bytes=None, stream=None):
    wb = _nbytes(workspace) if workspace_bytes is None else workspace_bytes
    _check(lib().ttt_la_parallel_fwd_shard_outputs(
        ctypes.byref(desc), _ptr(q), _ptr(W1), _ptr(prior), int(n_prior), _ptr(out),
        _ptr(S_final), _ptr(workspace), wb, _stream(stream)))


def ttt_la_parallel_momentum_fwd(desc, q, k, v, eta, alpha, W0, W2, W1, out, S_final,
                                 workspace, workspace_bytes=None, stream=None):
    wb = _nbytes(workspace) if workspace_bytes is None else workspace_bytes
    _check(lib().ttt_la_parallel_momentum_fwd(
        ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(eta), _ptr(alpha), _ptr(W0),
        _ptr(W2), _ptr(W1), _ptr(out), _ptr(S_final), _ptr(workspace), wb, _stream(stream)))


def ttt_la_parallel_bwd(desc, q, k, v, eta, W0, W2, W1, dout, dS_final, dq, dk, dv, deta, dW0,
                        dW2, dW1, workspace, workspace_bytes=None, stream=None):
    wb = _nbytes(workspace) if workspace_bytes is None else workspace_bytes
    _check(lib().ttt_la_parallel_bwd(
        ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(eta), _ptr(W0), _ptr(W2), _ptr(W1),
        _ptr(dout), _ptr(dS_final), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(deta), _ptr(dW0),
        _ptr(dW2), _ptr(dW1), _ptr(workspace), wb, _stream(stream)))


def ttt_linear_attn_fwd(desc, q, k, v, eta, S0, out, S_final, workspace, workspace_bytes=None,
                        stream=None):
    wb = _nbytes(workspace) if workspace_bytes is None else workspace_bytes
    _check(lib().ttt_linear_attn_fwd(
        ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(eta), _ptr(S0), _ptr(out),
        _ptr(S_final), _ptr(workspace), wb, _stream(stream)))


def ttt_la_parallel_fwd_noalloc(desc, q, k, v, eta, W0, W2, W1, out, S_final, stream=None):
    """Parallel form using the library's built-in scratch instead of a caller workspace,
    for callers that cannot allocate device memory (see include/ttt.h)."""
    _check(lib().ttt_la_parallel_fwd_noalloc(
        ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(eta), _ptr(W0), _ptr(W2), _ptr(W1),
        _ptr(out), _ptr(S_final), _stream(stream)))


def ttt_lact_recurrent_fwd(desc, q, k, v, eta, alpha, W0, W2, W1, out, W0_out, W2_out, W1_out,
                           M_io, workspace, workspace_bytes=None, stream=None):
    wb = _nbytes(workspace) if workspace_bytes is None else workspace_bytes
    _check(lib().ttt_lact_recurrent_fwd(
        ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(eta), _ptr(alpha), _ptr(W0),
        _ptr(W2), _ptr(W1), _ptr(out), _ptr(W0_out), _ptr(W2_out), _ptr(W1_out), _ptr(M_io),
        _ptr(workspace), wb, _stream(stream)))


def ttt_lm_target_workspace_bytes(N: int, d: int) -> int:
    return int(lib().ttt_lm_target_workspace_bytes(N, d))


def ttt_lm_target(N, d, X0, conv_w, W_target, vbar, workspace, workspace_bytes=None,
                  stream=None):
    wb = _nbytes(workspace) if workspace_bytes is None else workspace_bytes
    _check(lib().ttt_lm_target(N, d, _ptr(X0), _ptr(conv_w), _ptr(W_target), _ptr(vbar),
                               _ptr(workspace), wb, _stream(stream)))


def ttt_last_device_status(stream=None):
    _check(lib().ttt_last_device_status(_stream(stream)))


def ttt_set_debug_checks(flags: int):
    _check(lib().ttt_set_debug_checks(int(flags)))


def ttt_get_debug_checks() -> int:
    return int(lib().ttt_get_debug_checks())


def ttt_debug_check_workspace(desc, path, workspace, workspace_bytes=None, stream=None):
    wb = _nbytes(workspace) if workspace_bytes is None else workspace_bytes
    _check(lib().ttt_debug_check_workspace(ctypes.byref(desc), int(path), _ptr(workspace), wb,
                                           _stream(stream)))


def ttt_debug_wait_timeout(timeout_ns: int, stream=None):
    _check(lib().ttt_debug_wait_timeout(int(timeout_ns), _stream(stream)))


def ttt_trace_enable(capacity: int):
    _check(lib().ttt_trace_enable(int(capacity)))


def ttt_trace_disable():
    _check(lib().ttt_trace_disable())


def ttt_trace_count() -> int:
    return int(lib().ttt_trace_count())


def ttt_trace_get(index: int):
    """(kernel name, milliseconds) of trace record ``index``."""
    name = ctypes.c_char_p()
    ms = ctypes.c_float()
    _check(lib().ttt_trace_get(int(index), ctypes.byref(name), ctypes.byref(ms)))
    return name.value.decode(), float(ms.value)


def ttt_status_str(status: int) -> str:
    return lib().ttt_status_str(status).decode()


def ttt_last_error_message() -> str:
    return lib().ttt_last_error_message().decode(errors="replace")


def ttt_version() -> int:
    return int(lib().ttt_version())
