"""ctypes binding of libssmscan (include/ssmscan.h).

Argument marshalling only: every step of the layer core runs in the
library's CUDA kernels. PyTorch supplies device memory and the stream. There
is no CPU fallback: a missing library or a CPU tensor raises.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libssmscan.so")

SSM_OK = 0
SSM_ERR_INVALID_ARG = 1
SSM_ERR_UNSUPPORTED = 2
SSM_ERR_CUDA = 3
SSM_ERR_TIMEOUT = 4
SSM_ERR_INJECTED = 5
SSM_DTYPE_F32 = 0
SSM_DTYPE_BF16 = 1

_vp = ctypes.c_void_p
_i = ctypes.c_int
_sz = ctypes.c_size_t


class SsmError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"libssmscan status {status}: {msg}")
        self.status = status


class ssm_scan_params(ctypes.Structure):
    _fields_ = [
        ("struct_size", _sz),
        ("B", _i), ("D", _i), ("L", _i), ("N", _i),
        ("dtype", _i),
        ("u", _vp), ("delta", _vp), ("z", _vp),
        ("A", _vp), ("Dskip", _vp), ("delta_bias", _vp),
        ("Bm", _vp), ("Cm", _vp),
        ("delta_softplus", _i),
        ("seq_idx", _vp), ("cu_seqlens", _vp), ("n_docs", _i),
        ("n_splits", _i),
        ("out", _vp), ("final_state", _vp),
        ("workspace", _vp), ("workspace_bytes", _sz),
        ("initial_state", _vp),
        ("discretization", _i),
        ("state_complex", _i),
    ]


class ssm_scan_grads(ctypes.Structure):
    _fields_ = [
        ("struct_size", _sz),
        ("dout", _vp), ("du", _vp), ("ddelta", _vp), ("dz", _vp),
        ("dA", _vp), ("dB", _vp), ("dC", _vp), ("dD", _vp), ("ddelta_bias", _vp),
        ("deterministic", _i),
        ("dinitial_state", _vp),
        ("dfinal_state", _vp),
        ("workspace", _vp), ("workspace_bytes", _sz),
    ]


class ssm_ssd_params(ctypes.Structure):
    _fields_ = [
        ("struct_size", _sz),
        ("B", _i), ("L", _i), ("H", _i), ("P", _i), ("G", _i), ("N", _i),
        ("dtype", _i),
        ("x", _vp), ("dt_raw", _vp), ("A", _vp), ("Bm", _vp), ("Cm", _vp),
        ("D", _vp), ("dt_bias", _vp), ("dt_softplus", _i), ("seq_idx", _vp),
        ("y", _vp), ("final_state", _vp), ("status", _vp),
        ("chunk_states", _vp),
    ]


class ssm_ssd_grads(ctypes.Structure):
    _fields_ = [
        ("struct_size", _sz),
        ("dy", _vp), ("dx", _vp), ("ddt_raw", _vp), ("dA", _vp),
        ("dB", _vp), ("dC", _vp), ("dD", _vp), ("ddt_bias", _vp),
    ]


class ssm_decode_params(ctypes.Structure):
    _fields_ = [
        ("struct_size", _sz),
        ("B", _i), ("D", _i), ("N", _i), ("W", _i),
        ("dtype", _i),
        ("x", _vp), ("conv_state", _vp), ("conv_w", _vp), ("conv_bias", _vp),
        ("delta", _vp), ("z", _vp), ("Bm", _vp), ("Cm", _vp),
        ("A", _vp), ("Dskip", _vp), ("delta_bias", _vp),
        ("delta_softplus", _i),
        ("state", _vp), ("out", _vp), ("u_out", _vp),
    ]


class ssm_debug_info(ctypes.Structure):
    _fields_ = [
        ("struct_size", _sz),
        ("failures", ctypes.c_ulonglong),
        ("site", _i),
        ("offset", ctypes.c_longlong), ("count", ctypes.c_longlong), ("extent", ctypes.c_longlong),
        ("site_name", ctypes.c_char * 48),
    ]


_lib = None

EXPORTS = ("ssm_last_error", "ssm_abi_version", "ssm_conv1d_fwd", "ssm_conv1d_bwd_workspace_size",
           "ssm_conv1d_bwd", "ssm_conv1d_bwd_noalloc", "ssm_scan_workspace_size", "ssm_scan_fwd",
           "ssm_scan_bwd", "ssm_scan_bwd_workspace_size", "ssm_scan_status", "ssm_probe_ex2_rate", "ssm_decode_step",
           "ssm_conv1d_scan_fwd", "ssm_scan_fwd_summary", "ssm_scan_bwd_summary",
           "ssm_state_carry", "ssm_conv1d_fwd_ctx", "ssm_conv1d_bwd_ctx", "ssm_ssd_fwd",
           "ssm_ssd_bwd", "ssm_debug_report", "ssm_debug_selftest")


def load(path: str | None = None):
    """Load libssmscan.so (built in-tree by build.py; env SSM_LIBRARY may name
    another build of it); raises if it is missing."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or os.environ.get("SSM_LIBRARY") or LIB_PATH
    if not os.path.exists(p):
        raise ImportError(f"{p} is missing: build it with `python -m selective_state_space_35_b200.build`"
                          " (the package has no CPU fallback)")
    L = ctypes.CDLL(p)
    L.ssm_last_error.restype = ctypes.c_char_p
    L.ssm_last_error.argtypes = []
    L.ssm_abi_version.restype = _i
    L.ssm_abi_version.argtypes = []
    L.ssm_conv1d_fwd.restype = _i
    L.ssm_conv1d_fwd.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp]
    L.ssm_conv1d_bwd_workspace_size.restype = _i
    L.ssm_conv1d_bwd_workspace_size.argtypes = [_i, _i, _i, _i, ctypes.POINTER(_sz)]
    L.ssm_conv1d_bwd.restype = _i
    L.ssm_conv1d_bwd.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i,
                                 _vp, _sz, _vp]
    L.ssm_conv1d_bwd_noalloc.restype = _i
    L.ssm_conv1d_bwd_noalloc.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i,
                                         _i, _i, _vp]
    L.ssm_scan_workspace_size.restype = _i
    L.ssm_scan_workspace_size.argtypes = [ctypes.POINTER(ssm_scan_params), ctypes.POINTER(_sz)]
    L.ssm_scan_fwd.restype = _i
    L.ssm_scan_fwd.argtypes = [ctypes.POINTER(ssm_scan_params), _vp]
    L.ssm_scan_bwd.restype = _i
    L.ssm_scan_bwd.argtypes = [ctypes.POINTER(ssm_scan_params), ctypes.POINTER(ssm_scan_grads), _vp]
    L.ssm_scan_bwd_workspace_size.restype = _i
    L.ssm_scan_bwd_workspace_size.argtypes = [ctypes.POINTER(ssm_scan_params),
                                              ctypes.POINTER(ssm_scan_grads), ctypes.POINTER(_sz)]
    L.ssm_scan_status.restype = _i
    L.ssm_scan_status.argtypes = [ctypes.POINTER(ssm_scan_params), ctypes.POINTER(_i), _vp]
    L.ssm_probe_ex2_rate.restype = _i
    L.ssm_probe_ex2_rate.argtypes = [_vp, _sz, ctypes.POINTER(ctypes.c_double), _vp]
    L.ssm_conv1d_scan_fwd.restype = _i
    L.ssm_conv1d_scan_fwd.argtypes = [ctypes.POINTER(ssm_scan_params), _vp, _vp, _vp, _vp]
    L.ssm_decode_step.restype = _i
    L.ssm_decode_step.argtypes = [ctypes.POINTER(ssm_decode_params), _vp]
    L.ssm_ssd_fwd.restype = _i
    L.ssm_ssd_fwd.argtypes = [ctypes.POINTER(ssm_ssd_params), _vp]
    L.ssm_ssd_bwd.restype = _i
    L.ssm_ssd_bwd.argtypes = [ctypes.POINTER(ssm_ssd_params), ctypes.POINTER(ssm_ssd_grads), _vp]
    L.ssm_scan_fwd_summary.restype = _i
    L.ssm_scan_fwd_summary.argtypes = [ctypes.POINTER(ssm_scan_params), _vp, _vp, _vp, _vp]
    L.ssm_scan_bwd_summary.restype = _i
    L.ssm_scan_bwd_summary.argtypes = [ctypes.POINTER(ssm_scan_params), _vp, _vp, _vp, _vp, _vp]
    L.ssm_state_carry.restype = _i
    L.ssm_state_carry.argtypes = [_vp, _vp, _i, _i, _i, _vp, _vp, _vp, _i, _vp, _i, _i, _i, _vp]
    L.ssm_conv1d_fwd_ctx.restype = _i
    L.ssm_conv1d_fwd_ctx.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp]
    L.ssm_conv1d_bwd_ctx.restype = _i
    L.ssm_conv1d_bwd_ctx.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                     _vp, _i, _i, _i, _i, _i, _i, _vp, _sz, _vp]
    L.ssm_debug_report.restype = _i
    L.ssm_debug_report.argtypes = [ctypes.POINTER(ssm_debug_info), _i]
    L.ssm_debug_selftest.restype = _i
    L.ssm_debug_selftest.argtypes = [_vp, _sz, _vp]
    if path is None:
        _lib = L
    return L


def check(status: int) -> None:
    if status != SSM_OK:
        raise SsmError(status, load().ssm_last_error().decode(errors="replace"))


# Raw entry points with the ABI's own names (pointer-level).
def ssm_last_error() -> str:
    return load().ssm_last_error().decode(errors="replace")


def ssm_abi_version() -> int:
    return load().ssm_abi_version()


def ssm_conv1d_fwd(*args) -> int:
    return load().ssm_conv1d_fwd(*args)


def ssm_conv1d_bwd_workspace_size(B, D, L, W) -> int:
    n = _sz(0)
    check(load().ssm_conv1d_bwd_workspace_size(B, D, L, W, ctypes.byref(n)))
    return n.value


def ssm_conv1d_bwd(*args) -> int:
    return load().ssm_conv1d_bwd(*args)


def ssm_conv1d_bwd_noalloc(*args) -> int:
    return load().ssm_conv1d_bwd_noalloc(*args)


def ssm_scan_workspace_size(params: ssm_scan_params) -> int:
    n = _sz(0)
    check(load().ssm_scan_workspace_size(ctypes.byref(params), ctypes.byref(n)))
    return n.value


def ssm_scan_bwd_workspace_size(params: ssm_scan_params, grads: ssm_scan_grads) -> int:
    n = _sz(0)
    check(load().ssm_scan_bwd_workspace_size(ctypes.byref(params), ctypes.byref(grads),
                                             ctypes.byref(n)))
    return n.value


def ssm_scan_status(params: ssm_scan_params, stream) -> int:
    v = _i(0)
    check(load().ssm_scan_status(ctypes.byref(params), ctypes.byref(v), stream))
    return v.value


def ssm_probe_ex2_rate(sink, sink_floats: int, stream) -> float:
    r = ctypes.c_double(0.0)
    check(load().ssm_probe_ex2_rate(sink, sink_floats, ctypes.byref(r), stream))
    return r.value


def _ref(x):
    return None if x is None else ctypes.byref(x)


def ssm_scan_fwd(params: ssm_scan_params, stream) -> int:
    return load().ssm_scan_fwd(_ref(params), stream)


def ssm_scan_bwd(params: ssm_scan_params, grads: ssm_scan_grads, stream) -> int:
    return load().ssm_scan_bwd(_ref(params), _ref(grads), stream)


def ssm_conv1d_scan_fwd(params: ssm_scan_params, x, conv_w, conv_bias, stream) -> int:
    return load().ssm_conv1d_scan_fwd(_ref(params), x, conv_w, conv_bias, stream)


def ssm_decode_step(params: ssm_decode_params, stream) -> int:
    return load().ssm_decode_step(_ref(params), stream)


def ssm_scan_fwd_summary(params: ssm_scan_params, seq_prev, decay, state_end, stream) -> int:
    return load().ssm_scan_fwd_summary(_ref(params), seq_prev, decay, state_end, stream)


def ssm_scan_bwd_summary(params: ssm_scan_params, dout, seq_prev, decay, adj_start, stream) -> int:
    return load().ssm_scan_bwd_summary(_ref(params), dout, seq_prev, decay, adj_start, stream)


def ssm_state_carry(*args) -> int:
    return load().ssm_state_carry(*args)


def ssm_conv1d_fwd_ctx(*args) -> int:
    return load().ssm_conv1d_fwd_ctx(*args)


def ssm_conv1d_bwd_ctx(*args) -> int:
    return load().ssm_conv1d_bwd_ctx(*args)


def ssm_ssd_fwd(params: ssm_ssd_params, stream) -> int:
    return load().ssm_ssd_fwd(ctypes.byref(params), stream)


def ssm_ssd_bwd(params: ssm_ssd_params, grads: ssm_ssd_grads, stream) -> int:
    return load().ssm_ssd_bwd(ctypes.byref(params), ctypes.byref(grads), stream)


def ssm_debug_report(info, reset) -> int:
    return load().ssm_debug_report(info, reset)


def ssm_debug_selftest(buf, n, stream) -> int:
    return load().ssm_debug_selftest(buf, n, stream)
