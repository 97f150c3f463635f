"""ctypes binding of ``libhyena.so``: the C entry points under the same names.

Argument marshalling only. Every function takes plain integers for device
pointers and streams and returns the library's status code, exactly as the C
ABI in ``include/hyena.h`` does. There is no fallback: if the shared library
is missing or fails to load, importing this module raises.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
# HYENA_LIBRARY=checked loads the index-checking debug build (libhyena_checked.so)
LIB_PATH = os.path.join(_PKG, "libhyena_checked.so" if os.environ.get("HYENA_LIBRARY") == "checked"
                        else "libhyena.so")

HYENA_MAX_ORDER = 8
HYENA_F32, HYENA_BF16 = 0, 1
(HYENA_OK, HYENA_ERR_INVALID_ARG, HYENA_ERR_UNSUPPORTED, HYENA_ERR_ALIGNMENT,
 HYENA_ERR_WORKSPACE, HYENA_ERR_CUDA, HYENA_ERR_NOMEM) = range(7)
HYENA_PATH_CTA, HYENA_PATH_CLUSTER, HYENA_PATH_2D, HYENA_PATH_STAGED = 0, 1, 2, 3
HYENA_LAYOUT_BDL, HYENA_LAYOUT_BLD = 0, 1
HYENA_PLAN_RADIX3 = 1

STATUS_NAMES = {
    HYENA_OK: "HYENA_OK", HYENA_ERR_INVALID_ARG: "HYENA_ERR_INVALID_ARG",
    HYENA_ERR_UNSUPPORTED: "HYENA_ERR_UNSUPPORTED", HYENA_ERR_ALIGNMENT: "HYENA_ERR_ALIGNMENT",
    HYENA_ERR_WORKSPACE: "HYENA_ERR_WORKSPACE", HYENA_ERR_CUDA: "HYENA_ERR_CUDA",
    HYENA_ERR_NOMEM: "HYENA_ERR_NOMEM",
}

# Every symbol include/hyena.h declares (checked by the CPU test suite).
EXPORTED = (
    "hyena_plan_create", "hyena_plan_destroy", "hyena_plan_info", "hyena_workspace_bytes",
    "hyena_implicit_filter", "hyena_filter_spectrum", "hyena_forward", "hyena_status_string",
    "hyena_forward_no_alloc", "hyena_forward_host_workspace_bytes", "hyena_forward_host",
    "hyena_forward_gated", "hyena_plan_set_layout", "hyena_plan_device_errors", "hyena_plan_create_ex",
    "hyena_launch_count", "hyena_debug_fail_allocation", "hyena_debug_plan_resources",
    "hyena_filter_spectrum_ws", "hyena_filter_spectrum_workspace_bytes",
)


class hyena_implicit_params_t(ctypes.Structure):
    _fields_ = [
        ("W1", ctypes.c_void_p), ("b1", ctypes.c_void_p),
        ("W2", ctypes.c_void_p), ("b2", ctypes.c_void_p),
        ("W3", ctypes.c_void_p), ("b3", ctypes.c_void_p),
        ("window", ctypes.c_void_p),
        ("width", ctypes.c_int32), ("num_freqs", ctypes.c_int32),
        ("omega0", ctypes.c_float), ("omega_hidden", ctypes.c_float),
    ]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError("libhyena.so not built (%s); run __graft_entry__.build() or "
                          "python -m long_convolution_sequence_hyena_b200.build" % LIB_PATH)
    lib = ctypes.CDLL(LIB_PATH)
    p, i64, i32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
    sig = {
        "hyena_plan_create": ([ctypes.POINTER(p), i32, ctypes.POINTER(i64), i64, i32, i32, i32], i32),
        "hyena_plan_destroy": ([p], i32),
        "hyena_plan_info": ([p, ctypes.POINTER(i64), ctypes.POINTER(i64), ctypes.POINTER(i32)], i32),
        "hyena_workspace_bytes": ([p, i64], sz),
        "hyena_implicit_filter": ([p, ctypes.POINTER(hyena_implicit_params_t), p, p], i32),
        "hyena_filter_spectrum": ([p, p, ctypes.POINTER(hyena_implicit_params_t), p, p], i32),
        "hyena_forward": ([p, i64, p, ctypes.POINTER(p), p, p, p, p, sz, p], i32),
        "hyena_status_string": ([i32], ctypes.c_char_p),
        "hyena_forward_no_alloc": ([p, i64, p, ctypes.POINTER(p), p, p, p, p], i32),
        "hyena_forward_host_workspace_bytes": ([p, i64], sz),
        "hyena_forward_host": ([p, i64, p, ctypes.POINTER(p), p, p, p, p, sz, p], i32),
        "hyena_forward_gated": ([p, i64, p, p, ctypes.POINTER(p), p, p, p, p, sz, p], i32),
        "hyena_plan_set_layout": ([p, i32], i32),
        "hyena_plan_device_errors": ([p, ctypes.POINTER(i32), i32], i32),
        "hyena_plan_create_ex": ([ctypes.POINTER(p), i32, ctypes.POINTER(i64), i64, i32, i32, i32, i32], i32),
        "hyena_launch_count": ([ctypes.POINTER(i64)], i32),
        "hyena_debug_fail_allocation": ([i32], i32),
        "hyena_debug_plan_resources": ([ctypes.POINTER(i64)], i32),
        "hyena_filter_spectrum_ws": ([p, p, ctypes.POINTER(hyena_implicit_params_t), p, p, sz, p], i32),
        "hyena_filter_spectrum_workspace_bytes": ([p], sz),
    }
    for name, (args, res) in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    return lib


lib = _load()


def hyena_status_string(status: int) -> str:
    return lib.hyena_status_string(status).decode()


def hyena_plan_create(ndim: int, shape, channels: int, order: int, io_dtype: int, causal: int):
    """Returns (status, plan handle as int or None)."""
    out = ctypes.c_void_p()
    arr = (ctypes.c_int64 * len(shape))(*shape)
    st = lib.hyena_plan_create(ctypes.byref(out), ndim, arr, channels, order, io_dtype, causal)
    return st, out.value


def hyena_plan_create_ex(ndim: int, shape, channels: int, order: int, io_dtype: int, causal: int, flags: int):
    """Returns (status, plan handle as int or None)."""
    out = ctypes.c_void_p()
    arr = (ctypes.c_int64 * len(shape))(*shape)
    st = lib.hyena_plan_create_ex(ctypes.byref(out), ndim, arr, channels, order, io_dtype, causal, flags)
    return st, out.value


def hyena_plan_destroy(plan) -> int:
    return lib.hyena_plan_destroy(plan)


def hyena_plan_set_layout(plan, layout: int) -> int:
    return lib.hyena_plan_set_layout(plan, layout)


def hyena_plan_device_errors(plan, clear: bool = False):
    """Returns (status, device error word); synchronises with the device."""
    f = ctypes.c_int()
    st = lib.hyena_plan_device_errors(plan, ctypes.byref(f), 1 if clear else 0)
    return st, f.value


def hyena_launch_count() -> int:
    """Kernels the library has enqueued in this process so far."""
    n = ctypes.c_int64()
    st = lib.hyena_launch_count(ctypes.byref(n))
    if st != HYENA_OK:
        raise RuntimeError("hyena_launch_count: %d" % st)
    return n.value


def hyena_debug_plan_resources() -> int:
    """Device buffers, streams and host objects all live plans hold (test hook)."""
    n = ctypes.c_int64()
    st = lib.hyena_debug_plan_resources(ctypes.byref(n))
    if st != HYENA_OK:
        raise RuntimeError("hyena_debug_plan_resources: %d" % st)
    return n.value


def hyena_plan_info(plan):
    """Returns (status, fft_len, spectrum_elems, path)."""
    m, s, path = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int()
    st = lib.hyena_plan_info(plan, ctypes.byref(m), ctypes.byref(s), ctypes.byref(path))
    return st, m.value, s.value, path.value


def hyena_workspace_bytes(plan, batch: int) -> int:
    return lib.hyena_workspace_bytes(plan, batch)


def hyena_implicit_filter(plan, params, h_out: int, stream: int = 0) -> int:
    return lib.hyena_implicit_filter(plan, ctypes.byref(params) if params is not None else None, h_out, stream)


def hyena_filter_spectrum(plan, h, params, H_out: int, stream: int = 0) -> int:
    return lib.hyena_filter_spectrum(plan, h, ctypes.byref(params) if params is not None else None, H_out, stream)


def hyena_filter_spectrum_ws(plan, h, params, H_out: int, workspace, ws_bytes: int, stream: int = 0) -> int:
    return lib.hyena_filter_spectrum_ws(plan, h, ctypes.byref(params) if params is not None else None, H_out,
                                        workspace, ws_bytes, stream)


def hyena_forward(plan, batch: int, v: int, gates, H: int, Dskip, y: int, workspace=None, ws_bytes: int = 0,
                  stream: int = 0) -> int:
    garr = None if gates is None else (ctypes.c_void_p * len(gates))(*gates)
    return lib.hyena_forward(plan, batch, v, garr, H, Dskip, y, workspace, ws_bytes, stream)


def hyena_forward_gated(plan, batch: int, q: int, k: int, gates, H: int, Dskip, y: int, workspace=None,
                        ws_bytes: int = 0, stream: int = 0) -> int:
    """The gate sandwich: z^0 = q SiLU(k), z^n = SiLU(x^n) (K^n * z^{n-1} + Dskip^n z^{n-1})."""
    garr = None if gates is None else (ctypes.c_void_p * len(gates))(*gates)
    return lib.hyena_forward_gated(plan, batch, q, k, garr, H, Dskip, y, workspace, ws_bytes, stream)


def hyena_forward_no_alloc(plan, batch: int, v: int, gates, H: int, Dskip, y: int, stream: int = 0) -> int:
    """hyena_forward without a workspace argument: the staged path's scratch is the library's
    own fixed device array (for callers that cannot allocate device memory)."""
    garr = None if gates is None else (ctypes.c_void_p * len(gates))(*gates)
    return lib.hyena_forward_no_alloc(plan, batch, v, garr, H, Dskip, y, stream)


def hyena_forward_host_workspace_bytes(plan, batch: int) -> int:
    return lib.hyena_forward_host_workspace_bytes(plan, batch)


def hyena_forward_host(plan, batch: int, v_host: int, gates_host, H: int, Dskip, y_host: int, workspace,
                       ws_bytes: int, stream: int = 0) -> int:
    """hyena_forward on page-locked host activations (v, gates, y): the library copies them in
    and out, pipelined over the batch."""
    garr = None if gates_host is None else (ctypes.c_void_p * len(gates_host))(*gates_host)
    return lib.hyena_forward_host(plan, batch, v_host, garr, H, Dskip, y_host, workspace, ws_bytes, stream)
