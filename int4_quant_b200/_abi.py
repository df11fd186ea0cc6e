"""ctypes binding of the C ABI in ``include/arnq.h`` (library ``libarnq.so``).

Argument marshalling only: each function has the C entry point's name and
arguments, accepts device pointers as ints, torch tensors (their
``data_ptr()``) or None (NULL), and returns the C status code.  All
validation and all computation happen in the library.

The library is loaded on first use.  If it is missing this raises at once:
there is no other implementation to fall back to.
"""
from __future__ import annotations

import ctypes
import os
import re
import threading

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libarnq.so")
HEADER = os.path.join(os.path.dirname(PKG), "include", "arnq.h")

# --- constants mirrored from include/arnq.h ------------------------------------
ARNQ_OK = 0
ARNQ_ERR_NULL_PTR = 1
ARNQ_ERR_EMPTY = 2
ARNQ_ERR_SHAPE = 3
ARNQ_ERR_DTYPE = 4
ARNQ_ERR_MASK = 5
ARNQ_ERR_EPS = 6
ARNQ_ERR_ALIGN = 7
ARNQ_ERR_WORKSPACE = 8
ARNQ_ERR_CUDA = 9
ARNQ_ERR_PLAN = 10
ARNQ_ERR_DEVICE_TIMEOUT = 11

ARNQ_BF16, ARNQ_FP16 = 0, 1
ARNQ_INT8, ARNQ_INT4, ARNQ_INT4_INT32 = 0, 1, 2
ARNQ_MASK_ABSENT = -1
ARNQ_MASK_Y1, ARNQ_MASK_Y2 = 1, 2
ARNQ_MAX_N = 131072

ARNQ_KERNEL_AUTO, ARNQ_KERNEL_DIRECT, ARNQ_KERNEL_STAGED = 0, 1, 2
ARNQ_STATIC_SCRATCH_BYTES = 4096
ARNQ_WORKSPACE_BYTES = 256


class arnq_plan(ctypes.Structure):
    _fields_ = [(name, ctypes.c_int32) for name in
                ("kernel", "cluster", "threads", "units", "stages", "ctas_per_sm", "grid",
                 "vector", "wait_limit_us", "test_hold_bytes", "early_params")]

    def as_dict(self):
        return {f: getattr(self, f) for f, _ in self._fields_}


class arnq_workspace_status(ctypes.Structure):
    _fields_ = [("code", ctypes.c_int32), ("reserved", ctypes.c_int32), ("row", ctypes.c_int64)]


class ArnqError(RuntimeError):
    def __init__(self, status: int, where: str = ""):
        self.status = status
        super().__init__(f"{where}: {arnq_status_string(status)} (status {status})")


_lock = threading.Lock()
_lib = None

_p, _i64, _i32, _f32, _sz = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float,
                             ctypes.c_size_t)
_SIGS = {
    "arnq_status_string": ([_i32], ctypes.c_char_p),
    "arnq_selected_outputs": ([_i32, _i32, _i32, _p, _p], _i32),
    "arnq_workspace_size": ([_i64, _i64, _i32, _i32, _i32, _i32, _i32, _p], _i32),
    "arnq_run": ([_p, _p, _p, _p, _p, _p, _i64, _i64, _i32, _f32, _i32, _i32, _p, _p, _p, _p,
                  _p, _p, _sz, _p], _i32),
    "arnq_run_v1": ([_p, _p, _p, _p, _p, _i64, _i64, _i32, _f32, _i32, _p, _p, _p, _p, _p, _p,
                     _sz, _p], _i32),
    "arnq_rms_norm_dynamic_quant": ([_p, _p, _p, _p, _i64, _i64, _i32, _f32, _i32, _p, _p, _p,
                                     _sz, _p], _i32),
    "arnq_make_plan": ([_p, _p, _p, _p, _p, _p, _i64, _i64, _i32, _i32, _i32, _p, _p, _p, _p],
                       _i32),
    "arnq_run_planned": ([_p, _p, _p, _p, _p, _p, _i64, _i64, _i32, _f32, _i32, _i32, _p, _p, _p,
                          _p, _p, _p, _sz, _p, _p], _i32),
    "arnq_run_static_scratch": ([_p, _p, _p, _p, _p, _p, _i64, _i64, _i32, _f32, _i32, _i32, _p, _p,
                                 _p, _p, _p, _p], _i32),
}


def lib() -> ctypes.CDLL:
    """Loads libarnq.so (once).  Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(
                    f"{LIB_PATH} is missing: build it with `python -m int4_quant_b200.build` "
                    "(there is no fallback implementation)")
            L = ctypes.CDLL(LIB_PATH)
            for name, (args, res) in _SIGS.items():
                f = getattr(L, name)
                f.argtypes = args
                f.restype = res
            _lib = L
    return _lib


def header_functions(path: str = HEADER):
    """Names of the functions include/arnq.h declares."""
    with open(path) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(arnq_\w+)\s*\(", text)))


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x or None
    dp = getattr(x, "data_ptr", None)
    if dp is not None:
        return dp() or None
    raise TypeError(f"not a pointer: {type(x)!r}")


def _stream(s):
    if s is None:
        return None
    if isinstance(s, int):
        return s or None
    return getattr(s, "cuda_stream", None) or None


# --- the C entry points, same names -------------------------------------------

def arnq_status_string(status: int) -> str:
    return lib().arnq_status_string(int(status)).decode()


def arnq_selected_outputs(out_mask: int, has_smooth1: bool, has_smooth2: bool):
    """Returns (status, y1_on, y2_on)."""
    a, b = ctypes.c_int(0), ctypes.c_int(0)
    st = lib().arnq_selected_outputs(int(out_mask), int(bool(has_smooth1)),
                                     int(bool(has_smooth2)), ctypes.addressof(a),
                                     ctypes.addressof(b))
    return st, bool(a.value), bool(b.value)


def arnq_workspace_size(rows, n, dt, qdt, out_mask, has_smooth1, has_smooth2):
    """Returns (status, bytes)."""
    out = ctypes.c_size_t(0)
    st = lib().arnq_workspace_size(int(rows), int(n), int(dt), int(qdt), int(out_mask),
                                   int(bool(has_smooth1)), int(bool(has_smooth2)),
                                   ctypes.addressof(out))
    return st, out.value


def arnq_run(x1, x2, gamma, beta, smooth1, smooth2, rows, n, dt, eps, out_mask, qdt, y1, scale1,
             y2, scale2, x_out, workspace, workspace_bytes, stream) -> int:
    return lib().arnq_run(_ptr(x1), _ptr(x2), _ptr(gamma), _ptr(beta), _ptr(smooth1),
                          _ptr(smooth2), int(rows), int(n), int(dt), float(eps), int(out_mask),
                          int(qdt), _ptr(y1), _ptr(scale1), _ptr(y2), _ptr(scale2), _ptr(x_out),
                          _ptr(workspace), int(workspace_bytes), _stream(stream))


def arnq_run_v1(x1, x2, gamma, smooth1, smooth2, rows, n, dt, eps, qdt, y1, scale1, y2, scale2,
                x_out, workspace, workspace_bytes, stream) -> int:
    return lib().arnq_run_v1(_ptr(x1), _ptr(x2), _ptr(gamma), _ptr(smooth1), _ptr(smooth2),
                             int(rows), int(n), int(dt), float(eps), int(qdt), _ptr(y1),
                             _ptr(scale1), _ptr(y2), _ptr(scale2), _ptr(x_out), _ptr(workspace),
                             int(workspace_bytes), _stream(stream))


def arnq_rms_norm_dynamic_quant(x, gamma, beta, smooth, rows, n, dt, eps, qdt, y, scale,
                                workspace, workspace_bytes, stream) -> int:
    return lib().arnq_rms_norm_dynamic_quant(_ptr(x), _ptr(gamma), _ptr(beta), _ptr(smooth),
                                             int(rows), int(n), int(dt), float(eps), int(qdt),
                                             _ptr(y), _ptr(scale), _ptr(workspace),
                                             int(workspace_bytes), _stream(stream))


def arnq_make_plan(x1, x2, gamma, beta, smooth1, smooth2, rows, n, dt, out_mask, qdt, y1, y2,
                   x_out, plan: arnq_plan | None = None):
    """Returns (status, plan)."""
    plan = plan if plan is not None else arnq_plan()
    st = lib().arnq_make_plan(_ptr(x1), _ptr(x2), _ptr(gamma), _ptr(beta), _ptr(smooth1),
                              _ptr(smooth2), int(rows), int(n), int(dt), int(out_mask), int(qdt),
                              _ptr(y1), _ptr(y2), _ptr(x_out), ctypes.addressof(plan))
    return st, plan


def arnq_run_planned(x1, x2, gamma, beta, smooth1, smooth2, rows, n, dt, eps, out_mask, qdt, y1,
                     scale1, y2, scale2, x_out, workspace, workspace_bytes, stream,
                     plan: arnq_plan) -> int:
    return lib().arnq_run_planned(_ptr(x1), _ptr(x2), _ptr(gamma), _ptr(beta), _ptr(smooth1),
                                  _ptr(smooth2), int(rows), int(n), int(dt), float(eps),
                                  int(out_mask), int(qdt), _ptr(y1), _ptr(scale1), _ptr(y2),
                                  _ptr(scale2), _ptr(x_out), _ptr(workspace),
                                  int(workspace_bytes), _stream(stream),
                                  ctypes.addressof(plan))


def arnq_run_static_scratch(x1, x2, gamma, beta, smooth1, smooth2, rows, n, dt, eps, out_mask, qdt,
                            y1, scale1, y2, scale2, x_out, stream) -> int:
    return lib().arnq_run_static_scratch(_ptr(x1), _ptr(x2), _ptr(gamma), _ptr(beta),
                                         _ptr(smooth1), _ptr(smooth2), int(rows), int(n), int(dt),
                                         float(eps), int(out_mask), int(qdt), _ptr(y1),
                                         _ptr(scale1), _ptr(y2), _ptr(scale2), _ptr(x_out),
                                         _stream(stream))
