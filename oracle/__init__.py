"""CPU oracle for the fused add + RMSNorm + dynamic-quant operator.

TEST INFRASTRUCTURE ONLY.  The product package never imports this module; only
``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py``
do.  The arithmetic lives in ``arnq_oracle.c`` (plain C, fp64); this file only
compiles it with gcc and marshals numpy arrays through ctypes.

Every 16-bit floating-point array crosses this boundary as its raw bit
pattern (``numpy.uint16``); ``dtype`` says how to read it ("bf16" or "fp16").
The operator definitions followed are those of the CANN pages
"aclnnAddRmsNormDynamicQuantV2" (Formula and Constraints sections) and
"aclnnRmsNormDynamicQuant" (formula section); see the C file's header.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "arnq_oracle.c")
_LIB = os.path.join(_HERE, "libarnq_oracle.so")

# The oracle's own status codes (see arnq_oracle.c).
ORC_OK, ORC_BAD_MASK, ORC_EMPTY, ORC_BAD_SHAPE, ORC_NULL, ORC_BAD_ARG = range(6)
DTYPES = {"bf16": 0, "fp16": 1}
QDTYPES = {"int8": 0, "int4": 1, "int4_int32": 2}
QMAX = {"int8": 127, "int4": 7, "int4_int32": 7}


def _code_array(rows, n, qdtype):
    """Output array of one quantized output: int8 [rows, n], packed uint8
    [rows, n/2], or uint32 words [rows, n/8] of eight INT4 codes."""
    if qdtype == "int8":
        return np.zeros((rows, n), np.int8)
    if qdtype == "int4_int32":
        return np.zeros((rows, n // 8 if n % 8 == 0 else 0), np.uint32)
    return np.zeros((rows, n // 2), np.uint8)


def build(force: bool = False) -> str:
    """Compile the oracle with gcc into a shared object next to the source."""
    if not force and os.path.exists(_LIB) and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC):
        return _LIB
    cmd = ["gcc", "-O2", "-std=c11", "-Wall", "-Wextra", "-fPIC", "-shared",
           "-ffp-contract=off", "-fno-fast-math", "-o", _LIB, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    return _LIB


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        p, i64, i32, f32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float
        L.orc_add_rms_norm_dynamic_quant_v2.argtypes = [
            p, p, p, p, p, p, i64, i64, i32, f32, i32, i32, p, p, p, p, p, p, p, p]
        L.orc_add_rms_norm_dynamic_quant_v2.restype = i32
        L.orc_rms_norm_dynamic_quant.argtypes = [p, p, p, p, i64, i64, i32, f32, i32, p, p, p, p]
        L.orc_rms_norm_dynamic_quant.restype = i32
        L.orc_selected_outputs.argtypes = [i32, i32, i32, p, p]
        L.orc_selected_outputs.restype = i32
        L.orc_decode16.argtypes = [ctypes.c_uint16, i32]
        L.orc_decode16.restype = ctypes.c_double
        L.orc_encode16_rne.argtypes = [f32, i32]
        L.orc_encode16_rne.restype = ctypes.c_uint16
        L.orc_round_half_even.argtypes = [ctypes.c_double]
        L.orc_round_half_even.restype = ctypes.c_double
        L.orc_add_round.argtypes = [ctypes.c_uint16, ctypes.c_uint16, i32]
        L.orc_add_round.restype = ctypes.c_uint16
        L.orc_decode16_array.argtypes = [p, i64, i32, p]
        L.orc_decode16_array.restype = None
        L.orc_encode16_array.argtypes = [p, i64, i32, p]
        L.orc_encode16_array.restype = None
        L.orc_add_round_array.argtypes = [p, p, i64, i32, p]
        L.orc_add_round_array.restype = None
        _lib = L
    return _lib


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data


def _u16(a, shape=None) -> Optional[np.ndarray]:
    if a is None:
        return None
    a = np.ascontiguousarray(a, dtype=np.uint16)
    if shape is not None:
        assert a.shape == shape, (a.shape, shape)
    return a


def mask_code(mask) -> int:
    """None -> -1 (absent); (m0, m1) -> bit0 = m0, bit1 = m1."""
    if mask is None:
        return -1
    m0, m1 = mask
    return (1 if m0 else 0) | (2 if m1 else 0)


def selected_outputs(mask, has_s1: bool, has_s2: bool):
    """Returns (status, y1_on, y2_on) per the Formula and Constraints sections."""
    a, b = ctypes.c_int(0), ctypes.c_int(0)
    st = lib().orc_selected_outputs(mask_code(mask), int(has_s1), int(has_s2),
                                    ctypes.byref(a), ctypes.byref(b))
    return st, bool(a.value), bool(b.value)


def add_rms_norm_dynamic_quant_v2(x1, x2, gamma, beta=None, smooth1=None, smooth2=None, *,
                                  eps: float, mask=None, qdtype: str = "int8",
                                  dtype: str = "bf16", debug: bool = False) -> dict:
    """Runs the oracle of aclnnAddRmsNormDynamicQuantV2 on [rows, n] bit patterns.

    Returns a dict with "status", and, when it is ORC_OK: "x_out" (uint16 bits),
    "y1"/"scale1" and "y2"/"scale2" (None when not produced; codes are int8
    [rows, n], packed uint8 [rows, n/2], or for qdtype "int4_int32" uint32
    [rows, n/8] words of eight codes), "clamp_hits", and with debug=True
    the fp64 "in1"/"in2" arrays.
    """
    x1 = _u16(x1)
    rows, n = x1.shape if x1.ndim == 2 else (0, 0)
    x2 = _u16(x2, x1.shape)
    gamma, beta = _u16(gamma, (n,)), _u16(beta, (n,))
    smooth1, smooth2 = _u16(smooth1, (n,)), _u16(smooth2, (n,))
    st, on1, on2 = selected_outputs(mask, smooth1 is not None, smooth2 is not None)
    out = {"status": st, "y1": None, "scale1": None, "y2": None, "scale2": None,
           "x_out": None, "in1": None, "in2": None, "clamp_hits": 0}
    if st != ORC_OK:
        return out
    x_out = np.zeros((rows, n), np.uint16)
    y1 = _code_array(rows, n, qdtype) if on1 else None
    s1 = np.zeros((rows,), np.float32) if on1 else None
    y2 = _code_array(rows, n, qdtype) if on2 else None
    s2 = np.zeros((rows,), np.float32) if on2 else None
    in1 = np.zeros((rows, n), np.float64) if debug else None
    in2 = np.zeros((rows, n), np.float64) if debug else None
    hits = ctypes.c_int64(0)
    st = lib().orc_add_rms_norm_dynamic_quant_v2(
        _ptr(x1), _ptr(x2), _ptr(gamma), _ptr(beta), _ptr(smooth1), _ptr(smooth2),
        rows, n, DTYPES[dtype], float(eps), mask_code(mask), QDTYPES[qdtype],
        _ptr(y1), _ptr(s1), _ptr(y2), _ptr(s2), _ptr(x_out), _ptr(in1), _ptr(in2),
        ctypes.addressof(hits))
    out.update(status=st, x_out=x_out, y1=y1, scale1=s1, y2=y2, scale2=s2, in1=in1, in2=in2,
               clamp_hits=hits.value)
    return out


def rms_norm_dynamic_quant(x, gamma, beta=None, smooth=None, *, eps: float,
                           qdtype: str = "int8", dtype: str = "bf16", debug: bool = False) -> dict:
    """Runs the oracle of aclnnRmsNormDynamicQuant (no add, one output)."""
    x = _u16(x)
    rows, n = x.shape if x.ndim == 2 else (0, 0)
    gamma, beta, smooth = _u16(gamma, (n,)), _u16(beta, (n,)), _u16(smooth, (n,))
    y = _code_array(rows, n, qdtype)
    scale = np.zeros((rows,), np.float32)
    dbg = np.zeros((rows, n), np.float64) if debug else None
    hits = ctypes.c_int64(0)
    st = lib().orc_rms_norm_dynamic_quant(
        _ptr(x), _ptr(gamma), _ptr(beta), _ptr(smooth), rows, n, DTYPES[dtype], float(eps),
        QDTYPES[qdtype], _ptr(y), _ptr(scale), _ptr(dbg), ctypes.addressof(hits))
    return {"status": st, "y": y, "scale": scale, "in": dbg, "clamp_hits": hits.value}


def decode16(bits: np.ndarray, dtype: str) -> np.ndarray:
    bits = np.ascontiguousarray(bits, dtype=np.uint16).ravel()
    out = np.zeros(bits.shape, np.float64)
    lib().orc_decode16_array(_ptr(bits), bits.size, DTYPES[dtype], _ptr(out))
    return out


def encode16(values: np.ndarray, dtype: str) -> np.ndarray:
    f = np.ascontiguousarray(values, dtype=np.float32).ravel()
    out = np.zeros(f.shape, np.uint16)
    lib().orc_encode16_array(_ptr(f), f.size, DTYPES[dtype], _ptr(out))
    return out


def add_round(a: np.ndarray, b: np.ndarray, dtype: str) -> np.ndarray:
    a = np.ascontiguousarray(a, dtype=np.uint16).ravel()
    b = np.ascontiguousarray(b, dtype=np.uint16).ravel()
    out = np.zeros(a.shape, np.uint16)
    lib().orc_add_round_array(_ptr(a), _ptr(b), a.size, DTYPES[dtype], _ptr(out))
    return out


def round_half_even(v: float) -> float:
    return lib().orc_round_half_even(float(v))

