"""ctypes wrapper of oracle/cmx.c: the MX block quantiser and decoder of oracle/mx.py
restated in C.  TEST INFRASTRUCTURE ONLY.

Same rules, same value tables (taken from oracle.mx), same results: pinned bit-exact
against ``oracle.mx.quantize_mx`` / ``dequantize_mx`` by ``tests/test_oracle_mx.py``.  It exists so that the
parity tests at the Kimi-K3 shapes can quantise many experts' weights quickly.  ``build()``
compiles it with gcc into ``oracle/_cmx.so`` (it is built on first use when missing).
"""
import ctypes
import os
import subprocess

import numpy as np

from . import mx

_HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(_HERE, "cmx.c")
LIB = os.path.join(_HERE, "_cmx.so")
_lib = None


def build(force=False):
    """Compile cmx.c into _cmx.so (plain gcc, -O2, no fast-math)."""
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        tmp = LIB + ".tmp%d" % os.getpid()
        subprocess.run(["gcc", "-O2", "-fPIC", "-shared", "-fno-fast-math", SRC, "-o", tmp, "-lm"], check=True)
        os.replace(tmp, LIB)
    return LIB


def _load():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        f = L.mx_quantize_f32
        f.argtypes = [ctypes.c_void_p, ctypes.c_long, ctypes.c_long, ctypes.c_void_p, ctypes.c_int, ctypes.c_int,
                      ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p]
        f.restype = None
        g = L.mx_dequantize_f64
        g.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_long, ctypes.c_long, ctypes.c_void_p, ctypes.c_int,
                      ctypes.c_void_p]
        g.restype = None
        _lib = L
    return _lib


_FORMATS = {"e2m1": (mx._E2M1_POS, mx.E2M1_EMAX, 0x8), "e4m3": (mx._E4M3_POS, mx.E4M3_EMAX, 0x80)}


def quantize_mx_f32(values, fmt):
    """quantize_mx for fp32 values [..., K] (K % 32 == 0): (codes uint8 [..., K], scale
    bytes uint8 [..., K/32]), equal to oracle.mx.quantize_mx(values, fmt)."""
    v = np.ascontiguousarray(values, dtype=np.float32)
    K = v.shape[-1]
    if K % mx.BLOCK:
        raise ValueError("last dimension must be a multiple of 32")
    pos, emax, sign_bit = _FORMATS[fmt]
    pos = np.ascontiguousarray(pos, dtype=np.float64)
    rows = v.size // K
    codes = np.empty(v.shape, dtype=np.uint8)
    scales = np.empty(v.shape[:-1] + (K // mx.BLOCK,), dtype=np.uint8)
    _load().mx_quantize_f32(v.ctypes.data, rows, K, pos.ctypes.data, len(pos), emax, sign_bit,
                            codes.ctypes.data, scales.ctypes.data)
    return codes, scales


def dequantize_mx_f64(codes, scales, fmt):
    """dequantize_mx: exact fp64 values of MX codes [..., K] with scale bytes [..., K/32],
    equal to oracle.mx.dequantize_mx(codes, scales, fmt)."""
    c = np.ascontiguousarray(codes, dtype=np.uint8)
    sc = np.ascontiguousarray(scales, dtype=np.uint8)
    K = c.shape[-1]
    table, mask = (mx.E2M1_TABLE, 15) if fmt == "e2m1" else (mx.E4M3_TABLE, 255)
    table = np.ascontiguousarray(table, dtype=np.float64)
    out = np.empty(c.shape, dtype=np.float64)
    _load().mx_dequantize_f64(c.ctypes.data, sc.ctypes.data, c.size // K, K, table.ctypes.data, mask,
                              out.ctypes.data)
    return out
