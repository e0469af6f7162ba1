"""ctypes front of ``attn_oracle.c`` (the threaded fp64 C oracle).

TEST INFRASTRUCTURE ONLY: imported by tests, the smoke check and bench.py's
CPU legs, never by the product path.

``build()`` compiles the C file with gcc into ``liboracle_attn.so`` next to
it; ``attention_fwd`` / ``attention_pairs`` take numpy arrays (or CPU torch
tensors) holding the exact input values and return float64 results.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attn_oracle.c")
_LIB = os.path.join(_HERE, "liboracle_attn.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle (plain gcc, -O2, pthreads)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread",
                               _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        i64, i32, f64p = ctypes.c_int64, ctypes.c_int, ctypes.POINTER(ctypes.c_double)
        f32p, i32p = ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ctypes.c_int)
        lib.oracle_attn_fwd.restype = ctypes.c_int
        lib.oracle_attn_fwd.argtypes = [f32p, f32p, f32p, f64p, f64p,
                                        i32, i32, i32, i32, i32p, i32, i32,
                                        i64, i64, i64, i64, i64, i64, i64, i64, i64,
                                        ctypes.c_double, i32, i32, i32p, i32]
        _lib = lib
    return _lib


def _as_f32(x):
    if hasattr(x, "detach"):
        x = x.detach().to("cpu").float().numpy()
    return np.asarray(x, dtype=np.float32)


def _ptr(a, ct):
    return a.ctypes.data_as(ctypes.POINTER(ct))


def attention_fwd(q, k, v, skv_lens, scale: float, causal: bool, nthreads: int | None = None,
                  pairs=None):
    """q [B,Hq,Sq,dk], k [B,Hkv,S,dk], v [B,Hkv,S,dv] (strided views allowed:
    the innermost dimension must be contiguous).  Returns float64
    (out [B,Hq,Sq,dv], lse [B,Hq,Sq]); with ``pairs`` (a list of (b, h)) only
    those heads are computed and the rest of the outputs stay NaN."""
    lib = _load()
    qf, kf, vf = _as_f32(q), _as_f32(k), _as_f32(v)
    # keep views; float32 arrays from torch/numpy conversions may be copies,
    # which is fine as long as strides are in elements
    for a in (qf, kf, vf):
        if a.strides[-1] != 4:
            raise ValueError("innermost dimension must be contiguous")
    B, Hq, Sq, dk = qf.shape
    Hkv, dv = kf.shape[1], vf.shape[-1]
    skv = np.ascontiguousarray(np.asarray(skv_lens, dtype=np.int32))
    out = np.full((B, Hq, Sq, dv), np.nan)
    lse = np.full((B, Hq, Sq), np.nan)

    def st(a):
        return [s // 4 for s in a.strides[:3]]

    # base pointers must address element [0,0,0,0] of possibly offset views
    qs, ks, vs = st(qf), st(kf), st(vf)
    rows_arr = None
    nrows = 0
    if pairs is not None:
        rows_arr = np.ascontiguousarray(np.asarray(pairs, dtype=np.int32).reshape(-1, 2))
        nrows = rows_arr.shape[0]
    nthreads = nthreads or os.cpu_count() or 1
    rc = lib.oracle_attn_fwd(
        ctypes.cast(qf.__array_interface__["data"][0], ctypes.POINTER(ctypes.c_float)),
        ctypes.cast(kf.__array_interface__["data"][0], ctypes.POINTER(ctypes.c_float)),
        ctypes.cast(vf.__array_interface__["data"][0], ctypes.POINTER(ctypes.c_float)),
        _ptr(out, ctypes.c_double), _ptr(lse, ctypes.c_double),
        B, Hq, Hkv, Sq, _ptr(skv, ctypes.c_int), dk, dv,
        *qs, *ks, *vs, float(scale), int(bool(causal)), int(nthreads),
        _ptr(rows_arr, ctypes.c_int) if rows_arr is not None else None, nrows)
    if rc != 0:
        raise ValueError("oracle_attn_fwd rejected its arguments")
    return out, lse
