"""ctypes loader for the plain-C fp64 full-state oracle (``c/gdn_fullstate.c``).

TEST INFRASTRUCTURE: used by the tests (cross-checked against ``gdn``) and by
the benchmark's CPU-baseline leg, which times it on the host cores.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Dict, List, Optional, Sequence

import numpy as np

from .gdn import to_f64

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "c", "gdn_fullstate.c")
_LIB = os.path.join(_HERE, "c", "libgdn_oracle.so")
_lib: Optional[ctypes.CDLL] = None


def build(force: bool = False) -> str:
    """Compile the C oracle with gcc (fp64, no FMA contraction, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fopenmp", "-fPIC",
               "-shared", _SRC, "-o", _LIB + ".tmp", "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def _load() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.POINTER
        lib.gdn_oracle_beam_decode.restype = ctypes.c_int
        lib.gdn_oracle_beam_decode.argtypes = [
            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            P(ctypes.c_int32), P(ctypes.c_double),
            P(ctypes.c_double), P(ctypes.c_double), P(ctypes.c_double),
            P(ctypes.c_double), P(ctypes.c_double), P(ctypes.c_int32),
            P(ctypes.c_double), P(ctypes.c_double), ctypes.c_int]
        lib.gdn_oracle_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def max_threads() -> int:
    return int(_load().gdn_oracle_threads())


def _ptr(a: np.ndarray, ct):
    return a.ctypes.data_as(ctypes.POINTER(ct))


def beam_decode_fullstate(S0, steps: Sequence[Dict], nthreads: int = 0) -> List[Dict[str, np.ndarray]]:
    """Same contract as ``gdn.beam_decode_fullstate`` (o and delta per step)."""
    lib = _load()
    S0 = np.ascontiguousarray(to_f64(S0))
    R, H, dv, dk = S0.shape
    T = len(steps)
    Ws = np.array([int(np.asarray(s["parents"]).shape[-1]) for s in steps], dtype=np.int32)

    def cat(key, f64=True):
        parts = [to_f64(s[key]).reshape(-1) if f64 else
                 np.asarray(s[key], dtype=np.int32).reshape(-1) for s in steps]
        if not parts:
            return np.zeros(1, dtype=np.float64 if f64 else np.int32)
        return np.ascontiguousarray(np.concatenate(parts))

    q, k, v = cat("q"), cat("k"), cat("v")
    g, beta = cat("g"), cat("beta")
    par = cat("parents", f64=False)
    o = np.zeros_like(v)
    delta = np.zeros_like(v)
    rc = lib.gdn_oracle_beam_decode(
        R, H, dk, dv, T, _ptr(Ws, ctypes.c_int32), _ptr(S0, ctypes.c_double),
        _ptr(q, ctypes.c_double), _ptr(k, ctypes.c_double), _ptr(v, ctypes.c_double),
        _ptr(g, ctypes.c_double), _ptr(beta, ctypes.c_double), _ptr(par, ctypes.c_int32),
        _ptr(o, ctypes.c_double), _ptr(delta, ctypes.c_double), int(nthreads))
    if rc == -2:
        raise ValueError("parent index out of range")
    if rc != 0:
        raise RuntimeError(f"C oracle failed with code {rc}")
    out, off = [], 0
    for t in range(T):
        n = R * int(Ws[t]) * H * dv
        shp = (R, int(Ws[t]), H, dv)
        out.append({"o": o[off:off + n].reshape(shp), "delta": delta[off:off + n].reshape(shp)})
        off += n
    return out
