"""fp64 CPU oracle for kernelized linear attention (test infrastructure).

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this package.  The product path (the CUDA library and its
Python binding) never touches it, and it shares no code with them.

The arithmetic lives in ``la_oracle.c`` (plain C, double precision, one head
at a time, OpenMP across heads); this module compiles it with gcc on first
use and marshals numpy arrays to it.  Inputs are converted to float64 first,
so a bf16 tensor enters the oracle with exactly the values the GPU reads.

Functions (all arrays [B, H, N, D] contiguous, D innermost):
  forward(q, k, v, causal, phi)            -> o, S_final, z_final
  quadratic(q, k, v, causal, phi)          -> o   (small N only)
  backward(q, k, v, dO, causal, phi)       -> dq, dk, dv
  decode_step(S, z, q, k, v, phi)          -> o   (updates S, z in place)
  phi_map(x, phi), dphi_map(x, phi)        -> elementwise feature map / slope
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

PHI_ELU1 = 0
PHI_RELU_EPS = 1

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "la_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile la_oracle.c into liboracle.so next to it (gcc, -fopenmp)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-fno-fast-math", "-ffp-contract=off", "-fopenmp",
           "-fPIC", "-shared", "-std=c11", _SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P = ctypes.POINTER(ctypes.c_double)
            i64 = ctypes.c_int64
            ci = ctypes.c_int
            lib.oracle_forward.argtypes = [P, P, P, P, P, P, i64, i64, i64, i64, ci, ci]
            lib.oracle_quadratic.argtypes = [P, P, P, P, i64, i64, i64, i64, ci, ci]
            lib.oracle_backward.argtypes = [P, P, P, P, P, P, P, i64, i64, i64, i64, ci, ci]
            lib.oracle_decode_step.argtypes = [P, P, P, P, P, P, i64, i64, i64, ci]
            lib.oracle_set_threads.argtypes = [ci]
            lib.oracle_max_threads.restype = ci
            for fn in ("oracle_forward", "oracle_quadratic", "oracle_backward",
                       "oracle_decode_step", "oracle_set_threads"):
                getattr(lib, fn).restype = None
            _lib = lib
    return _lib


def _f64(x) -> np.ndarray:
    """Exact float64 copy of a numpy array or a (CPU/GPU) torch tensor."""
    if not isinstance(x, np.ndarray):
        x = x.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(x, dtype=np.float64)


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def set_threads(n: int) -> None:
    _load().oracle_set_threads(int(n))


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def _shape4(q):
    if q.ndim != 4:
        raise ValueError("expected [B, H, N, D]")
    return q.shape


def forward(q, k, v, causal: bool, phi: int = PHI_ELU1):
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, N, D = _shape4(q)
    o = np.empty_like(q)
    S = np.empty((B, H, D, D))
    z = np.empty((B, H, D))
    _load().oracle_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(S), _ptr(z),
                           B, H, N, D, int(bool(causal)), int(phi))
    return o, S, z


def quadratic(q, k, v, causal: bool, phi: int = PHI_ELU1):
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, N, D = _shape4(q)
    o = np.empty_like(q)
    _load().oracle_quadratic(_ptr(q), _ptr(k), _ptr(v), _ptr(o),
                             B, H, N, D, int(bool(causal)), int(phi))
    return o


def backward(q, k, v, dO, causal: bool, phi: int = PHI_ELU1):
    q, k, v, dO = _f64(q), _f64(k), _f64(v), _f64(dO)
    B, H, N, D = _shape4(q)
    dq, dk, dv = np.empty_like(q), np.empty_like(q), np.empty_like(q)
    _load().oracle_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(dO), _ptr(dq), _ptr(dk),
                            _ptr(dv), B, H, N, D, int(bool(causal)), int(phi))
    return dq, dk, dv


def decode_step(S: np.ndarray, z: np.ndarray, q, k, v, phi: int = PHI_ELU1):
    """One in-place step on float64 arrays S [B,H,D,D], z [B,H,D]; q,k,v [B,H,D]."""
    if S.dtype != np.float64 or not S.flags.c_contiguous:
        raise TypeError("S must be a C-contiguous float64 array (updated in place)")
    if z.dtype != np.float64 or not z.flags.c_contiguous:
        raise TypeError("z must be a C-contiguous float64 array (updated in place)")
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, D = q.shape
    o = np.empty_like(q)
    _load().oracle_decode_step(_ptr(S), _ptr(z), _ptr(q), _ptr(k), _ptr(v), _ptr(o),
                               B, H, D, int(phi))
    return o


def phi_map(x, phi: int = PHI_ELU1) -> np.ndarray:
    """The elementwise feature map on float64 values (elu+1 or relu+1e-6)."""
    x = _f64(x)
    if phi == PHI_ELU1:
        return np.where(x > 0, x + 1.0, np.exp(np.minimum(x, 0.0)))
    return np.maximum(x, 0.0) + 1e-6


def dphi_map(x, phi: int = PHI_ELU1) -> np.ndarray:
    x = _f64(x)
    if phi == PHI_ELU1:
        return np.where(x > 0, 1.0, np.exp(np.minimum(x, 0.0)))
    return np.where(x > 0, 1.0, 0.0)
